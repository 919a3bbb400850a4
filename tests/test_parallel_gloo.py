"""Batch sharding of the IA layer over ranks, on CPU with 2 gloo ranks.

Each rank runs a stand-in for the library on its own batch slice (the fp64
oracle, on the host: test infrastructure); the test checks that the shards
cover every (b,h) sequence exactly once, that the reassembled outputs equal
the unsharded run, and that the all-reduced dDelta equals the one-rank sum
over the whole batch."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from ssm_token_mixer_b200.parallel import batch_shard


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_fwd_bwd(q, k, v, delta, dO, M):
    import oracle
    g = oracle.backward(q, k, v, delta, dO, M)
    return {key: torch.from_numpy(np.asarray(g[key])).clone() for key in ("o", "dq", "dk", "dv", "dDelta")}


def _oracle_prefill(q, k, v, delta, M):
    import oracle
    r = oracle.forward(q, k, v, delta, M, want_state=False)
    return {"o": torch.from_numpy(r["o"]).clone()}


def _worker(rank, world, port, B, q_out):
    import datetime

    import torch.distributed as dist

    from ssm_token_mixer_b200 import parallel, synthetic
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        inp = synthetic.layer_inputs(B, 2, 24, 4, 3, "f32", seed=11, with_grad=True)
        loc = {n: parallel.local_rows(inp[n]) for n in ("q", "k", "v", "dO")}
        lo, hi = parallel.batch_shard(B, rank, world)
        r = parallel.fwd_bwd_sharded(loc["q"], loc["k"], loc["v"], inp["delta"], loc["dO"], 4,
                                     compute=_oracle_fwd_bwd)
        p = parallel.prefill_sharded(loc["q"], loc["k"], loc["v"], inp["delta"], 4, compute=_oracle_prefill)
        full = {n: parallel.gather_batch(r[n], B) for n in ("o", "dq", "dk", "dv")}
        full_o = parallel.gather_batch(p["o"], B)
        q_out.put((rank, lo, hi, {n: t.numpy() for n, t in full.items()}, full_o.numpy(),
                   r["dDelta"].numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("B", [3, 4])
def test_sharded_training_matches_one_rank(B, oracle_mod):
    from ssm_token_mixer_b200 import synthetic
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, B, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    # the shards cover every batch row once, in order
    rows = [i for _, lo, hi, *_ in res for i in range(lo, hi)]
    assert rows == list(range(B))
    inp = synthetic.layer_inputs(B, 2, 24, 4, 3, "f32", seed=11, with_grad=True)
    one = _oracle_fwd_bwd(inp["q"], inp["k"], inp["v"], inp["delta"], inp["dO"], 4)
    one_o = _oracle_prefill(inp["q"], inp["k"], inp["v"], inp["delta"], 4)["o"].numpy()
    for rank, lo, hi, full, full_o, dD in res:
        for n in ("o", "dq", "dk", "dv"):
            np.testing.assert_allclose(full[n], one[n].numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(full_o, one_o, rtol=0, atol=1e-12)
        # every rank holds the whole batch's dDelta: the sum of the shards' partial sums
        np.testing.assert_allclose(dD, one["dDelta"].numpy(), rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("B,world", [(8, 8), (8, 3), (2, 4), (96, 7)])
def test_batch_shard_covers_exactly(B, world):
    spans = [batch_shard(B, r, world) for r in range(world)]
    assert [i for lo, hi in spans for i in range(lo, hi)] == list(range(B))
    sizes = [hi - lo for lo, hi in spans]
    assert max(sizes) - min(sizes) <= 1
