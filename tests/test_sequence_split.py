"""One sequence split along N: the composition law behind it, the split over
2 and 3 gloo ranks on CPU, and, on the GPU, ia_state_carry and the split run
through the library in one process.

The recurrence is linear in its state, so after a span of L tokens a carried
state S0 has become lambda^L S0 plus what the span builds from zero (summary
sec. A.2: parallel passes over pieces with sequential state passing between
them).  The pins below check that law on the fp64 oracle against a plain
fp64 restatement of lambda^L = exp(L Delta A) written here; the gloo test
runs the ranks' compute with the oracle (test infrastructure) and the
composition with that restatement."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from ssm_token_mixer_b200 import synthetic
from ssm_token_mixer_b200.parallel import sequence_span


def lam_pow(delta, M, L, A=None):
    """lambda^L [H, M] complex: exp(L Delta_h(m) A_m), A = S4D-Lin when None."""
    d = np.asarray(delta, dtype=np.float64)
    a = (np.asarray(A, dtype=np.float64).reshape(M, 2) @ np.array([1.0, 1j]) if A is not None
         else -0.5 + 1j * np.pi * np.arange(M))
    dh = d[:, None] if d.ndim == 1 else d
    return np.exp(L * dh * a[None, :])


def compose(local, delta, M, L, B, H, d_xi, d_v, carry_in=None, A=None):
    """lambda^L carry_in + local over flat fp64 states (the library's layout)."""
    loc = np.asarray(local, dtype=np.float64)
    out = loc.copy()
    if carry_in is None:
        return out
    c = np.asarray(carry_in, dtype=np.float64).view(np.complex128)
    o = out.view(np.complex128)
    lp = lam_pow(delta, M, L, A)                     # [H, M]
    n1, n2 = B * H * M * d_xi, B * H * M * d_v
    o[:n1] += (c[:n1].reshape(B, H, M, d_xi) * lp[None, :, :, None]).ravel()
    o[n1:n1 + n2] += (c[n1:n1 + n2].reshape(B, H, M, d_v) * lp[None, :, :, None]).ravel()
    o[n1 + n2:] += (c[n1 + n2:].reshape(B, H, M) * lp[None]).ravel()
    return out


@pytest.mark.parametrize("per_mode", [False, True])
def test_state_composition_law_on_the_oracle(oracle_mod, per_mode):
    # forward over N1 + N2 from S0 == compose(forward over N2 from zero,
    # carry_in = forward over N1 from S0), for the final state; o over the
    # second span from that carry equals the tail of the whole run
    B, H, M, dx, dv, N1, N2 = 2, 2, 6, 5, 3, 37, 29
    inp = synthetic.layer_inputs(B, H, N1 + N2, dx, dv, "f32", seed=5)
    delta = inp["delta"] if not per_mode else \
        torch.from_numpy(np.exp(np.random.default_rng(6).uniform(np.log(1e-3), np.log(1e-1), (H, M))))
    s0 = np.random.default_rng(7).normal(size=oracle_mod.state_len(B, H, M, dx, dv))
    sl = lambda x, a, b: x[:, :, a:b]
    whole = oracle_mod.forward(inp["q"], inp["k"], inp["v"], delta, M, state_in=s0)
    first = oracle_mod.forward(*(sl(inp[n], 0, N1) for n in ("q", "k", "v")), delta, M, state_in=s0)
    local = oracle_mod.forward(*(sl(inp[n], N1, N1 + N2) for n in ("q", "k", "v")), delta, M)
    c = compose(local["state"], delta, M, N2, B, H, dx, dv, carry_in=first["state"])
    np.testing.assert_allclose(c, whole["state"], rtol=1e-10, atol=1e-12)
    tail = oracle_mod.forward(*(sl(inp[n], N1, N1 + N2) for n in ("q", "k", "v")), delta, M,
                              state_in=first["state"])
    np.testing.assert_allclose(tail["o"], whole["o"][:, :, N1:], rtol=1e-10, atol=1e-12)
    # a wrong decay length breaks it (the pin is sensitive to L)
    bad = compose(local["state"], delta, M, N2 + 1, B, H, dx, dv, carry_in=first["state"])
    assert np.abs(bad - whole["state"]).max() > 1e-6


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_compute(q, k, v, delta, M, A=None, state_in=None, want_state=False):
    import oracle
    r = oracle.forward(q, k, v, delta, M, A=A, state_in=None if state_in is None else state_in.numpy())
    return {"o": torch.from_numpy(r["o"]).clone(), "state": torch.from_numpy(r["state"]).clone()}


def _carry(local, delta, M, L, B, H, d_xi, d_v, carry_in=None, A=None):
    return torch.from_numpy(compose(local.numpy(), delta.numpy(), M, L, B, H, d_xi, d_v,
                                    carry_in=None if carry_in is None else carry_in.numpy()))


def _worker(rank, world, port, N, q_out):
    import datetime

    import torch.distributed as dist

    from ssm_token_mixer_b200 import parallel
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        inp = synthetic.layer_inputs(2, 2, N, 4, 3, "f32", seed=12)
        lo, hi = parallel.sequence_span(N, rank, world)
        span = {n: inp[n][:, :, lo:hi].contiguous() for n in ("q", "k", "v")}
        r = parallel.prefill_sequence_sharded(span["q"], span["k"], span["v"], inp["delta"], 4, want_state=True,
                                              compute=_oracle_compute, carry=_carry)
        q_out.put((rank, lo, hi, r["o"].numpy(), r["state"].numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,N", [(2, 50), (3, 61)])
def test_sequence_split_over_ranks_matches_one_rank(oracle_mod, world, N):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, N, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    assert [t for _, lo, hi, *_ in res for t in range(lo, hi)] == list(range(N))
    inp = synthetic.layer_inputs(2, 2, N, 4, 3, "f32", seed=12)
    one = oracle_mod.forward(inp["q"], inp["k"], inp["v"], inp["delta"], 4)
    o = np.concatenate([r[3] for r in res], axis=2)
    np.testing.assert_allclose(o, one["o"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res[-1][4], one["state"], rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("N,world", [(100, 3), (7, 7), (64, 5)])
def test_sequence_span_covers_exactly(N, world):
    spans = [sequence_span(N, r, world) for r in range(world)]
    assert [t for lo, hi in spans for t in range(lo, hi)] == list(range(N))


@pytest.mark.gpu
@pytest.mark.parametrize("per_mode,with_A,L", [(False, False, 0), (False, False, 1), (True, False, 64),
                                               (False, True, 1000), (True, True, 7168)])
def test_state_carry_on_the_gpu(per_mode, with_A, L):
    # ia_state_carry against the fp64 restatement above, on random states
    import ssm_token_mixer_b200 as ia
    from gpu_common import device
    dev = device()
    B, H, M, dx, dv = 3, 2, 64, 128, 64
    rng = np.random.default_rng(L + 3 * per_mode + with_A)
    delta = np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), (H, M) if per_mode else (H,))).astype(np.float32)
    A = None
    if with_A:
        A = np.stack([-rng.uniform(0.1, 1.0, M), rng.uniform(0, 200, M)], 1).astype(np.float32).ravel()
    n = 2 * B * H * M * (dx + dv + 1)
    loc = rng.normal(size=n).astype(np.float32)
    cin = rng.normal(size=n).astype(np.float32)
    g = lambda x: None if x is None else torch.from_numpy(x).to(dev)
    out = ia.state_carry(g(loc), g(delta), M, L, B, H, dx, dv, carry_in=g(cin), A=g(A))
    ia.check_device_errors()
    ref = compose(loc, delta, M, L, B, H, dx, dv, carry_in=cin, A=A)
    assert np.abs(out.cpu().double().numpy() - ref).max() / np.abs(ref).max() < 1e-6
    # in place (out aliasing carry_in), and no carry at all
    c2 = g(cin)
    ia.state_carry(g(loc), g(delta), M, L, B, H, dx, dv, carry_in=c2, A=g(A), out=c2)
    assert torch.equal(c2.cpu(), out.cpu())
    only = ia.state_carry(g(loc), g(delta), M, L, B, H, dx, dv, A=g(A))
    assert torch.equal(only.cpu(), torch.from_numpy(loc))


@pytest.mark.gpu
@pytest.mark.parametrize("dx,dv,dtype", [(64, 64, "bf16"), (128, 128, "bf16"), (16, 12, "f32")])
def test_sequence_split_through_the_library(oracle_mod, dx, dv, dtype):
    # the ranks of a sequence split, emulated in one process on one GPU: each
    # span from zero, carries composed by ia_state_carry, each span again from
    # its carry; the spans' outputs and the last end state against the oracle
    import ssm_token_mixer_b200 as ia
    from gpu_common import device
    from parity import TOL_BF16, TOL_F32, slice_rel
    dev = device()
    B, H, M, N, world = 2, 3, 64 if dtype == "bf16" else 8, 333, 3
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    inp = synthetic.layer_inputs(B, H, N, dx, dv, dtype, seed=17 + dx)
    g = lambda x: x.to(dev)
    spans = [sequence_span(N, r, world) for r in range(world)]
    part = lambda n, lo, hi: g(inp[n][:, :, lo:hi].contiguous())
    local = [ia.prefill_fwd(part("q", lo, hi), part("k", lo, hi), part("v", lo, hi), g(inp["delta"]), M,
                            want_state=True)["state"] for lo, hi in spans]
    outs, carry = [], None
    for r, (lo, hi) in enumerate(spans):
        if r == 1:
            carry = local[0]
        elif r > 1:
            carry = ia.state_carry(local[r - 1], g(inp["delta"]), M, spans[r - 1][1] - spans[r - 1][0], B, H, dx,
                                   dv, carry_in=carry)
        res = ia.prefill_fwd(part("q", lo, hi), part("k", lo, hi), part("v", lo, hi), g(inp["delta"]), M,
                             state_in=carry, want_state=True)
        outs.append(res["o"].cpu())
    ia.check_device_errors()
    ref = oracle_mod.forward(inp["q"], inp["k"], inp["v"], inp["delta"], M)
    assert slice_rel(torch.cat(outs, dim=2), ref["o"], (-2, -1)) < tol
    st = res["state"].cpu().double().numpy()
    assert np.abs(st - ref["state"]).max() / np.abs(ref["state"]).max() < tol
