"""Data-parallel execution of the IA layer across GPUs (one process per GPU).

The layer's (b,h) sequences are independent (each carries its own recurrent
state), so forward, backward and decode shard over the batch with no
communication on the data path: every rank runs the library on its own
batch slice.  The one exchange is in training, where Delta is a per-head
parameter shared by the whole batch: its gradient dDelta [H] is the sum over
all sequences, so the ranks add their partial sums with one all-reduce.

A single sequence too long for one GPU can also be split along N (the
summary's sec. A.2 parallel passes with sequential state passing, across
GPUs): each rank runs its span from a zero state, the ranks exchange their
local end states with one all-gather, each rank composes its carry-in with
the library's ia_state_carry (lambda^L S + S_local), and runs its span again
from that carry.

This module is the plumbing around the library calls: which batch rows or
tokens a rank owns, the collectives over a torch.distributed process group
(NCCL on GPUs), and a gather for callers that want the whole batch back.
The compute itself is the library's (the ``compute`` and ``carry``
arguments exist so that host tests can substitute stand-ins).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def _world(group=None):
    if dist.is_available() and dist.is_initialized():
        return dist.get_rank(group), dist.get_world_size(group)
    return 0, 1


def batch_shard(B: int, rank: int, world: int):
    """Contiguous rows [lo, hi) of a batch of B that `rank` of `world` owns.
    Shards differ in size by at most one row; with B < world some are empty."""
    if B < 0 or world <= 0 or not 0 <= rank < world:
        raise ValueError(f"bad shard request B={B} rank={rank} world={world}")
    per, extra = divmod(B, world)
    lo = rank * per + min(rank, extra)
    return lo, lo + per + (1 if rank < extra else 0)


def local_rows(x: torch.Tensor, group=None) -> torch.Tensor:
    """This rank's batch slice of a [B, ...] tensor (a view, no copy)."""
    rank, world = _world(group)
    lo, hi = batch_shard(x.shape[0], rank, world)
    return x.narrow(0, lo, hi - lo)


def prefill_sharded(q, k, v, delta, M, group=None, compute=None, **kw):
    """Prefill of this rank's sequences.  q, k, v are the rank's own batch
    slice; no collective is needed (the outputs stay sharded)."""
    if compute is None:
        import ssm_token_mixer_b200 as ia
        compute = ia.prefill_fwd
    return compute(q, k, v, delta, M, **kw)


def fwd_bwd_sharded(q, k, v, delta, dO, M, group=None, compute=None, **kw):
    """Training step of this rank's sequences, then one all-reduce (sum) of
    dDelta [H] over the group so that every rank holds the gradient of the
    whole global batch.  dq, dk, dv stay sharded."""
    if compute is None:
        import ssm_token_mixer_b200 as ia
        compute = ia.fwd_bwd
    r = compute(q, k, v, delta, dO, M, **kw)
    _, world = _world(group)
    if world > 1:
        dist.all_reduce(r["dDelta"], op=dist.ReduceOp.SUM, group=group)
    return r


def gather_batch(x: torch.Tensor, B: int, group=None) -> torch.Tensor:
    """Reassemble a [B, ...] tensor from every rank's batch slice (for
    evaluation and tests; not on the training path).  Uneven slices are
    padded to the largest for the all_gather and trimmed afterwards."""
    rank, world = _world(group)
    if world == 1:
        return x
    sizes = [batch_shard(B, r, world) for r in range(world)]
    most = max(hi - lo for lo, hi in sizes)
    pad = x.new_zeros((most,) + tuple(x.shape[1:]))
    pad[: x.shape[0]] = x
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[: hi - lo] for p, (lo, hi) in zip(parts, sizes)], dim=0)


def sequence_span(N: int, rank: int, world: int):
    """Contiguous tokens [lo, hi) of a sequence of N that `rank` owns (rank
    order is sequence order); spans differ in length by at most one."""
    return batch_shard(N, rank, world)


def prefill_sequence_sharded(q, k, v, delta, M, group=None, A=None, state_in=None, want_state=False,
                             compute=None, carry=None):
    """Prefill of sequences split along N over the ranks of `group`: q, k, v
    [B,H,N_r,d] are this rank's span (rank r holds the r-th span).  Rank 0
    runs once (from state_in); every other rank runs its span from a zero
    state, all ranks all-gather those end states and the span lengths, and
    rank r composes its carry-in C_r = lambda^(L_{r-1}) C_{r-1} + S_{r-1}
    (C_1 = rank 0's end state) and runs its span again from C_r.  Returns
    this rank's dict(o, state, ...): o for its span; with want_state the last
    rank's state is the end state of the whole sequence."""
    import ssm_token_mixer_b200 as ia
    compute = compute or ia.prefill_fwd
    carry = carry or ia.state_carry
    rank, world = _world(group)
    if world == 1:
        return compute(q, k, v, delta, M, A=A, state_in=state_in, want_state=want_state)
    B, H, n_local, d_xi = q.shape
    d_v = v.shape[-1]
    first = compute(q, k, v, delta, M, A=A, state_in=state_in if rank == 0 else None, want_state=True)
    local = first["state"]
    states = [torch.empty_like(local) for _ in range(world)]
    dist.all_gather(states, local, group=group)
    n_t = torch.tensor([n_local], dtype=torch.int64, device=local.device)
    lengths = [torch.empty_like(n_t) for _ in range(world)]
    dist.all_gather(lengths, n_t, group=group)
    if rank == 0:
        return first
    c = states[0]
    for p in range(1, rank):
        c = carry(states[p], delta, M, int(lengths[p].item()), B, H, d_xi, d_v, carry_in=c, A=A)
    return compute(q, k, v, delta, M, A=A, state_in=c, want_state=want_state)
