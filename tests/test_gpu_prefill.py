"""Prefill parity on the GPU: the CUDA path (through the C-ABI) against the
fp64 oracle on the same seeded inputs.  Bars: 1e-4 for fp32 inputs, 2e-2
for bf16 inputs, normwise per (b,h) slice on num and den separately (o where
den is away from zero) -- see parity.py."""
import numpy as np
import pytest
import torch

import ssm_token_mixer_b200 as ia
from gpu_common import device, gpu_prefill, state_slices
from parity import TOL_BF16, TOL_F32, report, slice_rel
from ssm_token_mixer_b200 import synthetic
from ssm_token_mixer_b200.workloads import WORKLOADS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    return device()


def oracle_state(oracle_mod, st, B, H, M, dx, dv):
    U, G, e = oracle_mod.split_state(st, B, H, M, dx, dv)
    return U, G, e


def check_state(st_gpu, st_ref, B, H, M, dx, dv, tol):
    s = st_gpu.double().numpy()
    n1, n2 = 2 * B * H * M * dx, 2 * B * H * M * dv
    Ug = s[:n1].view(np.complex128).reshape(B, H, M, dx)
    Gg = s[n1:n1 + n2].view(np.complex128).reshape(B, H, M, dv)
    eg = s[n1 + n2:].view(np.complex128).reshape(B, H, M)
    Ur, Gr, er = st_ref
    assert slice_rel(Ug, Ur, (-2, -1)) < tol
    assert slice_rel(Gg, Gr, (-2, -1)) < tol
    assert slice_rel(eg, er, (-1,)) < tol


def test_tiny_f32_workload(oracle_mod, dev):
    w = WORKLOADS["tiny_f32"]
    inp = synthetic.workload_inputs(w)
    r = gpu_prefill(inp, w.M, dev)
    ref = oracle_mod.forward(inp["q"], inp["k"], inp["v"], inp["delta"], w.M)
    rep = report(r["num"], r["den"], r["o"], ref)
    assert max(rep.values()) < TOL_F32, rep
    check_state(r["state"], oracle_mod.split_state(ref["state"], w.B, w.H, w.M, w.d_xi, w.d_v),
                w.B, w.H, w.M, w.d_xi, w.d_v, TOL_F32)


@pytest.mark.parametrize("dx,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("N", [1, 37, 64, 200])
def test_tensor_core_prefill_small(oracle_mod, dev, dx, dv, N):
    B, H, M = 2, 3, 64
    inp = synthetic.layer_inputs(B, H, N, dx, dv, "bf16", seed=7 * N + dx + dv)
    r = gpu_prefill(inp, M, dev)
    ref = oracle_mod.forward(inp["q"], inp["k"], inp["v"], inp["delta"], M)
    rep = report(r["num"], r["den"], r["o"], ref)
    assert max(rep.values()) < TOL_BF16, rep
    check_state(r["state"], oracle_mod.split_state(ref["state"], B, H, M, dx, dv), B, H, M, dx, dv,
                TOL_BF16)


@pytest.mark.parametrize("B,H,dx,dv", [(1, 3, 64, 64), (3, 5, 64, 64), (3, 1, 128, 128), (5, 3, 128, 64)])
def test_tensor_core_odd_batch_times_heads(oracle_mod, dev, B, H, dx, dv):
    # odd B*H on the tensor-core path: heads change between streams at
    # arbitrary CTA boundaries, whole streams or ranges as the planner picks
    M, N = 64, 150
    assert ia.prefill_path(B, H, N, dx, dv, M, "bf16") == "tensor_core"
    inp = synthetic.layer_inputs(B, H, N, dx, dv, "bf16", seed=13 * B + H + dx + dv)
    r = gpu_prefill(inp, M, dev)
    ref = oracle_mod.forward(inp["q"], inp["k"], inp["v"], inp["delta"], M)
    rep = report(r["num"], r["den"], r["o"], ref)
    assert max(rep.values()) < TOL_BF16, rep
    check_state(r["state"], oracle_mod.split_state(ref["state"], B, H, M, dx, dv), B, H, M, dx, dv, TOL_BF16)


@pytest.mark.parametrize("M", [1, 16, 48, 96])
def test_bf16_prefill_other_mode_counts(oracle_mod, dev, M):
    # bf16 inputs with M != 64 take the sequential CUDA-core path: same
    # tolerance as the tensor-core path, which only M = 64 runs
    B, H, N, d = 2, 3, 130, 64
    assert ia.prefill_path(B, H, N, d, d, M, "bf16") == "sequential"
    inp = synthetic.layer_inputs(B, H, N, d, d, "bf16", seed=300 + M)
    r = gpu_prefill(inp, M, dev)
    ref = oracle_mod.forward(inp["q"], inp["k"], inp["v"], inp["delta"], M)
    rep = report(r["num"], r["den"], r["o"], ref)
    assert max(rep.values()) < TOL_BF16, rep
    check_state(r["state"], oracle_mod.split_state(ref["state"], B, H, M, d, d), B, H, M, d, d, TOL_BF16)


def test_tensor_core_long_ragged_sequence(oracle_mod, dev):
    # few (b,h) pairs and a long ragged sequence: the planner spreads the
    # chunks over many CTAs, so most ranges start inside the sequence and
    # take their carried state from the look-back
    B, H, N, d, M = 1, 2, 1000, 64, 64
    assert ia.prefill_grid(B, H, N, d, d, M, "bf16") > 2
    inp = synthetic.layer_inputs(B, H, N, d, d, "bf16", seed=11)
    r = gpu_prefill(inp, M, dev)
    ref = oracle_mod.forward(inp["q"], inp["k"], inp["v"], inp["delta"], M)
    rep = report(r["num"], r["den"], r["o"], ref)
    assert max(rep.values()) < TOL_BF16, rep
    check_state(r["state"], oracle_mod.split_state(ref["state"], B, H, M, d, d), B, H, M, d, d, TOL_BF16)


@pytest.mark.parametrize("dtype,tol", [("bf16", TOL_BF16), ("f32", TOL_F32)])
def test_state_in_and_split_prefill(oracle_mod, dev, dtype, tol):
    # P13 on the GPU path: prefill(N1) -> state -> prefill(N2, state_in) == prefill(N1+N2)
    B, H, d, M = 2, 2, 64, 64
    N1, N2 = 130, 300
    inp = synthetic.layer_inputs(B, H, N1 + N2, d, d, dtype, seed=21)
    first = {k: (v[:, :, :N1].contiguous() if k != "delta" else v) for k, v in inp.items()}
    second = {k: (v[:, :, N1:].contiguous() if k != "delta" else v) for k, v in inp.items()}
    r1 = gpu_prefill(first, M, dev)
    r2 = gpu_prefill(second, M, dev, state_in=r1["state"].to(dev))
    ref = oracle_mod.forward(inp["q"], inp["k"], inp["v"], inp["delta"], M)
    num = torch.cat([r1["num"], r2["num"]], dim=2)
    den = torch.cat([r1["den"], r2["den"]], dim=2)
    o = torch.cat([r1["o"], r2["o"]], dim=2)
    rep = report(num, den, o, ref)
    assert max(rep.values()) < tol, rep
    check_state(r2["state"], oracle_mod.split_state(ref["state"], B, H, M, d, d), B, H, M, d, d, tol)


@pytest.mark.parametrize("dx,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("grid", [1, 2, 5, 7, 13, 29, 60])
def test_chunk_pass_ranges(oracle_mod, dev, monkeypatch, dx, dv, grid):
    # The chunk pass gives every CTA an equal range of the (stream, chunk)
    # space.  Forcing the grid exercises every kind of range: many whole
    # streams of different heads in one CTA (grid 1), ranges that start
    # inside a stream and take their state from one or several predecessors,
    # single-piece ranges inside a stream that publish an inclusive state for
    # the next, and ragged last chunks -- all from a carried state_in, with
    # the end state checked too.
    B, H, M = 2, 3, 64
    N0, N = 75, 300                   # 5 chunks per stream, the last one ragged
    inp = synthetic.layer_inputs(B, H, N0 + N, dx, dv, "bf16", seed=31 + grid + dx + dv)
    head = {k: (v[:, :, :N0].contiguous() if k != "delta" else v) for k, v in inp.items()}
    st = gpu_prefill(head, M, dev)["state"].to(dev)
    tail = {k: (v[:, :, N0:].contiguous() if k != "delta" else v) for k, v in inp.items()}
    monkeypatch.setenv("IA_PREFILL_GRID", str(grid))
    total = B * H * (dv // 64) * ((N + 63) // 64)
    assert ia.prefill_grid(B, H, N, dx, dv, M, "bf16") == min(grid, total)
    r = gpu_prefill(tail, M, dev, state_in=st)
    ref = oracle_mod.forward(inp["q"], inp["k"], inp["v"], inp["delta"], M)
    ref_tail = {"num": ref["num"][:, :, N0:], "den": ref["den"][:, :, N0:], "o": ref["o"][:, :, N0:]}
    rep = report(r["num"], r["den"], r["o"], ref_tail)
    assert max(rep.values()) < TOL_BF16, rep
    check_state(r["state"], oracle_mod.split_state(ref["state"], B, H, M, dx, dv), B, H, M, dx, dv, TOL_BF16)


@pytest.mark.parametrize("grid", [20, 37])
def test_look_back_across_many_predecessors(oracle_mod, dev, monkeypatch, grid):
    # One stream of 40 chunks (the last one ragged) over 20 or 37 CTAs: a
    # range's carry sums the published states of up to 36 predecessors, more
    # than the eight awaited per round, so the look-back takes several rounds
    # (and single-piece CTAs publish inclusive states that cut later ones
    # short), from a nonzero state_in.
    B, H, M, dx, dv = 1, 1, 64, 64, 64
    N0, N = 50, 64 * 39 + 23
    inp = synthetic.layer_inputs(B, H, N0 + N, dx, dv, "bf16", seed=400 + grid)
    head = {k: (v[:, :, :N0].contiguous() if k != "delta" else v) for k, v in inp.items()}
    st = gpu_prefill(head, M, dev)["state"].to(dev)
    tail = {k: (v[:, :, N0:].contiguous() if k != "delta" else v) for k, v in inp.items()}
    monkeypatch.setenv("IA_PREFILL_GRID", str(grid))
    assert ia.prefill_grid(B, H, N, dx, dv, M, "bf16") == grid
    r = gpu_prefill(tail, M, dev, state_in=st)
    ref = oracle_mod.forward(inp["q"], inp["k"], inp["v"], inp["delta"], M)
    ref_tail = {"num": ref["num"][:, :, N0:], "den": ref["den"][:, :, N0:], "o": ref["o"][:, :, N0:]}
    rep = report(r["num"], r["den"], r["o"], ref_tail)
    assert max(rep.values()) < TOL_BF16, rep
    check_state(r["state"], oracle_mod.split_state(ref["state"], B, H, M, dx, dv), B, H, M, dx, dv, TOL_BF16)


def test_first_token_returns_v(dev):
    # P3 on the GPU path: o_1 = v_1 whatever q_1 and k_1
    inp = synthetic.layer_inputs(3, 4, 70, 64, 64, "bf16", seed=3)
    r = gpu_prefill(inp, 64, dev)
    v1 = inp["v"][:, :, 0].float()
    assert slice_rel(r["o"][:, :, 0], v1, (-1,)) < 1e-2


def test_tensor_core_matches_cuda_core_path(dev, monkeypatch):
    inp = synthetic.layer_inputs(2, 2, 190, 64, 64, "bf16", seed=5)
    r_tc = gpu_prefill(inp, 64, dev)
    monkeypatch.setenv("IA_PREFILL_SIMT", "1")
    r_ref = gpu_prefill(inp, 64, dev)
    assert slice_rel(r_tc["num"], r_ref["num"], (-2, -1)) < TOL_BF16
    assert slice_rel(r_tc["den"], r_ref["den"], (-1,)) < TOL_BF16


def test_deterministic_rerun(dev):
    inp = synthetic.layer_inputs(2, 2, 300, 64, 64, "bf16", seed=9)
    a = gpu_prefill(inp, 64, dev)
    b = gpu_prefill(inp, 64, dev)
    assert torch.equal(a["o"], b["o"]) and torch.equal(a["state"], b["state"])


@pytest.mark.parametrize("name", ["prefill_125m", "prefill_1p3b", "prefill_1p3b_7168"])
def test_full_size_workloads_sampled(oracle_mod, dev, name):
    w = WORKLOADS[name]
    inp = synthetic.workload_inputs(w)
    r = gpu_prefill(inp, w.M, dev)
    assert torch.isfinite(r["o"]).all()
    rng = np.random.default_rng(0)
    picks = [(int(rng.integers(w.B)), int(rng.integers(w.H))) for _ in range(3)]
    picks.append((w.B - 1, w.H - 1))
    for b, h in picks:
        ref = oracle_mod.forward(inp["q"][b:b + 1, h:h + 1], inp["k"][b:b + 1, h:h + 1],
                                 inp["v"][b:b + 1, h:h + 1], inp["delta"][h:h + 1], w.M)
        rep = report(r["num"][b:b + 1, h:h + 1], r["den"][b:b + 1, h:h + 1],
                     r["o"][b:b + 1, h:h + 1], ref)
        assert max(rep.values()) < TOL_BF16, (b, h, rep)
        U, G, e = oracle_mod.split_state(ref["state"], 1, 1, w.M, w.d_xi, w.d_v)
        Ug, Gg, eg = state_slices(r["state"], w.B, w.H, w.M, w.d_xi, w.d_v, [(b, h)])
        assert slice_rel(Ug, U, (-2, -1)) < TOL_BF16 and slice_rel(Gg, G, (-2, -1)) < TOL_BF16
        assert slice_rel(eg, e, (-1,)) < TOL_BF16
