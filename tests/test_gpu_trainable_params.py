"""Trainable S4D parameters on the GPU: one Delta per (head, mode) and the
gradient of A (the summary's sec. 3.2 S4D recurrence, whose A and step train
with the model).  Every entry point takes delta [H,M] as well as [H] and a
general A; the training step returns dDelta in delta's shape and dA [M]
complex.  All checked against the fp64 oracle, whose per-mode Delta and dA
are pinned by finite differences, the tangent/adjoint test and an mpmath
brute force."""
import numpy as np
import pytest
import torch

import ssm_token_mixer_b200 as ia
from gpu_common import device
from parity import TOL_BF16, TOL_F32, report, slice_rel
from ssm_token_mixer_b200 import synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    return device()


def modes_params(H, M, seed):
    """Delta [H,M] in the S4D-Lin step range and a general decaying A [2M]."""
    g = torch.Generator().manual_seed(seed)
    delta = torch.exp(np.log(2e-2) + torch.rand(H, M, generator=g) * (np.log(1.2e-1) - np.log(2e-2)))
    A = torch.empty(2 * M)
    A[0::2] = -0.2 - 0.6 * torch.rand(M, generator=g)
    A[1::2] = np.pi * torch.arange(M) + 0.7 * torch.rand(M, generator=g)
    return delta.float(), A.float()


def vec_rel(x, r):
    return float(np.abs(x.double().numpy() - r).max() / np.abs(r).max())


@pytest.mark.parametrize("dtype,dx,dv,M,tol", [("bf16", 64, 64, 64, TOL_BF16), ("bf16", 128, 128, 64, TOL_BF16),
                                               ("f32", 16, 16, 8, TOL_F32)])
def test_prefill_per_mode_delta_and_A(oracle_mod, dev, dtype, dx, dv, M, tol):
    B, H, N = 2, 3, 150
    inp = synthetic.layer_inputs(B, H, N, dx, dv, dtype, seed=60 + dx)
    delta, A = modes_params(H, M, 61)
    r = ia.prefill_fwd(inp["q"].to(dev), inp["k"].to(dev), inp["v"].to(dev), delta.to(dev), M, A=A.to(dev),
                       want_num_den=True, want_state=True)
    ia.check_device_errors()
    ref = oracle_mod.forward(inp["q"], inp["k"], inp["v"], delta, M, A=A)
    rep = report(r["num"].cpu(), r["den"].cpu(), r["o"].cpu(), ref)
    assert max(rep.values()) < tol, rep
    st = r["state"].cpu().double().numpy()
    assert np.abs(st - ref["state"]).max() / np.abs(ref["state"]).max() < tol


@pytest.mark.parametrize("dx,grid", [(64, 14), (128, 25)])
def test_look_back_with_per_mode_delta_and_A(oracle_mod, dev, monkeypatch, dx, grid):
    # ranges that start inside a stream compose their carry with
    # lambda_m^(C d) from each mode's own Delta and A
    B, H, M, N = 1, 2, 64, 64 * 20 + 17
    inp = synthetic.layer_inputs(B, H, N, dx, dx, "bf16", seed=90 + dx)
    delta, A = modes_params(H, M, 91)
    monkeypatch.setenv("IA_PREFILL_GRID", str(grid))
    assert ia.prefill_grid(B, H, N, dx, dx, M, "bf16") == grid
    r = ia.prefill_fwd(inp["q"].to(dev), inp["k"].to(dev), inp["v"].to(dev), delta.to(dev), M, A=A.to(dev),
                       want_num_den=True, want_state=True)
    ia.check_device_errors()
    ref = oracle_mod.forward(inp["q"], inp["k"], inp["v"], delta, M, A=A)
    rep = report(r["num"].cpu(), r["den"].cpu(), r["o"].cpu(), ref)
    assert max(rep.values()) < TOL_BF16, rep
    st = r["state"].cpu().double().numpy()
    assert np.abs(st - ref["state"]).max() / np.abs(ref["state"]).max() < TOL_BF16


def test_decode_per_mode_delta_and_A(oracle_mod, dev):
    B, H, d, M = 4, 3, 128, 64
    pre = synthetic.layer_inputs(B, H, 70, d, d, "bf16", seed=62)
    delta, A = modes_params(H, M, 63)
    ref = oracle_mod.forward(pre["q"], pre["k"], pre["v"], delta, M, A=A)
    state_ref = ref["state"]
    state = torch.from_numpy(state_ref.astype(np.float32)).to(dev)
    for step in range(2):
        q, k, v = synthetic.decode_token(B, H, d, d, "bf16", step=step)
        r = ia.decode_step(q.to(dev), k.to(dev), v.to(dev), delta.to(dev), state, M, A=A.to(dev),
                           want_num_den=True)
        ia.check_device_errors()
        _, num_r, den_r, state_ref = oracle_mod.decode_step(q, k, v, delta, M, state_ref, A=A)
        assert slice_rel(r["num"].cpu(), num_r, (-1,)) < 1e-4
        assert np.abs(r["den"].cpu().double().numpy() - den_r).max() / np.abs(den_r).max() < 1e-4


@pytest.mark.parametrize("path,dtype,d,M,tol", [("tensor_core", "bf16", 64, 64, TOL_BF16),
                                                ("sequential", "f32", 16, 8, TOL_F32),
                                                ("sequential", "bf16", 128, 64, TOL_BF16)])
@pytest.mark.parametrize("per_mode", [True, False])
def test_training_step_gradients_of_delta_and_A(oracle_mod, dev, path, dtype, d, M, tol, per_mode):
    B, H, N = 2, 3, 150
    inp = synthetic.layer_inputs(B, H, N, d, d, dtype, seed=64 + d, with_grad=True)
    delta, A = modes_params(H, M, 65)
    if not per_mode:
        delta = delta[:, 0].contiguous()
    assert ia.fwd_bwd_path(B, H, N, d, d, M, dtype) == path
    g = {k: v.to(dev) for k, v in inp.items()}
    r = ia.fwd_bwd(g["q"], g["k"], g["v"], delta.to(dev), g["dO"], M, A=A.to(dev))
    ia.check_device_errors()
    ref = oracle_mod.backward(inp["q"], inp["k"], inp["v"], delta, inp["dO"], M, A=A)
    for key in ("dq", "dk", "dv"):
        assert slice_rel(r[key].cpu(), ref[key], (-2, -1)) < tol, key
    assert tuple(r["dDelta"].shape) == tuple(delta.shape)
    assert vec_rel(r["dDelta"].cpu(), ref["dDelta"]) < tol
    assert vec_rel(r["dA"].cpu(), ref["dA"]) < tol


def test_parameter_gradients_are_reproducible(dev):
    # dDelta and dA come from a fixed-order reduction, not from atomics: two
    # runs give the same bits
    inp = synthetic.layer_inputs(4, 4, 300, 64, 64, "bf16", seed=66, with_grad=True)
    delta, A = modes_params(4, 64, 67)
    g = {k: v.to(dev) for k, v in inp.items()}
    runs = [ia.fwd_bwd(g["q"], g["k"], g["v"], delta.to(dev), g["dO"], 64, A=A.to(dev)) for _ in range(2)]
    ia.check_device_errors()
    assert torch.equal(runs[0]["dDelta"], runs[1]["dDelta"]) and torch.equal(runs[0]["dA"], runs[1]["dA"])
