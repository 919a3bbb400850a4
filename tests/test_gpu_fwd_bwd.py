"""Training-step parity on the GPU: o, dq, dk, dv, dDelta and dA against the
oracle's reverse-mode adjoint (itself pinned by finite differences and the
tangent/adjoint dot-product test)."""
import numpy as np
import pytest
import torch

import ssm_token_mixer_b200 as ia
from gpu_common import device
from parity import TOL_BF16, TOL_F32, slice_rel
from ssm_token_mixer_b200 import synthetic
from ssm_token_mixer_b200.workloads import WORKLOADS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    return device()


def run(inp, M, dev):
    d = {k: v.to(dev) for k, v in inp.items()}
    r = ia.fwd_bwd(d["q"], d["k"], d["v"], d["delta"], d["dO"], M)
    ia.check_device_errors()
    return {k: v.cpu() for k, v in r.items()}


def vec_rel(x, r):
    x = x.double().numpy() if hasattr(x, "double") else np.asarray(x)
    return float(np.abs(x - r).max() / np.abs(r).max())


def compare(r, g, tol):
    assert slice_rel(r["dq"], g["dq"], (-2, -1)) < tol
    assert slice_rel(r["dk"], g["dk"], (-2, -1)) < tol
    assert slice_rel(r["dv"], g["dv"], (-2, -1)) < tol
    dd = vec_rel(r["dDelta"], g["dDelta"])
    assert dd < tol, dd
    da = vec_rel(r["dA"], g["dA"])
    assert da < tol, da


@pytest.mark.parametrize("dtype,tol", [("f32", TOL_F32), ("bf16", TOL_BF16)])
def test_fwd_bwd_small(oracle_mod, dev, dtype, tol):
    B, H, N, d, M = 2, 3, 150, 16, 8
    inp = synthetic.layer_inputs(B, H, N, d, d, dtype, seed=31, with_grad=True)
    r = run(inp, M, dev)
    g = oracle_mod.backward(inp["q"], inp["k"], inp["v"], inp["delta"], inp["dO"], M)
    assert slice_rel(r["o"], g["o"], (-2, -1)) < tol
    compare(r, g, tol)


def test_fwd_bwd_training_shape_reduced_batch(oracle_mod, dev):
    w = WORKLOADS["train_350m"]
    inp = synthetic.workload_inputs(w, B=1)
    r = run(inp, w.M, dev)
    g = oracle_mod.backward(inp["q"], inp["k"], inp["v"], inp["delta"], inp["dO"], w.M)
    compare(r, g, TOL_BF16)


@pytest.mark.parametrize("N", [64, 150, 333])
def test_fwd_bwd_tensor_core_path(oracle_mod, dev, N):
    # bf16, M = 64, d = 64 runs the tensor-core reverse-mode kernel; ragged N
    B, H, d, M = 2, 3, 64, 64
    inp = synthetic.layer_inputs(B, H, N, d, d, "bf16", seed=41 + N, with_grad=True)
    r = run(inp, M, dev)
    g = oracle_mod.backward(inp["q"], inp["k"], inp["v"], inp["delta"], inp["dO"], M)
    assert slice_rel(r["o"], g["o"], (-2, -1)) < TOL_BF16
    compare(r, g, TOL_BF16)


def test_fwd_bwd_tensor_core_matches_cuda_core(dev, monkeypatch):
    inp = synthetic.layer_inputs(2, 2, 200, 64, 64, "bf16", seed=77, with_grad=True)
    r_tc = run(inp, 64, dev)
    monkeypatch.setenv("IA_BWD_SIMT", "1")
    r_ref = run(inp, 64, dev)
    for key in ("dq", "dk", "dv"):
        assert slice_rel(r_tc[key], r_ref[key], (-2, -1)) < TOL_BF16, key
    dd = (r_tc["dDelta"] - r_ref["dDelta"]).abs().max() / r_ref["dDelta"].abs().max()
    assert dd.item() < TOL_BF16
