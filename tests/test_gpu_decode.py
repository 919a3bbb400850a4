"""Decode-step parity on the GPU against the oracle's decode step, plus the
prefill-then-decode identity (P12) on the GPU path itself."""
import numpy as np
import pytest
import torch

import ssm_token_mixer_b200 as ia
from gpu_common import device, gpu_prefill
from parity import TOL_BF16, TOL_F32, slice_rel
from ssm_token_mixer_b200 import synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    return device()


@pytest.mark.parametrize("split", ["default", "1", "2", "4", "8"])
@pytest.mark.parametrize("B", [1, 16, 64])
def test_decode_steps_match_oracle(oracle_mod, dev, monkeypatch, B, split):
    # every cluster size (1, 2, 4 or 8 CTAs per (b,h), each taking a range of
    # the modes, rank 0 adding the partials) is forced at every batch size,
    # besides the default choice
    if split != "default":
        monkeypatch.setenv("IA_DECODE_SPLIT", split)
    H, d, M, N0 = 16, 128, 64, 96
    pre = synthetic.layer_inputs(B, H, N0, d, d, "bf16", seed=1004)
    ref = oracle_mod.forward(pre["q"], pre["k"], pre["v"], pre["delta"], M)
    state_ref = ref["state"]
    state = torch.from_numpy(state_ref.astype(np.float32)).to(dev)
    delta = pre["delta"].to(dev)
    for step in range(3):
        q, k, v = synthetic.decode_token(B, H, d, d, "bf16", step=step)
        r = ia.decode_step(q.to(dev), k.to(dev), v.to(dev), delta, state, M, want_num_den=True)
        ia.check_device_errors()
        o_r, num_r, den_r, state_ref = oracle_mod.decode_step(q, k, v, pre["delta"], M, state_ref)
        assert slice_rel(r["num"].cpu(), num_r, (-1,)) < 1e-4
        dr = np.abs(r["den"].cpu().double().numpy() - den_r).max() / np.abs(den_r).max()
        assert dr < 1e-4
    assert np.abs(state.cpu().double().numpy() - state_ref).max() / np.abs(state_ref).max() < 1e-4


def test_decode_f32_odd_shapes(oracle_mod, dev):
    B, H, dx, dv, M = 3, 5, 18, 10, 7
    st = np.zeros(oracle_mod.state_len(B, H, M, dx, dv))
    state = torch.zeros(st.size, dtype=torch.float32, device=dev)
    delta = torch.tensor([0.01, 0.05, 0.002, 0.09, 0.03])
    for step in range(4):
        q, k, v = (torch.randn(B, H, n, generator=torch.Generator().manual_seed(step * 3 + i))
                   for i, n in enumerate((dx, dx, dv)))
        r = ia.decode_step(q.to(dev), k.to(dev), v.to(dev), delta.to(dev), state, M)
        o_r, _, _, st = oracle_mod.decode_step(q, k, v, delta, M, st)
        assert slice_rel(r["o"].cpu(), o_r, (-1,)) < TOL_F32


def test_prefill_then_decode_equals_longer_prefill(dev):
    # P12 on the GPU path: prefill(N) then k decode steps == prefill(N + k)
    B, H, d, M, N, K = 2, 4, 128, 64, 150, 3
    inp = synthetic.layer_inputs(B, H, N + K, d, d, "bf16", seed=77)
    head = {k_: (v[:, :, :N].contiguous() if k_ != "delta" else v) for k_, v in inp.items()}
    full = gpu_prefill(inp, M, dev)
    part = gpu_prefill(head, M, dev)
    state = part["state"].to(dev)
    delta = inp["delta"].to(dev)
    for t in range(N, N + K):
        r = ia.decode_step(inp["q"][:, :, t].contiguous().to(dev), inp["k"][:, :, t].contiguous().to(dev),
                           inp["v"][:, :, t].contiguous().to(dev), delta, state, M, want_num_den=True)
        assert slice_rel(r["num"].cpu(), full["num"][:, :, t], (-1,)) < TOL_BF16
    s1, s2 = state.cpu().double().numpy(), full["state"].double().numpy()
    assert np.abs(s1 - s2).max() / np.abs(s2).max() < TOL_BF16


def test_decode_graph_capture(dev):
    B, H, d, M = 4, 16, 128, 64
    state = torch.zeros(ia.state_bytes(B, H, M, d, d) // 4, dtype=torch.float32, device=dev)
    q, k, v = (x.to(dev) for x in synthetic.decode_token(B, H, d, d, "bf16", step=0))
    delta = torch.full((H,), 0.01, device=dev)
    o = torch.empty(B, H, d, device=dev)
    ia.decode_step(q, k, v, delta, state, M, o=o)      # warm-up (cluster attribute set)
    torch.cuda.synchronize()
    state.zero_()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            ia.decode_step(q, k, v, delta, state, M, o=o, stream=s)
    state.zero_()
    g.replay()
    torch.cuda.synchronize()
    o1 = o.clone()
    state.zero_()
    ia.decode_step(q, k, v, delta, state, M, o=o)
    torch.cuda.synchronize()
    assert torch.equal(o1, o)
    assert torch.allclose(o1, v.float(), rtol=1e-2, atol=1e-2)   # first token from zero state: o = v
