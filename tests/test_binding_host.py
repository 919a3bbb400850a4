"""Argument checks of the Python binding, on the CPU.

The library receives raw pointers and cannot see tensor sizes, so the binding
checks every tensor against the shape before calling it.  Here the four
compute entry points are replaced by recorders (the size queries still go to
the real library): valid calls, in the patterns the GPU tests and bench.py
use, must reach the entry point with the right sizes; invalid ones must raise
before it.  No kernel runs and no device memory is touched.
"""
import ctypes

import pytest
import torch

import ssm_token_mixer_b200 as ia

COMPUTE = ("ia_prefill_fwd", "ia_prefill_fwd_static", "ia_fwd_bwd", "ia_decode_step")


class RecordingLib:
    def __init__(self, real):
        self.real = real
        self.calls = []

    def __getattr__(self, name):
        if name in COMPUTE:
            def entry(*args):
                self.calls.append((name, args))
                return 0
            return entry
        return getattr(self.real, name)


@pytest.fixture
def rec(monkeypatch):
    from ssm_token_mixer_b200 import build
    build.build()
    lib = RecordingLib(ia.load_library())
    monkeypatch.setattr(ia, "load_library", lambda: lib)
    monkeypatch.setattr(ia, "_stream", lambda stream: None)
    return lib


@pytest.fixture
def any_device(monkeypatch):
    # lets CPU tensors stand for device tensors once shapes and dtypes are checked
    monkeypatch.setattr(ia, "_cuda_device", lambda named: torch.device("cpu"))


def seq(B, H, N, dx, dv, dt=torch.bfloat16, grad=False):
    t = {"q": torch.empty(B, H, N, dx, dtype=dt), "k": torch.empty(B, H, N, dx, dtype=dt),
         "v": torch.empty(B, H, N, dv, dtype=dt), "delta": torch.full((H,), 0.01)}
    if grad:
        t["dO"] = torch.empty(B, H, N, dv, dtype=dt)
    return t


def tok(B, H, dx, dv, dt=torch.bfloat16):
    return torch.empty(B, H, dx, dtype=dt), torch.empty(B, H, dx, dtype=dt), torch.empty(B, H, dv, dtype=dt)


def test_bench_and_test_call_patterns_reach_the_library(rec, any_device):
    # prefill leg: 125M shape with caller-owned o and workspace
    t = seq(8, 12, 2048, 64, 64)
    o = torch.empty(8, 12, 2048, 64, dtype=torch.float32)
    need = ia.prefill_workspace_bytes(8, 12, 2048, 64, 64, 64, "bf16")
    ws = torch.empty(max(need, 1), dtype=torch.uint8)
    ia.prefill_fwd(t["q"], t["k"], t["v"], t["delta"], 64, o=o, workspace=ws)
    name, args = rec.calls[-1]
    assert name == "ia_prefill_fwd" and args[-2].value == ws.numel()
    # training leg: 350M shape, workspace sized by the query, passed in bytes
    t = seq(8, 16, 2048, 64, 64, grad=True)
    need = ia.fwd_bwd_workspace_bytes(8, 16, 2048, 64, 64, 64, "bf16")
    ws = torch.empty(need, dtype=torch.uint8)
    r = ia.fwd_bwd(t["q"], t["k"], t["v"], t["delta"], t["dO"], 64, workspace=ws)
    assert rec.calls[-1][0] == "ia_fwd_bwd" and rec.calls[-1][1][-2].value == need
    assert r["dq"].shape == (8, 16, 2048, 64) and r["dDelta"].shape == (16,)
    # decode leg: prefix prefill with state, then steps on the returned state
    t = seq(16, 16, 100, 128, 128)
    pre = ia.prefill_fwd(t["q"], t["k"], t["v"], t["delta"], 64, want_state=True)
    assert pre["state"].numel() * 4 == ia.state_bytes(16, 16, 64, 128, 128)
    o = torch.empty(16, 16, 128, dtype=torch.float32)
    ia.decode_step(*tok(16, 16, 128, 128), t["delta"], pre["state"].clone(), 64, o=o)
    assert rec.calls[-1][0] == "ia_decode_step"
    # fp32 inputs with odd sizes, a carried state and the no-allocation entry point
    t = seq(3, 5, 37, 18, 10, dt=torch.float32)
    st = torch.zeros(ia.state_bytes(3, 5, 7, 18, 10) // 4)
    r = ia.prefill_fwd(t["q"], t["k"], t["v"], t["delta"], 7, state_in=st, want_num_den=True, want_state=True)
    assert r["num"].shape == (3, 5, 37, 10) and r["den"].shape == (3, 5, 37)
    ia.decode_step(*tok(3, 5, 18, 10, torch.float32), t["delta"], st, 7, want_num_den=True)
    t = seq(1, 4, 130, 128, 128)
    ia.prefill_fwd_static(t["q"], t["k"], t["v"], t["delta"], 64, want_num_den=True, want_state=True)
    assert rec.calls[-1][0] == "ia_prefill_fwd_static"
    # an explicit S4D matrix: M complex values as 2M floats
    t = seq(1, 2, 10, 16, 16)
    ia.prefill_fwd(t["q"], t["k"], t["v"], t["delta"], 8, A=torch.zeros(8, 2))
    assert [c[0] for c in rec.calls].count("ia_prefill_fwd") == 4


@pytest.mark.parametrize("bad,err", [
    (lambda t: t.update(k=torch.empty(2, 3, 50, 8, dtype=torch.bfloat16)), ValueError),   # k shorter than q
    (lambda t: t.update(v=torch.empty(2, 3, 49, 16, dtype=torch.bfloat16)), ValueError),  # v one token short
    (lambda t: t.update(v=torch.empty(2, 3, 64, 16, dtype=torch.float32)), TypeError),    # dtype mix
    (lambda t: t.update(delta=torch.full((2,), 0.01)), ValueError),                       # one Delta per head
    (lambda t: t.update(delta=torch.full((3,), 0.01, dtype=torch.float64)), TypeError),
    (lambda t: t.update(q=torch.empty(2, 3, 64, 16, dtype=torch.float16),
                        k=torch.empty(2, 3, 64, 16, dtype=torch.float16),
                        v=torch.empty(2, 3, 64, 16, dtype=torch.float16)), TypeError),    # fp16 inputs
    (lambda t: t.update(q=torch.empty(3, 64, 16, dtype=torch.bfloat16)), ValueError),     # missing batch dim
    (lambda t: t.update(A=torch.zeros(7, 2)), ValueError),                                # M = 8 modes
    (lambda t: t.update(o=torch.empty(2, 3, 64, 8)), ValueError),
    (lambda t: t.update(o=torch.empty(2, 3, 64, 16, dtype=torch.bfloat16)), TypeError),
    (lambda t: t.update(state_in=torch.zeros(10)), ValueError),
    (lambda t: t.update(state_in=torch.zeros(ia.state_bytes(2, 3, 8, 16, 16) // 8, dtype=torch.float64)),
     TypeError),
])
def test_prefill_rejects_inconsistent_tensors(rec, any_device, bad, err):
    t = seq(2, 3, 64, 16, 16)
    t.update(A=None, o=None, state_in=None)
    bad(t)
    with pytest.raises(err):
        ia.prefill_fwd(t["q"], t["k"], t["v"], t["delta"], 8, A=t["A"], o=t["o"], state_in=t["state_in"])
    assert rec.calls == []


def test_training_and_decode_reject_inconsistent_tensors(rec, any_device):
    t = seq(2, 3, 64, 16, 16, grad=True)
    with pytest.raises(ValueError):
        ia.fwd_bwd(t["q"], t["k"], t["v"], t["delta"], t["dO"][:, :, :32], 8)
    with pytest.raises(TypeError):
        ia.fwd_bwd(t["q"], t["k"], t["v"], t["delta"], t["dO"].float(), 8)
    q, k, v = tok(2, 3, 16, 16)
    st = torch.zeros(ia.state_bytes(2, 3, 8, 16, 16) // 4)
    with pytest.raises(ValueError):      # state of another shape
        ia.decode_step(q, k, v, t["delta"], st[:-2], 8)
    with pytest.raises(ValueError):      # a sequence instead of one token
        ia.decode_step(t["q"], t["k"], t["v"], t["delta"], st, 8)
    with pytest.raises(ValueError):
        ia.decode_step(q, k, v[:, :2], t["delta"], st, 8)
    with pytest.raises(ValueError):
        ia.decode_step(q, k, v, t["delta"], st, 8, o=torch.empty(2, 3, 8))
    assert rec.calls == []


def test_host_tensors_are_refused_before_the_library(rec):
    # correct shapes and dtypes, but in host memory: the library would
    # dereference these pointers on the GPU, so the binding refuses them
    t = seq(1, 2, 40, 16, 16, grad=True)
    with pytest.raises(ValueError, match="CUDA"):
        ia.prefill_fwd(t["q"], t["k"], t["v"], t["delta"], 8)
    with pytest.raises(ValueError, match="CUDA"):
        ia.fwd_bwd(t["q"], t["k"], t["v"], t["delta"], t["dO"], 8)
    with pytest.raises(ValueError, match="CUDA"):
        ia.prefill_fwd_static(t["q"], t["k"], t["v"], t["delta"], 8)
    q, k, v = tok(1, 2, 16, 16)
    with pytest.raises(ValueError, match="CUDA"):
        ia.decode_step(q, k, v, t["delta"], torch.zeros(ia.state_bytes(1, 2, 8, 16, 16) // 4), 8)
    assert rec.calls == []


def test_workspace_size_is_passed_in_bytes(rec, any_device):
    t = seq(1, 2, 40, 64, 64)
    need = ia.prefill_workspace_bytes(1, 2, 40, 64, 64, 64, "bf16")
    ws = torch.empty((need + 3) // 4, dtype=torch.float32)     # any dtype: the size is counted in bytes
    ia.prefill_fwd(t["q"], t["k"], t["v"], t["delta"], 64, workspace=ws)
    assert rec.calls[-1][1][-2].value == ws.numel() * 4 >= need
