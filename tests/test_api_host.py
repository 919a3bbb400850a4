"""C-ABI contract checks that need no GPU: the library loads, exports every
symbol include/ia.h declares, and rejects bad arguments on the host before
any launch (no compute call is made here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from ssm_token_mixer_b200 import build
    build.build()
    import ssm_token_mixer_b200 as ia
    return ia.load_library()


def declared_symbols():
    syms = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            syms |= set(re.findall(r"IA_API\s+[\w\s\*]+?\b(ia_\w+)\s*\(", text))
    return syms


def test_exports_every_declared_symbol(lib):
    syms = declared_symbols()
    assert {"ia_prefill_fwd", "ia_fwd_bwd", "ia_decode_step"} <= syms
    for s in syms:
        assert hasattr(lib, s), s


def shape(B=2, H=3, N=100, dx=64, dv=64, M=64, dt=1):
    import ssm_token_mixer_b200 as ia
    return ia.IAShape(B, H, N, dx, dv, M, dt)


FAKE = ctypes.c_void_p(0x10000)      # aligned, never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p(0x10008)


def prefill(lib, s, q=FAKE, o=FAKE, state_in=None, state_out=None, ws=None, wsb=0):
    return lib.ia_prefill_fwd(ctypes.byref(s) if s is not None else None, q, FAKE, FAKE, FAKE, None,
                              state_in, o, None, None, state_out, ws, ctypes.c_size_t(wsb), None)


def test_state_bytes(lib):
    s = shape(B=2, H=3, dx=5, dv=7, M=11)
    assert lib.ia_state_bytes(ctypes.byref(s)) == 8 * 2 * 3 * 11 * (5 + 7 + 1)


def test_invalid_arguments(lib):
    assert prefill(lib, None) == 1
    for bad in (dict(B=0), dict(H=-1), dict(N=0), dict(dx=0), dict(M=0), dict(dt=7)):
        assert prefill(lib, shape(**bad)) == 1, bad
    assert prefill(lib, shape(), q=None) == 1
    assert prefill(lib, shape(), o=None) == 1
    assert prefill(lib, shape(), q=MISALIGNED) == 1
    assert prefill(lib, shape(), state_in=FAKE, state_out=FAKE) == 1


def test_workspace_checked_before_launch(lib):
    s = shape()
    need = lib.ia_prefill_workspace_bytes(ctypes.byref(s))
    assert need > 0                                     # tensor-core path uses tables
    assert prefill(lib, s) == 3
    assert prefill(lib, s, ws=FAKE, wsb=need - 1) == 3
    fb = lib.ia_fwd_bwd_workspace_bytes(ctypes.byref(s))
    rc = lib.ia_fwd_bwd(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE,
                        FAKE, FAKE, ctypes.c_size_t(fb - 1), None)
    assert rc == 3


def test_decode_validation(lib):
    s = shape(dx=63)
    rc = lib.ia_decode_step(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, None, None, None)
    assert rc == 2
    rc = lib.ia_decode_step(ctypes.byref(shape()), FAKE, FAKE, FAKE, FAKE, None, None, FAKE, None, None, None)
    assert rc == 1


def test_injected_launch_failure(lib, monkeypatch):
    # every entry point, given valid arguments, reports the injected launch
    # failure after its checks and launches nothing (no pointer is touched)
    monkeypatch.setenv("IA_INJECT_LAUNCH_FAILURE", "1")
    s = shape(dt=0, dx=16, dv=16, M=4)                 # CUDA-core path: no workspace
    assert prefill(lib, s) == 4
    rc = lib.ia_decode_step(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, None, None, None)
    assert rc == 4
    need = lib.ia_fwd_bwd_workspace_bytes(ctypes.byref(s))
    rc = lib.ia_fwd_bwd(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                        FAKE, ctypes.c_size_t(need), None)
    assert rc == 4
    t = shape(B=1, H=2, N=100, dx=64, dv=64, M=64, dt=1)   # the no-allocation entry point: bf16, M = 64
    rc = lib.ia_prefill_fwd_static(ctypes.byref(t), FAKE, FAKE, FAKE, FAKE, None, None, FAKE, None, None,
                                   None, None)
    assert rc == 4
    # without the switch, argument errors still come first
    monkeypatch.setenv("IA_INJECT_LAUNCH_FAILURE", "0")
    assert prefill(lib, shape(B=0)) == 1


def test_no_alloc_head_limit_and_shape_checks(lib, monkeypatch):
    # The limit follows the table size: 99 heads of 20,992 bytes fit the
    # 2 MiB array after its 256-byte alignment allowance.  H = 99 passes every
    # check (the injected failure then stops it before any launch), H = 100
    # is refused as too large for the array.
    assert lib.ia_prefill_static_max_heads() == 99
    monkeypatch.setenv("IA_INJECT_LAUNCH_FAILURE", "1")

    def static(s):
        return lib.ia_prefill_fwd_static(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, None, None, FAKE, None,
                                         None, None, None)
    assert static(shape(B=1, H=99, N=64, dx=64, dv=64, M=64, dt=1)) == 4
    assert static(shape(B=1, H=100, N=64, dx=64, dv=64, M=64, dt=1)) == 3
    # the same shape checks as ia_prefill_fwd: B*H beyond int range is invalid
    assert static(shape(B=1 << 16, H=1 << 16, N=64, dx=64, dv=64, M=64, dt=1)) == 1
    assert prefill(lib, shape(B=1 << 16, H=1 << 16, N=64)) == 1
    assert static(shape(B=1, H=2, N=64, dx=32, dv=64, M=64, dt=1)) == 2   # not a tensor-core shape


def test_path_queries(lib):
    def paths(**kw):
        s = shape(**kw)
        return lib.ia_prefill_path(ctypes.byref(s)), lib.ia_fwd_bwd_path(ctypes.byref(s))
    TC, SEQ = 1, 2
    assert paths(B=8, H=12, N=2048, dx=64, dv=64, M=64, dt=1) == (TC, TC)
    assert paths(B=4, H=16, N=2048, dx=128, dv=128, M=64, dt=1) == (TC, SEQ)   # d = 128 training: CUDA cores
    assert paths(B=1, H=2, N=256, dx=16, dv=16, M=16, dt=0) == (SEQ, SEQ)     # fp32 inputs
    assert paths(B=1, H=2, N=256, dx=64, dv=64, M=32, dt=1) == (SEQ, SEQ)     # M != 64
    assert paths(B=0) == (0, 0)


def test_selftest_argument_checks(lib):
    assert lib.ia_selftest_wait_expiry(ctypes.c_ulonglong(1000000), None, None) == 1
    assert lib.ia_selftest_wait_expiry(ctypes.c_ulonglong(10), FAKE, None) == 1          # limit too short
    assert lib.ia_selftest_wait_expiry(ctypes.c_ulonglong(2 * 10 ** 9), FAKE, None) == 1  # above one second
    assert lib.ia_selftest_wait_expiry(ctypes.c_ulonglong(1000000), ctypes.c_void_p(0x10004), None) == 1


def test_status_strings(lib):
    for code in range(7):
        assert lib.ia_status_string(code).startswith(b"IA_")
    assert b"unknown" in lib.ia_status_string(99)


def test_missing_library_fails_loudly(monkeypatch):
    import ssm_token_mixer_b200 as ia
    monkeypatch.setattr(ia, "_lib", None)
    monkeypatch.setattr(ia, "_LIB_PATH", "/nonexistent/libia.so")
    with pytest.raises(RuntimeError):
        ia.load_library()


def _segments(lib, s, monkeypatch):
    """Segments per sequence of the tensor-core plan, read from the workspace
    size: each boundary between segments keeps one carried state per (b,h)."""
    ws = lib.ia_prefill_workspace_bytes(ctypes.byref(s))
    monkeypatch.setenv("IA_PREFILL_SEGMENTS", "1")
    ws1 = lib.ia_prefill_workspace_bytes(ctypes.byref(s))
    monkeypatch.delenv("IA_PREFILL_SEGMENTS")
    per_bh = lib.ia_state_bytes(ctypes.byref(s)) // (s.B * s.H)
    extra = ws - ws1
    assert extra % (s.B * s.H * per_bh) == 0
    return 1 + extra // (s.B * s.H * per_bh)


@pytest.mark.parametrize("B,H,N,d,nseg", [
    (8, 12, 2048, 64, 1),    # 125M prefill: 96 sequences, one pass
    (8, 16, 2048, 64, 1),    # 350M training shape: 128 sequences
    (4, 16, 2048, 128, 2),   # 1.3B prefill: 64 sequences of 32 chunks -> 2 x 16 chunks on 128 CTAs
    (1, 16, 7168, 128, 9),   # 1.3B long context: 16 x 112 chunks -> 9 x 13 chunks on 144 CTAs
])
def test_segment_plan_on_148_sms(lib, monkeypatch, B, H, N, d, nseg):
    # With no GPU the planner assumes a B200's 148 SMs.  Splitting pays when
    # the sequences alone leave SMs idle: a state-only pass and the carry scan
    # then precede the full pass (4 launches instead of tables + full pass).
    s = shape(B=B, H=H, N=N, dx=d, dv=d, M=64, dt=1)
    assert _segments(lib, s, monkeypatch) == nseg
    assert lib.ia_prefill_launches(ctypes.byref(s)) == (4 if nseg > 1 else 2)


def test_segment_override_and_cuda_core_path(lib, monkeypatch):
    s = shape(B=8, H=12, N=2048, dx=64, dv=64, M=64, dt=1)
    monkeypatch.setenv("IA_PREFILL_SEGMENTS", "4")
    assert lib.ia_prefill_launches(ctypes.byref(s)) == 4
    monkeypatch.delenv("IA_PREFILL_SEGMENTS")
    # fp32 inputs run the sequential CUDA-core kernel: one launch, no segments
    assert lib.ia_prefill_launches(ctypes.byref(shape(B=1, H=2, N=256, dx=16, dv=16, M=16, dt=0))) == 1
