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
                        FAKE, FAKE, FAKE, ctypes.c_size_t(fb - 1), None)
    assert rc == 3


def test_delta_per_mode_flag_checked(lib):
    s = shape()
    s.delta_per_mode = 2                                # only 0 ([H]) and 1 ([H,M]) are defined
    assert prefill(lib, s) == 1
    assert lib.ia_state_bytes(ctypes.byref(s)) == 0
    s.delta_per_mode = 1
    assert prefill(lib, s) == 3                         # valid: fails later, on the missing workspace


def test_decode_validation(lib):
    s = shape(dx=63)
    rc = lib.ia_decode_step(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, None, None, None)
    assert rc == 2
    rc = lib.ia_decode_step(ctypes.byref(shape()), FAKE, FAKE, FAKE, FAKE, None, None, FAKE, None, None, None)
    assert rc == 1
    # rows past 256 entries, or mode parameters past shared memory, are refused
    for bad in (shape(dx=258), shape(dv=258), shape(M=12000)):
        rc = lib.ia_decode_step(ctypes.byref(bad), FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, None, None, None)
        assert rc == 2


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
                        None, FAKE, ctypes.c_size_t(need), None)
    assert rc == 4
    assert lib.ia_selftest_wait_expiry(ctypes.c_ulonglong(1000000), FAKE, None) == 4
    t = shape(B=1, H=2, N=100, dx=64, dv=64, M=64, dt=1)   # the no-allocation entry point: bf16, M = 64
    rc = lib.ia_prefill_fwd_static(ctypes.byref(t), FAKE, FAKE, FAKE, FAKE, None, None, FAKE, None, None,
                                   None, None)
    assert rc == 4
    # the optional parts: token-serial (fp32, no workspace) and tensor-core
    # (bf16 stabilisation + bidirectional, with its workspace) forms
    import ssm_token_mixer_b200 as ia
    opt = ia.IAOptions()
    opt.gain = FAKE
    opt.eps = 1e-6
    rc = lib.ia_prefill_fwd_ex(ctypes.byref(s), ctypes.byref(opt), FAKE, FAKE, FAKE, FAKE, None, None, FAKE,
                               None, None, None, None, ctypes.c_size_t(0), None)
    assert rc == 4
    opt.bidirectional = 1
    assert lib.ia_prefill_ex_path(ctypes.byref(t), ctypes.byref(opt)) == 1
    need = lib.ia_prefill_ex_workspace_bytes(ctypes.byref(t), ctypes.byref(opt))
    rc = lib.ia_prefill_fwd_ex(ctypes.byref(t), ctypes.byref(opt), FAKE, FAKE, FAKE, FAKE, None, None, FAKE,
                               None, None, None, FAKE, ctypes.c_size_t(need), None)
    assert rc == 4
    opt.bidirectional = 0
    rc = lib.ia_decode_step_ex(ctypes.byref(s), ctypes.byref(opt), FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE,
                               None, None, None)
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


@pytest.mark.parametrize("B,H,N,dx,dv,grid,splits", [
    (8, 12, 2048, 64, 64, 96, False),      # 125M prefill: 96 whole sequences beat 144 ranges and their state-only chains
    (8, 16, 2048, 64, 64, 128, False),     # 350M training shape: 128 whole streams beat 148 ranges of 27.7
    (4, 16, 2048, 128, 128, 128, False),   # 1.3B prefill: 64 sequences x 2 value blocks, whole streams
    (1, 16, 7168, 128, 128, 148, True),    # 1.3B long context: 32 streams x 112 chunks over 148 SMs
    (37, 4, 256, 64, 64, 148, False),      # 148 streams of 4 chunks: one whole stream per SM
    (1, 2, 200, 64, 64, 2, False),         # 2 streams of 4 chunks: pieces shorter than 4 do not pay
])
def test_chunk_pass_plan_on_148_sms(lib, B, H, N, dx, dv, grid, splits):
    # With no GPU the planner assumes a B200's 148 SMs.  Each CTA takes an
    # equal range of the (stream, chunk) space; when a range starts inside a
    # stream the workspace also holds the look-back states (two per CTA).
    # (the planner's cost model may trade a few CTAs for better-aligned ranges)
    s = shape(B=B, H=H, N=N, dx=dx, dv=dv, M=64, dt=1)
    got = lib.ia_prefill_grid(ctypes.byref(s))
    assert (grid - 8 <= got <= grid) if splits else got == grid
    assert lib.ia_prefill_launches(ctypes.byref(s)) == 2
    tables = H * 20992 + 256
    ws = lib.ia_prefill_workspace_bytes(ctypes.byref(s))
    per_cta = 2 * (128 * (dx + 64) + 128) * 4 + 4
    assert ws == (tables + got * per_cta + 256 if splits else tables)


def test_grid_override_and_cuda_core_path(lib, monkeypatch):
    s = shape(B=8, H=12, N=2048, dx=64, dv=64, M=64, dt=1)
    monkeypatch.setenv("IA_PREFILL_GRID", "7")
    assert lib.ia_prefill_grid(ctypes.byref(s)) == 7
    monkeypatch.setenv("IA_PREFILL_GRID", "100000")
    assert lib.ia_prefill_grid(ctypes.byref(s)) == 148     # at most one CTA per SM
    monkeypatch.delenv("IA_PREFILL_GRID")
    # fp32 inputs run the sequential CUDA-core kernel: one launch, no chunk-pass grid
    t = shape(B=1, H=2, N=256, dx=16, dv=16, M=16, dt=0)
    assert lib.ia_prefill_launches(ctypes.byref(t)) == 1
    assert lib.ia_prefill_grid(ctypes.byref(t)) == 0


def test_token_serial_segments_follow_the_workspace():
    # the token-serial form's segment count: at most one per 64 tokens, at
    # most the planned count, and only as many as the workspace holds (none
    # given: one CTA per (b,h)); the tensor-core form is always 1
    import ssm_token_mixer_b200 as ia
    B, H, N, d, M = 1, 2, 357, 16, 8
    need = ia.prefill_ex_workspace_bytes(B, H, N, d, d, M, "f32", selective=True)
    full = ia.prefill_ex_segments(B, H, N, d, d, M, "f32", need, selective=True)
    assert 2 <= full <= N // 64
    assert ia.prefill_ex_segments(B, H, N, d, d, M, "f32", 0, selective=True) == 1
    assert ia.prefill_ex_segments(B, H, N, d, d, M, "f32", need - 1, selective=True) == full - 1
    assert ia.prefill_ex_segments(B, H, 127, d, d, M, "f32", 1 << 30, selective=True) == 1
    # bytes grow by one end state per extra segment, plus a step sum per segment with delta_t
    per_seg = B * H * M * (2 * d + 1) * 8
    assert need == 16 + (full - 1) * per_seg + B * H * full * 8
    plain = ia.prefill_ex_workspace_bytes(B, H, N, d, d, M, "f32", readout=True)
    assert plain == 16 + (ia.prefill_ex_segments(B, H, N, d, d, M, "f32", plain, readout=True) - 1) * per_seg
    assert ia.prefill_ex_segments(B, H, 4096, 64, 64, 64, "bf16", 1 << 30, norm=True) == 1   # tensor cores


def test_optional_parts_path_selection_and_readout_workspace():
    # host logic only: which kernels ia_prefill_fwd_ex runs, and the W'
    # operands (32 KB per head) in the tensor-core form's workspace
    import ssm_token_mixer_b200 as ia
    B, H, N = 2, 3, 300
    tc = lambda dx, **kw: ia.prefill_ex_path(B, H, N, dx, 64, 64, "bf16", **kw)
    assert tc(64, readout=True) == tc(64, readout=True, norm=True, bidirectional=True) == "tensor_core"
    assert tc(128, readout=True) == "sequential"          # W' does not fit beside the d_xi = 128 tiles
    assert tc(64, selective=True) == tc(64, selective=True, readout=True) == "sequential"
    assert ia.prefill_ex_path(B, H, N, 64, 64, 64, "f32", readout=True) == "sequential"
    plain = ia.prefill_ex_workspace_bytes(B, H, N, 64, 64, 64, "bf16", norm=True)
    with_w = ia.prefill_ex_workspace_bytes(B, H, N, 64, 64, 64, "bf16", norm=True, readout=True)
    assert with_w - plain == H * 32768
