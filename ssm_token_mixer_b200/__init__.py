"""Interdomain Attention (IA) layer hot path for NVIDIA B200 -- Python binding.

This module only marshals torch tensors (device memory and the current CUDA
stream) into the C-ABI of ``lib/libia.so`` (declared in ``include/ia.h``);
every step of the layer runs in that library's sm_100a kernels.  There is no
CPU or PyTorch fallback: if the library is missing or a call fails, the call
raises.

Entry points (same names as the C-ABI):
  prefill_fwd(q, k, v, delta, M, ...)   causal prefill, returns o (+ num, den, state)
  fwd_bwd(q, k, v, delta, dO, M, ...)   training step: o, dq, dk, dv, dDelta
  decode_step(q, k, v, delta, state, M)  one recurrent step, state updated in place
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["IAError", "load_library", "state_bytes", "prefill_workspace_bytes",
           "fwd_bwd_workspace_bytes", "prefill_path", "fwd_bwd_path", "prefill_static_max_heads",
           "prefill_fwd", "prefill_fwd_static", "prefill_fwd_ex", "fwd_bwd", "decode_step",
           "decode_step_ex", "check_device_errors",
           "selftest_wait_expiry", "set_launch_events", "library_path", "IA_F32", "IA_BF16"]

IA_F32, IA_BF16 = 0, 1
_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "lib", "libia.so")
_lib = None

STATUS = {0: "IA_OK", 1: "IA_ERR_INVALID_ARG", 2: "IA_ERR_UNSUPPORTED", 3: "IA_ERR_WORKSPACE",
          4: "IA_ERR_CUDA", 5: "IA_ERR_TIMEOUT", 6: "IA_ERR_PARAM_RANGE"}
PATHS = {0: None, 1: "tensor_core", 2: "sequential"}


class IAError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        msg = _lib.ia_status_string(status).decode() if _lib else STATUS.get(status, str(status))
        if _lib and status == 4:   # IA_ERR_CUDA: name the CUDA error behind it
            msg += f" ({_lib.ia_last_cuda_error_string().decode()}, code {_lib.ia_last_cuda_error()})"
        super().__init__(f"{where}: {msg}")


class IAShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int),
                ("d_xi", ctypes.c_int), ("d_v", ctypes.c_int), ("M", ctypes.c_int),
                ("in_dtype", ctypes.c_int), ("delta_per_mode", ctypes.c_int)]


class IAOptions(ctypes.Structure):
    _fields_ = [("delta_t", ctypes.c_void_p), ("gain", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("eps", ctypes.c_float), ("W", ctypes.c_void_p), ("bidirectional", ctypes.c_int)]


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libia.so (built by ssm_token_mixer_b200.build); raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                           "`python -m ssm_token_mixer_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(_LIB_PATH)
    P, S = ctypes.c_void_p, ctypes.POINTER(IAShape)
    for name in ("ia_state_bytes", "ia_prefill_workspace_bytes", "ia_fwd_bwd_workspace_bytes"):
        getattr(lib, name).restype = ctypes.c_size_t
        getattr(lib, name).argtypes = [S]
    for name in ("ia_prefill_launches", "ia_prefill_grid", "ia_prefill_path", "ia_fwd_bwd_path"):
        getattr(lib, name).restype = ctypes.c_int
        getattr(lib, name).argtypes = [S]
    lib.ia_prefill_static_max_heads.restype = ctypes.c_int
    lib.ia_prefill_static_max_heads.argtypes = []
    lib.ia_selftest_wait_expiry.restype = ctypes.c_int
    lib.ia_selftest_wait_expiry.argtypes = [ctypes.c_ulonglong, P, P]
    lib.ia_prefill_fwd.restype = ctypes.c_int
    lib.ia_prefill_fwd.argtypes = [S] + [P] * 10 + [P, ctypes.c_size_t, P]
    lib.ia_prefill_fwd_static.restype = ctypes.c_int
    lib.ia_prefill_fwd_static.argtypes = [S] + [P] * 10 + [P]
    lib.ia_fwd_bwd.restype = ctypes.c_int
    lib.ia_fwd_bwd.argtypes = [S] + [P] * 12 + [P, ctypes.c_size_t, P]
    lib.ia_decode_step.restype = ctypes.c_int
    lib.ia_decode_step.argtypes = [S] + [P] * 9 + [P]
    O = ctypes.POINTER(IAOptions)
    lib.ia_prefill_fwd_ex.restype = ctypes.c_int
    lib.ia_prefill_fwd_ex.argtypes = [S, O] + [P] * 10 + [P, ctypes.c_size_t, P]
    lib.ia_prefill_ex_workspace_bytes.restype = ctypes.c_size_t
    lib.ia_prefill_ex_workspace_bytes.argtypes = [S, O]
    lib.ia_prefill_ex_path.restype = ctypes.c_int
    lib.ia_prefill_ex_path.argtypes = [S, O]
    lib.ia_prefill_ex_segments.restype = ctypes.c_int
    lib.ia_prefill_ex_segments.argtypes = [S, O, P, ctypes.c_size_t]
    lib.ia_decode_step_ex.restype = ctypes.c_int
    lib.ia_decode_step_ex.argtypes = [S, O] + [P] * 9 + [P]
    lib.ia_state_carry.restype = ctypes.c_int
    lib.ia_state_carry.argtypes = [S, P, P, ctypes.c_longlong, P, P, P, P]
    lib.ia_set_launch_events.restype = ctypes.c_int
    lib.ia_set_launch_events.argtypes = [P, P]
    lib.ia_check_device_errors.restype = ctypes.c_int
    lib.ia_check_device_errors.argtypes = [P]
    lib.ia_status_string.restype = ctypes.c_char_p
    lib.ia_status_string.argtypes = [ctypes.c_int]
    lib.ia_last_cuda_error.restype = ctypes.c_int
    lib.ia_last_cuda_error.argtypes = []
    lib.ia_last_cuda_error_string.restype = ctypes.c_char_p
    lib.ia_last_cuda_error_string.argtypes = []
    _lib = lib
    return lib


def _dtype_code(t):
    if t.dtype == torch.float32:
        return IA_F32
    if t.dtype == torch.bfloat16:
        return IA_BF16
    raise TypeError(f"unsupported input dtype {t.dtype} (float32 or bfloat16)")


def make_shape(B, H, N, d_xi, d_v, M, dtype, delta_per_mode=False) -> IAShape:
    code = dtype if isinstance(dtype, int) else (IA_BF16 if dtype in (torch.bfloat16, "bf16") else IA_F32)
    return IAShape(int(B), int(H), int(N), int(d_xi), int(d_v), int(M), code, int(bool(delta_per_mode)))


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(status, where):
    if status != 0:
        raise IAError(status, where)


def state_bytes(B, H, M, d_xi, d_v) -> int:
    return int(load_library().ia_state_bytes(ctypes.byref(make_shape(B, H, 1, d_xi, d_v, M, IA_F32))))


def prefill_workspace_bytes(B, H, N, d_xi, d_v, M, dtype) -> int:
    return int(load_library().ia_prefill_workspace_bytes(ctypes.byref(make_shape(B, H, N, d_xi, d_v, M, dtype))))


def prefill_launches(B, H, N, d_xi, d_v, M, dtype) -> int:
    return int(load_library().ia_prefill_launches(ctypes.byref(make_shape(B, H, N, d_xi, d_v, M, dtype))))


def prefill_grid(B, H, N, d_xi, d_v, M, dtype) -> int:
    """CTAs of the tensor-core chunk pass for this shape (0 off that path)."""
    return int(load_library().ia_prefill_grid(ctypes.byref(make_shape(B, H, N, d_xi, d_v, M, dtype))))


def prefill_path(B, H, N, d_xi, d_v, M, dtype):
    """'tensor_core' or 'sequential': the kernels ia_prefill_fwd runs for this shape."""
    return PATHS[load_library().ia_prefill_path(ctypes.byref(make_shape(B, H, N, d_xi, d_v, M, dtype)))]


def fwd_bwd_path(B, H, N, d_xi, d_v, M, dtype):
    """'tensor_core' or 'sequential': the reverse-pass kernels ia_fwd_bwd runs for this shape."""
    return PATHS[load_library().ia_fwd_bwd_path(ctypes.byref(make_shape(B, H, N, d_xi, d_v, M, dtype)))]


def state_carry(local, delta, M, L, B, H, d_xi, d_v, carry_in=None, A=None, out=None, stream=None):
    """lambda^L * carry_in + local over whole states (flat fp32, the
    ia_state_bytes layout; see ia_state_carry): the state before a span
    decayed across it plus what the span built from zero.  Returns out."""
    lib = load_library()
    dpm = _check_delta(delta, H, M)
    shp = make_shape(B, H, 1, d_xi, d_v, M, "f32", dpm)
    n = lib.ia_state_bytes(ctypes.byref(shp)) // 4
    _need("local", local, dtype=torch.float32, numel=n)
    if carry_in is not None:
        _need("carry_in", carry_in, dtype=torch.float32, numel=n)
    if A is not None:
        _need("A", A, dtype=torch.float32, numel=2 * int(M))
    dev = _cuda_device([("local", local), ("delta", delta), ("carry_in", carry_in), ("A", A), ("out", out)])
    if out is None:
        out = torch.empty_like(local)
    else:
        _need("out", out, dtype=torch.float32, numel=n)
    rc = lib.ia_state_carry(ctypes.byref(shp), _ptr(delta), _ptr(A), int(L), _ptr(carry_in), _ptr(local),
                            _ptr(out), _stream(stream))
    _check(rc, "ia_state_carry")
    return out


def _presence_options(norm, selective, readout, bidirectional):
    """Options whose arrays are placeholder addresses: for the queries, which
    test only which parts are present and read no array."""
    opt = IAOptions()
    some = ctypes.c_void_p(256)
    if selective:
        opt.delta_t = some
    if norm:
        opt.gain = some
    if readout:
        opt.W = some
    opt.eps = 1e-6
    opt.bidirectional = int(bool(bidirectional))
    return opt


def prefill_ex_path(B, H, N, d_xi, d_v, M, dtype, norm=False, selective=False, readout=False,
                    bidirectional=False):
    """'tensor_core' or 'sequential': the kernels ia_prefill_fwd_ex runs for this
    shape and these optional parts."""
    opt = _presence_options(norm, selective, readout, bidirectional)
    shp = make_shape(B, H, N, d_xi, d_v, M, dtype)
    return PATHS[load_library().ia_prefill_ex_path(ctypes.byref(shp), ctypes.byref(opt))]


def prefill_ex_segments(B, H, N, d_xi, d_v, M, dtype, workspace_bytes, norm=False, selective=False,
                        readout=False, bidirectional=False) -> int:
    """Segments per sequence ia_prefill_fwd_ex runs with a workspace of that
    many bytes (0 bytes: none given): 1 for the tensor-core form and a single
    token-serial pass."""
    opt = _presence_options(norm, selective, readout, bidirectional)
    shp = make_shape(B, H, N, d_xi, d_v, M, dtype)
    ws = ctypes.c_void_p(16) if workspace_bytes else None   # only the pointer's presence counts
    return int(load_library().ia_prefill_ex_segments(ctypes.byref(shp), ctypes.byref(opt), ws,
                                                     ctypes.c_size_t(workspace_bytes)))


def prefill_ex_workspace_bytes(B, H, N, d_xi, d_v, M, dtype, norm=False, selective=False, readout=False,
                               bidirectional=False) -> int:
    """Workspace bytes ia_prefill_fwd_ex needs for this shape and these parts."""
    opt = _presence_options(norm, selective, readout, bidirectional)
    shp = make_shape(B, H, N, d_xi, d_v, M, dtype)
    return int(load_library().ia_prefill_ex_workspace_bytes(ctypes.byref(shp), ctypes.byref(opt)))


def prefill_static_max_heads() -> int:
    return int(load_library().ia_prefill_static_max_heads())


def fwd_bwd_workspace_bytes(B, H, N, d_xi, d_v, M, dtype) -> int:
    return int(load_library().ia_fwd_bwd_workspace_bytes(ctypes.byref(make_shape(B, H, N, d_xi, d_v, M, dtype))))


def _workspace(nbytes, device, workspace):
    if nbytes == 0:
        return None
    if workspace is not None:
        return workspace
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


# The library receives raw device pointers and cannot see tensor sizes, so the
# binding checks every tensor against the shape before the call: a short or
# misplaced buffer is an error here rather than an out-of-bounds access on the
# GPU.  Shapes and dtypes are checked first, the device last.
def _need(name, t, shape=None, dtype=None, numel=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, got {type(t).__name__}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} has {t.numel()} elements, expected {numel}")


def _cuda_device(named):
    """The one CUDA device all given tensors live on (None entries skipped)."""
    dev = None
    for name, t in named:
        if t is None:
            continue
        if t.device.type != "cuda":
            raise ValueError(f"{name} is on {t.device}; the library takes CUDA tensors")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the other tensors on {dev}")
    return dev


def _check_delta(delta, H, M):
    """delta [H] (one step per head) or [H,M] (one per head and mode), fp32.
    Returns True for the per-mode form."""
    _need("delta", delta, dtype=torch.float32)
    if tuple(delta.shape) == (H,):
        return False
    if tuple(delta.shape) == (H, int(M)):
        return True
    raise ValueError(f"delta has shape {tuple(delta.shape)}, expected ({H},) or ({H}, {int(M)})")


def _check_sequence_args(q, k, v, delta, M, A, dO=None):
    """q, k [B,H,N,d_xi], v and dO [B,H,N,d_v] in one input dtype, delta [H]
    or [H,M] fp32, A [M] complex as 2M fp32 (or None).  Returns (B, H, N, d_xi, d_v)."""
    _need("q", q)
    if q.dim() != 4:
        raise ValueError(f"q must be [B,H,N,d_xi], got shape {tuple(q.shape)}")
    _dtype_code(q)
    B, H, N, d_xi = q.shape
    _need("k", k, (B, H, N, d_xi), q.dtype)
    _need("v", v, dtype=q.dtype)
    if v.dim() != 4 or tuple(v.shape[:3]) != (B, H, N):
        raise ValueError(f"v must be [B,H,N,d_v] = [{B},{H},{N},d_v], got {tuple(v.shape)}")
    d_v = v.shape[3]
    _check_delta(delta, H, M)
    if A is not None:
        _need("A", A, dtype=torch.float32, numel=2 * int(M))
    if dO is not None:
        _need("dO", dO, (B, H, N, d_v), q.dtype)
    return B, H, N, d_xi, d_v


def _check_token_args(q, k, v, delta, M, A):
    """Decode: q, k [B,H,d_xi], v [B,H,d_v].  Returns (B, H, d_xi, d_v)."""
    _need("q", q)
    if q.dim() != 3:
        raise ValueError(f"q must be [B,H,d_xi], got shape {tuple(q.shape)}")
    _dtype_code(q)
    B, H, d_xi = q.shape
    _need("k", k, (B, H, d_xi), q.dtype)
    _need("v", v, dtype=q.dtype)
    if v.dim() != 3 or tuple(v.shape[:2]) != (B, H):
        raise ValueError(f"v must be [B,H,d_v] = [{B},{H},d_v], got {tuple(v.shape)}")
    _check_delta(delta, H, M)
    if A is not None:
        _need("A", A, dtype=torch.float32, numel=2 * int(M))
    return B, H, d_xi, v.shape[2]


def prefill_fwd(q, k, v, delta, M, A=None, state_in=None, want_num_den=False, want_state=False,
                o=None, workspace=None, stream=None):
    """Causal IA prefill.  q,k [B,H,N,d_xi], v [B,H,N,d_v] (fp32 or bf16), delta [H] fp32.

    Returns dict with o [B,H,N,d_v] fp32 and, on request, num, den, state (flat fp32)."""
    lib = load_library()
    B, H, N, d_xi, d_v = _check_sequence_args(q, k, v, delta, M, A)
    shp = make_shape(B, H, N, d_xi, d_v, M, _dtype_code(q), delta.dim() == 2)
    n_state = lib.ia_state_bytes(ctypes.byref(shp)) // 4
    if state_in is not None:
        _need("state_in", state_in, dtype=torch.float32, numel=n_state)
    if o is not None:
        _need("o", o, (B, H, N, d_v), torch.float32)
    if workspace is not None:
        _need("workspace", workspace)
    dev = _cuda_device([("q", q), ("k", k), ("v", v), ("delta", delta), ("A", A), ("state_in", state_in),
                        ("o", o), ("workspace", workspace)])
    if o is None:
        o = torch.empty(B, H, N, d_v, dtype=torch.float32, device=dev)
    num = torch.empty_like(o) if want_num_den else None
    den = torch.empty(B, H, N, dtype=torch.float32, device=dev) if want_num_den else None
    st = torch.empty(n_state, dtype=torch.float32, device=dev) if want_state else None
    need = lib.ia_prefill_workspace_bytes(ctypes.byref(shp))
    ws = _workspace(need, dev, workspace)
    rc = lib.ia_prefill_fwd(ctypes.byref(shp), _ptr(q), _ptr(k), _ptr(v), _ptr(delta), _ptr(A),
                            _ptr(state_in), _ptr(o), _ptr(num), _ptr(den), _ptr(st), _ptr(ws),
                            ctypes.c_size_t(_nbytes(ws)), _stream(stream))
    _check(rc, "ia_prefill_fwd")
    return {"o": o, "num": num, "den": den, "state": st}


def prefill_fwd_static(q, k, v, delta, M, A=None, state_in=None, want_num_den=False,
                       want_state=False, o=None, stream=None):
    """prefill_fwd for callers that cannot allocate device memory: the library
    keeps its scratch in a fixed per-GPU array instead of a workspace (see
    ia_prefill_fwd_static in include/ia.h).  Output tensors are still the
    caller's; pass `o` (and use want_* = False) to allocate nothing here."""
    lib = load_library()
    B, H, N, d_xi, d_v = _check_sequence_args(q, k, v, delta, M, A)
    shp = make_shape(B, H, N, d_xi, d_v, M, _dtype_code(q), delta.dim() == 2)
    n_state = lib.ia_state_bytes(ctypes.byref(shp)) // 4
    if state_in is not None:
        _need("state_in", state_in, dtype=torch.float32, numel=n_state)
    if o is not None:
        _need("o", o, (B, H, N, d_v), torch.float32)
    dev = _cuda_device([("q", q), ("k", k), ("v", v), ("delta", delta), ("A", A), ("state_in", state_in),
                        ("o", o)])
    if o is None:
        o = torch.empty(B, H, N, d_v, dtype=torch.float32, device=dev)
    num = torch.empty_like(o) if want_num_den else None
    den = torch.empty(B, H, N, dtype=torch.float32, device=dev) if want_num_den else None
    st = torch.empty(n_state, dtype=torch.float32, device=dev) if want_state else None
    rc = lib.ia_prefill_fwd_static(ctypes.byref(shp), _ptr(q), _ptr(k), _ptr(v), _ptr(delta), _ptr(A),
                                   _ptr(state_in), _ptr(o), _ptr(num), _ptr(den), _ptr(st), _stream(stream))
    _check(rc, "ia_prefill_fwd_static")
    return {"o": o, "num": num, "den": den, "state": st}


def fwd_bwd(q, k, v, delta, dO, M, A=None, workspace=None, stream=None):
    """Forward + reverse mode from a zero state: returns dict(o, dq, dk, dv, dDelta, dA).

    delta is [H] (one step per head) or [H,M] (one per head and mode); dDelta
    has its shape.  dA [2M] holds (dL/dRe A_m, dL/dIm A_m), for A as given or
    for the S4D-Lin default when A is None."""
    lib = load_library()
    B, H, N, d_xi, d_v = _check_sequence_args(q, k, v, delta, M, A, dO=dO)
    shp = make_shape(B, H, N, d_xi, d_v, M, _dtype_code(q), delta.dim() == 2)
    if workspace is not None:
        _need("workspace", workspace)
    dev = _cuda_device([("q", q), ("k", k), ("v", v), ("delta", delta), ("A", A), ("dO", dO),
                        ("workspace", workspace)])
    o = torch.empty(B, H, N, d_v, dtype=torch.float32, device=dev)
    dq = torch.empty(B, H, N, d_xi, dtype=torch.float32, device=dev)
    dk = torch.empty_like(dq)
    dv = torch.empty(B, H, N, d_v, dtype=torch.float32, device=dev)
    dD = torch.empty(tuple(delta.shape), dtype=torch.float32, device=dev)
    dA = torch.empty(2 * int(M), dtype=torch.float32, device=dev)
    need = lib.ia_fwd_bwd_workspace_bytes(ctypes.byref(shp))
    ws = _workspace(need, dev, workspace)
    rc = lib.ia_fwd_bwd(ctypes.byref(shp), _ptr(q), _ptr(k), _ptr(v), _ptr(delta), _ptr(A), _ptr(dO),
                        _ptr(o), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dD), _ptr(dA), _ptr(ws),
                        ctypes.c_size_t(_nbytes(ws)), _stream(stream))
    _check(rc, "ia_fwd_bwd")
    return {"o": o, "dq": dq, "dk": dk, "dv": dv, "dDelta": dD, "dA": dA}


def decode_step(q, k, v, delta, state, M, A=None, o=None, want_num_den=False, stream=None):
    """One decode step.  q,k [B,H,d_xi], v [B,H,d_v]; state (flat fp32) updated in place."""
    lib = load_library()
    B, H, d_xi, d_v = _check_token_args(q, k, v, delta, M, A)
    shp = make_shape(B, H, 1, d_xi, d_v, M, _dtype_code(q), delta.dim() == 2)
    _need("state", state, dtype=torch.float32, numel=lib.ia_state_bytes(ctypes.byref(shp)) // 4)
    if o is not None:
        _need("o", o, (B, H, d_v), torch.float32)
    dev = _cuda_device([("q", q), ("k", k), ("v", v), ("delta", delta), ("A", A), ("state", state), ("o", o)])
    if o is None:
        o = torch.empty(B, H, d_v, dtype=torch.float32, device=dev)
    num = torch.empty_like(o) if want_num_den else None
    den = torch.empty(B, H, dtype=torch.float32, device=dev) if want_num_den else None
    rc = lib.ia_decode_step(ctypes.byref(shp), _ptr(q), _ptr(k), _ptr(v), _ptr(delta), _ptr(A),
                            _ptr(state), _ptr(o), _ptr(num), _ptr(den), _stream(stream))
    _check(rc, "ia_decode_step")
    return {"o": o, "num": num, "den": den}


def _options(named_shapes, delta_t, gain, bias, eps, W, bidirectional, B, H, M, d_xi, d_v, tokens):
    """Check the optional parts and build the C options struct."""
    if delta_t is not None:
        _need("delta_t", delta_t, (B, H) + tokens, torch.float32)
    for name, t in (("gain", gain), ("bias", bias)):
        if t is not None:
            _need(name, t, (H, d_xi + d_v), torch.float32)
    if W is not None:
        _need("W", W, dtype=torch.float32, numel=2 * H * int(M) * int(M))
    opt = IAOptions(_ptr(delta_t), _ptr(gain), _ptr(bias), float(eps), _ptr(W), int(bool(bidirectional)))
    return opt


def prefill_fwd_ex(q, k, v, M, delta=None, A=None, delta_t=None, gain=None, bias=None, eps=1e-6, W=None,
                   bidirectional=False, state_in=None, want_num_den=False, want_state=False, stream=None,
                   workspace=None, o=None):
    """The layer with its optional parts (see ia_prefill_fwd_ex in include/ia.h):
    delta_t [B,H,N] a step per token, gain/bias [H, d_xi+d_v] the RMSNorm on the
    SSM input, W [H,M,M,2] (re, im) the complex readout matrix, bidirectional
    the two-direction layer.  workspace: a uint8 device tensor of at least
    prefill_ex_workspace_bytes (allocated here when None).  Returns dict(o,
    num, den, state)."""
    lib = load_library()
    _need("q", q)
    if q.dim() != 4:
        raise ValueError(f"q must be [B,H,N,d_xi], got shape {tuple(q.shape)}")
    B, H, N, d_xi = q.shape
    _need("k", k, (B, H, N, d_xi), q.dtype)
    _need("v", v, dtype=q.dtype)
    if v.dim() != 4 or tuple(v.shape[:3]) != (B, H, N):
        raise ValueError(f"v must be [B,H,N,d_v], got {tuple(v.shape)}")
    d_v = v.shape[3]
    dpm = _check_delta(delta, H, M) if delta is not None else False
    if delta is None and delta_t is None:
        raise ValueError("either delta or delta_t is needed")
    if A is not None:
        _need("A", A, dtype=torch.float32, numel=2 * int(M))
    shp = make_shape(B, H, N, d_xi, d_v, M, _dtype_code(q), dpm)
    n_state = lib.ia_state_bytes(ctypes.byref(shp)) // 4
    if state_in is not None:
        _need("state_in", state_in, dtype=torch.float32, numel=n_state)
    opt = _options(None, delta_t, gain, bias, eps, W, bidirectional, B, H, M, d_xi, d_v, (N,))
    dev = _cuda_device([("q", q), ("k", k), ("v", v), ("delta", delta), ("A", A), ("delta_t", delta_t),
                        ("gain", gain), ("bias", bias), ("W", W), ("state_in", state_in)])
    if o is None:
        o = torch.empty(B, H, N, d_v, dtype=torch.float32, device=dev)
    else:
        _need("o", o, (B, H, N, d_v), torch.float32)
    num = torch.empty_like(o) if want_num_den else None
    den = torch.empty(B, H, N, dtype=torch.float32, device=dev) if want_num_den else None
    st = torch.empty(n_state, dtype=torch.float32, device=dev) if want_state else None
    need = int(lib.ia_prefill_ex_workspace_bytes(ctypes.byref(shp), ctypes.byref(opt)))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev) if need else None
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rc = lib.ia_prefill_fwd_ex(ctypes.byref(shp), ctypes.byref(opt), _ptr(q), _ptr(k), _ptr(v), _ptr(delta),
                               _ptr(A), _ptr(state_in), _ptr(o), _ptr(num), _ptr(den), _ptr(st),
                               _ptr(workspace), nbytes, _stream(stream))
    _check(rc, "ia_prefill_fwd_ex")
    return {"o": o, "num": num, "den": den, "state": st}


def decode_step_ex(q, k, v, state, M, delta=None, A=None, delta_t=None, gain=None, bias=None, eps=1e-6,
                   W=None, want_num_den=False, stream=None):
    """One decode step with the optional parts; delta_t is [B,H] here."""
    lib = load_library()
    _need("q", q)
    if q.dim() != 3:
        raise ValueError(f"q must be [B,H,d_xi], got shape {tuple(q.shape)}")
    B, H, d_xi = q.shape
    _need("k", k, (B, H, d_xi), q.dtype)
    _need("v", v, dtype=q.dtype)
    d_v = v.shape[2]
    dpm = _check_delta(delta, H, M) if delta is not None else False
    if delta is None and delta_t is None:
        raise ValueError("either delta or delta_t is needed")
    shp = make_shape(B, H, 1, d_xi, d_v, M, _dtype_code(q), dpm)
    _need("state", state, dtype=torch.float32, numel=lib.ia_state_bytes(ctypes.byref(shp)) // 4)
    opt = _options(None, delta_t, gain, bias, eps, W, False, B, H, M, d_xi, d_v, ())
    dev = _cuda_device([("q", q), ("k", k), ("v", v), ("delta", delta), ("A", A), ("state", state),
                        ("delta_t", delta_t), ("gain", gain), ("bias", bias), ("W", W)])
    o = torch.empty(B, H, d_v, dtype=torch.float32, device=dev)
    num = torch.empty_like(o) if want_num_den else None
    den = torch.empty(B, H, dtype=torch.float32, device=dev) if want_num_den else None
    rc = lib.ia_decode_step_ex(ctypes.byref(shp), ctypes.byref(opt), _ptr(q), _ptr(k), _ptr(v), _ptr(delta),
                               _ptr(A), _ptr(state), _ptr(o), _ptr(num), _ptr(den), _stream(stream))
    _check(rc, "ia_decode_step_ex")
    return {"o": o, "num": num, "den": den}


def set_launch_events(begin=None, end=None):
    """Bracket every later call's dominant kernel launch with two torch.cuda.Events
    (profiling aid); call with no arguments to stop."""
    b = ctypes.c_void_p(begin.cuda_event) if begin is not None else None
    e = ctypes.c_void_p(end.cuda_event) if end is not None else None
    _check(load_library().ia_set_launch_events(b, e), "ia_set_launch_events")


def check_device_errors(stream=None):
    """Synchronise the stream and raise if a device-side bounded wait expired
    (IA_ERR_TIMEOUT) or a tensor-core call met an out-of-range Delta
    (IA_ERR_PARAM_RANGE); the flag is cleared either way."""
    _check(load_library().ia_check_device_errors(_stream(stream)), "ia_check_device_errors")


def selftest_wait_expiry(limit_ns, device=None, stream=None):
    """Run the library's bounded-wait self-test kernel (see include/ia.h) and
    return its six u64 results: per waiter, completed flag and ns waited."""
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    out = torch.zeros(6, dtype=torch.int64, device=dev)
    _check(load_library().ia_selftest_wait_expiry(ctypes.c_ulonglong(int(limit_ns)), _ptr(out), _stream(stream)),
           "ia_selftest_wait_expiry")
    return out
