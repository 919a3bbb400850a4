"""fp64 CPU oracle for the Interdomain Attention (IA) layer -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py``
(``cpu_baseline`` and ``--impl reference``) may import this package.  The
product path (``ssm_token_mixer_b200``) never does; it fails loudly when its
CUDA library is missing instead of falling back here.

The arithmetic lives in ``ia_oracle.c`` (plain C, fp64, OpenMP over the
independent (batch, head) sequences).  This module only builds that file with
gcc and marshals numpy arrays to it.  What is computed, and which passage of
the paper "Interdomain Attention: Beyond Token-Level Key-Value Memory" each
routine follows, is stated in ``ia_oracle.c``.

Pins (tests/test_oracle_pins.py) tie every routine here to something other
than itself: brute-force quadratic form, closed forms, special cases that
reduce to textbook averages, finite differences and a tangent/adjoint
dot-product test.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ia_oracle.c")
_LIB = os.path.join(_HERE, "libia_oracle.so")
_lib = None


def compile_source(src: str, out: str) -> str:
    """Compile an oracle source file into a shared library at ``out`` with the
    oracle's flags (gcc, -O2, OpenMP, IEEE fp64 with no contraction).  The
    mutation test uses it to build copies that carry a planted mistake."""
    tmp = out + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-fno-fast-math", "-ffp-contract=off", src, "-o", tmp, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile ia_oracle.c into libia_oracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "ia_oracle.h"))
    ):
        compile_source(_SRC, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i = ctypes.c_int
        lib.iao_state_len.restype = ctypes.c_long
        lib.iao_state_len.argtypes = [i] * 5
        lib.iao_params.argtypes = [i, ctypes.c_double, P, P, P]
        lib.iao_forward.argtypes = [i] * 6 + [P] * 4 + [i] + [P] * 6
        lib.iao_forward_features.argtypes = [i] * 6 + [P] * 10
        lib.iao_decode_step.argtypes = [i] * 5 + [P] * 4 + [i] + [P] * 5
        lib.iao_brute.argtypes = [i] * 6 + [P] * 4 + [i] + [P] * 4
        lib.iao_backward.argtypes = [i] * 6 + [P] * 4 + [i] + [P] * 8
        lib.iao_jvp.argtypes = [i] * 6 + [P] * 4 + [i] + [P] * 7
        lib.iao_forward_ex.argtypes = [i] * 6 + [P] * 3 + [i, P, i] + [P] * 4 + [ctypes.c_double] + [P] * 6
        lib.iao_num_threads.restype = i
        for name in ("iao_params", "iao_forward", "iao_forward_features", "iao_decode_step",
                     "iao_brute", "iao_backward", "iao_jvp", "iao_forward_ex"):
            getattr(lib, name).restype = i
        _lib = lib
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor (any dtype, any device) -> exact fp64
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(x):
    return None if x is None else x.ctypes.data_as(ctypes.c_void_p)


def _dpm(delta):
    """1 if delta holds one value per head and mode ([H,M]), 0 for one per head ([H])."""
    return 1 if delta.ndim == 2 else 0


def _check(rc, name):
    if rc != 0:
        raise RuntimeError(f"oracle {name} failed with code {rc}")


def num_threads() -> int:
    return int(_load().iao_num_threads())


def state_len(B, H, M, d_xi, d_v) -> int:
    return int(_load().iao_state_len(B, H, M, d_xi, d_v))


def split_state(state, B, H, M, d_xi, d_v):
    """View a flat state buffer as complex (U [B,H,M,d_xi], Gamma [B,H,M,d_v], eta [B,H,M])."""
    s = np.asarray(state, dtype=np.float64)
    n1, n2, n3 = 2 * B * H * M * d_xi, 2 * B * H * M * d_v, 2 * B * H * M
    U = s[:n1].view(np.complex128).reshape(B, H, M, d_xi)
    G = s[n1:n1 + n2].view(np.complex128).reshape(B, H, M, d_v)
    e = s[n1 + n2:n1 + n2 + n3].view(np.complex128).reshape(B, H, M)
    return U, G, e


def params(M, delta, A=None):
    """lambda_m, b_m (complex [M]) for one head."""
    lam = np.zeros(2 * M)
    b = np.zeros(2 * M)
    A = _f64(A)
    _check(_load().iao_params(M, float(delta), _p(A), _p(lam), _p(b)), "params")
    return lam.view(np.complex128), b.view(np.complex128)


def forward(q, k, v, delta, M, A=None, state_in=None, want_state=True):
    """Sequential recurrence.  q,k [B,H,N,d_xi], v [B,H,N,d_v], delta [H] or [H,M], M modes.

    Returns dict(o, num, den, state) in fp64 (state flat, see split_state)."""
    q, k, v, delta, A, state_in = map(_f64, (q, k, v, delta, A, state_in))
    return _forward(q, k, v, delta, A, state_in, want_state, M)


def _forward(q, k, v, delta, A, state_in, want_state, M):
    B, H, N, d_xi = q.shape
    d_v = v.shape[-1]
    o = np.zeros((B, H, N, d_v))
    num = np.zeros((B, H, N, d_v))
    den = np.zeros((B, H, N))
    st = np.zeros(state_len(B, H, M, d_xi, d_v)) if want_state else None
    rc = _load().iao_forward(B, H, N, d_xi, d_v, M, _p(q), _p(k), _p(v), _p(delta), _dpm(delta), _p(A),
                             _p(state_in), _p(o), _p(num), _p(den), _p(st))
    _check(rc, "forward")
    return {"o": o, "num": num, "den": den, "state": st}


def forward_features(fq, fk, v, lam, b, state_in=None):
    """Recurrence on already-mapped features with explicit lambda/b tables [H,M] complex."""
    fq, fk, v, state_in = map(_f64, (fq, fk, v, state_in))
    lam = np.ascontiguousarray(np.asarray(lam, dtype=np.complex128)).view(np.float64)
    b = np.ascontiguousarray(np.asarray(b, dtype=np.complex128)).view(np.float64)
    B, H, N, d_xi = fq.shape
    d_v = v.shape[-1]
    M = lam.size // (2 * H)
    o = np.zeros((B, H, N, d_v))
    num = np.zeros((B, H, N, d_v))
    den = np.zeros((B, H, N))
    st = np.zeros(state_len(B, H, M, d_xi, d_v))
    rc = _load().iao_forward_features(B, H, N, d_xi, d_v, M, _p(fq), _p(fk), _p(v), _p(lam),
                                      _p(b), _p(state_in), _p(o), _p(num), _p(den), _p(st))
    _check(rc, "forward_features")
    return {"o": o, "num": num, "den": den, "state": st}


def decode_step(q, k, v, delta, M, state, A=None):
    """One decode step; q,k [B,H,d_xi], v [B,H,d_v]; returns (o, num, den, new_state)."""
    q, k, v, delta, A = map(_f64, (q, k, v, delta, A))
    st = np.array(_f64(state), copy=True)
    B, H, d_xi = q.shape
    d_v = v.shape[-1]
    o = np.zeros((B, H, d_v))
    num = np.zeros((B, H, d_v))
    den = np.zeros((B, H))
    rc = _load().iao_decode_step(B, H, d_xi, d_v, M, _p(q), _p(k), _p(v), _p(delta), _dpm(delta), _p(A),
                                 _p(st), _p(o), _p(num), _p(den))
    _check(rc, "decode_step")
    return o, num, den, st


def brute(q, k, v, delta, M, A=None):
    q, k, v, delta, A = map(_f64, (q, k, v, delta, A))
    B, H, N, d_xi = q.shape
    d_v = v.shape[-1]
    o = np.zeros((B, H, N, d_v))
    num = np.zeros((B, H, N, d_v))
    den = np.zeros((B, H, N))
    rc = _load().iao_brute(B, H, N, d_xi, d_v, M, _p(q), _p(k), _p(v), _p(delta), _dpm(delta), _p(A),
                           _p(o), _p(num), _p(den))
    _check(rc, "brute")
    return {"o": o, "num": num, "den": den}


def backward(q, k, v, delta, dO, M, A=None):
    """Reverse mode from a zero state: returns dict(o, dq, dk, dv, dDelta, dA).

    dDelta has delta's shape ([H] or [H,M]); dA is [2M] as (dL/dRe A_m,
    dL/dIm A_m) pairs, summed over batch, heads and time."""
    q, k, v, delta, dO, A = map(_f64, (q, k, v, delta, dO, A))
    B, H, N, d_xi = q.shape
    d_v = v.shape[-1]
    o = np.zeros((B, H, N, d_v))
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dD = np.zeros(delta.shape)
    dA = np.zeros(2 * M)
    rc = _load().iao_backward(B, H, N, d_xi, d_v, M, _p(q), _p(k), _p(v), _p(delta), _dpm(delta), _p(A),
                              _p(dO), _p(o), _p(dq), _p(dk), _p(dv), _p(dD), _p(dA))
    _check(rc, "backward")
    return {"o": o, "dq": dq, "dk": dk, "dv": dv, "dDelta": dD, "dA": dA}


def jvp(q, k, v, delta, tq, tk, tv, tdelta, M, A=None, tA=None):
    """Output tangent along (tq, tk, tv, tdelta[, tA]); tdelta has delta's shape,
    tA is [2M] (re, im) pairs or None."""
    q, k, v, delta, tq, tk, tv, tdelta, A, tA = map(_f64, (q, k, v, delta, tq, tk, tv, tdelta, A, tA))
    B, H, N, d_xi = q.shape
    d_v = v.shape[-1]
    to = np.zeros((B, H, N, d_v))
    rc = _load().iao_jvp(B, H, N, d_xi, d_v, M, _p(q), _p(k), _p(v), _p(delta), _dpm(delta), _p(A),
                         _p(tq), _p(tk), _p(tv), _p(tdelta), _p(tA), _p(to))
    _check(rc, "jvp")
    return to


def forward_ex(q, k, v, M, delta=None, A=None, delta_t=None, gain=None, bias=None, eps=1e-6, W=None,
               state_in=None, map_features=True):
    """The layer with its optional parts (see iao_forward_ex): RMSNorm gain and
    bias [H, d_xi+d_v] on the SSM input, a step per token delta_t [B,H,N], a
    complex readout matrix W [H,M,M] (complex array or [H,M,M,2] reals).
    Returns dict(o, num, den, state)."""
    q, k, v, delta, A, delta_t, gain, bias, state_in = map(
        _f64, (q, k, v, delta, A, delta_t, gain, bias, state_in))
    if W is not None:
        W = np.asarray(W)
        W = np.ascontiguousarray(W.astype(np.complex128) if np.iscomplexobj(W) else
                                 W.reshape(W.shape[:-1] + (2,)).astype(np.float64).view(np.complex128)[..., 0])
        W = W.view(np.float64)
    B, H, N, d_xi = q.shape
    d_v = v.shape[-1]
    o = np.zeros((B, H, N, d_v))
    num = np.zeros((B, H, N, d_v))
    den = np.zeros((B, H, N))
    st = np.zeros(state_len(B, H, M, d_xi, d_v))
    dpm = 0 if delta is None else _dpm(delta)
    rc = _load().iao_forward_ex(B, H, N, d_xi, d_v, M, _p(q), _p(k), _p(v), 1 if map_features else 0,
                                _p(delta), dpm, _p(A), _p(delta_t), _p(gain), _p(bias), float(eps), _p(W),
                                _p(state_in), _p(o), _p(num), _p(den), _p(st))
    _check(rc, "forward_ex")
    return {"o": o, "num": num, "den": den, "state": st}


def forward_bidirectional(q, k, v, M, **kw):
    """The bidirectional layer (summary sec. 5.2: Caduceus-IA keeps Caduceus'
    bidirectional handling): the causal layer on the sequence plus the causal
    layer on the time-reversed sequence, reversed back: o = f(x) + flip(f(flip x)).
    Per-token arrays in kw (delta_t) are reversed with the inputs."""
    fwd = forward_ex(q, k, v, M, **kw)["o"]
    flip = lambda x: None if x is None else np.ascontiguousarray(np.flip(_f64(x), axis=2))
    kw_r = dict(kw)
    if kw.get("delta_t") is not None:
        kw_r["delta_t"] = flip(kw["delta_t"])
    rev = forward_ex(flip(q), flip(k), flip(v), M, **kw_r)["o"]
    return fwd + np.flip(rev, axis=2)
