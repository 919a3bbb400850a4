"""Seeded synthetic inputs for the IA layer -- random draws only.

This module holds none of the layer's arithmetic; both the CUDA path's tests
and the oracle read the same tensors from here.  Recipe (all on a CPU
``torch.Generator``):

1. ``delta`` [H]: log-uniform on [1e-3, 1e-1] (the S4D-Lin step range),
   ``exp(log(1e-3) + U(0,1) * (log(1e-1) - log(1e-3)))`` in fp32;
2. ``q, k`` [B,H,N,d_xi] then ``v`` [B,H,N,d_v]: standard normal fp32, cast to
   bf16 for bf16 workloads (the cast is the input; it is not counted as error);
3. ``dO`` [B,H,N,d_v] (training only): standard normal, cast like v.

Decode steps draw their per-step q, k, v from seed ``2000 + step``.
"""
import math

import torch

LOG_DMIN = math.log(1e-3)
LOG_DMAX = math.log(1e-1)


def _dtype(name):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def make_delta(H, gen):
    u = torch.rand(H, generator=gen, dtype=torch.float32)
    return torch.exp(LOG_DMIN + u * (LOG_DMAX - LOG_DMIN))


def layer_inputs(B, H, N, d_xi, d_v, dtype="bf16", seed=0, with_grad=False):
    """Returns dict(delta, q, k, v[, dO]) as CPU tensors in the input dtype."""
    gen = torch.Generator().manual_seed(seed)
    dt = _dtype(dtype)
    out = {"delta": make_delta(H, gen)}
    out["q"] = torch.randn(B, H, N, d_xi, generator=gen).to(dt)
    out["k"] = torch.randn(B, H, N, d_xi, generator=gen).to(dt)
    out["v"] = torch.randn(B, H, N, d_v, generator=gen).to(dt)
    if with_grad:
        out["dO"] = torch.randn(B, H, N, d_v, generator=gen).to(dt)
    return out


def workload_inputs(w, B=None, N=None, with_grad=None):
    """Inputs for a Workload, optionally with a different batch or length."""
    return layer_inputs(B or w.B, w.H, N or w.N, w.d_xi, w.d_v, w.dtype, w.seed,
                        with_grad=(w.kind == "fwd_bwd") if with_grad is None else with_grad)


def decode_token(B, H, d_xi, d_v, dtype="bf16", step=0):
    """q, k [B,H,d_xi] and v [B,H,d_v] for one decode step."""
    gen = torch.Generator().manual_seed(2000 + step)
    dt = _dtype(dtype)
    q = torch.randn(B, H, d_xi, generator=gen).to(dt)
    k = torch.randn(B, H, d_xi, generator=gen).to(dt)
    v = torch.randn(B, H, d_v, generator=gen).to(dt)
    return q, k, v
