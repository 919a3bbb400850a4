"""Shared helpers for the GPU parity tests (test infrastructure)."""
import numpy as np
import torch

import ssm_token_mixer_b200 as ia
from ssm_token_mixer_b200 import build


def device():
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda:0")


def to_dev(inp, dev):
    return {k: v.to(dev) for k, v in inp.items()}


def gpu_prefill(inp, M, dev, state_in=None, **kw):
    d = to_dev(inp, dev)
    r = ia.prefill_fwd(d["q"], d["k"], d["v"], d["delta"], M, want_num_den=True, want_state=True,
                       state_in=state_in, **kw)
    ia.check_device_errors()
    return {k: (v.cpu() if v is not None else None) for k, v in r.items()}


def pick(inp, bh_list, H):
    """Sub-batch of (b,h) slices as [n,1,N,d] tensors plus their deltas."""
    out = {}
    for key in ("q", "k", "v", "dO"):
        if key in inp:
            out[key] = torch.stack([inp[key][b, h] for b, h in bh_list])[:, None]
    out["delta"] = None
    return out


def state_slices(state, B, H, M, dx, dv, bh_list):
    """Flat state -> complex U, G, eta for the listed (b,h), each [n,1,...]."""
    s = state.double().numpy() if hasattr(state, "numpy") else np.asarray(state)
    n1, n2 = 2 * B * H * M * dx, 2 * B * H * M * dv
    U = s[:n1].view(np.complex128).reshape(B, H, M, dx)
    G = s[n1:n1 + n2].view(np.complex128).reshape(B, H, M, dv)
    e = s[n1 + n2:n1 + n2 + 2 * B * H * M].view(np.complex128).reshape(B, H, M)
    idx = tuple(np.array(x) for x in zip(*bh_list))
    return U[idx][:, None], G[idx][:, None], e[idx][:, None]
