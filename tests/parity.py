"""Error measures for comparing the CUDA path with the fp64 oracle.

Readings of 'max relative error' (the bar is 1e-4 for fp32 inputs and 2e-2
for bf16 inputs, checked on num and den separately): normwise per (b,h)
slice, max|x - r| / max|r|.  o = num/den is compared only where
|den| >= 1e-3 max|den| in the slice, because den is a signed sum (the
readout weights can be negative) and o is ill-conditioned near its zeros.
"""
import numpy as np

TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def to_np(x):
    if hasattr(x, "detach"):
        return x.detach().double().cpu().numpy()
    x = np.asarray(x)
    return x.astype(np.complex128) if np.iscomplexobj(x) else x.astype(np.float64)


def slice_rel(x, r, axes):
    """max over leading (b,h) slices of max|x-r| / max|r| reduced over `axes`."""
    x, r = to_np(x), to_np(r)
    err = np.max(np.abs(x - r), axis=axes)
    ref = np.max(np.abs(r), axis=axes)
    return float(np.max(err / np.maximum(ref, 1e-300)))


def o_rel(o, o_ref, den_ref):
    """Normwise error of o over the rows whose |den| is not near a zero crossing."""
    o, o_ref, den_ref = to_np(o), to_np(o_ref), to_np(den_ref)
    worst = 0.0
    for idx in np.ndindex(*o.shape[:-2]):
        d = np.abs(den_ref[idx])
        keep = d >= 1e-3 * d.max()
        if keep.any():
            e = np.max(np.abs(o[idx][keep] - o_ref[idx][keep])) / np.max(np.abs(o_ref[idx][keep]))
            worst = max(worst, float(e))
    return worst


def report(num, den, o, ref):
    """Dict of the three measures for prefill outputs [B,H,N,...] vs oracle dict."""
    return {"num": slice_rel(num, ref["num"], (-2, -1)),
            "den": slice_rel(den, ref["den"], (-1,)),
            "o": o_rel(o, ref["o"], ref["den"])}
