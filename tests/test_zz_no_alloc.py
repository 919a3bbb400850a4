"""ia_prefill_fwd_static: the prefill for callers that cannot allocate device
memory (a plugin inside another framework's memory pool, or a serving loop
that must not reach cudaMalloc/cudaFree because they can synchronise the
device).  It keeps its scratch in a fixed array inside the library, so this
file checks, through the C-ABI, that two calls in a row -- different shapes,
so the second one reads whatever the first left in the shared array -- give
the same results as ia_prefill_fwd within the bf16 parity bar, and that a
problem too large for the array is refused before any launch.

Kept in a file of its own that pytest collects last."""
import pytest
import torch

import ssm_token_mixer_b200 as ia
from gpu_common import device
from parity import TOL_BF16, slice_rel
from ssm_token_mixer_b200 import synthetic

pytestmark = pytest.mark.gpu


def test_static_scratch_prefill_matches_workspace_entry_point():
    dev = device()
    cases = [(2, 3, 300, 64, 64, 101), (1, 4, 130, 128, 128, 202)]   # two calls in a row
    for B, H, N, dx, dv, seed in cases:
        inp = synthetic.layer_inputs(B, H, N, dx, dv, "bf16", seed=seed)
        q, k, v, delta = (inp[n].to(dev) for n in ("q", "k", "v", "delta"))
        ref = ia.prefill_fwd(q, k, v, delta, 64, want_num_den=True, want_state=True)
        got = ia.prefill_fwd_static(q, k, v, delta, 64, want_num_den=True, want_state=True)
        ia.check_device_errors()
        assert slice_rel(got["num"].cpu(), ref["num"].cpu(), (-2, -1)) < TOL_BF16
        assert slice_rel(got["den"].cpu(), ref["den"].cpu(), (-1,)) < TOL_BF16
        st_err = (got["state"] - ref["state"]).abs().max() / ref["state"].abs().max()
        assert st_err.item() < TOL_BF16
        keep = ref["den"].abs() >= 1e-3 * ref["den"].abs().amax(dim=-1, keepdim=True)
        diff = (got["o"] - ref["o"]).abs()[keep]
        assert (diff.max() / ref["o"].abs()[keep].max()).item() < TOL_BF16


def test_static_scratch_refuses_too_many_heads():
    dev = device()
    H = 128                                         # 128 x 21.5 KB of tables > 2 MiB
    inp = synthetic.layer_inputs(1, H, 64, 64, 64, "bf16", seed=1)
    q, k, v, delta = (inp[n].to(dev) for n in ("q", "k", "v", "delta"))
    with pytest.raises(ia.IAError) as err:
        ia.prefill_fwd_static(q, k, v, delta, 64)
    assert err.value.status == 3
