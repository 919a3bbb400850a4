"""ia_prefill_fwd_static: the prefill for callers that cannot allocate device
memory (a plugin inside another framework's memory pool, or a serving loop
that must not reach cudaMalloc/cudaFree because they can synchronise the
device).  It keeps its scratch in a fixed array inside the library, so this
file checks, through the C-ABI, that two calls in a row -- different shapes,
so the second one reads whatever the first left in the shared array -- give
the same results as ia_prefill_fwd and as the fp64 oracle within the bf16
parity bar, and that a problem too large for the array is refused before any
launch while the largest one it holds runs.

Kept in a file of its own that pytest collects last."""
import pytest
import torch

import ssm_token_mixer_b200 as ia
from gpu_common import device
from parity import TOL_BF16, report, slice_rel
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


def test_static_scratch_prefill_matches_oracle(oracle_mod):
    dev = device()
    B, H, N, d = 1, 3, 200, 64
    inp = synthetic.layer_inputs(B, H, N, d, d, "bf16", seed=303)
    q, k, v, delta = (inp[n].to(dev) for n in ("q", "k", "v", "delta"))
    for _ in range(2):                              # two calls in a row share the array
        got = ia.prefill_fwd_static(q, k, v, delta, 64, want_num_den=True)
        ia.check_device_errors()
        r = report(got["num"].cpu(), got["den"].cpu(), got["o"].cpu(),
                   oracle_mod.forward(inp["q"], inp["k"], inp["v"], inp["delta"], 64, want_state=False))
        assert max(r.values()) < TOL_BF16, r


def test_static_scratch_head_limit():
    dev = device()
    H = ia.prefill_static_max_heads()               # 99 heads of tables fill the 2 MiB array
    for heads, ok in ((H, True), (H + 1, False)):
        inp = synthetic.layer_inputs(1, heads, 64, 64, 64, "bf16", seed=1)
        q, k, v, delta = (inp[n].to(dev) for n in ("q", "k", "v", "delta"))
        if ok:
            got = ia.prefill_fwd_static(q, k, v, delta, 64)
            ia.check_device_errors()
            ref = ia.prefill_fwd(q, k, v, delta, 64)
            assert slice_rel(got["o"].cpu(), ref["o"].cpu(), (-2, -1)) < TOL_BF16
        else:
            with pytest.raises(ia.IAError) as err:
                ia.prefill_fwd_static(q, k, v, delta, 64)
            assert err.value.status == 3
