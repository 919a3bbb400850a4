"""Failure reporting on the GPU, with no fault, trap or hang.

- The bounded waits' expiry path: a small library kernel waits on shared
  barriers that nothing completes, with a short limit, and nothing else in
  flight.  The kernel must return, the abortable wait with the full limit
  must give up as soon as its neighbour raises the abort flag, and
  ia_check_device_errors must report IA_ERR_TIMEOUT once, then clear it.
- The tensor-core path's fp16 range: a Delta whose decay factor over half a
  chunk exceeds the limit stated in include/ia.h must be reported as
  IA_ERR_PARAM_RANGE (and cleared), while in-range Deltas report nothing.
"""
import pytest
import torch

import ssm_token_mixer_b200 as ia
from gpu_common import device
from ssm_token_mixer_b200 import synthetic

pytestmark = pytest.mark.gpu

IA_ERR_TIMEOUT, IA_ERR_PARAM_RANGE = 5, 6


def test_bounded_wait_expiry_reports_and_clears():
    dev = device()
    ia.check_device_errors()                       # start from a clear flag
    limit = 2_000_000                              # 2 ms
    out = ia.selftest_wait_expiry(limit, device=dev).cpu().tolist()
    with pytest.raises(ia.IAError) as err:
        ia.check_device_errors()
    assert err.value.status == IA_ERR_TIMEOUT
    ia.check_device_errors()                       # cleared: no error the second time
    done = out[0::2]
    waited = out[1::2]
    assert done == [0, 0, 0]                       # no barrier ever completed
    assert limit <= waited[0] < 200 * limit        # plain wait: expired after its limit
    assert limit <= waited[1] < 200 * limit        # abortable wait: expired and raised the abort flag
    assert waited[2] < 200 * limit < 10 ** 9       # full-limit wait: left on the abort, long before 1 s
    # the context is still usable
    x = torch.ones(4, device=dev)
    assert float((x * 2).sum()) == 8.0


@pytest.mark.parametrize("bad", [0.5, 2.0, -0.05])
def test_out_of_range_delta_is_reported(bad):
    dev = device()
    inp = synthetic.layer_inputs(1, 2, 130, 64, 64, "bf16", seed=7)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    ia.check_device_errors()
    ok = torch.tensor([0.1, 0.2], dtype=torch.float32, device=dev)
    ia.prefill_fwd(q, k, v, ok, 64)
    ia.check_device_errors()                       # in range: nothing reported
    delta = torch.tensor([0.05, bad], dtype=torch.float32, device=dev)
    ia.prefill_fwd(q, k, v, delta, 64)
    with pytest.raises(ia.IAError) as err:
        ia.check_device_errors()
    assert err.value.status == IA_ERR_PARAM_RANGE
    ia.check_device_errors()                       # cleared


def test_cuda_core_path_has_no_delta_limit():
    # fp32 inputs run the fp32 sequential kernel, which takes any Delta > 0
    dev = device()
    inp = synthetic.layer_inputs(1, 2, 40, 16, 16, "f32", seed=8)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    delta = torch.tensor([0.5, 2.0], dtype=torch.float32, device=dev)
    r = ia.prefill_fwd(q, k, v, delta, 16)
    ia.check_device_errors()
    assert torch.isfinite(r["o"]).all()
