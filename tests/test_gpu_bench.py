"""The end-to-end measurement of bench.py on the GPU: the stream of batches
whose copies in and out overlap the neighbouring steps' compute must still
hand every step's full output back to the host."""
import pytest
import torch

import bench
import ssm_token_mixer_b200 as ia
from gpu_common import device
from ssm_token_mixer_b200 import synthetic
from ssm_token_mixer_b200.workloads import Workload

pytestmark = pytest.mark.gpu


def test_pipelined_end_to_end_returns_each_steps_output():
    dev = device()
    w = Workload("e2e_check", 2, 3, 333, 64, 64, 64, "bf16", 77)
    inp = synthetic.workload_inputs(w)
    delta = inp["delta"].to(dev)
    need = ia.prefill_workspace_bytes(w.B, w.H, w.N, w.d_xi, w.d_v, w.M, "bf16")
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    host_in = tuple(inp[n].pin_memory() for n in ("q", "k", "v"))
    host_out = [torch.full((w.B, w.H, w.N, w.d_v), float("nan")).pin_memory() for _ in range(2)]
    ms = bench.e2e_pipelined(torch, ia, dev, w, host_in, host_out, delta, ws, steps=5, warmup=3)
    assert ms > 0
    ref = ia.prefill_fwd(*(x.to(dev) for x in host_in), delta, w.M)["o"].cpu()
    for out in host_out:   # both buffers hold a completed step's o
        assert torch.equal(out, ref)
