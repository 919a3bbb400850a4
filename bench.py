#!/usr/bin/env python
"""Throughput of the IA layer hot path on B200, one JSON line on stdout.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one call of the layer over one batch of synthetic, seeded input
with the inputs already resident in HBM.  The headline value is the prefill
forward of the 125M-layer shape (B=8, H=12, N=2048, d_xi=d_v=64, M=64, bf16
inputs): every row of the forward path (parameter tables, feature map, chunk
Gram/decay contractions, carried-state reads, readout, chunk carries) runs in
each step.  The same line carries, as separate legs timed the same way, the
training step (forward + reverse mode, 350M-layer shape), the graphed decode
step (1.3B-layer shape, B = 1/16/64) and a long-context prefill (1.3B-layer
shape, B=1, N=7168) whose 16 sequences the planner splits into segments, so
its steps also run the state-only pass and the inter-segment carry scan.

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events
on the launching stream, with the L2 flushed (a 256 MB write) between steps
outside the events; a barrier and a device synchronise on both sides; the
max over ranks.  The dominant kernel of each leg is timed alone through the
library's launch events.  For N > 1 (torchrun) every rank runs the same
per-GPU workload with no data-path collective (weak scaling).

--impl reference times the fp64 CPU oracle (the only other implementation of
the method available here) on the host cores, on a bounded sample of the same
workload, and prints the same line with "impl": "reference".
"""
import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "IA layer tokens/s (fwd, fwd+bwd, decode) and % of tensor/HBM roofline on 1 B200"
CHUNK = 64
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------- algorithmic work
def flops_fwd(dx, dv, M):
    """Per token per head, as the chunkwise algorithm issues it with C = 64 tiles."""
    C = CHUNK
    return (2 * C * dx + 4 * C * M + 4 * M * dx + 4 * C * M + 2 * C * dv + 2 * C + 4 * M * dv
            + 4 * M + 4 * M * (dx + dv) + 4 * M)


def bytes_fwd(dx, dv, s_in=2):
    """Read q, k, v once and write o in fp32, per token per head."""
    return (2 * dx + dv) * s_in + 4 * dv


def bytes_fwd_bwd(dx, dv, s_in=2):
    return bytes_fwd(dx, dv, s_in) + (2 * dx + dv) * s_in + s_in * dv + 4 * dv + 4 * (2 * dx + dv)


def bytes_decode(dx, dv, M):
    """Per (b,h): read and write the fp32 complex state, read q, k, v, write o."""
    return 2 * 8 * M * (dx + dv + 1) + 2 * (2 * dx + dv) + 4 * dv


# ---------------------------------------------------------------- distributed helpers
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def shard_units(n_units, rank, world):
    """Contiguous share [lo, hi) of n_units for this rank (weak scaling uses the full n per rank)."""
    per = n_units // world
    extra = n_units % world
    lo = rank * per + min(rank, extra)
    return lo, lo + per + (1 if rank < extra else 0)


def max_over_ranks(x, device=None):
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def rank_workload(w, rank, world, scaling):
    """This rank's workload and the batch the whole job processes.  Weak
    scaling: every rank runs the full workload (its own batch of the same
    size); strong: the workload's batch is split over the ranks."""
    import dataclasses
    if scaling == "weak" or world == 1:
        return w, world * w.B
    if w.B < world:
        raise SystemExit(f"--scaling strong needs B >= ranks ({w.name}: B={w.B}, {world} ranks)")
    lo, hi = shard_units(w.B, rank, world)
    return dataclasses.replace(w, B=hi - lo), w.B


# ---------------------------------------------------------------- environment
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler(threading.Thread):
    """Samples SM clock and clock-event reasons through NVML every 5 ms."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks",
               0x10: "sync_boost"}

    def __init__(self, index):
        super().__init__(daemon=True)
        self.index = index
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._halt = threading.Event()
        self.ok = False

    def run(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            self.ok = True
            while not self._halt.is_set():
                self.samples.append(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                r = get_r(h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
                time.sleep(0.005)
        except Exception:   # NVML missing: report no clock data rather than failing the bench
            self.ok = False

    def stop(self):
        self._halt.set()
        self.join(timeout=2)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def recorded_traffic(profile_name, kernel_src):
    """dram bytes per launch from a committed ncu summary, if the kernel is unchanged since."""
    p = os.path.join(ROOT, "profiles", profile_name)
    if not os.path.exists(p):
        return None
    text = open(p).read()
    m = re.search(r"traffic_bytes_per_launch:\s*(\d+)", text)
    h = re.search(r"kernel_source_sha256:\s*([0-9a-f]{64})", text)
    if not m or not h:
        return None
    src = os.path.join(ROOT, kernel_src)
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != h.group(1):
        return None
    return int(m.group(1))


# ---------------------------------------------------------------- timing core
class Timer:
    def __init__(self, dev):
        import torch
        self.torch = torch
        self.dev = dev
        self.flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
        self.s = torch.cuda.Event(enable_timing=True)
        self.e = torch.cuda.Event(enable_timing=True)
        self.kb = torch.cuda.Event(enable_timing=True)
        self.ke = torch.cuda.Event(enable_timing=True)
        st = torch.cuda.current_stream()
        for ev in (self.kb, self.ke):   # create the underlying CUDA events
            ev.record(st)
        torch.cuda.synchronize()

    def flush(self):
        self.flush_buf.fill_(1)

    def run(self, fn, steps, warmup, kernel_events=True, flush=True):
        """Returns (list of step ms, list of dominant-kernel ms)."""
        import ssm_token_mixer_b200 as ia
        torch = self.torch
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        if kernel_events:
            ia.set_launch_events(self.kb, self.ke)
        steps_ms, kern_ms = [], []
        st = torch.cuda.current_stream()
        try:
            for _ in range(steps):
                if flush:
                    self.flush()
                self.s.record(st)
                fn()
                self.e.record(st)
                torch.cuda.synchronize()
                steps_ms.append(self.s.elapsed_time(self.e))
                if kernel_events:
                    kern_ms.append(self.kb.elapsed_time(self.ke))
        finally:
            if kernel_events:
                ia.set_launch_events()
        ia.check_device_errors()
        return steps_ms, kern_ms

    def run_batch(self, fn, steps, warmup):
        """K steps back to back between one pair of events (no per-step
        synchronize): for work whose inputs already exceed L2.  Returns the
        per-step ms list (the mean, K times)."""
        import ssm_token_mixer_b200 as ia
        torch = self.torch
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        st = torch.cuda.current_stream()
        self.s.record(st)
        for _ in range(steps):
            fn()
        self.e.record(st)
        torch.cuda.synchronize()
        ia.check_device_errors()
        t = self.s.elapsed_time(self.e)
        return [t / steps] * steps


def roofline(bytes_per_launch, flops_per_launch, kern_ms, peaks, peak_kind, traffic, sustained):
    hbm = float(peaks["hbm_gbs"])
    tc = float(peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"])
    t = statistics.mean(kern_ms) * 1e-3
    ai = flops_per_launch / bytes_per_launch
    ridge = tc * 1e12 / (hbm * 1e9)
    out = {"bound": "hbm" if ai < ridge else "tensor"}
    if out["bound"] == "hbm":
        ach = bytes_per_launch / t / 1e9
        out.update(achieved=ach, peak=hbm, unit="GB/s", frac=ach / hbm)
    else:
        ach = flops_per_launch / t / 1e12
        out.update(achieved=ach, peak=tc, unit="TFLOP/s", frac=ach / tc)
    out["traffic"] = traffic
    out["peak_source"] = f"{peak_kind} ({'sustained' if sustained else 'burst'} tensor peak for the ridge)"
    out["tensor_frac"] = flops_per_launch / t / (tc * 1e12)
    out["kernel_ms"] = statistics.mean(kern_ms)
    return out


def e2e_pipelined(torch, ia, dev, w, host_in, host_out, delta, ws, steps, warmup):
    """Total ms of `steps` prefills fed from pinned host memory (after `warmup`
    untimed ones): H2D of a step's q, k, v on one stream, the prefill on a
    second, D2H of its o on a third, two device buffers per side, events
    between them; timed from the first copy in to the last copy out."""
    qh, kh, vh = host_in
    cin, comp, cout = (torch.cuda.Stream(device=dev) for _ in range(3))
    bufs = [tuple(torch.empty(x.shape, dtype=x.dtype, device=dev) for x in host_in) for _ in range(2)]
    outs = [torch.empty(host_out[0].shape, dtype=torch.float32, device=dev) for _ in range(2)]
    ev = lambda: torch.cuda.Event()
    inputs_in = [ev(), ev()]     # set b's inputs have landed
    inputs_free = [ev(), ev()]   # the prefill that read set b is done
    out_ready = [ev(), ev()]     # o of set b is complete
    out_free = [ev(), ev()]      # o of set b has been copied out
    for e in inputs_free + out_free:
        e.record(comp)

    def run(n):
        for i in range(n):
            b = i % 2
            q, k, v = bufs[b]
            with torch.cuda.stream(cin):
                cin.wait_event(inputs_free[b])
                q.copy_(qh, non_blocking=True)
                k.copy_(kh, non_blocking=True)
                v.copy_(vh, non_blocking=True)
                inputs_in[b].record(cin)
            comp.wait_event(inputs_in[b])
            comp.wait_event(out_free[b])
            ia.prefill_fwd(q, k, v, delta, w.M, o=outs[b], workspace=ws, stream=comp)
            inputs_free[b].record(comp)
            out_ready[b].record(comp)
            with torch.cuda.stream(cout):
                cout.wait_event(out_ready[b])
                host_out[b].copy_(outs[b], non_blocking=True)
                out_free[b].record(cout)

    run(warmup)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(cin)
    run(steps)
    t1.record(cout)   # after the last copy out
    torch.cuda.synchronize()
    ia.check_device_errors()
    return t0.elapsed_time(t1)


# ---------------------------------------------------------------- legs
def leg_prefill(dev, w, steps, warmup, timer, peaks, peak_kind, rank, world, cpu_leg,
                profile="tc_prefill_d64_125m.md", job_B=None):
    """Prefill of one workload: step time, the chunk pass timed live, e2e, and
    the oracle on the full batch."""
    import torch
    import ssm_token_mixer_b200 as ia
    from ssm_token_mixer_b200 import synthetic
    inp = synthetic.workload_inputs(w)
    q, k, v, delta = (inp[n].to(dev) for n in ("q", "k", "v", "delta"))
    o = torch.empty(w.B, w.H, w.N, w.d_v, dtype=torch.float32, device=dev)
    need = ia.prefill_workspace_bytes(w.B, w.H, w.N, w.d_xi, w.d_v, w.M, "bf16")
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    fn = lambda: ia.prefill_fwd(q, k, v, delta, w.M, o=o, workspace=ws)
    barrier(dev)
    torch.cuda.synchronize()
    step_ms, kern_ms = timer.run(fn, steps, warmup)
    torch.cuda.synchronize()
    barrier(dev)
    total = max_over_ranks(sum(step_ms), dev)
    tokens = w.B * w.N
    job_tokens = (job_B or world * w.B) * w.N
    value = job_tokens * steps / (total * 1e-3)
    launches = ia.prefill_launches(w.B, w.H, w.N, w.d_xi, w.d_v, w.M, "bf16")
    fl = flops_fwd(w.d_xi, w.d_v, w.M) * tokens * w.H
    by = bytes_fwd(w.d_xi, w.d_v) * tokens * w.H
    traffic = recorded_traffic(profile, "ssm_token_mixer_b200/csrc/ia_prefill_tc.cu")
    rf = roofline(by, fl, kern_ms, peaks, peak_kind, traffic, sustained=False)
    # the chunk pass starts under the table kernel (programmatic dependent
    # launch), so its events bracket both: an upper bound on its time
    rf["kernel"] = "chunk pass, timed from the table kernel it overlaps"
    rf["launches_per_step"] = launches
    step_s = total / steps * 1e-3
    rf["step"] = {"achieved_gbs": by / step_s / 1e9, "frac_hbm": by / step_s / 1e9 / float(peaks["hbm_gbs"])}
    # end to end through the public API with host buffers: every step copies
    # its q, k, v in from pinned host memory, runs the prefill and copies o
    # out, as a stream of batches would: the input copy of step i+1 and the
    # output copy of step i-1 run on their own streams (the two copy engines)
    # while step i computes, with two device buffers for each side
    qh, kh, vh = (x.pin_memory() for x in (inp["q"], inp["k"], inp["v"]))
    ohs = [torch.empty(o.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    e2e_total = max_over_ranks(e2e_pipelined(torch, ia, dev, w, (qh, kh, vh), ohs, delta, ws, steps, warmup), dev)
    res = {
        "workload": f"{w.name} (B{w.B} H{w.H} N{w.N} d_xi{w.d_xi} d_v{w.d_v} M{w.M}, bf16 inputs)",
        "value": value, "unit": "tokens/s", "ms_per_step": total / steps, "roofline": rf,
        "launches_per_step": launches, "gpu_launches": launches * steps,
        "e2e": {"value": job_tokens * steps / (e2e_total * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(sum(x.numel() * x.element_size() for x in (qh, kh, vh))),
                "d2h_bytes_per_step": int(ohs[0].numel() * 4),
                "schedule": "copies in and out overlapped with the neighbouring steps' compute (two buffers)"},
        "algorithmic": {"flops": fl, "bytes": by},
    }
    if cpu_leg and rank == 0 and world == 1:
        import oracle
        t0 = time.perf_counter()
        oracle.forward(inp["q"], inp["k"], inp["v"], inp["delta"], w.M, want_state=False)
        dt = time.perf_counter() - t0
        res["cpu_baseline"] = {"value": tokens / dt, "unit": "tokens/s", "cores": oracle.num_threads(),
                               "kind": "oracle",
                               "sample": f"full {w.name} batch (B{w.B} H{w.H} N{w.N}), one pass, fp64 "
                                         f"sequential recurrence, OpenMP over (b,h), {dt:.1f} s"}
    return res


def leg_prefill_long(dev, w, steps, warmup, timer, peaks, peak_kind, rank, world):
    """Long-context prefill of few sequences: the planner splits them into
    segments, so a step runs the table prologue, the state-only pass, the
    carry scan and the full chunk pass (the dominant kernel, timed live)."""
    import torch
    import ssm_token_mixer_b200 as ia
    from ssm_token_mixer_b200 import synthetic
    inp = synthetic.workload_inputs(w)
    q, k, v, delta = (inp[n].to(dev) for n in ("q", "k", "v", "delta"))
    o = torch.empty(w.B, w.H, w.N, w.d_v, dtype=torch.float32, device=dev)
    need = ia.prefill_workspace_bytes(w.B, w.H, w.N, w.d_xi, w.d_v, w.M, "bf16")
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    fn = lambda: ia.prefill_fwd(q, k, v, delta, w.M, o=o, workspace=ws)
    barrier(dev)
    step_ms, kern_ms = timer.run(fn, steps, warmup)
    barrier(dev)
    total = max_over_ranks(sum(step_ms), dev)
    tokens = w.B * w.N
    launches = ia.prefill_launches(w.B, w.H, w.N, w.d_xi, w.d_v, w.M, "bf16")
    fl = flops_fwd(w.d_xi, w.d_v, w.M) * tokens * w.H
    by = bytes_fwd(w.d_xi, w.d_v) * tokens * w.H
    traffic = recorded_traffic("tc_prefill_1p3b_7168.md", "ssm_token_mixer_b200/csrc/ia_prefill_tc.cu")
    rf = roofline(by, fl, kern_ms, peaks, peak_kind, traffic, sustained=False)
    rf["kernel"] = "chunk pass over 148 ranges with their state-only chains and look-back, timed from the table kernel it overlaps"
    step_s = total / steps * 1e-3
    rf["step"] = {"achieved_gbs": by / step_s / 1e9, "frac_hbm": by / step_s / 1e9 / float(peaks["hbm_gbs"])}
    return {"workload": f"{w.name} (B{w.B} H{w.H} N{w.N} d_xi{w.d_xi} d_v{w.d_v} M{w.M}, bf16 inputs)",
            "value": world * tokens * steps / (total * 1e-3), "unit": "tokens/s",
            "ms_per_step": total / steps, "steps": steps, "launches_per_step": launches,
            "gpu_launches": launches * steps, "roofline": rf}


def leg_fwd_bwd(dev, w, steps, warmup, timer, peaks, peak_kind, rank, world, cpu_leg, job_B=None):
    """Training step; with several ranks each step ends with the all-reduce
    of dDelta over NCCL (the one exchange data-parallel training needs)."""
    import torch
    import ssm_token_mixer_b200 as ia
    from ssm_token_mixer_b200 import parallel, synthetic
    inp = synthetic.workload_inputs(w)
    d = {n: inp[n].to(dev) for n in ("q", "k", "v", "delta", "dO")}
    need = ia.fwd_bwd_workspace_bytes(w.B, w.H, w.N, w.d_xi, w.d_v, w.M, "bf16")
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    fn = lambda: parallel.fwd_bwd_sharded(d["q"], d["k"], d["v"], d["delta"], d["dO"], w.M, workspace=ws)
    barrier(dev)
    step_ms, kern_ms = timer.run(fn, steps, warmup)
    barrier(dev)
    total = max_over_ranks(sum(step_ms), dev)
    tokens = w.B * w.N
    # the dominant kernel is the reverse pass: its own algorithmic work is the
    # step's minus the forward's (re-read q, k, v; read dO, o; write dq, dk, dv;
    # two forward-sized contraction chains by the convention of 3x forward flops)
    fl_step = 3 * flops_fwd(w.d_xi, w.d_v, w.M) * tokens * w.H
    by_step = bytes_fwd_bwd(w.d_xi, w.d_v) * tokens * w.H
    fl = 2 * flops_fwd(w.d_xi, w.d_v, w.M) * tokens * w.H
    by = (bytes_fwd_bwd(w.d_xi, w.d_v) - bytes_fwd(w.d_xi, w.d_v)) * tokens * w.H
    traffic = recorded_traffic("tc_bwd_350m.md", "ssm_token_mixer_b200/csrc/ia_bwd_tc.cu")
    rf = roofline(by, fl, kern_ms, peaks, peak_kind, traffic, sustained=False)
    rf["kernel"] = "reverse pass (tc_bwd_kernel)"
    step_s = total / steps * 1e-3
    rf["step"] = {"algorithmic_bytes": by_step, "algorithmic_flops": fl_step,
                  "achieved_gbs": by_step / step_s / 1e9, "frac_hbm": by_step / step_s / 1e9 / float(peaks["hbm_gbs"])}
    launches = ia.prefill_launches(w.B, w.H, w.N, w.d_xi, w.d_v, w.M, "bf16") + 1
    res = {"workload": f"{w.name} (B{w.B} H{w.H} N{w.N} d_xi{w.d_xi} d_v{w.d_v} M{w.M}, bf16 inputs)",
           "value": (job_B or world * w.B) * w.N * steps / (total * 1e-3), "unit": "tokens/s",
           "ms_per_step": total / steps, "steps": steps, "gpu_launches": launches * steps,
           "roofline": rf}
    if cpu_leg and rank == 0 and world == 1:
        import oracle
        sub = synthetic.workload_inputs(w, B=1)
        t0 = time.perf_counter()
        oracle.backward(sub["q"], sub["k"], sub["v"], sub["delta"], sub["dO"], w.M)
        dt = time.perf_counter() - t0
        res["cpu_baseline"] = {"value": w.N / dt, "unit": "tokens/s", "cores": oracle.num_threads(),
                               "kind": "oracle", "sample": f"batch element 0 of {w.name} (H{w.H} N{w.N}), "
                                                           f"forward + reverse mode, {dt:.1f} s"}
    return res


def leg_decode(dev, w, steps, warmup, timer, peaks, peak_kind, rank, world, cpu_leg):
    import torch
    import ssm_token_mixer_b200 as ia
    from ssm_token_mixer_b200 import synthetic
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    out = {"workload": f"{w.name} (H{w.H} d_xi{w.d_xi} d_v{w.d_v} M{w.M}, bf16 q/k/v, fp32 state, "
                       f"state after a 7168-token prefill)", "unit": "tokens/s", "batches": {}}
    for B in w.decode_batches:
        sb = ia.state_bytes(B, w.H, w.M, w.d_xi, w.d_v)
        R = max(2, math.ceil(4 * l2 / sb))
        # prefix state: GPU prefill of 7168 seeded random tokens at this batch
        g = torch.Generator(device=dev).manual_seed(w.seed)
        Np = 7168
        qp = torch.randn(B, w.H, Np, w.d_xi, device=dev, generator=g).bfloat16()
        kp = torch.randn(B, w.H, Np, w.d_xi, device=dev, generator=g).bfloat16()
        vp = torch.randn(B, w.H, Np, w.d_v, device=dev, generator=g).bfloat16()
        delta = synthetic.make_delta(w.H, torch.Generator().manual_seed(w.seed)).to(dev)
        pre = ia.prefill_fwd(qp, kp, vp, delta, w.M, want_state=True)
        del qp, kp, vp
        states = [pre["state"].clone() for _ in range(R)]
        toks = [tuple(x.to(dev) for x in synthetic.decode_token(B, w.H, w.d_xi, w.d_v, "bf16", step=i))
                for i in range(steps)]
        o = torch.empty(B, w.H, w.d_v, dtype=torch.float32, device=dev)
        # the K timed steps captured in one CUDA graph, each step with its own
        # inputs and state replica: kernel after kernel inside a graph, as a
        # layer's decode kernel runs inside a per-token graph of a whole model;
        # for comparison the same steps as K graphs of one step each
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for i in range(3):   # warm-up outside capture
                ia.decode_step(*toks[i % len(toks)], delta, states[i % R], w.M, o=o, stream=s)
        torch.cuda.current_stream().wait_stream(s)
        loop = torch.cuda.CUDAGraph()
        with torch.cuda.graph(loop, stream=s):
            for i in range(steps):
                ia.decode_step(*toks[i], delta, states[i % R], w.M, o=o, stream=s)
        graphs = []
        for i in range(steps):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=s):
                ia.decode_step(*toks[i], delta, states[i % R], w.M, o=o, stream=s)
            graphs.append(gr)
        torch.cuda.synchronize()
        it = iter(range(10 ** 9))
        fn = lambda: graphs[next(it) % steps].replay()
        barrier(dev)
        # the K steps run back to back (a decode loop); the state replicas
        # rotate through more than L2, so no flush is needed between them.
        # Warm-up: W replays of the K-step graph.
        t_loop = timer.run_batch(loop.replay, 1, max(1, warmup))[0]
        step_ms = [t_loop / steps] * steps
        per_graph_ms = timer.run_batch(fn, steps, warmup)
        barrier(dev)
        total = max_over_ranks(sum(step_ms), dev)
        by = bytes_decode(w.d_xi, w.d_v, w.M) * B * w.H
        rf = roofline(by, 2 * by, step_ms, peaks, peak_kind, None, sustained=False)
        rf["bound"] = "hbm"
        rf["achieved"] = by / (statistics.mean(step_ms) * 1e-3) / 1e9
        rf["unit"] = "GB/s"
        rf["peak"] = float(peaks["hbm_gbs"])
        rf["frac"] = rf["achieved"] / rf["peak"]
        rf.pop("tensor_frac", None)
        rf["note"] = (f"the K steps in one captured graph, between two events (kernel only); "
                      f"{R} state replicas rotate so each step reads HBM")
        entry = {"value": world * B * steps / (total * 1e-3), "ms_per_step": total / steps,
                 "ms_per_step_one_graph_per_step": statistics.mean(per_graph_ms),
                 "roofline": rf, "gpu_launches": steps}
        # end to end with host buffers (no graph): H2D q,k,v, step, D2H o
        hq = [tuple(x.pin_memory() for x in synthetic.decode_token(B, w.H, w.d_xi, w.d_v, "bf16", step=i))
              for i in range(steps)]
        oh = torch.empty(o.shape, dtype=torch.float32).pin_memory()
        dq, dk, dvv = (torch.empty_like(x) for x in toks[0])
        it2 = iter(range(10 ** 9))

        def e2e():
            i = next(it2) % steps
            dq.copy_(hq[i][0], non_blocking=True)
            dk.copy_(hq[i][1], non_blocking=True)
            dvv.copy_(hq[i][2], non_blocking=True)
            ia.decode_step(dq, dk, dvv, delta, states[i % R], w.M, o=o)
            oh.copy_(o, non_blocking=True)

        e2e_ms, _ = timer.run(e2e, steps, warmup, kernel_events=False, flush=False)
        e2e_total = max_over_ranks(sum(e2e_ms), dev)
        entry["e2e"] = {"value": world * B * steps / (e2e_total * 1e-3), "unit": "tokens/s",
                        "h2d_bytes_per_step": int(sum(x.numel() * x.element_size() for x in hq[0])),
                        "d2h_bytes_per_step": int(oh.numel() * 4)}
        out["batches"][str(B)] = entry
        del graphs, loop, states, pre
        torch.cuda.empty_cache()
    if cpu_leg and rank == 0 and world == 1:
        import numpy as np
        import oracle
        B = max(w.decode_batches)
        st = np.zeros(oracle.state_len(B, w.H, w.M, w.d_xi, w.d_v))
        delta = synthetic.make_delta(w.H, __import__("torch").Generator().manual_seed(w.seed))
        t0 = time.perf_counter()
        n = 3
        for i in range(n):
            q, k, v = synthetic.decode_token(B, w.H, w.d_xi, w.d_v, "bf16", step=i)
            _, _, _, st = oracle.decode_step(q, k, v, delta, w.M, st)
        dt = time.perf_counter() - t0
        out["cpu_baseline"] = {"value": B * n / dt, "unit": "tokens/s", "cores": oracle.num_threads(),
                               "kind": "oracle", "sample": f"{n} decode steps at B={B}, {dt:.2f} s"}
    return out


def leg_optional_parts(dev, w, steps, warmup, timer, peaks, peak_kind, rank, world):
    """The layer's optional parts (RMSNorm on the SSM input, a step per token,
    the complex readout matrix, the bidirectional layer) through
    ia_prefill_fwd_ex on the same workload: the tensor-core chunk pass where
    the parts allow it, else the token-serial CUDA-core kernel over segments
    of each sequence in two passes around a carry.  Each part is timed alone
    and some together."""
    import torch
    import ssm_token_mixer_b200 as ia
    from ssm_token_mixer_b200 import synthetic
    inp = synthetic.workload_inputs(w)
    q, k, v, delta = (inp[n].to(dev) for n in ("q", "k", "v", "delta"))
    g = torch.Generator().manual_seed(w.seed + 500)
    D = w.d_xi + w.d_v
    parts = {
        "selective": {"delta_t": torch.exp(math.log(5e-3) + torch.rand(w.B, w.H, w.N, generator=g) *
                                           (math.log(1e-1) - math.log(5e-3))).to(dev)},
        "norm": {"gain": (0.5 + torch.rand(w.H, D, generator=g)).to(dev),
                 "bias": (0.3 * torch.randn(w.H, D, generator=g)).to(dev)},
        "readout": {"W": (torch.randn(w.H, w.M, w.M, 2, generator=g) / math.sqrt(w.M)).to(dev)},
        "bidirectional": {"bidirectional": True},
    }
    parts["norm+bidirectional"] = {**parts["norm"], **parts["bidirectional"]}
    parts["all"] = {**parts["selective"], **parts["norm"], **parts["readout"]}
    tokens = w.B * w.N
    by = bytes_fwd(w.d_xi, w.d_v) * tokens * w.H
    out = {"workload": f"{w.name} (B{w.B} H{w.H} N{w.N} d_xi{w.d_xi} d_v{w.d_v} M{w.M}, bf16 inputs)",
           "unit": "tokens/s",
           "kernel": "ia_prefill_fwd_ex: the tensor-core chunk pass with a prologue (and, bidirectional, a "
                     "second pass and an epilogue) where the parts allow it, else the token-serial CUDA-core "
                     "layer; `path` per part", "parts": {}}
    for name, kw in parts.items():
        d = None if "delta_t" in kw else delta
        present = dict(norm="gain" in kw, selective="delta_t" in kw, readout="W" in kw,
                       bidirectional=bool(kw.get("bidirectional")))
        path = ia.prefill_ex_path(w.B, w.H, w.N, w.d_xi, w.d_v, w.M, "bf16", **present)
        need = ia.prefill_ex_workspace_bytes(w.B, w.H, w.N, w.d_xi, w.d_v, w.M, "bf16", **present)
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev) if need else None
        o = torch.empty(w.B, w.H, w.N, w.d_v, dtype=torch.float32, device=dev)
        fn = lambda: ia.prefill_fwd_ex(q, k, v, w.M, delta=d, workspace=ws, o=o, **kw)
        barrier(dev)
        step_ms, kern_ms = timer.run(fn, steps, warmup)
        barrier(dev)
        total = max_over_ranks(sum(step_ms), dev)
        passes = 2 if kw.get("bidirectional") else 1
        rf = roofline(by * passes, flops_fwd(w.d_xi, w.d_v, w.M) * tokens * w.H * passes, kern_ms, peaks,
                      peak_kind, None, sustained=False)
        # tensor cores: the prologue, the W' conversion, a table kernel and a chunk pass per direction,
        # the epilogue; token-serial: one pass per direction, or pass 1, the carry (past two segments)
        # and pass 2
        nseg = ia.prefill_ex_segments(w.B, w.H, w.N, w.d_xi, w.d_v, w.M, "bf16", need, **present)
        launches = ((1 if present["norm"] or present["bidirectional"] else 0) + (1 if present["readout"] else 0) +
                    passes * 2 + (1 if present["bidirectional"] else 0)) if path == "tensor_core" else \
            passes * (1 if nseg == 1 else 2 if nseg == 2 else 3)
        out["parts"][name] = {"value": world * tokens * steps / (total * 1e-3), "ms_per_step": total / steps,
                              "path": path, "segments": nseg, "roofline": rf, "gpu_launches": launches * steps}
    return out


def workload_config(w, scaling="weak"):
    """The JSON line's config: the workload and how it is timed (both arms)."""
    return {"workload": f"{w.name} prefill (B{w.B} H{w.H} N{w.N} d_xi{w.d_xi} d_v{w.d_v} M{w.M}, "
                        f"bf16 inputs, fp32 state/output)",
            "l2": "flushed (256 MB write) between timed steps",
            "per_gpu": "each rank runs the full workload (weak scaling)" if scaling == "weak" else
                       "the batch is split over the ranks (strong scaling); decode and the long prefill "
                       "stay per rank"}


# ---------------------------------------------------------------- reference arm (oracle)
def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    from ssm_token_mixer_b200 import synthetic
    from ssm_token_mixer_b200.workloads import WORKLOADS
    w = WORKLOADS[args.workload]
    inp = synthetic.workload_inputs(w)          # the full batch per step, as the GPU arm
    ms = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle.forward(inp["q"], inp["k"], inp["v"], inp["delta"], w.M, want_state=False)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            ms.append(dt * 1e3)
    value = w.B * w.N * len(ms) / (sum(ms) * 1e-3)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(ms),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"full {w.name} batch (B{w.B} H{w.H} N{w.N}) per step, fp64 sequential "
                                   f"recurrence, OpenMP over the (b,h) sequences on the host cores"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ---------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--legs", default="prefill,prefill_1p3b,fwd_bwd,decode,prefill_long,optional_parts",
                    help="comma list of legs to run (prefill is the headline)")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--workload", default="prefill_125m", help="headline prefill workload")
    ap.add_argument("--scaling", choices=["weak", "strong"], default="weak",
                    help="weak: every rank runs the full batch; strong: the batch is split over the ranks")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist
    rank, world, local = dist_env()
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from ssm_token_mixer_b200 import build
    from ssm_token_mixer_b200.workloads import WORKLOADS
    if rank == 0:
        build.build()
    barrier(dev)
    peaks, peak_kind = load_peaks()
    timer = Timer(dev)
    legs = [x for x in args.legs.split(",") if x]
    clocks = ClockSampler(dev.index)
    clocks.start()
    w = WORKLOADS[args.workload]
    line = {"metric": METRIC, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": args.scaling, "vs_baseline": None,
            "dtype": "f16xf16->f32 (bf16 inputs)", "data": "synthetic (seeded N(0,1) q/k/v, log-uniform Delta)",
            "config": workload_config(w, args.scaling)}
    w_loc, job_B = rank_workload(w, rank, world, args.scaling)
    cpu = not args.no_cpu
    try:
        if "prefill" in legs:
            r = leg_prefill(dev, w_loc, args.steps, args.warmup, timer, peaks, peak_kind, rank, world, cpu,
                            job_B=job_B)
            line.update(value=r["value"], ms_per_step=r["ms_per_step"], roofline=r["roofline"],
                        e2e=r["e2e"], gpu_launches=r["gpu_launches"])
            if "cpu_baseline" in r:
                line["cpu_baseline"] = r["cpu_baseline"]
            line["algorithmic_per_step"] = r["algorithmic"]
        extra_launches = 0
        if "prefill_1p3b" in legs:
            wl, jb = rank_workload(WORKLOADS["prefill_1p3b"], rank, world, args.scaling)
            r = leg_prefill(dev, wl, args.steps, args.warmup, timer, peaks, peak_kind,
                            rank, world, cpu, profile="tc_prefill_1p3b.md", job_B=jb)
            r.pop("algorithmic", None)
            line["prefill_1p3b"] = r
            extra_launches += r["gpu_launches"]
        if "fwd_bwd" in legs:
            wl, jb = rank_workload(WORKLOADS["train_350m"], rank, world, args.scaling)
            r = leg_fwd_bwd(dev, wl, args.steps, args.warmup, timer, peaks, peak_kind,
                            rank, world, cpu, job_B=jb)
            line["fwd_bwd"] = r
            extra_launches += r["gpu_launches"]
        if "decode" in legs:
            r = leg_decode(dev, WORKLOADS["decode_1p3b"], args.steps, args.warmup, timer, peaks, peak_kind,
                           rank, world, cpu)
            line["decode"] = r
        if "prefill_long" in legs:
            r = leg_prefill_long(dev, WORKLOADS["prefill_1p3b_7168"], args.steps, args.warmup, timer, peaks,
                                 peak_kind, rank, world)
            line["prefill_long"] = r
            extra_launches += r["gpu_launches"]
        if "optional_parts" in legs:
            r = leg_optional_parts(dev, WORKLOADS["prefill_125m"], min(args.steps, 3), 3, timer, peaks,
                                   peak_kind, rank, world)
            line["optional_parts"] = r
            extra_launches += sum(p["gpu_launches"] for p in r["parts"].values())
        line["gpu_launches_all_legs"] = line.get("gpu_launches", 0) + extra_launches + sum(
            b["gpu_launches"] for b in line.get("decode", {}).get("batches", {}).values())
    finally:
        line["clocks"] = clocks.stop()
    if "value" not in line:
        line["value"] = None
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
