"""Host-side checks of bench.py's measurement arithmetic (no GPU).

The algorithmic work per token per head is fixed by the chunkwise algorithm
with C = 64 tiles; the expected constants below are the worked values for the
125M (d = 64) and 1.3B (d = 128) layer shapes with M = 64 modes."""
import hashlib
import os

import pytest

import bench


@pytest.mark.parametrize("d,flops,bytes_fwd,bytes_train", [
    (64, 115_328, 640, 2_176),
    (128, 197_248, 1_280, None),
])
def test_algorithmic_work_per_token_head(d, flops, bytes_fwd, bytes_train):
    assert bench.flops_fwd(d, d, 64) == flops
    assert bench.bytes_fwd(d, d) == bytes_fwd
    if bytes_train is not None:
        assert bench.bytes_fwd_bwd(d, d) == bytes_train


def test_decode_bytes_per_head():
    # read + write of the complex fp32 state (U, Gamma, eta), q, k, v in bf16, o in fp32
    state = 8 * 64 * (128 + 128 + 1)
    assert bench.bytes_decode(128, 128, 64) == 2 * state + 2 * (2 * 128 + 128) + 4 * 128


def test_roofline_picks_the_binding_resource():
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 100.0, "bf16_tflops_sustained": 80.0}
    # 1 GB moved with little arithmetic in 2 ms: memory-bound at 500 GB/s
    r = bench.roofline(1e9, 1e9, [2.0, 2.0], peaks, "test", None, sustained=False)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(500.0) and r["frac"] == pytest.approx(0.5)
    # arithmetic intensity above the ridge (100e12 / 1000e9 = 100 flop/B): tensor-bound
    r = bench.roofline(1e6, 1e12, [20.0], peaks, "test", 123, sustained=True)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(50.0) and r["frac"] == pytest.approx(50.0 / 80.0)
    assert r["traffic"] == 123 and r["kernel_ms"] == pytest.approx(20.0)


def test_recorded_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("// kernel\n")
    digest = hashlib.sha256(src.read_bytes()).hexdigest()
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "k.md").write_text(
        "kernel_source_sha256: %s\ntraffic_bytes_per_launch: 4242\n" % digest)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("k.md", "kernel.cu") == 4242
    src.write_text("// kernel, changed since the capture\n")
    assert bench.recorded_traffic("k.md", "kernel.cu") is None
    assert bench.recorded_traffic("missing.md", "kernel.cu") is None


def test_reference_arm_reports_the_gpu_arms_config(capsys, monkeypatch):
    # the oracle arm times one batch element per step on the host cores and
    # labels its line with the same workload config as the GPU arm
    import argparse
    import json
    from ssm_token_mixer_b200.workloads import WORKLOADS
    monkeypatch.delenv("RANK", raising=False)
    args = argparse.Namespace(steps=1, warmup=0, gpus=1, workload="prefill_125m")
    assert bench.run_reference(args) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["config"] == bench.workload_config(WORKLOADS["prefill_125m"])
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["e2e"]["value"] == line["value"] == line["cpu_baseline"]["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1


def test_rank_workload_weak_and_strong():
    import bench
    from ssm_token_mixer_b200.workloads import WORKLOADS
    w = WORKLOADS["prefill_125m"]
    assert bench.rank_workload(w, 0, 1, "strong") == (w, 8)
    assert bench.rank_workload(w, 1, 4, "weak") == (w, 32)          # every rank: the full batch of 8
    parts = [bench.rank_workload(w, r, 3, "strong") for r in range(3)]
    assert [p[0].B for p in parts] == [3, 3, 2] and {p[1] for p in parts} == {8}
    with pytest.raises(SystemExit):
        bench.rank_workload(WORKLOADS["prefill_1p3b_7168"], 0, 2, "strong")   # B = 1 cannot split
