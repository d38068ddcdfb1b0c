"""Host arithmetic of bench.py (CPU): the FLOP model, the step's branch-layer count, the
throughput formula, the clock and power record, and the traffic record's source check.

The FLOP figures are pinned to the algorithmic work of the 1024^2 workload: per branch-block
GEMMs 2 (4 D^2 + 3 D F) N and attention 4 N^2 D, 83 branch-blocks per step when layer 22 is
skipped on the unconditional branch (84 on step 0, outside the skip window [0.01, 1.0])."""
import hashlib
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_flop_model_1024():
    N, D, F = 4608, 3072, 8192
    fl = bench.flops_per_branch_layer(N)
    gemm = fl["gemm_qkv"] + fl["gemm_oproj"] + fl["gemm_gateup"] + fl["gemm_down"]
    assert gemm == pytest.approx(2 * (4 * D * D + 3 * D * F) * N, rel=1e-12)
    assert gemm == pytest.approx(1.0437e12, rel=1e-4)
    assert fl["attention"] == pytest.approx(2.609e11, rel=1e-3)
    per_step = 83 * (gemm + fl["attention"])
    assert per_step == pytest.approx(1.0828e14, rel=1e-4)


def test_branch_layers_follow_skip_window():
    # step 0 (p = 0) is outside [0.01, 1.0]: both branches run all 42 layers
    assert bench.step_branch_layers(0) == 84
    for step in (1, 25, 49):
        assert bench.step_branch_layers(step) == 83


def test_job_throughput_counts_all_ranks():
    # 50 steps, 2 forwards each, on 4 ranks in 5 s of device time -> 80 forwards/s
    out = bench.job_throughput(50, 4, 5000.0)
    value = out[0] if isinstance(out, tuple) else out
    assert value == pytest.approx(80.0)


def test_clock_summary_with_power():
    c = bench.ClockSampler(0)
    c.lines = ["1410, 1965, 998.5, Not Active, Not Active, Not Active, Active",
               "1430, 1965, 990.0, Not Active, Not Active, Not Active, Active",
               "1420, 1965, 980.0, Not Active, Not Active, Not Active, Not Active",
               "garbage line"]
    s = c.summary()
    assert s["sm_mhz"] == 1420
    assert s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]
    assert s["samples"] == 3
    assert s["power_w"] == pytest.approx(990.0)


def test_clock_summary_empty():
    c = bench.ClockSampler(0)
    assert c.summary() is None


def test_traffic_record_checks_its_sources(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel source v1\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    digest = hashlib.sha256(b"kernel source v1\n").hexdigest()
    rec = {"k": {"dram_bytes_per_launch": 12345, "sources": ["k.cu"], "source_sha256": digest}}
    (prof / "kernel_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_traffic("k") == 12345
    assert bench.kernel_traffic("missing") is None
    src.write_text("kernel source v2\n")  # the kernel changed since the counters were taken
    assert bench.kernel_traffic("k") is None


def test_committed_traffic_records_are_well_formed():
    recs = json.load(open(os.path.join(ROOT, "profiles", "kernel_traffic.json")))
    for name, rec in recs.items():
        if name.startswith("_"):
            continue
        assert rec["dram_bytes_per_launch"] > 0
        assert all(os.path.exists(os.path.join(ROOT, f)) for f in rec["sources"])
        assert os.path.exists(os.path.join(ROOT, rec["summary"]))


def test_reference_arm_line_names_its_extrapolation(capsys):
    """bench.py --impl reference: the oracle on one branch-block per timed step, the JSON line says
    that the step figure is extrapolated and what was timed."""
    import argparse
    import json

    bench.run_reference(argparse.Namespace(steps=1, warmup=0, gpus=1))
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["extrapolated"] is True
    assert line["steps"] == 1 and line["warmup"] == 0
    assert "branch-block" in line["timed_per_step"] and line["dtype"] == "f64"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["value"] > 0 and line["e2e"]["value"] == line["value"]
