"""Host-side logic of bench.py (no GPU): roofline selection, the traffic lookup's gating, the
configuration record of sweeps and the throughput arithmetic."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from free_block_sparse_02_b200 import configs  # noqa: E402

PEAKS = {"hbm_gbs": 6557.4, "bf16_tflops": 1629.0, "bf16_tflops_sustained": 1374.6}


def test_assignment_roofline_is_the_binding_one():
    """13B-DiT layer: 4 C_p d = 65,536 flops (two bf16 terms of W) and 2d + 4 = 260 bytes per
    key, so the tensor time (flops / peak) exceeds the HBM time; the mid-size shape (d = 64,
    C_p = 64) is HBM-bound."""
    big = bench.km_rooflines(configs.workload(2), 0.378, 0.244, PEAKS)
    assert big["assignment"]["bound"] == "tensor" and big["assignment"]["unit"] == "TFLOP/s"
    assert big["assignment"]["other"]["unit"] == "GB/s"
    keys = 24 * 118800
    assert big["assignment"]["achieved"] == pytest.approx(keys * 4 * 128 * 128 / 0.378e-3 / 1e12)
    assert big["update"]["bound"] == "hbm"
    assert big["update"]["achieved"] == pytest.approx(keys * 260 / 0.244e-3 / 1e9)
    mid = bench.km_rooflines(configs.workload(1), 0.0205, 0.0246, PEAKS)
    assert mid["assignment"]["bound"] == "hbm"
    assert bench.km_rooflines(configs.workload(1), 0.0, 0.0, PEAKS) == {}


def test_whole_loop_kmeans_is_reported_per_iteration():
    """Mid-size call, key side as one launch of 24 iterations in 0.5 ms: time per iteration,
    and the scoring's tensor flops (4 C_p d per key per iteration) against the sustained peak."""
    w = configs.workload(1)
    r = bench.km_loop_roofline(w, 0.5, [16, 24, 15], PEAKS)["loop"]
    assert r["bound"] == "latency" and r["iterations"] == 24
    assert r["ms_per_iteration"] == pytest.approx(0.5 / 24)
    keys = 8 * 16384
    assert r["tensor"]["achieved"] == pytest.approx(keys * 4 * 64 * 64 * 24 / 0.5e-3 / 1e12)
    assert r["tensor"]["peak"] == PEAKS["bf16_tflops_sustained"]
    assert r["hbm_bytes"] == keys * 2 * 64  # the keys are read from HBM once per call


def test_profiled_traffic_is_only_reported_for_the_profiled_configuration():
    w = configs.workload(1)
    assert bench.profiled_traffic(w.replace(P=64)) is None
    assert bench.profiled_traffic(configs.scaled_down(w, heads=2)) is None
    assert bench.profiled_traffic(configs.workload(0)) is None  # no profile of the tiny call


def test_sweep_settings_are_recorded_in_the_config():
    w = configs.workload(1).replace(probe_mode=configs.PROBE_RANDOM, correction=configs.CORRECTION_MEAN,
                                    trunc_rank=8, lam=1.0, recipe="field")
    c = bench.workload_config(w)
    assert c["probes"] == "random" and c["correction"] == "mean" and c["trunc_rank"] == 8 and c["lam"] == 1.0
    assert c["generator"].startswith("smooth random field")
    assert bench.workload_config(configs.workload(2))["generator"].endswith("+ 3D RoPE")


def test_whole_job_throughput_counts_every_rank():
    flops = configs.workload(1).dense_flops()
    one = bench.whole_job_tflops(1, flops, 3.2)
    assert one == pytest.approx(flops / 3.2e-3 / 1e12)
    assert bench.whole_job_tflops(4, flops, 3.2) == pytest.approx(4 * one)


def test_source_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    a = "// header\nint f(int x) {  /* twice */\n  return 2 * x;  // doubled\n}\n"
    b = "int f(int x) {\n\n  return 2 * x;\n}\n/* a new note\n spanning lines */\n"
    c = "int f(int x) {\n  return 3 * x;\n}\n"
    for name, text in (("a.cu", a), ("b.cu", b), ("c.cu", c)):
        (tmp_path / name).write_text(text)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.source_hash("a.cu") == bench.source_hash("b.cu")
    assert bench.source_hash("a.cu") != bench.source_hash("c.cu")


def test_attention_flops_count_the_probe_rows():
    w = configs.workload(2)
    pairs = 69_700_000_000
    assert bench.attention_flops(w, pairs) == pytest.approx(4 * 128 * (pairs + 24 * 512 * 118800))
    assert bench.attention_flops(w.replace(P=0), pairs) == pytest.approx(4 * 128 * pairs)


def test_oracle_sample_extrapolates_from_measured_parts():
    w = configs.workload(0)
    s = bench.OracleSample(w)
    for i in range(3):
        assert s.step(i) > 0
    assert s.t_part > 0 and len(s.t_sparse) == 3
    assert s.s_per_call() == pytest.approx(
        w.B * w.H * (s.t_part + s.slices * sum(s.t_sparse) / 3 + sum(s.t_rest) / 3))
    assert "extrapolated" in s.describe()
