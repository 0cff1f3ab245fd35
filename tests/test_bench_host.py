"""Host-side logic of bench.py (no GPU): roofline selection, the traffic lookup's gating, the
configuration record of sweeps and the throughput arithmetic."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from free_block_sparse_02_b200 import configs  # noqa: E402

PEAKS = {"hbm_gbs": 6557.4, "bf16_tflops": 1629.0}


def test_assignment_roofline_is_the_binding_one():
    """13B-DiT layer: 6 C_p d = 98,304 flops and 2d + 4 = 260 bytes per key, so the tensor time
    (flops / peak) exceeds the HBM time; the mid-size shape (d = 64, C_p = 64) is HBM-bound."""
    big = bench.km_rooflines(configs.workload(2), 0.378, 0.244, PEAKS)
    assert big["assignment"]["bound"] == "tensor" and big["assignment"]["unit"] == "TFLOP/s"
    assert big["assignment"]["other"]["unit"] == "GB/s"
    keys = 24 * 118800
    assert big["assignment"]["achieved"] == pytest.approx(keys * 6 * 128 * 128 / 0.378e-3 / 1e12)
    assert big["update"]["bound"] == "hbm"
    assert big["update"]["achieved"] == pytest.approx(keys * 260 / 0.244e-3 / 1e9)
    mid = bench.km_rooflines(configs.workload(1), 0.0205, 0.0246, PEAKS)
    assert mid["assignment"]["bound"] == "hbm"
    assert bench.km_rooflines(configs.workload(1), 0.0, 0.0, PEAKS) == {}


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
