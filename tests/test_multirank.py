"""Multi-rank host logic of the benchmark on CPU: two gloo ranks on 127.0.0.1.

Each GPU runs its own independent operator call (heads and calls never exchange data), so the
only cross-rank step is the max over ranks of the per-step device times.  These tests run that
step with the gloo backend, check the whole-job throughput arithmetic, and check that every
rank draws its own inputs.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from free_block_sparse_02_b200 import configs, gen  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r reports step times (1 + r, 10 - r, 3): the job's step is as slow as its slowest rank
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 3.0], world)
        w = configs.scaled_down(configs.workload(1), heads=1, grid=(4, 8, 16))
        q, _, _ = gen.make_qkv(w, variant=rank)
        out[rank] = (got, float(q.float().sum()))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_max_over_ranks_and_per_rank_inputs_with_two_gloo_ranks():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1]
    for r in range(world):
        assert res[r][0] == [2.0, 10.0, 3.0]
    assert res[0][1] != res[1][1], "each rank must run its own independent call"


def test_max_over_ranks_single_rank_is_identity():
    assert bench.max_over_ranks([1.5, 2.5], 1) == [1.5, 2.5]


def test_whole_job_throughput_counts_every_rank():
    w = configs.workload(1)
    f = w.dense_flops()
    one = bench.whole_job_tflops(1, f, 4.0)
    assert np.isclose(one, f / 4e-3 / 1e12)
    assert np.isclose(bench.whole_job_tflops(8, f, 4.0), 8 * one)
