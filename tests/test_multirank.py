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


# ---------------------------------------------------------------- one call split by heads
from free_block_sparse_02_b200 import shard as SH  # noqa: E402
from oracle import sparsepr_oracle as O  # noqa: E402


def test_head_ranges_are_contiguous_balanced_and_cover_every_head():
    for bh in range(0, 41):
        for world in range(1, 9):
            rs = [SH.head_range(bh, world, r) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == bh
            assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
            sizes = [b - a for a, b in rs]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 0
    assert SH.head_range(24, 8, 3) == (9, 12)       # the 13B-DiT layer: 3 heads per GPU
    assert SH.head_range(40, 8, 7) == (35, 40)
    with pytest.raises(ValueError):
        SH.head_range(4, 2, 2)


def _shard_case(probe_mode):
    return configs.scaled_down(configs.workload(1), heads=3, grid=(2, 8, 16), s=32, n_kgroups=8, n_qgroups=6,
                               P=16, km_iters=4, probe_mode=probe_mode)


def _oracle_heads(w, q, k, v, bh0, bh1, seed_heads_from=0):
    """The oracle on heads [bh0, bh1) as a call whose heads are numbered from seed_heads_from."""
    out = []
    for bh in range(bh0, bh1):
        r = O.call_head(q[bh], k[bh], v[bh], w, bh - seed_heads_from)
        out.append((r["klabels"], r["qlabels"], r["route"], r["probes"], r["O"]))
    return out


def _shard_rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        res = {}
        for mode in (configs.PROBE_STRATIFIED, configs.PROBE_RANDOM):
            w = _shard_case(mode)
            Q, K, V = gen.make_qkv(w)
            wl, bh0, bh1 = SH.shard_workload(w, world, rank)
            # the rank's slice of the one call, run as its own call of B = 1, H = bh1 - bh0
            q, k, v = (gen.as_f64(SH.local_slice(x, bh0, bh1))[0] for x in (Q, K, V))
            local = [None] * (bh1 - bh0)
            for i in range(bh1 - bh0):
                r = O.call_head(q[i], k[i], v[i], wl, i)
                local[i] = (r["klabels"], r["qlabels"], r["route"], r["probes"], r["O"])
            gathered = [None] * world
            dist.all_gather_object(gathered, (bh0, bh1, local))
            res[mode] = gathered
        out[rank] = res
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_head_sharded_call_on_two_gloo_ranks_equals_the_single_rank_call():
    """Two gloo ranks split one 3-head call (2 does not divide 3): each runs its heads as a call of
    its own with the seed advanced to its first head.  The assembled labels, routes, probe rows
    (stratified and random) and outputs equal the single-process oracle call's, head by head."""
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_shard_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1]
    for mode in (configs.PROBE_STRATIFIED, configs.PROBE_RANDOM):
        w = _shard_case(mode)
        Q, K, V = gen.make_qkv(w)
        q, k, v = (gen.as_f64(x).reshape(-1, w.N, w.d) for x in (Q, K, V))
        whole = _oracle_heads(w, q, k, v, 0, w.B * w.H)
        assembled = []
        for bh0, bh1, local in res[0][mode]:
            assert len(local) == bh1 - bh0
            assembled.extend(local)
        assert [(a, b) for a, b, _ in res[0][mode]] == [(0, 1), (1, 3)]
        assert len(assembled) == len(whole)
        for (kl, ql, rt, pr, o), (kl0, ql0, rt0, pr0, o0) in zip(assembled, whole):
            assert np.array_equal(kl, kl0) and np.array_equal(ql, ql0)
            assert np.array_equal(rt, rt0) and np.array_equal(pr, pr0)
            assert np.array_equal(o, o0)
    # and the seed offset matters: numbering the second rank's heads from 0 without it differs
    w = _shard_case(configs.PROBE_RANDOM)
    Q, K, V = gen.make_qkv(w)
    q, k, v = (gen.as_f64(x).reshape(-1, w.N, w.d) for x in (Q, K, V))
    wrong = O.call_head(q[1], k[1], v[1], w, 0)
    right = O.call_head(q[1], k[1], v[1], w, 1)
    assert not np.array_equal(wrong["probes"], right["probes"])
