#!/usr/bin/env python
"""Throughput of the SparsePR per-call sparse attention operator on B200.

One step = one whole operator call (plan: response-coupled partitioning, routing, probes;
attention: block-sparse + dense probe rows; fit_apply: weighted ridge + residual add) over
one batch of seeded synthetic video-latent Q/K/V of the chosen workload (default: the
13B-DiT-720p-shaped layer, B=1 H=24 N=118800 d=128 at 22% density, the largest single-GPU
configuration at that density).

  python bench.py [--gpus N --steps K --warmup W] [--workload I] [--shard heads] [--impl reference]

Prints one JSON line (rank 0).  `value` is dense-equivalent TFLOPS of all ranks
(4*B*H*N^2*d per call / device time); `ms_per_step` is milliseconds per call (max over
ranks).  With N > 1 (torchrun) every rank runs its own independent call on its own inputs
(weak scaling, no collective on the data path); with --shard heads the ranks split ONE call by
heads (strong scaling; --gather adds an NCCL all-gather of the output inside the timed region).
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from free_block_sparse_02_b200 import configs, gen  # noqa: E402

METRIC = "SparsePR ms/call & dense-equiv TFLOPS at 22% density; % bf16 TC peak"
L2_FLUSH_BYTES = 256 << 20
KM_W_TERMS = 2  # bf16 terms of the group weights in the k-means assignment's products
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(values, world, device=None):
    """Element-wise max of `values` over all ranks (one all_reduce MAX; identity at world 1).
    Per-step device times are combined this way: the job takes as long as its slowest rank."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def sum_over_ranks(values, world, device=None):
    """Element-wise sum of `values` over all ranks (identity at world 1)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return [float(x) for x in t]


def whole_job_tflops(world, flops_per_call, ms_per_call):
    """Throughput of the whole job: every rank runs one independent call of `flops_per_call`
    (dense-equivalent) per step, and a step lasts `ms_per_call` (the max over ranks)."""
    return world * flops_per_call / (ms_per_call * 1e-3) / 1e12


def _strip_comments(text: str) -> str:
    """C/C++/CUDA source without comments, trailing blanks and empty lines: the code a
    profile's counters belong to (a comment edit does not void them)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(ln.rstrip() for ln in text.splitlines() if ln.strip())


def source_hash(*rel):
    """sha256 of the given sources (paths relative to the repository root), comments stripped."""
    import hashlib
    h = hashlib.sha256()
    for r in rel:
        with open(os.path.join(ROOT, r), encoding="utf-8") as f:
            h.update(_strip_comments(f.read()).encode())
    return h.hexdigest()


ATTN_SOURCES = ("free_block_sparse_02_b200/csrc/attention_sm100.cu", "free_block_sparse_02_b200/csrc/sm100.cuh")


def profiled_traffic(w):
    """DRAM read + write bytes per attention launch from the committed ncu summary of this
    workload, or None when there is none or the attention code changed since it was taken."""
    import re
    if w != configs.workload(w.index):  # a sweep or a cut of the workload: not what was profiled
        return None
    path = os.path.join(ROOT, "profiles", f"attn_tc_kernel_{w.name}.md")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        text = f.read()
    m = re.search(r"^dram_bytes_per_launch:\s*(\d+)", text, re.M)
    h = re.search(r"^source_sha256:\s*([0-9a-f]{64})", text, re.M)
    if not m or not h or h.group(1) != source_hash(*ATTN_SOURCES):
        return None
    return int(m.group(1))


def workload_config(w, extra=None):
    c = {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "density": w.density, "s": w.s,
         "n_kgroups": w.n_kgroups, "n_qgroups": w.n_qgroups, "P": w.P,
         "probes": ["uniform", "stratified", "random"][w.probe_mode], "km_iters": w.km_iters, "km_tol": w.km_tol,
         "lam": w.lam, "correction": "mean" if w.correction == 1 else "affine", "trunc_rank": w.trunc_rank,
         "key_rank": w.key_rank,
         "generator": (f"clustered Gaussian tiles {w.tile} on grid {w.grid}" if w.recipe == "tiles" else
                       f"smooth random field, length scales {w.field_ell}, logit contrast {w.field_tau}, "
                       f"value offset {w.value_offset}, on grid {w.grid}") + (" + 3D RoPE" if w.rope else "")}
    if extra:
        c.update(extra)
    return c


# ------------------------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of this GPU's clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={uuid}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def output_quality(S, w, Q, K, V, O_main, main_probes, dev, n_eval=2048):
    """Normalised output error of the call (Table 2's metric) on n_eval strided rows per head,
    its probe rows excluded, against exact dense rows from a second operator whose n_eval
    uniform probe rows are computed densely; and the same error for the semantic partition
    without repair (Table 2's baseline), giving the error reduction.  Outside the timed region."""
    import numpy as np
    ev = min(n_eval, w.N, 4096)
    dense_op = S.SparsePR(w, device=dev, P=ev, probe_mode=configs.PROBE_UNIFORM, repair=0)
    dense_op(Q, K, V)
    ref = dense_op.query(S.Q_ODENSE).astype(np.float64)          # [BH, ev, d]
    rows = dense_op.query(S.Q_PROBES)                            # [BH, ev] ascending tokens
    del dense_op
    sem = S.SparsePR(w, device=dev, partition=configs.PARTITION_SEMANTIC, repair=0)
    O_sem = sem(Q, K, V, out_dtype=O_main.dtype)
    torch.cuda.synchronize(dev)
    BH = w.B * w.H
    # the uniform evaluation rows are the same in every head: gather them on the device
    idx = torch.from_numpy(rows[0].astype(np.int64)).to(dev)
    assert (rows == rows[0][None, :]).all()
    O1 = O_main.reshape(BH, w.N, w.d).index_select(1, idx).float().cpu().numpy().astype(np.float64)
    O0 = O_sem.reshape(BH, w.N, w.d).index_select(1, idx).float().cpu().numpy().astype(np.float64)
    sem_probes = sem.query(S.Q_PROBES)
    del sem, O_sem
    e1, e0 = [], []
    for h in range(BH):
        keep = ~np.isin(rows[h], main_probes[h]) & ~np.isin(rows[h], sem_probes[h])
        r = ref[h][keep]
        den = np.linalg.norm(r, axis=1) + 1e-8
        e1.append(np.linalg.norm(O1[h][keep] - r, axis=1) / den)
        e0.append(np.linalg.norm(O0[h][keep] - r, axis=1) / den)
    e1, e0 = np.concatenate(e1), np.concatenate(e0)
    return {"mean_err": float(e1.mean()), "p99_err": float(np.percentile(e1, 99)),
            "semantic_no_repair_mean_err": float(e0.mean()),
            "error_reduction": float(1.0 - e1.mean() / e0.mean()),
            "eval_rows": f"{ev} strided rows per head minus probe rows; output dtype of the call"}


QUALITY_NOTE_TILES = ("clustered-tile inputs have independent N(0,1) values: the residual of a dropped key group "
                      "is an average of unrelated noise, which no affine map of the sparse output predicts, so "
                      "the fitted correction can raise the error on them (a property of these inputs, not a "
                      "parity result); quality_field shows the same operator on smooth-field inputs")


def km_rooflines(w, asg_ms, upd_ms, pk):
    """Rooflines of one key k-means assignment and one update launch (first iteration of the
    call).  Both read every key once (2 d bytes, bf16) and write (assignment) or read (update)
    its label (4 bytes).  The assignment also runs the tensor-core products of every key with
    the two bf16 terms (hi, mid) of the C_p (padded) group weights, 2 x 2 x C_p x d flops per
    key: at the large shapes that, not HBM, is its bound, and it is reported against the bf16
    peak with the HBM fraction beside it.  The update is HBM-bound."""
    units = w.B * w.H * w.N
    by = units * (2 * w.d + 4)
    cp = (w.n_kgroups + 15) // 16 * 16
    fl = units * KM_W_TERMS * 2 * cp * w.d
    out = {}
    if asg_ms > 0:
        s = asg_ms * 1e-3
        tpk = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])  # inside a long step
        t_hbm, t_tc = by / (pk["hbm_gbs"] * 1e9), fl / (tpk * 1e12)
        hbm = {"achieved": by / s / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": by / s / 1e9 / pk["hbm_gbs"]}
        tc = {"achieved": fl / s / 1e12, "peak": tpk, "unit": "TFLOP/s", "frac": fl / s / 1e12 / tpk}
        main, other = (tc, hbm) if t_tc >= t_hbm else (hbm, tc)
        out["assignment"] = {"bound": "tensor" if t_tc >= t_hbm else "hbm", **main, "ms": asg_ms, "traffic": None,
                             "other": other,
                             "algorithmic": f"{units} keys x (2d + 4) bytes = {by} bytes and x {2 * KM_W_TERMS} C_p d = "
                                            f"{fl} flops per launch"}
    if upd_ms > 0:
        a = by / (upd_ms * 1e-3) / 1e9
        out["update"] = {"bound": "hbm", "achieved": a, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": a / pk["hbm_gbs"], "ms": upd_ms, "traffic": None,
                         "algorithmic": f"{units} keys x (2d + 4) bytes = {by} bytes per launch"}
    return out


def km_loop_roofline(w, loop_ms, k_iters, pk):
    """The key k-means of a mid-size call as one launch (every Lloyd iteration; the keys stay in
    shared memory, read from HBM once).  Its time is set by the per-iteration chain (scoring,
    fp64 re-decision, group sums, two head barriers, the centroid step), not by a throughput
    roofline: reported per iteration, with the tensor-core flops of the scoring against the bf16
    peak for scale."""
    units = w.B * w.H * w.N
    cp = (w.n_kgroups + 15) // 16 * 16
    it = max(k_iters) if k_iters else 0
    fl = units * KM_W_TERMS * 2 * cp * w.d * it
    tpk = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
    s = loop_ms * 1e-3
    return {"loop": {"bound": "latency", "ms": loop_ms, "iterations": it,
                     "ms_per_iteration": loop_ms / it if it else None,
                     "tensor": {"achieved": fl / s / 1e12 if s > 0 else None, "peak": tpk, "unit": "TFLOP/s",
                                "frac": fl / s / 1e12 / tpk if s > 0 else None},
                     "hbm_bytes": units * 2 * w.d,
                     "algorithmic": f"{units} keys read once ({units * 2 * w.d} bytes); {it} iterations of "
                                    f"{2 * KM_W_TERMS} C_p d flops per key on the tensor cores"}}


def attention_flops(w, sparse_pairs):
    """Algorithmic flops of one attention launch: 4 d per executed query-key pair, counting the
    block-sparse pairs of every row and the probe rows' dense pairs (P N per head), which the
    same launch computes.  Padding rows and masked keys are not counted."""
    return 4.0 * w.d * (sparse_pairs + w.B * w.H * w.P * w.N)


# ------------------------------------------------------------------------------------ CPU baseline
def _oracle_cores():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=os.cpu_count())
    except Exception:
        return os.cpu_count()


class OracleSample:
    """The fp64 oracle, as it stands, on a bounded sample of one call of workload `w`.

    One head's partition (steps 1-5 and the probe choice: call_head without outputs) runs once
    and is timed.  A step then runs the oracle's output steps on that partition: the
    block-sparse attention of one slice of the query groups (groups g with g mod S = step mod S,
    S = min(8, C_q) slices, so S consecutive steps cover every group once), the probe rows'
    dense attention, the ridge fit, its restriction to the residual span and the corrected
    output.  The time of a whole call is estimated as
        B * H * (partition + S * mean block-sparse slice time + mean time of the rest),
    every term measured; it is an extrapolation over heads and slices, and says so."""

    def __init__(self, w, head=0):
        import numpy as np
        from oracle import sparsepr_oracle as O
        self.O, self.np, self.w = O, np, w
        b, h = divmod(head, w.H)
        Q, K, V = gen.make_qkv(w, heads=[(b, h)])
        self.q, self.k, self.v = (gen.as_f64(x)[b, h] for x in (Q, K, V))
        t0 = time.perf_counter()
        self.r = O.call_head(self.q, self.k, self.v, w, head, compute_outputs=False)
        self.t_part = time.perf_counter() - t0
        self.slices = max(1, min(8, w.n_qgroups))
        self.t_sparse, self.t_rest = [], []

    def step(self, i, record=True):
        O, np, r = self.O, self.np, self.r
        sel = (np.arange(self.w.n_qgroups) % self.slices) == (i % self.slices)
        route = r["route"] & sel[:, None]
        t0 = time.perf_counter()
        osp = O.sparse_attention(self.q, self.k, self.v, r["qlabels"], r["klabels"], route)
        t1 = time.perf_counter()
        p, wts = r["probes"], r["weights"]
        od = O.attention(self.q[p], self.k, self.v)
        if len(p):
            A, _ = O.ridge_fit(osp[p], od, wts, self.w.lam)
            A = O.restrict_to_residual_span(A, od - osp[p], wts)
        else:
            A = np.zeros((self.w.d + 1, self.w.d))
        out = O.apply_correction(osp, A)
        out[p] = od
        t2 = time.perf_counter()
        if record:
            self.t_sparse.append(t1 - t0)
            self.t_rest.append(t2 - t1)
        return t2 - t0

    def s_per_call(self):
        per_head = self.t_part + self.slices * statistics.mean(self.t_sparse) + statistics.mean(self.t_rest)
        return self.w.B * self.w.H * per_head

    def describe(self):
        return (f"head 0 of {self.w.B * self.w.H}: its partition once ({self.t_part:.1f} s), then per step the "
                f"block-sparse attention of 1/{self.slices} of its query groups (a different slice each step) "
                f"plus its probe rows, ridge fit and correction; call time extrapolated as "
                f"{self.w.B * self.w.H} x (partition + {self.slices} x slice + rest)")


def oracle_baseline(w):
    """cpu_baseline: the oracle's partition of one head plus one output step (about 10-30 s of
    CPU work at the large shapes), extrapolated to the call."""
    s = OracleSample(w)
    s.step(0)
    per_call = s.s_per_call()
    return {"value": w.dense_flops() / per_call / 1e12, "unit": "TFLOPS", "cores": _oracle_cores(), "kind": "oracle",
            "sample": s.describe() + " (one step)", "s_per_call_extrapolated": per_call}


def run_reference(args, w, world, rank):
    if rank != 0:
        return
    t_start = time.perf_counter()
    s = OracleSample(w)
    for i in range(args.warmup):
        s.step(i, record=False)
    t0 = time.perf_counter()
    steps = [s.step(args.warmup + i) for i in range(args.steps)]
    timed = time.perf_counter() - t0
    per_call = s.s_per_call()
    val = w.dense_flops() / per_call / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOPS", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(steps) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, {"l2": "n/a (CPU)"}),
            "oracle_s_per_call_extrapolated": per_call,
            "oracle_partition_s_per_head": s.t_part,
            "cpu_baseline": {"kind": "oracle", "cores": _oracle_cores(), "value": val, "unit": "TFLOPS",
                             "sample": s.describe()},
            "e2e": {"value": val, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "timed_s": timed, "wall_s": time.perf_counter() - t_start}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------ GPU arm
def _rank_inputs(w, world, rank, shard):
    """(local workload, Q, K, V on the CPU, bh0, bh1).  Replicas: every rank draws the whole call
    from its own generator variant.  Head shards: the rank draws only its heads of the one call
    (variant 0) and runs them as a call of B = 1 with the seed of its first head."""
    from free_block_sparse_02_b200 import shard as SH
    if not shard or world == 1:
        Q, K, V = gen.make_qkv(w, variant=rank if not shard else 0)
        return w, Q, K, V, 0, w.B * w.H
    wl, bh0, bh1 = SH.shard_workload(w, world, rank)
    if wl is None:
        raise SystemExit(f"--shard heads: rank {rank} of {world} has no head of the {w.B * w.H}-head call")
    Q, K, V = gen.make_qkv(w, variant=0, heads=[divmod(bh, w.H) for bh in range(bh0, bh1)])
    return wl, *(SH.local_slice(x, bh0, bh1).contiguous() for x in (Q, K, V)), bh0, bh1


def run_ours(args, w, world, rank, local):
    from free_block_sparse_02_b200 import _lib as S
    import torch.distributed as dist

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    S.load()
    shard = args.shard == "heads" and world > 1
    wl, Qc, Kc, Vc, bh0, bh1 = _rank_inputs(w, world, rank, args.shard == "heads")
    Q, K, V = Qc.to(dev), Kc.to(dev), Vc.to(dev)
    op = S.SparsePR(wl, device=dev)
    O = torch.empty(Q.shape, dtype=Q.dtype, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    gather = None
    if shard and args.gather:
        per = -(-w.B * w.H // world)
        gather = (torch.zeros((per, w.N, w.d), dtype=Q.dtype, device=dev),
                  torch.empty((world * per, w.N, w.d), dtype=Q.dtype, device=dev))

    def step():
        op(Q, K, V, O=O)
        if gather is not None:
            gather[0][:bh1 - bh0].copy_(O.reshape(bh1 - bh0, w.N, w.d))
            dist.all_gather_into_tensor(gather[1], gather[0])

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    st = op.stats()
    pairs = sum(s["sparse_pairs"] for s in st)
    realised = statistics.mean(s["density"] for s in st)
    part_stats = {"k_iters": [s["k_iters"] for s in st], "q_iters": [s["q_iters"] for s in st],
                  "k_refined": sum(s["k_refined"] for s in st), "q_refined": sum(s["q_refined"] for s in st),
                  "span_rank": [s["span_rank"] for s in st], "fit_retries": sum(s["fit_retries"] for s in st)}

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    # the first key k-means assignment and update launches of each timed call (tensor-core path)
    km_ev = {kid: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)] for kid in (1, 2, 3)}
    for a, b in kev + km_ev[1] + km_ev[2] + km_ev[3]:  # torch creates the CUDA event on first record
        a.record(stream)
        b.record(stream)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local)
    launches0 = S.launch_count()
    for i in range(args.steps):
        flush.zero_()                         # L2 flush between timed steps, outside the events
        op.set_kernel_events(*kev[i])
        for kid in (1, 2, 3):
            op.set_kernel_events(*km_ev[kid][i], kernel=kid)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    launches = S.launch_count() - launches0
    clk = clocks.stop()
    op.set_kernel_events(None, None)
    for kid in (1, 2, 3):
        op.set_kernel_events(None, None, kernel=kid)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    kern_ms = [a.elapsed_time(b) for a, b in kev]
    # the k-means hooks bracket the first assignment and update of the per-iteration tensor-core
    # path (bf16 inputs, at most 256 padded key groups; above that the key k-means runs on the
    # CUDA cores and the events stay unset), or, when the whole key loop runs in one launch, that
    # launch
    km_loop = int(op.query(S.Q_KM_PATH)[0]) == 1
    tc_km = wl.dtype == configs.BF16 and (wl.n_kgroups + 15) // 16 * 16 <= 256 and not km_loop
    asg_ms = statistics.mean(a.elapsed_time(b) for a, b in km_ev[1]) if tc_km else 0.0
    upd_ms = statistics.mean(a.elapsed_time(b) for a, b in km_ev[2]) if tc_km else 0.0
    loop_ms = statistics.mean(a.elapsed_time(b) for a, b in km_ev[3]) if km_loop else 0.0
    ms = statistics.mean(step_ms)
    kms = statistics.mean(kern_ms)
    ms_max, kms_max, asg_ms, upd_ms, loop_ms = max_over_ranks([ms, kms, asg_ms, upd_ms, loop_ms], world, dev)
    # attention roofline per rank: this rank's launch, the slowest rank's time
    kflops = attention_flops(wl, pairs)
    kflops_min, = [-x for x in max_over_ranks([-kflops], world, dev)]
    # executed pairs of the whole job (block-sparse and probe rows, all ranks)
    executed, = sum_over_ranks([kflops], world, dev)

    # end to end through the public API with host buffers (pinned), copies inside the region
    Qh, Kh, Vh = Qc.pin_memory(), Kc.pin_memory(), Vc.pin_memory()
    Oh = torch.empty(O.shape, dtype=O.dtype).pin_memory()
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    for i in range(args.steps + 1):
        flush.zero_()
        if i > 0:
            e2e_ev[i - 1][0].record(stream)
        Q.copy_(Qh, non_blocking=True)
        K.copy_(Kh, non_blocking=True)
        V.copy_(Vh, non_blocking=True)
        op(Q, K, V, O=O)
        Oh.copy_(O, non_blocking=True)
        if i > 0:
            e2e_ev[i - 1][1].record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = statistics.mean(a.elapsed_time(b) for a, b in e2e_ev)
    e2e_ms, = max_over_ranks([e2e_ms], world, dev)

    if rank == 0:
        pk = peaks()
        # whole-job throughput: replicas run `world` calls per step, head shards one call
        job_flops = w.dense_flops() * (1 if shard else world)
        value = job_flops / (ms_max * 1e-3) / 1e12
        achieved = kflops / (kms_max * 1e-3) / 1e12
        # the kernel is timed inside a long step (a whole call, calls back to back under the
        # power cap): the sustained bf16 figure is its peak; the burst figure is given beside it
        peak = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
        burst = pk["bf16_tflops"]
        elt = Q.element_size()
        if shard:
            par = f"one call split by heads over {world} GPUs ({wl.H} or so heads each, no data-path collective" + \
                  (", NCCL all-gather of O inside the timed region)" if gather is not None else ")")
        else:
            par = f"{world} independent calls, one per GPU"
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
            "scaling": "strong" if shard else "weak",
            "vs_baseline": None, "dtype": "bf16" if w.dtype == configs.BF16 else "f32", "data": "synthetic",
            "config": workload_config(w, {"l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write)",
                                          "realised_density": realised, "parallelism": par}),
            "ms_per_call": ms_max,
            "executed_tflops": executed / (ms_max * 1e-3) / 1e12,
            "kernel_ms": {"block_sparse_attention": kms_max},
            "roofline": {"bound": "tensor", "kernel": "attn_tc_kernel: block-sparse attention and the dense probe "
                                                        "rows (the kernel the metric's % of bf16 peak refers to)",
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                         "traffic": profiled_traffic(wl),
                         "peak_source": f"{pk['source']} bf16 dense, sustained (the kernel runs inside a long "
                                        f"step), MEASURED_PEAKS.json",
                         "peak_burst": burst, "frac_of_burst": achieved / burst,
                         "algorithmic": f"4*d*(executed sparse pairs + P*N*heads) = {kflops:.4g} flop per launch "
                                        f"(rank 0; smallest over ranks {kflops_min:.4g})"},
            "roofline_kmeans": (km_rooflines(wl, asg_ms, upd_ms, pk) if tc_km else
                                km_loop_roofline(wl, loop_ms, part_stats["k_iters"], pk) if km_loop else None),
            "e2e": {"value": job_flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOPS",
                    "h2d_bytes_per_step": 3 * Q.numel() * elt, "d2h_bytes_per_step": O.numel() * O.element_size(),
                    "ms_per_step": e2e_ms},
            "gpu_launches": launches,
            "partition": part_stats,
            "clocks": clk,
        }
        if not args.no_quality:
            try:
                q = output_quality(S, wl, Q, K, V, O, op.query(S.Q_PROBES), dev)
                if wl.recipe == "tiles":
                    q["note"] = QUALITY_NOTE_TILES
                line["quality"] = q
            except Exception as exc:  # reported, never fatal: the timing above stands on its own
                line["quality"] = {"error": str(exc)[:200]}
            if world == 1 and wl.recipe == "tiles":
                try:
                    line["quality_field"] = field_quality(S, wl, dev)
                except Exception as exc:
                    line["quality_field"] = {"error": str(exc)[:200]}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = oracle_baseline(w)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def field_quality(S, w, dev, heads=2):
    """The same operator and error metric on smooth-field inputs of the workload's shape
    (`heads` heads): inputs whose block-sparse residual an affine map of the sparse output can
    predict, as the paper's model activations are."""
    wf = configs.scaled_down(w, heads=min(heads, w.H)).replace(recipe="field")
    Q, K, V = (x.to(dev) for x in gen.make_qkv(wf))
    op = S.SparsePR(wf, device=dev)
    O = op(Q, K, V)
    q = output_quality(S, wf, Q, K, V, O, op.query(S.Q_PROBES), dev)
    q["inputs"] = f"smooth random field on the workload's grid, {wf.H} heads"
    return q


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", type=int, default=2, help="index into configs.WORKLOADS")
    ap.add_argument("--shard", default="none", choices=["none", "heads"],
                    help="multi-GPU: independent calls per rank (none) or one call split by heads")
    ap.add_argument("--gather", action="store_true", help="--shard heads: all-gather O inside the timed region")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-quality", action="store_true", help="skip the output-error report (after the timing)")
    ap.add_argument("--heads", type=int, default=0,
                    help="run the workload on this many heads instead (a smaller case for profilers)")
    ap.add_argument("--density", type=float, default=0.0, help="override the density target (sweeps)")
    ap.add_argument("--probes", type=int, default=-1, help="override the probe budget P (sweeps)")
    ap.add_argument("--probe-mode", default=None, choices=["uniform", "stratified", "random"],
                    help="override the probe selection (Table 4 sweeps)")
    ap.add_argument("--correction", default=None, choices=["affine", "mean"],
                    help="override the correction family (Table 4 sweeps)")
    ap.add_argument("--lam", type=float, default=None, help="override the ridge lambda (>= 0 absolute)")
    ap.add_argument("--trunc-rank", type=int, default=0, help="restrict the map to the r leading residual directions")
    ap.add_argument("--key-rank", type=int, default=0, help="key-response rank r_K (Table C.1; 0 = full)")
    ap.add_argument("--kgroups", type=int, default=0, help="override the key-group count C_k")
    ap.add_argument("--qgroups", type=int, default=0, help="override the query-group count C_q")
    ap.add_argument("--sampled", type=int, default=0, help="override the sampled-query count s")
    ap.add_argument("--inputs", default="tiles", choices=["tiles", "field"],
                    help="input recipe: clustered Gaussian tiles (the workloads' own) or a smooth random field")
    args = ap.parse_args()
    world, rank, local = dist_env()
    w = configs.workload(args.workload)
    if args.heads > 0:
        w = configs.scaled_down(w, heads=args.heads)
    if args.density > 0:
        w = w.replace(density=args.density)
    if args.probes >= 0:
        w = w.replace(P=args.probes)
    if args.inputs != w.recipe:
        w = w.replace(recipe=args.inputs)
    if args.probe_mode is not None:
        w = w.replace(probe_mode={"uniform": configs.PROBE_UNIFORM, "stratified": configs.PROBE_STRATIFIED,
                                  "random": configs.PROBE_RANDOM}[args.probe_mode])
    if args.correction is not None:
        w = w.replace(correction=configs.CORRECTION_MEAN if args.correction == "mean" else configs.CORRECTION_AFFINE)
    if args.lam is not None:
        w = w.replace(lam=args.lam)
    if args.trunc_rank > 0:
        w = w.replace(trunc_rank=args.trunc_rank)
    if args.key_rank > 0:
        w = w.replace(key_rank=args.key_rank)
    if args.kgroups > 0:
        w = w.replace(n_kgroups=args.kgroups)
    if args.qgroups > 0:
        w = w.replace(n_qgroups=args.qgroups)
    if args.sampled > 0:
        w = w.replace(s=args.sampled)
    if args.impl == "reference":
        run_reference(args, w, world, rank)
    else:
        run_ours(args, w, world, rank, local)


if __name__ == "__main__":
    main()
