"""The large workloads at their full sizes, launched as the benchmark launches them (one call
over all heads, bf16 output), checked against the fp64 oracle on sampled heads and rows (needs
a B200).

Per checked head: the oracle's key and query groups equal the GPU's (up to the oracle's
near-ties), its routes, probes and weights equal the GPU's, and -- on the GPU's partition -- the
probe rows' dense outputs, 256 strided rows' block-sparse outputs, the fitted map and those rows'
corrected outputs match the oracle's, computed one row at a time (all N rows of a head would take
the oracle minutes each).  Workloads: the 13B-DiT-shaped layer (22% density), the 14B-DiT-shaped
layer at the two ends of its density sweep (15% and 30%), and the 8-call world-model stream at
its largest probe budget (P = 2048), every call warm-started from the previous one.
"""
import numpy as np
import pytest
import torch

from free_block_sparse_02_b200 import build, configs, gen
from free_block_sparse_02_b200 import _lib as S
from oracle import sparsepr_oracle as O
from test_gpu_parity import GAIN_CAP, _close, fit_matches, labels_match, oracle_routing_on, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    S.load()


def _sparse_rows(q, k, v, rows, qlabels, klabels, route):
    """Block-sparse attention output of the given rows only (the oracle's definition, row by row
    grouped by query group): each row attends to the keys of the groups its group keeps."""
    out = np.zeros((len(rows), v.shape[1]))
    for g in np.unique(qlabels[rows]):
        sel = np.flatnonzero(qlabels[rows] == g)
        keys = np.flatnonzero(route[g][klabels])
        out[sel] = O.attention(q[rows[sel]], k[keys], v[keys])
    return out


class GpuCall:
    """Everything the checks read back from one GPU call."""

    def __init__(self, op, out):
        self.kl, self.ql = op.query(S.Q_KLABELS), op.query(S.Q_QLABELS)
        self.route = op.query(S.Q_ROUTE).astype(bool)
        self.probes, self.pw = op.query(S.Q_PROBES), op.query(S.Q_PROBE_W)
        self.kc, self.qc = op.query(S.Q_KCENT), op.query(S.Q_QCENT)
        self.st, self.A = op.stats(), op.query(S.Q_FIT)
        self.osp, self.od = op.query(S.Q_OSP), op.query(S.Q_ODENSE)
        self.out = out


def check_head(w, g, h, q, k, v, warm=None, log=None, case="", n_rows=256):
    """Sampled checks of head h of one GPU call against the oracle.  Returns the oracle's warm
    state for the next call of a stream: its own when the partitions agree, else the GPU's
    centroids (a near-tie decided the other way; the next call then starts where the GPU's did)."""
    r = O.call_head(q, k, v, w, h, warm=warm, compute_outputs=False)
    labels_match(g.kl[h], r["kmeans_k"], f"{case} head {h} key groups")
    labels_match(g.ql[h], r["kmeans_q"], f"{case} head {h} query groups")
    same = np.array_equal(g.kl[h], r["klabels"]) and np.array_equal(g.ql[h], r["qlabels"])
    if same:
        ref_route, ref_probes, ref_w, ref_pairs = r["route"], r["probes"], r["weights"], r["sparse_pairs"]
    else:
        ref_route, ref_probes, ref_w, ref_pairs = oracle_routing_on(q, g.kl[h], g.ql[h], g.kc[h], w, h)
    assert np.array_equal(g.route[h], ref_route), f"{case} head {h} routes"
    assert np.array_equal(g.probes[h], ref_probes), f"{case} head {h} probes"
    np.testing.assert_allclose(g.pw[h], ref_w, rtol=1e-12)
    assert g.st[h]["sparse_pairs"] == ref_pairs
    p = g.probes[h]
    od = g.od[h].astype(np.float64)
    od_ref = O.attention(q[p], k, v)
    _close(f"{case} head {h} O_dense", od, od_ref, 2e-2, 1e-2)
    osp = g.osp[h].astype(np.float64)
    rows = (np.arange(n_rows) * w.N) // n_rows
    rows = rows[~np.isin(rows, p)]
    ref_sp = _sparse_rows(q, k, v, np.concatenate([rows, p]), g.ql[h], g.kl[h], g.route[h])
    ref_rows_sp, ref_p_sp = ref_sp[:len(rows)], ref_sp[len(rows):]
    _close(f"{case} head {h} O_sp rows", osp[rows], ref_rows_sp, 2e-2, 1e-2)
    _close(f"{case} head {h} O_sp probes", osp[p], ref_p_sp, 2e-2, 1e-2)
    # the fit on the GPU's own probe rows (both sides fp64)
    A_full, _ = O.ridge_fit(osp[p], od, g.pw[h], w.lam)
    A_ref = O.restrict_to_residual_span(A_full, od - osp[p], g.pw[h])
    fit_matches(g.A[h], A_full, A_ref, od - osp[p], g.pw[h], f"{case} head {h} fit")
    got = g.out[0, h].float().cpu().numpy().astype(np.float64)
    # corrected rows: the GPU's O_sp through the GPU's map, to the bf16 output's rounding
    _close(f"{case} head {h} apply", got[rows], O.apply_correction(osp[rows], g.A[h]), 2e-2, 1e-2)
    assert np.abs(got[p] - od).max() <= 2e-2, f"{case} head {h} probe rows"
    # end to end on the sampled rows: the oracle's rows through the oracle's own map; the bar is
    # the flat one up to a map gain of 1.1, the bar times the gain up to GAIN_CAP, and above the
    # cap the stages above (unscaled) carry the claim
    A_orc_full, _ = O.ridge_fit(ref_p_sp, od_ref, g.pw[h], w.lam)
    A_orc = O.restrict_to_residual_span(A_orc_full, od_ref - ref_p_sp, g.pw[h])
    ref_rows = O.apply_correction(ref_rows_sp, A_orc)
    A_lin = A_orc[:-1]
    gain_inf = 1.0 + np.abs(A_lin).sum(axis=0).max()
    gain_2 = 1.0 + np.linalg.norm(A_lin, 2)
    bar = "stage-only"
    if gain_inf <= 1.1 and gain_2 <= 1.1:
        bar = "flat"
        _close(f"{case} head {h} O rows", got[rows], ref_rows, 2e-2, 1e-2)
    elif gain_inf <= GAIN_CAP and gain_2 <= GAIN_CAP:
        bar = "scaled"
        _close(f"{case} head {h} O rows (bar x gain)", got[rows], ref_rows, 2e-2 * gain_inf, 1e-2 * gain_2)
    if log is not None:
        # the sampled rows' errors against the exact dense rows: the GPU's and the oracle's
        dense = O.attention(q[rows], k, v)
        log.append(dict(case=case, head=h, gain_inf=float(gain_inf), gain_2=float(gain_2), e2e=bar,
                        e2e_abs=float(np.abs(got[rows] - ref_rows).max()),
                        e2e_rl2=float(np.linalg.norm(got[rows] - ref_rows) / np.linalg.norm(ref_rows)), slack=0.0,
                        e_gpu=float(O.row_errors(got[rows], dense).mean()),
                        e_orc=float(O.row_errors(ref_rows, dense).mean())))
    if same:
        return O.warm_state(r)
    return O.WarmState(key_centroids=g.kc[h], query_centroids=g.qc[h])


def test_dit13b_full_size_sampled(parity_log):
    """The 13B-DiT-shaped layer (24 heads x 118,800 tokens, d = 128, 22%): first and last head."""
    w = configs.workload(2)
    Q, K, V = gen.make_qkv(w)
    op, out = run_gpu(w, Q, K, V, out_dtype=torch.bfloat16)
    g = GpuCall(op, out)
    for h in (0, w.H - 1):
        check_head(w, g, h, *(gen.as_f64(x[0, h]) for x in (Q, K, V)), log=parity_log, case="dit13b 22%")


@pytest.fixture(scope="module")
def dit14b_inputs():
    w = configs.workload(3)
    return w, gen.make_qkv(w)


@pytest.mark.parametrize("density", [0.15, 0.30])
def test_dit14b_density_ends_full_size_sampled(density, dit14b_inputs, parity_log):
    """The 14B-DiT-shaped layer (40 heads x 75,600 tokens, d = 128) at the two ends of its density
    sweep: first and last head."""
    w0, (Q, K, V) = dit14b_inputs
    w = w0.replace(density=density)
    op, out = run_gpu(w, Q, K, V, out_dtype=torch.bfloat16)
    g = GpuCall(op, out)
    for h in (0, w.H - 1):
        check_head(w, g, h, *(gen.as_f64(x[0, h]) for x in (Q, K, V)), log=parity_log,
                   case=f"dit14b {int(round(density * 100))}%")


def test_worldmodel_stream_full_size_p2048_sampled(parity_log):
    """The world-model stream (16 heads x 42,240 tokens, d = 128) at P = 2048: all 8 calls on one
    plan, calls 1-7 warm-started (2 Lloyd iterations) from the previous call's centroids; first
    and last head of every call, the oracle's warm-start chain followed alongside."""
    w = configs.workload(4).replace(P=2048)
    calls = gen.make_stream(w)
    op = S.SparsePR(w)
    warm = {h: None for h in (0, w.H - 1)}
    for c, (Q, K, V) in enumerate(calls):
        out = op(Q.cuda(), K.cuda(), V.cuda(), out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        op.sync()
        g = GpuCall(op, out)
        if c > 0:
            assert all(s["k_iters"] <= w.km_iters_warm and s["q_iters"] <= w.km_iters_warm for s in g.st)
        for h in warm:
            warm[h] = check_head(w, g, h, *(gen.as_f64(x[0, h]) for x in (Q, K, V)), warm=warm[h],
                                 log=parity_log, case=f"stream P=2048 call {c}")
