"""Failure paths of the operator on the GPU (needs a B200), made without faulting the GPU.

1. A ridge system that stays indefinite.  A partition installed from the host gives one probe
   row a large negative weight, so X^T W X + lambda I has a negative eigenvalue for every
   lambda the jitter retries reach: the fit must record three retries, return
   SPARSEPR_ERR_NUMERIC from sparsepr_sync, leave A = 0 (unprobed rows keep O_sp, probe rows
   O_dense), and the next call on the same plan must be clean and correct.
2. A bounded device-side wait that gives up.  The test hook sets the attention kernel's wait
   limit to a few hundred cycles, far below the latency of its first tile loads: the launch must
   give up, drain its copies, free its tensor memory and return, sparsepr_sync must return
   SPARSEPR_ERR_TIMEOUT, and, with the default limit restored, the next call on the same plan
   must be clean and correct.
3. The same for the barriers between the CTAs of one head in the whole-loop k-means launch:
   with a limit of one cycle the first CTA to reach a barrier gives up before the other fifteen
   arrive, every CTA of the launch leaves (the abort flag), every point is left in group 0, and
   the call reports SPARSEPR_ERR_TIMEOUT; the next call with the default limit is clean.
"""
import numpy as np
import pytest
import torch

from free_block_sparse_02_b200 import build, configs, gen
from free_block_sparse_02_b200 import _lib as S
from oracle import sparsepr_oracle as O
from test_gpu_parity import _close, compare_partition

pytestmark = pytest.mark.gpu

NUMERIC, TIMEOUT, INVALID, UNSUPPORTED = 5, 6, 1, 2


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    S.load()


def _workload():
    return configs.scaled_down(configs.workload(1), heads=2, grid=(4, 16, 32), s=64, n_kgroups=16, n_qgroups=12,
                               P=80, km_iters=6)


def _flat(x):
    return gen.as_f64(x).reshape(-1, x.shape[2], x.shape[3])


def _clean_call_matches_oracle(op, w, Q, K, V):
    """A normal call on the plan: no pending status, and the oracle's partition and outputs."""
    out = op(Q.cuda(), K.cuda(), V.cuda(), out_dtype=torch.float32)
    torch.cuda.synchronize()
    op.sync()
    qf, kf, vf = _flat(Q), _flat(K), _flat(V)
    res = O.call(qf[None], kf[None], vf[None], w)
    compare_partition(op, res, w, qf)
    osp = op.query(S.Q_OSP).astype(np.float64)
    got = out.cpu().numpy().reshape(-1, w.N, w.d)
    probes, pw = op.query(S.Q_PROBES), op.query(S.Q_PROBE_W)
    kl, ql, route = op.query(S.Q_KLABELS), op.query(S.Q_QLABELS), op.query(S.Q_ROUTE).astype(bool)
    for h in range(w.B * w.H):
        ref = O.outputs_given_partition(qf[h], kf[h], vf[h], ql[h], kl[h], route[h], probes[h], pw[h], w.lam)
        _close(f"head {h} O_sp after the failure", osp[h], ref["osp"], 2e-2, 1e-2)
        assert np.isfinite(got[h]).all()


def test_indefinite_ridge_reports_numeric_and_the_next_call_is_clean():
    w = _workload()
    Q, K, V = gen.make_qkv(w)
    qf, kf, vf = _flat(Q), _flat(K), _flat(V)
    parts = [O.call_head(qf[h], kf[h], vf[h], w, h, compute_outputs=False) for h in range(w.H)]
    weights = np.stack([r["weights"] for r in parts]).copy()
    weights[:, 0] = -1000.0 * w.P  # one probe row outweighs all the others with the wrong sign
    op = S.SparsePR(w)
    op.set_partition(np.stack([r["klabels"] for r in parts]), np.stack([r["qlabels"] for r in parts]),
                     np.stack([r["route"] for r in parts]), np.stack([r["probes"] for r in parts]), weights)
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    op.attention(Qd, Kd, Vd)
    out = op.fit_apply(out_dtype=torch.float32)
    with pytest.raises(S.SparsePRError) as e:
        op.sync()
    assert e.value.status == NUMERIC
    op.sync()  # the status word was cleared by the first sync
    st = op.stats()
    assert all(s["fit_retries"] == 3 for s in st), [s["fit_retries"] for s in st]
    assert not np.any(op.query(S.Q_FIT)), "a failed fit leaves A = 0"
    osp = op.query(S.Q_OSP)
    od = op.query(S.Q_ODENSE)
    got = out.cpu().numpy().reshape(-1, w.N, w.d)
    for h in range(w.H):
        p = parts[h]["probes"]
        unprobed = np.setdiff1d(np.arange(w.N), p)
        assert np.array_equal(got[h][unprobed], osp[h][unprobed]), "A = 0: unprobed rows keep O_sp"
        assert np.array_equal(got[h][p], od[h]), "probe rows keep their exact rows"
    _clean_call_matches_oracle(op, w, Q, K, V)
    assert all(s["fit_retries"] == 0 for s in op.stats())


def test_attention_wait_limit_gives_timeout_and_the_next_call_is_clean():
    w = _workload()
    Q, K, V = gen.make_qkv(w)
    op = S.SparsePR(w)
    with pytest.raises(S.SparsePRError) as e:
        op.set_wait_limit(100, kernel=1)  # only the attention launch takes the hook
    assert e.value.status == UNSUPPORTED
    with pytest.raises(S.SparsePRError) as e:
        op.set_wait_limit(-1)
    assert e.value.status == INVALID
    op.set_wait_limit(200)
    op(Q.cuda(), K.cuda(), V.cuda(), out_dtype=torch.float32)
    torch.cuda.synchronize()  # the launch returned: no wait was left spinning
    with pytest.raises(S.SparsePRError) as e:
        op.sync()
    assert e.value.status == TIMEOUT
    op.sync()  # cleared
    op.set_wait_limit(0)
    _clean_call_matches_oracle(op, w, Q, K, V)


def test_kmeans_loop_wait_limit_gives_timeout_and_the_next_call_is_clean():
    w = _workload()  # 2 heads of 2048 points: 16 CTAs per head in the whole-loop k-means
    Q, K, V = gen.make_qkv(w)
    op = S.SparsePR(w)
    assert list(op.query(S.Q_KM_PATH)) == [1, 1]
    op.set_wait_limit(1, kernel=S.KERNEL_KMEANS_LOOP)
    op(Q.cuda(), K.cuda(), V.cuda(), out_dtype=torch.float32)
    torch.cuda.synchronize()  # the launches returned: no barrier was left spinning
    with pytest.raises(S.SparsePRError) as e:
        op.sync()
    assert e.value.status == TIMEOUT
    op.sync()  # cleared
    assert not np.any(op.query(S.Q_KLABELS)) and not np.any(op.query(S.Q_QLABELS)), "aborted loops leave group 0"
    op.set_wait_limit(0, kernel=S.KERNEL_KMEANS_LOOP)
    _clean_call_matches_oracle(op, w, Q, K, V)
