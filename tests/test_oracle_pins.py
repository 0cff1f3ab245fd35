"""Pins of the fp64 oracle to things other than itself (CPU only).

Each test checks one oracle function, or a whole call from its own partition, against a closed
form, a library routine (torch SDPA, scikit-learn k-means, numpy lstsq and SVD, scipy orth),
brute force on a tiny input, or a hand-worked fixture under tests/golden/ whose derivation is
written in the fixture.  They are chosen so that a plausible slip (a dropped term, a wrong sign
or scale, a transposed operand, an off-by-one in a sampling formula, a swapped argument in the
call) fails at least one of them; test_oracle_mutations.py plants such slips and checks that.
"""
import json
import math
import os

import types

import numpy as np
import pytest
import scipy.linalg
import torch

from oracle import sparsepr_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- random draws
def test_splitmix64_published_vectors():
    for case in _gold("splitmix64_vectors.json")["cases"]:
        r = O.SplitMix64(case["seed"])
        assert [r.next() for _ in case["outputs"]] == case["outputs"]


def test_kmeans_init_ids_is_a_partial_fisher_yates():
    # Brute force: the same shuffle on an explicit full array.
    for n, c, seed in [(10, 10, 3), (1000, 16, 77), (37, 5, 2**63 + 11)]:
        arr = list(range(n))
        r = O.SplitMix64(seed)
        for i in range(c):
            j = i + r.next() % (n - i)
            arr[i], arr[j] = arr[j], arr[i]
        ids = O.kmeans_init_ids(n, c, seed)
        assert ids == arr[:c]
        assert len(set(ids)) == c and all(0 <= x < n for x in ids)
    assert sorted(O.kmeans_init_ids(50, 50, 9)) == list(range(50))


def test_stream_seeds_differ_per_head_and_stage():
    seeds = {O.stream_seed(5, bh, st) for bh in range(4) for st in range(2)}
    assert len(seeds) == 8


# ---------------------------------------------------------------- sampling
def test_sample_query_rows_formula():
    assert list(O.sample_query_rows(8, 8)) == list(range(8))
    assert list(O.sample_query_rows(10, 1)) == [5]
    assert list(O.sample_query_rows(10, 2)) == [2, 7]
    r = O.sample_query_rows(118800, 1024)
    assert np.all(np.diff(r) > 0) and r[0] >= 0 and r[-1] < 118800


# ---------------------------------------------------------------- attention
def _sdpa(q, k, v, mask=None):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))[None, None]
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=m)[0, 0].numpy()


def test_dense_attention_matches_torch_sdpa():
    rng = np.random.default_rng(0)
    q, k, v = rng.standard_normal((7, 16)), rng.standard_normal((23, 16)), rng.standard_normal((23, 5))
    np.testing.assert_allclose(O.attention(q * 3, k, v), _sdpa(q * 3, k, v), rtol=1e-12, atol=1e-12)


def test_dense_attention_special_cases():
    rng = np.random.default_rng(1)
    q, k = rng.standard_normal((4, 8)), rng.standard_normal((9, 8))
    v = np.tile(rng.standard_normal((1, 3)), (9, 1))
    np.testing.assert_allclose(O.attention(q, k, v), np.tile(v[:1], (4, 1)), rtol=0, atol=1e-14)
    np.testing.assert_allclose(O.attention(q, k[:1], v[:1] * 2), np.tile(v[:1] * 2, (4, 1)), atol=1e-14)
    # a key far more aligned than the others takes all the mass
    kk = np.zeros((3, 8)); kk[1, 0] = 1000.0
    qq = np.zeros((1, 8)); qq[0, 0] = 1.0
    vv = np.eye(3)
    np.testing.assert_allclose(O.attention(qq, kk, vv), [[0, 1, 0]], atol=1e-12)


def test_sparse_attention_matches_masked_sdpa():
    rng = np.random.default_rng(2)
    N, d = 40, 8
    q, k, v = rng.standard_normal((N, d)), rng.standard_normal((N, d)), rng.standard_normal((N, d))
    ql = rng.integers(0, 3, N)
    kl = rng.integers(0, 4, N)
    route = np.array([[1, 0, 1, 0], [0, 1, 0, 0], [1, 1, 1, 1]], dtype=bool)
    mask = route[ql][:, kl]
    np.testing.assert_allclose(O.sparse_attention(q, k, v, ql, kl, route), _sdpa(q, k, v, mask),
                               rtol=1e-12, atol=1e-12)
    full = np.ones((3, 4), dtype=bool)
    np.testing.assert_allclose(O.sparse_attention(q, k, v, ql, kl, full), O.attention(q, k, v), atol=1e-13)
    # a query group that keeps no key group has no keys to attend to: its rows are the empty sum, 0
    none = route.copy()
    none[1] = False
    out = O.sparse_attention(q, k, v, ql, kl, none)
    assert np.all(out[ql == 1] == 0.0)
    np.testing.assert_allclose(out[ql != 1], _sdpa(q, k, v, mask)[ql != 1], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- k-means
def _blobs(rng, n_per, centres, spread):
    pts = [c + spread * rng.standard_normal((n_per, centres.shape[1])) for c in centres]
    return np.concatenate(pts)


def test_lloyd_matches_scikit_learn():
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(3)
    X = _blobs(rng, 30, 4.0 * rng.standard_normal((6, 5)), 1.0)
    init = X[[0, 31, 62, 95, 130, 170]]
    res = O.lloyd(X, init, iters=100, tol=0.0)
    km = KMeans(n_clusters=6, init=init, n_init=1, max_iter=100, tol=0.0, algorithm="lloyd").fit(X)
    assert np.array_equal(res.labels, km.labels_)
    np.testing.assert_allclose(res.centroids, km.cluster_centers_, rtol=1e-12, atol=1e-12)


def test_lloyd_objective_non_increasing_and_fixed_point():
    rng = np.random.default_rng(4)
    X = rng.standard_normal((300, 4))
    res = O.lloyd(X, X[:12], iters=50, tol=0.0)
    J = np.array(res.objective)
    assert np.all(np.diff(J) <= 1e-9 * J[:-1])
    # J_0 is recorded at the first assignment: each point's squared distance to its nearest
    # initial centroid, by brute force
    J0 = sum(min(float(np.sum((x - c) ** 2)) for c in X[:12]) for x in X)
    assert J[0] == pytest.approx(J0, rel=1e-12)
    again = O.lloyd(X, res.centroids, iters=1, tol=0.0)
    assert np.array_equal(again.labels, res.labels)
    np.testing.assert_allclose(again.centroids, res.centroids, atol=1e-13)


def test_lloyd_recovers_generator_tiles():
    from free_block_sparse_02_b200 import configs, gen
    w = configs.workload(0)
    Q, K, V = gen.make_qkv(w)
    k = gen.as_f64(K)[0, 0]
    tiles = gen.token_tiles(w)
    first = [int(np.flatnonzero(tiles == t)[0]) for t in range(w.n_tiles)]
    res = O.lloyd(k, k[first], iters=20, tol=0.0)
    assert np.array_equal(res.labels, tiles)


def test_lloyd_empty_group_keeps_centroid_and_shadow():
    X = np.array([[0.0], [0.1], [10.0]])
    init = np.array([[0.0], [10.0], [100.0]])
    res = O.lloyd(X, init, iters=3, tol=0.0, shadow=X * 2, shadow_init=init * 2)
    assert list(res.labels) == [0, 0, 1]
    assert res.centroids[2, 0] == 100.0 and res.shadow[2, 0] == 200.0
    np.testing.assert_allclose(res.shadow[:2, 0], [0.1, 20.0])


def test_lloyd_tolerance_stop_rule():
    rng = np.random.default_rng(5)
    X = rng.standard_normal((400, 3))
    res = O.lloyd(X, X[:8], iters=100, tol=1e-2)
    J = res.objective
    assert res.n_iter == len(J)
    if res.n_iter < 100:
        assert J[-2] - J[-1] <= 1e-2 * J[-2]
    for a, b in zip(J[:-2], J[1:-1]):
        assert a - b > 1e-2 * a
    never = O.lloyd(X, X[:8], iters=7, tol=-1.0)
    assert never.n_iter == 7
    # tol = 0: the run ends at the first iteration that leaves the objective unchanged (a fixed
    # point of Lloyd's map gives bit-identical centroids, so the decrease is exactly 0)
    zero = O.lloyd(X, X[:8], iters=200, tol=0.0)
    assert zero.n_iter < 200 and zero.objective[-1] == zero.objective[-2]
    assert all(a > b for a, b in zip(zero.objective[:-2], zero.objective[1:-1]))
    # the earliest stop is at iteration 1: a start at a fixed point takes exactly two iterations
    assert O.lloyd(X, zero.centroids, iters=10, tol=0.0).n_iter == 2


def test_near_tie_margin_flags_equidistant_point():
    X = np.array([[0.0], [1.0], [2.0]])
    labels, d1, margin = O.assign(X, np.array([[0.0], [2.0]]))
    assert list(labels) == [0, 0, 1]          # the midpoint goes to the lower index
    assert margin[1] == 0.0 and margin[0] == np.inf
    # the margin is relative: x = 0.5 against centroids 0 and 2 has d1 = 0.25, d2 = 2.25
    _, _, m = O.assign(np.array([[0.5]]), np.array([[0.0], [2.0]]))
    assert m[0] == pytest.approx(8.0, rel=1e-15)
    # a near-tie at any iteration stays flagged: the midpoint ties only at the first assignment
    # (centroids 0 and 2), and after the update (0.5 and 2) it does not
    res = O.lloyd(X, np.array([[0.0], [2.0]]), iters=3, tol=-1.0)
    assert res.near_ties == [1, 0, 0] and list(res.near_tie_mask) == [False, True, False]


def test_key_response_kmeans_equals_metric_kmeans_in_key_space():
    """k-means on rows of F = K Qs^T / sqrt(d) equals Euclidean k-means on K L with
    L L^T = Qs^T Qs / d (a different space and a library k-means)."""
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(6)
    d, s = 6, 20
    K = _blobs(rng, 25, 3.0 * rng.standard_normal((5, d)), 0.7)
    Qs = rng.standard_normal((s, d))
    F = K @ Qs.T / math.sqrt(d)
    ids = [0, 26, 52, 77, 101]
    res = O.lloyd(F, F[ids], iters=60, tol=0.0, shadow=K, shadow_init=K[ids])
    L = np.linalg.cholesky(Qs.T @ Qs / d)
    Z = K @ L
    km = KMeans(n_clusters=5, init=Z[ids], n_init=1, max_iter=60, tol=0.0, algorithm="lloyd").fit(Z)
    assert np.array_equal(res.labels, km.labels_)
    # the shadow (key-space) centroids map onto the response-space centroids
    np.testing.assert_allclose(res.shadow @ Qs.T / math.sqrt(d), res.centroids, rtol=1e-10, atol=1e-10)


# ---------------------------------------------------------------- responses
def test_query_responses_and_rms():
    rng = np.random.default_rng(7)
    q, c = rng.standard_normal((5, 16)), rng.standard_normal((3, 16))
    R = O.query_responses(q, c)
    np.testing.assert_allclose(R[2, 1], float(q[2] @ c[1]) / 4.0, rtol=1e-14)
    Rt = O.rms_normalize(R)
    np.testing.assert_allclose(np.mean(Rt ** 2, axis=1), 1.0, rtol=1e-9)
    np.testing.assert_allclose(O.rms_normalize(7.5 * R), Rt, rtol=1e-10)  # the 1e-12 epsilon
    assert np.all(np.sign(Rt) == np.sign(R))
    assert np.all(O.rms_normalize(np.zeros((2, 3))) == 0.0)


# ---------------------------------------------------------------- routing
def test_route_group_hand_cases():
    g = _gold("routing_cases.json")
    S, m = np.array(g["scores"]), np.array(g["sizes"])
    for case in g["cases"]:
        assert O.route_group(S, m, case["fixed_k"], case["kappa"]) == case["expected"], case


def test_routing_scores_hand_case():
    c = _gold("routing_cases.json")["score_case"]
    S = O.routing_scores(np.array(c["R"]), np.array(c["qlabels"]), c["n_qgroups"], np.array(c["ksizes"]))
    np.testing.assert_allclose(S[0], c["expected_row0"], rtol=1e-15)
    assert np.all(np.isneginf(S[1]))


def test_routing_scores_pool_by_linearity():
    # mean of responses == response of the mean query (a different computation path)
    rng = np.random.default_rng(8)
    q, kc = rng.standard_normal((30, 8)), rng.standard_normal((4, 8))
    ql = rng.integers(0, 3, 30)
    m = np.array([3, 0, 5, 9])
    S = O.routing_scores(O.query_responses(q, kc), ql, 3, m)
    for g in range(3):
        qbar = q[ql == g].mean(axis=0)
        ref = kc @ qbar / math.sqrt(8) + np.log(np.where(m > 0, m, 1))
        np.testing.assert_allclose(S[g][m > 0], ref[m > 0], rtol=1e-12)
        assert np.isneginf(S[g][1])


def test_per_row_key_budget():
    # kappa*N + (s + Ck + P)*N == rho*N^2 : the target counts routing and probe pairs
    N, s, Ck, P = 16384, 256, 64, 128
    kap = O.per_row_key_budget(0.22, N, s, Ck, P)
    assert abs((kap + s + Ck + P) * N / N ** 2 - float(np.float32(0.22))) < 1e-12


# ---------------------------------------------------------------- probes
def test_probes_uniform_formula():
    t, w = O.probes_uniform(10, 2)
    assert list(t) == [2, 7] and list(w) == [1.0, 1.0]
    t, _ = O.probes_uniform(1024, 32)
    assert t[0] == 16 and t[-1] == 1008 and np.all(np.diff(t) == 32)


def test_probes_stratified_hand_cases():
    for c in _gold("stratified_probe_cases.json")["cases"]:
        t, w = O.probes_stratified(np.array(c["labels"]), c["n_qgroups"], c["P"])
        assert list(t) == c["tokens"]
        np.testing.assert_allclose(w, c["weights"], rtol=1e-14)


def test_probes_stratified_invariants():
    rng = np.random.default_rng(9)
    ql = rng.integers(0, 17, 5000)
    ql[ql == 3] = 4                       # an empty group
    t, w = O.probes_stratified(ql, 17, 128)
    assert len(t) == 128 and len(set(t.tolist())) == 128 and np.all(np.diff(t) > 0)
    np.testing.assert_allclose(w.sum(), 128.0, rtol=1e-13)
    n = np.bincount(ql, minlength=17)
    m = np.bincount(ql[t], minlength=17)
    assert np.all(np.abs(m - 128 * n / 5000) < 1.0 + 1e-12) and m[3] == 0


# ---------------------------------------------------------------- ridge and projection
def test_ridge_exact_when_residual_is_affine():
    rng = np.random.default_rng(10)
    P, d = 40, 6
    osp = rng.standard_normal((P, d))
    Btrue = rng.standard_normal((d + 1, d))
    od = osp + np.hstack([osp, np.ones((P, 1))]) @ Btrue
    A, lam = O.ridge_fit(osp, od, rng.uniform(0.5, 2.0, P), 0.0)
    assert lam == 0.0
    np.testing.assert_allclose(A, Btrue, rtol=1e-10, atol=1e-10)


def test_ridge_matches_augmented_lstsq():
    rng = np.random.default_rng(11)
    P, d = 25, 5
    osp, od, w = rng.standard_normal((P, d)), rng.standard_normal((P, d)), rng.uniform(0.2, 3.0, P)
    A, lam = O.ridge_fit(osp, od, w, -1.0)
    X = np.hstack([osp, np.ones((P, 1))])
    G = X.T @ (w[:, None] * X)
    assert lam == pytest.approx(1e-3 * np.trace(G) / (d + 1), rel=1e-14)
    Xa = np.vstack([np.sqrt(w)[:, None] * X, math.sqrt(lam) * np.eye(d + 1)])
    Ra = np.vstack([np.sqrt(w)[:, None] * (od - osp), np.zeros((d + 1, d))])
    ref = np.linalg.lstsq(Xa, Ra, rcond=None)[0]
    np.testing.assert_allclose(A, ref, rtol=1e-10, atol=1e-11)
    # normal equations: X^T W (R - X A) = lam A
    np.testing.assert_allclose(X.T @ (w[:, None] * ((od - osp) - X @ A)), lam * A, atol=1e-11)
    A1, lam1 = O.ridge_fit(osp, od, w, 1.0)
    assert lam1 == 1.0 and not np.allclose(A1, A)


def test_ridge_mean_only_special_case():
    rng = np.random.default_rng(12)
    P, d = 9, 4
    R, w = rng.standard_normal((P, d)), rng.uniform(0.5, 1.5, P)
    A, _ = O.weighted_ridge(np.ones((P, 1)), R, w, 0.0)
    np.testing.assert_allclose(A[0], (w[:, None] * R).sum(0) / w.sum(), rtol=1e-13)
    A, lam = O.weighted_ridge(np.ones((P, 1)), R, w, 2.0)
    np.testing.assert_allclose(A[0], (w[:, None] * R).sum(0) / (w.sum() + 2.0), rtol=1e-13)


def test_residual_span_projection():
    rng = np.random.default_rng(13)
    P, d = 5, 12                                     # rank-deficient: span has dimension 5
    R, w = rng.standard_normal((P, d)), rng.uniform(0.5, 1.5, P)
    U = O.residual_span_basis(R, w)
    assert U.shape == (d, P)
    Qo = scipy.linalg.orth(R.T)
    np.testing.assert_allclose(U @ U.T, Qo @ Qo.T, atol=1e-12)
    A = rng.standard_normal((d + 1, d))
    PA = O.restrict_to_residual_span(A, R, w)
    np.testing.assert_allclose(PA, A @ Qo @ Qo.T, atol=1e-12)
    np.testing.assert_allclose(O.restrict_to_residual_span(PA, R, w), PA, atol=1e-12)
    # the ridge solution already lies in the span: the projection leaves it unchanged
    osp = rng.standard_normal((P, d))
    A2, _ = O.ridge_fit(osp, osp + R, w, 0.5)
    np.testing.assert_allclose(O.restrict_to_residual_span(A2, R, w), A2, atol=1e-12)
    assert O.residual_span_basis(np.zeros((3, 4)), np.ones(3)).shape == (4, 0)


def test_apply_correction_and_row_errors():
    osp = np.array([[1.0, 2.0]])
    A = np.array([[1.0, 0.0], [0.0, 2.0], [0.5, -1.0]])
    np.testing.assert_allclose(O.apply_correction(osp, A), [[1 + 1 + 0.5, 2 + 4 - 1]])
    e = O.row_errors(np.array([[3.0, 4.0], [1.0, 1.0]]), np.array([[0.0, 0.0], [1.0, 1.0]]))
    np.testing.assert_allclose(e, [5.0 / 1e-8, 0.0])


# ---------------------------------------------------------------- whole call
class _Cfg:
    s, n_kgroups, n_qgroups, density, fixed_k, P, probe_mode = 16, 4, 4, 0.5, 0, 6, 1
    lam, km_iters, km_iters_warm, km_tol, seed = -1.0, 8, 2, 1e-4, 99


def _small_inputs(seed=14, N=96, d=8):
    rng = np.random.default_rng(seed)
    centres = 2.0 * rng.standard_normal((6, d))
    lab = np.repeat(np.arange(6), N // 6)
    q = centres[lab] + 0.5 * rng.standard_normal((N, d))
    k = centres[lab] + 0.5 * rng.standard_normal((N, d))
    return q, k, rng.standard_normal((N, d))


def test_call_with_every_group_kept_is_dense():
    q, k, v = _small_inputs()
    cfg = _Cfg()
    cfg.fixed_k = cfg.n_kgroups
    r = O.call_head(q, k, v, cfg, 0)
    dense = O.attention(q, k, v)
    np.testing.assert_allclose(r["osp"], dense, atol=1e-13)
    np.testing.assert_allclose(r["O"], dense, atol=1e-13)
    assert np.abs(r["A"]).max() < 1e-12
    N = q.shape[0]
    assert r["sparse_pairs"] == N * N
    assert r["density"] == pytest.approx(1.0 + (cfg.s + cfg.n_kgroups + cfg.P) / N)


def test_call_constant_values_are_exact():
    q, k, v = _small_inputs(15)
    v[:] = np.array([0.5, -1.0, 2.0, 0.0, 1.0, 3.0, -2.0, 0.25])
    r = O.call_head(q, k, v, _Cfg(), 0)
    np.testing.assert_allclose(r["O"], np.tile(v[:1], (q.shape[0], 1)), atol=1e-12)


def test_call_partition_is_consistent():
    q, k, v = _small_inputs(16)
    cfg = _Cfg()
    r = O.call_head(q, k, v, cfg, 3)
    assert np.array_equal(np.bincount(r["klabels"], minlength=4), r["ksizes"])
    # key-space centroids are the means of their groups' keys
    for j in range(4):
        if r["ksizes"][j]:
            np.testing.assert_allclose(r["kcent"][j], k[r["klabels"] == j].mean(0), atol=1e-13)
    assert np.all(r["route"].sum(1)[r["qsizes"] > 0] >= 1)
    assert np.all(r["O"][r["probes"]] == r["odense"])
    # warm start from the state of this call runs the warm iteration limit
    r2 = O.call_head(q, k, v, cfg, 3, warm=O.warm_state(r))
    assert r2["kmeans_k"].n_iter <= cfg.km_iters_warm
    assert np.array_equal(r2["klabels"], r["klabels"])


class _Cfg53(_Cfg):
    """Unequal group counts (5 key groups, 3 query groups), so that a swapped label array or
    group count in the call changes the result."""
    n_kgroups, n_qgroups = 5, 3


def test_call_routes_and_sparse_rows_follow_its_partition():
    """The later stages of a whole call, checked from the call's own partition by other routes,
    for the response-coupled and the semantic partition alike:
    - the routing scores by pooling: the response of the group's mean query to each key-group
      centroid (the member keys' means) plus ln m_j;
    - the per-row key budget by the density it must reach with the routing and probe pairs;
    - the block-sparse rows by torch SDPA under the mask route[g(q), j(k)];
    - the executed pairs and the realised density by counting that mask;
    - the stratified probes by their per-group counts."""
    q, k, v = _small_inputs(17)
    N, d = q.shape
    for partition in (0, 1):
        cfg = _Cfg53()
        cfg.partition = partition
        r = O.call_head(q, k, v, cfg, 1)
        kl, ql = r["klabels"], r["qlabels"]
        m = np.bincount(kl, minlength=cfg.n_kgroups)
        n = np.bincount(ql, minlength=cfg.n_qgroups)
        assert np.count_nonzero(m) > 1 and np.count_nonzero(n) > 1
        cent = np.array([k[kl == j].mean(0) if m[j] else np.zeros(d) for j in range(cfg.n_kgroups)])
        for g in np.flatnonzero(n):
            pooled = cent @ q[ql == g].mean(0) / math.sqrt(d) + np.log(np.maximum(m, 1))
            np.testing.assert_allclose(r["scores"][g][m > 0], pooled[m > 0], rtol=1e-12, atol=1e-12)
            assert np.all(np.isneginf(r["scores"][g][m == 0]))
        # the budget leaves room for s*N routing, C_k*N centroid and P*N probe pairs
        assert abs((r["kappa"] + cfg.s + cfg.n_kgroups + cfg.P) / N - float(np.float32(cfg.density))) < 1e-12
        mask = r["route"][ql][:, kl]
        np.testing.assert_allclose(r["osp"], _sdpa(q, k, v, mask), rtol=1e-12, atol=1e-12)
        # executed pairs counted on the mask, and the realised density they give with the
        # routing, centroid and probe pairs
        assert r["sparse_pairs"] == int(mask.sum())
        assert r["density"] == pytest.approx((cfg.s + cfg.n_kgroups + cfg.P) / N + mask.sum() / N ** 2, rel=1e-14)
        per_group = np.bincount(ql[r["probes"]], minlength=cfg.n_qgroups)
        assert per_group.sum() == cfg.P and np.all(np.abs(per_group - cfg.P * n / N) < 1.0)


def _fit_rows(r):
    X = np.hstack([r["osp"][r["probes"]], np.ones((len(r["probes"]), 1))])
    return X, r["odense"] - r["osp"][r["probes"]], r["weights"]


def test_call_fit_is_the_weighted_ridge_of_its_probe_residuals():
    """The map a whole call applies, checked from its own probe rows by other routes.
    - The ridge solution: augmented least squares (numpy lstsq) on X = [O_sp(p), 1],
      R = O_dense(p) - O_sp(p) and the call's probe weights, with lam the call reports.
    - The residual span: the right singular vectors of W^(1/2) R (numpy SVD) whose squared
      singular value is above 1e-10 of the largest.  With P < d that span is a proper subspace,
      so a projection on another one would show.
    - The map: the ridge solution times the projector on that span.  With a truncation rank r
      the projector is on the r leading vectors.
    - The mean-only family: no linear part, and the shrunk weighted mean residual, in the same
      span, as the intercept."""
    q, k, v = _small_inputs(18)
    cfg = _Cfg53()
    r = O.call_head(q, k, v, cfg, 0)
    X, R, w = _fit_rows(r)
    d = q.shape[1]
    assert len(w) < d and np.ptp(w) > 0            # a proper span and unequal weights
    lam = r["lam"]
    Xa = np.vstack([np.sqrt(w)[:, None] * X, math.sqrt(lam) * np.eye(d + 1)])
    Ra = np.vstack([np.sqrt(w)[:, None] * R, np.zeros((d + 1, d))])
    A_ridge = np.linalg.lstsq(Xa, Ra, rcond=None)[0]
    _, sv, Vt = np.linalg.svd(np.sqrt(w)[:, None] * R)
    V = Vt[:int(np.sum(sv ** 2 > 1e-10 * sv[0] ** 2))].T
    assert V.shape[1] < d
    scale = np.abs(A_ridge).max()
    np.testing.assert_allclose(r["A"], A_ridge @ V @ V.T, rtol=0, atol=1e-9 * scale)

    cfg.trunc_rank = 2
    rt = O.call_head(q, k, v, cfg, 0)
    assert np.array_equal(rt["probes"], r["probes"])
    np.testing.assert_allclose(rt["A"], A_ridge @ V[:, :2] @ V[:, :2].T, rtol=0, atol=1e-9 * scale)

    cfg.trunc_rank, cfg.correction = 0, 1
    rm = O.call_head(q, k, v, cfg, 0)
    assert not np.any(rm["A"][:-1])
    mean = (w[:, None] * R).sum(0) / (w.sum() + rm["lam"])
    np.testing.assert_allclose(rm["A"][-1], mean @ V @ V.T, rtol=0, atol=1e-12 * np.abs(mean).max())


def test_table2_error_reduction_arithmetic():
    t = _gold("table2_error_reduction.json")
    red = [100 * O.error_reduction(b, a) for a, b in zip(t["semantic_mean"], t["sparsepr_mean"])]
    lo, hi = t["stated_reduction_range_pct"]
    assert round(min(red), 1) == lo and round(max(red), 1) == hi
    # Figure 4(a): the gain of the response-coupled partition, SparsePR against the semantic
    # partition with the same probe repair, for the mean and the p99 error
    for ours, base, key in (("sparsepr_mean", "semantic_repair_mean", "fig4_mean_range_pct"),
                            ("sparsepr_p99", "semantic_repair_p99", "fig4_p99_range_pct")):
        red = [100 * O.error_reduction(a, b) for a, b in zip(t[ours], t[base])]
        assert [round(min(red), 1), round(max(red), 1)] == t[key], (key, red)


def test_repair_reduces_error_on_smooth_field_inputs():
    """On inputs whose sparse residual is affine-predictable (the smooth-field recipe), the
    whole oracle call reproduces what Table 2 and the abstract report: the probe-fitted repair
    lowers the mean unprobed-row error well below both the same partition without repair and the
    semantic partition without repair (the abstract's 61.6-90.5% reduction)."""
    from free_block_sparse_02_b200 import configs, gen
    w = configs.workload(0, recipe="field", probe_mode=configs.PROBE_STRATIFIED)
    Q, K, V = gen.make_qkv(w)
    q, k, v = (gen.as_f64(x)[0, 0] for x in (Q, K, V))
    dense = O.attention(q, k, v)
    err = {}
    for name, ww in (("sparsepr", w), ("no-repair", w.replace(repair=0)),
                     ("semantic", w.replace(partition=configs.PARTITION_SEMANTIC, repair=0))):
        r = O.call_head(q, k, v, ww, 0)
        err[name] = O.mean_error(r["O"], dense, np.setdiff1d(np.arange(w.N), r["probes"]))
    assert err["sparsepr"] < 0.6 * err["no-repair"]
    assert O.error_reduction(err["sparsepr"], err["semantic"]) > 0.5, err


def test_random_probes_are_the_seeded_fisher_yates_draw():
    """Random probe rows: P distinct rows of [0, N), ascending, weight 1; the same rows as a
    brute-force partial Fisher-Yates over an explicit array driven by the SplitMix64 outputs;
    a different head (or seed) gives a different draw; P = N gives every row."""
    N, P, seed = 500, 40, 77
    ids, w = O.probes_random(N, P, seed, bh=3)
    assert ids.shape == (P,) and np.all(np.diff(ids) > 0) and ids.min() >= 0 and ids.max() < N
    assert np.all(w == 1.0)
    rng = O.SplitMix64((seed + (1 << 63) + 2 * 3) & ((1 << 64) - 1))
    arr = list(range(N))
    for i in range(P):
        j = i + rng.next() % (N - i)
        arr[i], arr[j] = arr[j], arr[i]
    assert np.array_equal(ids, np.sort(arr[:P]))
    assert not np.array_equal(ids, O.probes_random(N, P, seed, bh=4)[0])
    assert np.array_equal(O.probes_random(64, 64, seed, bh=0)[0], np.arange(64))
    # the probe stream never coincides with a k-means stream of any head
    assert all(O.probe_stream_seed(seed, b) != O.stream_seed(seed, h, st)
               for b in range(8) for h in range(8) for st in (0, 1))


def test_mean_only_correction_is_the_weighted_mean_residual():
    """Table 4's mean-only family: no linear part and the weighted mean probe residual as the
    intercept (lambda = 0), shrunk by lambda otherwise, and the automatic lambda is 1e-3 of the
    weight sum."""
    rng = np.random.default_rng(11)
    osp, od = rng.standard_normal((30, 5)), rng.standard_normal((30, 5))
    w = rng.uniform(0.5, 2.0, 30)
    A, lam = O.mean_fit(osp, od, w, 0.0)
    assert lam == 0.0 and not np.any(A[:-1])
    np.testing.assert_allclose(A[-1], (w[:, None] * (od - osp)).sum(0) / w.sum(), rtol=1e-13)
    A1, _ = O.mean_fit(osp, od, w, 2.5)
    np.testing.assert_allclose(A1[-1], (w[:, None] * (od - osp)).sum(0) / (w.sum() + 2.5), rtol=1e-13)
    _, lam_auto = O.mean_fit(osp, od, w, -1.0)
    assert np.isclose(lam_auto, 1e-3 * w.sum(), rtol=1e-13)


def test_truncated_span_is_the_leading_right_singular_subspace():
    """Output truncation to rank r keeps the r leading eigenvectors of R^T W R, i.e. the r
    leading right singular vectors of W^(1/2) R (checked against the SVD); rank >= the
    numerical rank is the untruncated restriction; the projected map keeps exactly its part
    along those directions."""
    rng = np.random.default_rng(21)
    P, d = 40, 6
    R = rng.standard_normal((P, d)) @ np.diag([5.0, 3.0, 2.0, 1.0, 0.5, 0.1])
    w = rng.uniform(0.5, 2.0, P)
    _, _, Vt = np.linalg.svd(np.sqrt(w)[:, None] * R)
    for r in (1, 2, 4, 5):                          # 5: one direction fewer than the span
        U = O.residual_span_basis(R, w, r)
        assert U.shape == (d, r)
        np.testing.assert_allclose(U @ U.T, Vt[:r].T @ Vt[:r], atol=1e-12)
    A = rng.standard_normal((d + 1, d))
    np.testing.assert_allclose(O.restrict_to_residual_span(A, R, w, 2), A @ Vt[:2].T @ Vt[:2], atol=1e-12)
    np.testing.assert_allclose(O.restrict_to_residual_span(A, R, w, d), O.restrict_to_residual_span(A, R, w, 0),
                               atol=1e-12)


def test_mean_error_is_the_row_error_mean():
    rng = np.random.default_rng(3)
    O_, R_ = rng.standard_normal((6, 4)), rng.standard_normal((6, 4))
    rows = np.array([0, 2, 5])
    expect = np.mean([np.linalg.norm(O_[i] - R_[i]) / (np.linalg.norm(R_[i]) + 1e-8) for i in rows])
    assert np.isclose(O.mean_error(O_, R_, rows), expect, rtol=1e-14)


def test_repair_off_keeps_sparse_rows_and_exact_probes():
    w = types.SimpleNamespace(s=8, n_kgroups=4, n_qgroups=4, density=0.5, fixed_k=2, P=6, probe_mode=0,
                              lam=-1.0, km_iters=4, km_iters_warm=0, km_tol=-1.0, seed=5, repair=0)
    q, k, v = (np.random.default_rng(i).standard_normal((64, 8)) for i in range(3))
    r = O.call_head(q, k, v, w, 0)
    unprobed = np.setdiff1d(np.arange(64), r["probes"])
    assert np.array_equal(r["O"][unprobed], r["osp"][unprobed])
    assert np.array_equal(r["O"][r["probes"]], r["odense"])
    assert not np.any(r["A"])


def test_semantic_partition_is_kmeans_on_the_raw_inputs():
    """The semantic baseline's key groups are Lloyd's k-means of the raw keys (the same seeded
    initial points and limits), pinned against scikit-learn from those initial centroids."""
    from sklearn.cluster import KMeans
    w = types.SimpleNamespace(s=8, n_kgroups=5, n_qgroups=3, density=0.5, fixed_k=2, P=6, probe_mode=0,
                              lam=-1.0, km_iters=50, km_iters_warm=0, km_tol=-1.0, seed=9, partition=1,
                              repair=0)
    rng = np.random.default_rng(4)
    centres = 4 * rng.standard_normal((5, 8))
    k = centres[rng.integers(0, 5, 80)] + 0.3 * rng.standard_normal((80, 8))
    q = centres[rng.integers(0, 5, 80)] + 0.3 * rng.standard_normal((80, 8))
    v = rng.standard_normal((80, 8))
    r = O.call_head(q, k, v, w, 2)
    ids = O.kmeans_init_ids(80, 5, O.stream_seed(9, 2, 0))
    km = KMeans(n_clusters=5, init=k[ids], n_init=1, max_iter=50, tol=0.0, algorithm="lloyd").fit(k)
    assert np.array_equal(r["klabels"], km.labels_)
    ids = O.kmeans_init_ids(80, 3, O.stream_seed(9, 2, 1))
    kq = KMeans(n_clusters=3, init=q[ids], n_init=1, max_iter=50, tol=0.0, algorithm="lloyd").fit(q)
    assert np.array_equal(r["qlabels"], kq.labels_)


# ---------------------------------------------------------------- warm start (streaming calls)
class _WarmCfg:
    s, n_kgroups, n_qgroups, density, fixed_k, P, probe_mode = 16, 6, 5, 0.5, 0, 6, 1
    lam, km_tol, seed = -1.0, -1.0, 31

    def __init__(self, km_iters, km_iters_warm):
        self.km_iters, self.km_iters_warm = km_iters, km_iters_warm


def _rms_rows(C):
    return np.sqrt(np.mean(C * C, axis=1))


def test_warm_start_restarts_lloyd_where_the_previous_call_stopped():
    """On the same inputs, a call of a Lloyd iterations followed by a warm-started call of b
    iterations must end where one cold call of a + b iterations ends: the state of Lloyd's method
    is its centroids, and the warm start hands them over (keys in key space, re-projected through
    the sampled queries; queries in the previous call's response coordinates, unchanged).  The
    key groups have converged by iteration a, so both calls see the same response coordinates;
    the query groups have not, so the pin has teeth: a warm start that re-normalised the carried
    query centroids, or restarted from the seeded points, would end elsewhere."""
    q, k, v = _small_inputs(39)
    a, b = 4, 4
    ra = O.call_head(q, k, v, _WarmCfg(a, 0), 2, compute_outputs=False)
    rab = O.call_head(q, k, v, _WarmCfg(a + b, 0), 2, compute_outputs=False)
    # preconditions: keys converged by a; queries still moving between a and a + b; the carried
    # query centroids are not unit-RMS rows (re-normalising them would move them)
    assert np.array_equal(ra["klabels"], rab["klabels"])
    assert not np.array_equal(ra["qlabels"], rab["qlabels"])
    assert np.abs(_rms_rows(ra["qcent"]) - 1.0).max() > 1e-2
    rw = O.call_head(q, k, v, _WarmCfg(a, b), 2, warm=O.warm_state(ra), compute_outputs=False)
    assert rw["kmeans_k"].n_iter == b and rw["kmeans_q"].n_iter == b
    assert np.array_equal(rw["klabels"], rab["klabels"])
    assert np.array_equal(rw["qlabels"], rab["qlabels"])
    np.testing.assert_allclose(rw["kmeans_q"].objective, rab["kmeans_q"].objective[a:], rtol=1e-12)
    np.testing.assert_allclose(rw["qcent"], rab["qcent"], rtol=1e-12, atol=1e-12)
    # the same restart from re-normalised query centroids does not reproduce it
    bad = O.WarmState(key_centroids=ra["kcent"], query_centroids=O.rms_normalize(ra["qcent"]))
    rb = O.call_head(q, k, v, _WarmCfg(a, b), 2, warm=bad, compute_outputs=False)
    assert not np.allclose(rb["kmeans_q"].objective, rab["kmeans_q"].objective[a:], rtol=1e-9)


def test_warm_start_key_step_uses_the_current_calls_metric():
    """Call 2 sees new queries and keys.  With one warm iteration its key labels are the first
    assignment from the previous call's key-space centroids c_j, in call 2's response space:
    argmin_j (k_t - c_j)^T M2 (k_t - c_j) with M2 = Qs2^T Qs2 / d, evaluated here in key space (the
    metric identity, not the oracle's response-space projection).  The previous call's metric M1
    would give other labels on these inputs."""
    rng = np.random.default_rng(22)
    N, d = 120, 8
    q1, k1, v1 = rng.standard_normal((N, d)), rng.standard_normal((N, d)), rng.standard_normal((N, d))
    stretch = np.array([4.0, 0.25, 3.0, 0.5, 1.0, 2.0, 0.3, 1.5])
    q2, k2, v2 = q1 * stretch + 0.3 * rng.standard_normal((N, d)), rng.standard_normal((N, d)), v1
    cfg = _WarmCfg(6, 1)
    r1 = O.call_head(q1, k1, v1, cfg, 0, compute_outputs=False)
    r2 = O.call_head(q2, k2, v2, cfg, 0, warm=O.warm_state(r1), compute_outputs=False)
    C = r1["kcent"]
    rows = O.sample_query_rows(N, cfg.s)
    M2 = q2[rows].T @ q2[rows] / d
    M1 = q1[rows].T @ q1[rows] / d

    def labels_under(M):
        D = np.array([[(kt - c) @ M @ (kt - c) for c in C] for kt in k2])
        return np.argmin(D, axis=1)

    assert r2["kmeans_k"].n_iter == 1
    assert np.array_equal(r2["klabels"], labels_under(M2))
    assert not np.array_equal(labels_under(M1), labels_under(M2))


def test_warm_start_from_converged_centroids_is_a_fixed_point():
    """A call warm-started from the converged state of the same inputs keeps every label and the
    objectives after one iteration."""
    q, k, v = _small_inputs(23)
    r = O.call_head(q, k, v, _WarmCfg(60, 0), 1, compute_outputs=False, keep_history=True)
    hk, hq = r["kmeans_k"].label_history, r["kmeans_q"].label_history
    assert np.array_equal(hk[-1], hk[-2]) and np.array_equal(hq[-1], hq[-2])  # converged
    rw = O.call_head(q, k, v, _WarmCfg(60, 1), 1, warm=O.warm_state(r), compute_outputs=False)
    assert np.array_equal(rw["klabels"], r["klabels"]) and np.array_equal(rw["qlabels"], r["qlabels"])
    np.testing.assert_allclose(rw["kmeans_k"].objective[0], r["kmeans_k"].objective[-1], rtol=1e-12)
    np.testing.assert_allclose(rw["kmeans_q"].objective[0], r["kmeans_q"].objective[-1], rtol=1e-12)


# ---------------------------------------------------------------- key response rank (Table C.1 r_K)
def test_key_response_basis_is_the_best_rank_r_approximation():
    """Eckart-Young: projecting the responses on their r leading right singular vectors leaves
    exactly the energy of the trailing eigenvalues of F^T F (a separate symmetric eigensolver)."""
    rng = np.random.default_rng(41)
    F = rng.standard_normal((200, 12)) @ rng.standard_normal((12, 30))
    for r in (1, 5, 11):
        Vr = O.key_response_basis(F, r)
        assert Vr.shape == (30, r)
        np.testing.assert_allclose(Vr.T @ Vr, np.eye(r), atol=1e-12)
        resid = np.linalg.norm(F - F @ Vr @ Vr.T) ** 2
        ev = np.sort(np.linalg.eigvalsh(F.T @ F))[::-1]
        np.testing.assert_allclose(resid, ev[r:].sum(), rtol=1e-9, atol=1e-9 * ev[0])
    assert O.key_response_basis(F, 0) is None and O.key_response_basis(F, 30) is None


class _RankCfg(_WarmCfg):
    def __init__(self, key_rank):
        super().__init__(8, 0)
        self.key_rank = key_rank


def test_key_rank_at_or_above_the_response_rank_changes_nothing():
    """F = K Qs^T / sqrt(d) has rank <= d, so its d leading singular directions keep every
    distance: the key groups equal the unprojected ones."""
    q, k, v = _small_inputs(42)
    d = q.shape[1]
    full = O.call_head(q, k, v, _RankCfg(0), 0, compute_outputs=False)
    same = O.call_head(q, k, v, _RankCfg(d), 0, compute_outputs=False)
    assert np.array_equal(full["klabels"], same["klabels"])
    np.testing.assert_allclose(same["kmeans_k"].objective, full["kmeans_k"].objective, rtol=1e-9)


def test_key_rank_equals_metric_kmeans_in_key_space():
    """k-means on the rank-r response coordinates equals Euclidean k-means (scikit-learn) on the
    keys mapped by L Z_r, where M = Qs^T Qs / d = L L^T (Cholesky) and Z_r holds the r leading
    eigenvectors of L^T (K^T K) L: a different route through d x d matrices only."""
    from sklearn.cluster import KMeans
    q, k, v = _small_inputs(43, N=120, d=8)
    cfg = _RankCfg(3)
    r = O.call_head(q, k, v, cfg, 0, compute_outputs=False)
    d = q.shape[1]
    Qs = q[O.sample_query_rows(q.shape[0], cfg.s)]
    Lc = np.linalg.cholesky(Qs.T @ Qs / d)
    ev, Z = np.linalg.eigh(Lc.T @ (k.T @ k) @ Lc)
    Zr = Z[:, np.argsort(-ev)[:cfg.key_rank]]
    Y = k @ Lc @ Zr
    ids = O.kmeans_init_ids(q.shape[0], cfg.n_kgroups, O.stream_seed(cfg.seed, 0, 0))
    km = KMeans(n_clusters=cfg.n_kgroups, init=Y[ids], n_init=1, max_iter=cfg.km_iters, tol=0.0,
                algorithm="lloyd").fit(Y)
    assert np.array_equal(r["klabels"], km.labels_)
    # and the rank matters on these inputs
    assert not np.array_equal(r["klabels"], O.call_head(q, k, v, _RankCfg(0), 0, compute_outputs=False)["klabels"])
