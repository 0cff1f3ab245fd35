"""Plain float64 CPU oracle of the SparsePR per-call sparse attention operator.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or link this module:
only the tests, the package's smoke check and the benchmark's CPU-baseline leg use it.  It
shares no code, constant or helper with the CUDA path.

Source: Taghavi, Langari, Pandey, "Partition the Support, Reconstruct the Residual:
Training-Free Sparse Attention for Video Generation and World Models" (arXiv 2608.18484),
as given by its abstract (listing page and arXiv abstract page) and by the method section of
its project page "SparsePR: Training-Free Sparse Attention for Video Generation".  The pages
print no equation, so each step below is the plainest reading of the prose; every reading is
named in the function that makes it.

The operator, per (batch, head), in the abstract's order:
  1. sample s query rows; the key responses are F = K Q_s^T / sqrt(d)  (one row per key);
  2. k-means on the rows of F -> C_k paired K/V groups; key-group centroids in key space;
  3. query responses R = Q C^T / sqrt(d) to those centroids, per-query RMS normalised
     (Table D.1, "Per query RMS" column, the reference setting);
  4. k-means on the normalised responses -> C_q query groups that share one sparse route;
  5. routing: per query group the kept key groups, to a target executed-pair density that
     counts routing and exact probe pairs (project page, Results: the reported density
     counts the routing and the exact probe pairs too);
  6. block-sparse attention: each query attends only to the keys of its group's kept key
     groups (softmax over the retained keys only);
  7. exact dense attention on P probe rows (Table 4: uniform spatiotemporal or query-group
     stratified probes);
  8. weighted ridge fit of an affine map [O_sp, 1] -> O_dense - O_sp on the probe rows,
     restricted to the output subspace spanned by the probe residuals (arXiv abstract;
     project page, method column "Probe-Fitted Residual Reconstruction");
  9. the predicted residual is added to every unprobed row; probe rows keep their exact
     dense output.

All arithmetic is float64 on the exact values of the (bf16 or fp32) inputs.

Pinned by tests/test_oracle_pins.py against closed forms, library routines (torch SDPA,
scikit-learn k-means, numpy lstsq, scipy orth), brute force on tiny inputs and hand-worked
fixtures under tests/golden/.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence

import numpy as np

NEAR_TIE_REL = 1e-5          # relative distance margin below which a label is a near-tie
SPAN_REL_TOL = 1e-10         # eigenvalues below this fraction of the largest are not in the span
RMS_EPS = 1e-12
ERR_EPS = 1e-8               # Table D.1 caption: ||O_sp - O_dense|| / (||O_dense|| + 1e-8)

_MASK64 = (1 << 64) - 1


# ----------------------------------------------------------------------------------------------
# Random draws of the method: k-means initial points.
# ----------------------------------------------------------------------------------------------
class SplitMix64:
    """SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number generators",
    OOPSLA 2014), the counter-based generator used to draw k-means initial points:
    state += golden gamma; output = mix64 variant 13 of the state."""

    GAMMA = 0x9E3779B97F4A7C15

    def __init__(self, seed: int):
        self.state = seed & _MASK64

    def next(self) -> int:
        self.state = (self.state + self.GAMMA) & _MASK64
        z = self.state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        return z ^ (z >> 31)


def kmeans_init_ids(n_points: int, n_clusters: int, seed: int) -> List[int]:
    """n_clusters distinct point indices by a partial Fisher-Yates shuffle driven by
    SplitMix64(seed): for i = 0..C-1 swap slot i with slot i + (next() mod (n - i)).
    (Reading: the pages say only "seeded init"; this is the plain seeded choice of C
    distinct points.)"""
    if n_clusters > n_points:
        raise ValueError("more clusters than points")
    rng = SplitMix64(seed)
    slots: Dict[int, int] = {}
    out = []
    for i in range(n_clusters):
        j = i + rng.next() % (n_points - i)
        vi = slots.get(i, i)
        vj = slots.get(j, j)
        slots[i], slots[j] = vj, vi
        out.append(vj)
    return out


def stream_seed(seed: int, bh: int, stage: int) -> int:
    """Seed of the k-means draw of head bh: stage 0 = key groups, 1 = query groups."""
    return (seed + 2 * bh + stage) & _MASK64


def probe_stream_seed(seed: int, bh: int) -> int:
    """Seed of head bh's random probe rows: the k-means streams offset by 2^63, so that no
    k-means stream of any head coincides with it."""
    return (seed + (1 << 63) + 2 * bh) & _MASK64


# ----------------------------------------------------------------------------------------------
# Step 1: sampled query rows (abstract: keys are characterised by their responses to sampled
# queries).
# ----------------------------------------------------------------------------------------------
def sample_query_rows(N: int, s: int) -> np.ndarray:
    """Reading: s rows spread evenly over raster token order, row i = floor((2i+1) N / (2s))."""
    i = np.arange(s, dtype=np.int64)
    return ((2 * i + 1) * N) // (2 * s)


# ----------------------------------------------------------------------------------------------
# Steps 2 and 4: Lloyd's k-means.
# ----------------------------------------------------------------------------------------------
@dataclasses.dataclass
class KMeansResult:
    labels: np.ndarray            # int64 (n,)
    centroids: np.ndarray         # (C, D) feature-space centroids after the last update
    shadow: Optional[np.ndarray]  # (C, E) means of the shadow rows per group (key space)
    objective: List[float]        # J at every assignment
    n_iter: int
    near_ties: List[int]          # per iteration: points with relative margin < NEAR_TIE_REL
    near_tie_mask: np.ndarray     # bool (n,): near-tie at any iteration
    final_margin: np.ndarray      # relative margin (d2 - d1) / d1 at the last assignment
    stop_margin: float            # |(J_prev - J)/J_prev - tol| at the stop test (inf if none)
    label_history: List[np.ndarray]


def squared_distances(X: np.ndarray, C: np.ndarray) -> np.ndarray:
    """||x - c||^2 for every (row of X, row of C), by the expansion
    ||x||^2 - 2 x.c + ||c||^2 in float64 (matrix product as a library step)."""
    xx = np.einsum("ij,ij->i", X, X)
    cc = np.einsum("ij,ij->i", C, C)
    D = xx[:, None] - 2.0 * (X @ C.T) + cc[None, :]
    return np.maximum(D, 0.0)


def assign(X: np.ndarray, C: np.ndarray):
    """Nearest centroid, lowest index on exact ties; also the relative margin to the runner-up."""
    D = squared_distances(X, C)
    labels = np.argmin(D, axis=1)              # first minimum = lowest index
    n = X.shape[0]
    d1 = D[np.arange(n), labels]
    if C.shape[0] > 1:
        D2 = D.copy()
        D2[np.arange(n), labels] = np.inf
        d2 = D2.min(axis=1)
    else:
        d2 = np.full(n, np.inf)
    with np.errstate(divide="ignore", invalid="ignore"):
        margin = np.where(d1 > 0, (d2 - d1) / np.where(d1 > 0, d1, 1.0),
                          np.where(d2 > 0, np.inf, 0.0))
    return labels, d1, margin


def lloyd(X: np.ndarray, init_centroids: np.ndarray, iters: int, tol: float,
          shadow: Optional[np.ndarray] = None, shadow_init: Optional[np.ndarray] = None,
          keep_history: bool = False) -> KMeansResult:
    """Lloyd's iterations (Table C.1: iteration limit, tolerance 1e-4).

    Readings: squared Euclidean distance; ties go to the lowest centroid index; an empty
    group keeps its previous centroid (and shadow centroid); iteration it assigns, records
    J_it = sum of distances, updates the centroids, and stops early when it >= 1 and
    J_{it-1} - J_it <= tol * J_{it-1} (tol < 0: never early).  The final centroids are the
    means of the final groups.  `shadow` rows (the keys themselves) are averaged with the same
    labels, giving key-space centroids."""
    C = np.array(init_centroids, dtype=np.float64, copy=True)
    S = None if shadow is None else np.array(shadow_init, dtype=np.float64, copy=True)
    nC = C.shape[0]
    J_hist: List[float] = []
    ties: List[int] = []
    tie_mask = np.zeros(X.shape[0], dtype=bool)
    hist: List[np.ndarray] = []
    stop_margin = math.inf
    labels = np.zeros(X.shape[0], dtype=np.int64)
    margin = np.zeros(X.shape[0])
    it = 0
    for it in range(iters):
        labels, d1, margin = assign(X, C)
        J = float(d1.sum())
        J_hist.append(J)
        nt = margin < NEAR_TIE_REL
        ties.append(int(nt.sum()))
        tie_mask |= nt
        if keep_history:
            hist.append(labels.copy())
        counts = np.bincount(labels, minlength=nC)
        for j in range(nC):
            if counts[j] > 0:
                members = labels == j
                C[j] = X[members].mean(axis=0)
                if S is not None:
                    S[j] = shadow[members].mean(axis=0)
        if tol >= 0 and it >= 1:
            rel = (J_hist[-2] - J) / J_hist[-2] if J_hist[-2] != 0 else 0.0
            stop_margin = abs(rel - tol)
            if J_hist[-2] - J <= tol * J_hist[-2]:
                break
    return KMeansResult(labels=labels, centroids=C, shadow=S, objective=J_hist, n_iter=it + 1,
                        near_ties=ties, near_tie_mask=tie_mask, final_margin=margin,
                        stop_margin=stop_margin, label_history=hist)


def key_response_basis(F: np.ndarray, rank: int) -> Optional[np.ndarray]:
    """Table C.1 "Key response rank r_K" (48 in the paper's runs).  Reading: the N x s key
    responses are taken in the basis of their r_K leading right singular vectors (the best
    rank-r_K approximation of the response matrix, not centred), so k-means sees the r_K-dim
    coordinates F V_r.  Returns V_r (s x r), or None when rank is 0 (off) or not below the
    response matrix's rank bound min(N, s) (the projection would keep every distance)."""
    if rank <= 0 or rank >= min(F.shape):
        return None
    _, _, Vt = np.linalg.svd(F, full_matrices=False)
    return Vt[:rank].T


# ----------------------------------------------------------------------------------------------
# Step 3: query responses to the key-group centroids, per-query RMS normalisation.
# ----------------------------------------------------------------------------------------------
def query_responses(q: np.ndarray, key_centroids: np.ndarray) -> np.ndarray:
    """R = Q C^T / sqrt(d): responses (logits) of every query to every key-group centroid.
    Reading: a "response" is the scaled logit, not a probability."""
    d = q.shape[1]
    return (q @ key_centroids.T) / math.sqrt(d)


def rms_normalize(R: np.ndarray) -> np.ndarray:
    """Table D.1 "Per query RMS": r / sqrt(mean_j r_j^2 + 1e-12), no centring."""
    ms = np.mean(R * R, axis=1, keepdims=True)
    return R / np.sqrt(ms + RMS_EPS)


# ----------------------------------------------------------------------------------------------
# Step 5: routing.
# ----------------------------------------------------------------------------------------------
def routing_scores(R: np.ndarray, qlabels: np.ndarray, n_qgroups: int,
                   ksizes: np.ndarray) -> np.ndarray:
    """S[g, j] = mean over queries of group g of the raw response to key group j, plus ln m_j.

    Reading: the pooled response of the group is its members' mean logit; ln m_j is the
    first-order log-mass of a group of m_j similar keys; empty key groups score -inf."""
    Cq, Ck = n_qgroups, R.shape[1]
    S = np.full((Cq, Ck), -np.inf)
    with np.errstate(divide="ignore"):
        logm = np.where(ksizes > 0, np.log(np.maximum(ksizes, 1).astype(np.float64)), -np.inf)
    for g in range(Cq):
        rows = qlabels == g
        if rows.any():
            S[g] = R[rows].mean(axis=0) + logm
    return S


def per_row_key_budget(density: float, N: int, s: int, n_kgroups: int, P: int) -> float:
    """kappa = rho*N - (s + C_k + P): keys each query may attend to in the block-sparse pass
    so that (s*N routing + C_k*N centroid + P*N probe + sparse) pairs / N^2 = rho.
    rho is taken at the operator's float32 precision."""
    return float(np.float32(density)) * N - (s + n_kgroups + P)


def route_group(S_row: np.ndarray, ksizes: np.ndarray, fixed_k: int, kappa: float) -> List[int]:
    """Kept key groups of one query group (ascending ids).

    Key groups are visited by score, highest first (ties: lower id), empty ones skipped.
    fixed_k > 0: the first fixed_k are kept.  Otherwise the top one is always kept and each
    later group is kept iff it brings the running key count closer to kappa:
    |cum + m_j - kappa| < |cum - kappa|."""
    order = sorted((j for j in range(len(ksizes)) if ksizes[j] > 0), key=lambda j: (-S_row[j], j))
    chosen: List[int] = []
    if fixed_k > 0:
        chosen = order[:fixed_k]
    else:
        cum = 0.0
        for j in order:
            m = float(ksizes[j])
            if not chosen or abs(cum + m - kappa) < abs(cum - kappa):
                chosen.append(j)
                cum += m
    return sorted(chosen)


# ----------------------------------------------------------------------------------------------
# Steps 6 and 7: attention.
# ----------------------------------------------------------------------------------------------
def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """softmax(q k^T / sqrt(d)) v, row-wise, float64.  With no keys the rows are the empty sum, 0."""
    if k.shape[0] == 0:
        return np.zeros((q.shape[0], v.shape[1]))
    s = (q @ k.T) / math.sqrt(q.shape[1])
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p @ v


def sparse_attention(q, k, v, qlabels, klabels, route: np.ndarray) -> np.ndarray:
    """Each query attends only to the keys whose group its query group keeps (hard drop)."""
    out = np.zeros((q.shape[0], v.shape[1]))
    for g in range(route.shape[0]):
        rows = np.flatnonzero(qlabels == g)
        if rows.size == 0:
            continue
        keys = np.flatnonzero(route[g][klabels])
        out[rows] = attention(q[rows], k[keys], v[keys])
    return out


def probes_uniform(N: int, P: int):
    """Table 4 "Uniform spatiotemporal probes": rows floor((2i+1) N / (2P)), weight 1."""
    i = np.arange(P, dtype=np.int64)
    return ((2 * i + 1) * N) // (2 * P), np.ones(P)


def probes_random(N: int, P: int, seed: int, bh: int):
    """Table 4 "Random probes": P distinct rows drawn uniformly at random (the partial
    Fisher-Yates draw of the k-means initial points, on the head's probe stream), in ascending
    token order, weight 1 each."""
    ids = np.sort(np.array(kmeans_init_ids(N, P, probe_stream_seed(seed, bh)), dtype=np.int64))
    return ids, np.ones(P)


def select_probes(cfg, qlabels: np.ndarray, n_qgroups: int, N: int, bh: int):
    """The probe rows and weights of the configured mode: 0 uniform, 1 query-group stratified
    (the paper's reference setting), 2 random."""
    if cfg.probe_mode == 0:
        return probes_uniform(N, cfg.P)
    if cfg.probe_mode == 2:
        return probes_random(N, cfg.P, getattr(cfg, "seed", 0), bh)
    return probes_stratified(qlabels, n_qgroups, cfg.P)


def probes_stratified(qlabels: np.ndarray, n_qgroups: int, P: int):
    """Table 4 "Query group stratified probes" (the reference setting).

    Reading: group g gets m_g = floor(P n_g / N) probes plus one for the largest remainders
    (P n_g mod N, ties to the lower g) until P are placed; inside the group (members in token
    order) probe i sits at member floor((2i+1) n_g / (2 m_g)); its weight is n_g / m_g,
    scaled so the weights sum to P.  Probes are returned in ascending token order."""
    N = qlabels.shape[0]
    n = np.bincount(qlabels, minlength=n_qgroups).astype(np.int64)
    base = (P * n) // N
    rem = (P * n) % N
    extra = int(P - base.sum())
    order = sorted(range(n_qgroups), key=lambda g: (-int(rem[g]), g))
    m = base.copy()
    for g in order[:extra]:
        m[g] += 1
    toks, wts = [], []
    for g in range(n_qgroups):
        if m[g] == 0:
            continue
        members = np.flatnonzero(qlabels == g)
        for i in range(int(m[g])):
            toks.append(int(members[((2 * i + 1) * int(n[g])) // (2 * int(m[g]))]))
            wts.append(float(n[g]) / float(m[g]))
    toks = np.array(toks, dtype=np.int64)
    wts = np.array(wts)
    o = np.argsort(toks, kind="stable")
    toks, wts = toks[o], wts[o]
    if wts.size:
        wts = wts * (P / wts.sum())
    return toks, wts


# ----------------------------------------------------------------------------------------------
# Step 8: probe-fitted residual reconstruction.
# ----------------------------------------------------------------------------------------------
def ridge_lambda(G: np.ndarray, lam_cfg: float) -> float:
    """lam_cfg >= 0: absolute.  Otherwise 1e-3 * tr(X^T W X) / (d+1) (the operator's automatic
    scale; the paper's own runs use lambda = 1, Table 4 and Table D.2)."""
    return float(lam_cfg) if lam_cfg >= 0 else 1e-3 * float(np.trace(G)) / G.shape[0]


def ridge_fit(osp_p: np.ndarray, odense_p: np.ndarray, w: np.ndarray, lam_cfg: float):
    """Weighted ridge regression of the residual on [O_sp, 1] (arXiv abstract: "a call-specific
    affine correction"; Table 4 "full weighted ridge"): A = (X^T W X + lam I)^-1 X^T W R,
    X = [O_sp(p), 1], R = O_dense(p) - O_sp(p), W = diag(w); lam also penalises the intercept.
    Returns (A of shape (d+1, d), lam)."""
    P, d = osp_p.shape
    if P == 0:
        return np.zeros((d + 1, d)), 0.0
    X = np.hstack([osp_p, np.ones((P, 1))])
    return weighted_ridge(X, odense_p - osp_p, w, lam_cfg)


def weighted_ridge(X: np.ndarray, R: np.ndarray, w: np.ndarray, lam_cfg: float):
    """argmin_A sum_p w_p ||R_p - X_p A||^2 + lam ||A||_F^2 = (X^T W X + lam I)^-1 X^T W R.
    With X = ones((P, 1)) this is the mean-only correction family of Table 4."""
    WX = w[:, None] * X
    G = X.T @ WX
    lam = ridge_lambda(G, lam_cfg)
    A = np.linalg.solve(G + lam * np.eye(X.shape[1]), WX.T @ R)
    return A, lam


def residual_span_basis(R: np.ndarray, w: np.ndarray, rank: int = 0) -> np.ndarray:
    """Orthonormal basis (d, r) of the span of the probe residual rows: eigenvectors of
    R^T W R with eigenvalue above SPAN_REL_TOL of the largest (none if all are zero).
    rank > 0 truncates it to the `rank` eigenvectors of largest eigenvalue (Table D.2's output
    truncation; reading: the low-rank probe-residual subspace is the leading one)."""
    d = R.shape[1]
    Sg = R.T @ (w[:, None] * R)
    ev, U = np.linalg.eigh(Sg)
    top = ev.max() if ev.size else 0.0
    if not top > 0:
        return np.zeros((d, 0))
    keep = ev > SPAN_REL_TOL * top
    U, ev = U[:, keep], ev[keep]
    if rank > 0 and U.shape[1] > rank:
        U = U[:, np.argsort(-ev, kind="stable")[:rank]]
    return U


def restrict_to_residual_span(A: np.ndarray, R: np.ndarray, w: np.ndarray, rank: int = 0) -> np.ndarray:
    """Project the fitted map's outputs onto the probe-residual subspace (arXiv abstract page:
    the correction stays inside the span of the probe residuals): A <- A U U^T.
    Without truncation (rank 0) the ridge solution already lies in that span (each output of A
    is a combination of residual rows), so this is the identity up to rounding; with rank r the
    outputs keep only their part along the r leading residual directions."""
    U = residual_span_basis(R, w, rank)
    return A @ U @ U.T


def apply_correction(osp: np.ndarray, A: np.ndarray) -> np.ndarray:
    """O_sp + [O_sp, 1] A for every row."""
    return osp + osp @ A[:-1] + A[-1][None, :]


def row_errors(O: np.ndarray, Oref: np.ndarray) -> np.ndarray:
    """Normalised attention-output error per row (Table D.1 caption)."""
    return np.linalg.norm(O - Oref, axis=1) / (np.linalg.norm(Oref, axis=1) + ERR_EPS)


# ----------------------------------------------------------------------------------------------
# The whole call.
# ----------------------------------------------------------------------------------------------
@dataclasses.dataclass
class WarmState:
    key_centroids: np.ndarray     # (C_k, d) key space
    query_centroids: np.ndarray   # (C_q, C_k) normalised response space


def mean_fit(osp_p: np.ndarray, odense_p: np.ndarray, w: np.ndarray, lam_cfg: float):
    """Table 4 "Mean-only" correction family: the weighted ridge with the constant feature
    alone, A_lin = 0 and intercept (sum_p w_p + lam)^-1 sum_p w_p R_p (lam by the same rule on
    the 1 x 1 Gram).  Returns A of shape (d+1, d) and lam."""
    P, d = osp_p.shape
    A = np.zeros((d + 1, d))
    if P == 0:
        return A, 0.0
    Am, lam = weighted_ridge(np.ones((P, 1)), odense_p - osp_p, w, lam_cfg)
    A[-1] = Am[0]
    return A, lam


def outputs_given_partition(q, k, v, qlabels, klabels, route, probes, weights, lam_cfg, repair=1, correction=0,
                            trunc_rank=0):
    """Steps 6-9 for a given partition, route table and probe set (repair=0: no correction;
    unprobed rows keep their sparse output, probe rows their exact one; correction=1: the
    mean-only family instead of the affine map of [O_sp, 1]; trunc_rank r > 0: the map's outputs
    restricted to the r leading residual directions)."""
    osp = sparse_attention(q, k, v, qlabels, klabels, route)
    odense = attention(q[probes], k, v)
    if repair:
        fit = mean_fit if correction == 1 else ridge_fit
        A, lam = fit(osp[probes], odense, weights, lam_cfg)
        if len(probes):
            A = restrict_to_residual_span(A, odense - osp[probes], weights, trunc_rank)
    else:
        A, lam = np.zeros((q.shape[1] + 1, q.shape[1])), 0.0
    O = apply_correction(osp, A)
    O[probes] = odense
    return dict(osp=osp, odense=odense, A=A, lam=lam, O=O)


def call_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, cfg, bh: int,
              warm: Optional[WarmState] = None, keep_history: bool = False,
              compute_outputs: bool = True) -> dict:
    """One (batch, head) of one call.  cfg needs: s, n_kgroups, n_qgroups, density, fixed_k,
    P, probe_mode (0 uniform, 1 stratified, 2 random), lam, km_iters, km_iters_warm, km_tol,
    seed, and optionally partition (0 response-coupled, 1 semantic), repair (1 correct, 0 not),
    correction (0 affine map of [O_sp, 1], 1 mean-only), trunc_rank (0 none, r > 0 the r
    leading residual directions) and key_rank (0 none, r > 0 the key responses in their r
    leading right singular directions, Table C.1's r_K)."""
    if getattr(cfg, "partition", 0) == 1:
        return semantic_call_head(q, k, v, cfg, bh, compute_outputs=compute_outputs)
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N, d = q.shape
    scale = 1.0 / math.sqrt(d)
    Ck, Cq = cfg.n_kgroups, cfg.n_qgroups
    seed = getattr(cfg, "seed", 0)
    tol = float(np.float32(cfg.km_tol))  # the operator's tolerance is a float32 argument

    # 1-2: key responses to the sampled queries and paired K/V groups.
    rows = sample_query_rows(N, cfg.s)
    Qs = q[rows]
    F = (k @ Qs.T) * scale
    Vr = key_response_basis(F, getattr(cfg, "key_rank", 0))
    if Vr is not None:
        F = F @ Vr
    if warm is None:
        ids = kmeans_init_ids(N, Ck, stream_seed(seed, bh, 0))
        C0, S0, iters = F[ids], k[ids], cfg.km_iters
    else:
        C0 = (warm.key_centroids @ Qs.T) * scale
        if Vr is not None:
            C0 = C0 @ Vr
        S0, iters = warm.key_centroids, cfg.km_iters_warm
    kk = lloyd(F, C0, iters, tol, shadow=k, shadow_init=S0, keep_history=keep_history)
    klabels = kk.labels
    kcent = kk.shadow

    # 3-4: query responses to the key-group centroids, normalised, and query groups.
    R = query_responses(q, kcent)
    Rt = rms_normalize(R)
    if warm is None:
        ids = kmeans_init_ids(N, Cq, stream_seed(seed, bh, 1))
        C0q, iters = Rt[ids], cfg.km_iters
    else:
        C0q, iters = warm.query_centroids, cfg.km_iters_warm
    qq = lloyd(Rt, C0q, iters, tol, keep_history=keep_history)
    qlabels = qq.labels

    # 5: routing.
    m = np.bincount(klabels, minlength=Ck)
    n = np.bincount(qlabels, minlength=Cq)
    S = routing_scores(R, qlabels, Cq, m)
    kappa = per_row_key_budget(cfg.density, N, cfg.s, Ck, cfg.P)
    route = np.zeros((Cq, Ck), dtype=bool)
    for g in range(Cq):
        if n[g] > 0:
            route[g, route_group(S[g], m, cfg.fixed_k, kappa)] = True
    sparse_pairs = int(sum(int(n[g]) * int(m[route[g]].sum()) for g in range(Cq)))
    density = (cfg.s * N + Ck * N + cfg.P * N + sparse_pairs) / float(N) ** 2

    # 7: probes.
    probes, weights = select_probes(cfg, qlabels, Cq, N, bh)

    out = dict(sample_rows=rows, klabels=klabels, kcent=kcent, kmeans_k=kk, R=R, Rt=Rt,
               qlabels=qlabels, qcent=qq.centroids, kmeans_q=qq, ksizes=m, qsizes=n,
               scores=S, kappa=kappa, route=route, sparse_pairs=sparse_pairs, density=density,
               probes=probes, weights=weights)
    if compute_outputs:
        out.update(outputs_given_partition(q, k, v, qlabels, klabels, route, probes, weights, cfg.lam,
                                           repair=getattr(cfg, "repair", 1),
                                           correction=getattr(cfg, "correction", 0),
                                           trunc_rank=getattr(cfg, "trunc_rank", 0)))
    return out


def route_and_probe(q, klabels, qlabels, kcent, cfg, bh: int = 0):
    """Steps 5 and 7 for a given partition: routes, realised density and probes."""
    N = q.shape[0]
    Ck, Cq = cfg.n_kgroups, cfg.n_qgroups
    m = np.bincount(klabels, minlength=Ck)
    n = np.bincount(qlabels, minlength=Cq)
    S = routing_scores(query_responses(q, kcent), qlabels, Cq, m)
    kappa = per_row_key_budget(cfg.density, N, cfg.s, Ck, cfg.P)
    route = np.zeros((Cq, Ck), dtype=bool)
    for g in range(Cq):
        if n[g] > 0:
            route[g, route_group(S[g], m, cfg.fixed_k, kappa)] = True
    sparse_pairs = int(sum(int(n[g]) * int(m[route[g]].sum()) for g in range(Cq)))
    density = (cfg.s * N + Ck * N + cfg.P * N + sparse_pairs) / float(N) ** 2
    probes, weights = select_probes(cfg, qlabels, Cq, N, bh)
    return dict(ksizes=m, qsizes=n, scores=S, kappa=kappa, route=route, sparse_pairs=sparse_pairs,
                density=density, probes=probes, weights=weights)


def semantic_call_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, cfg, bh: int,
                       compute_outputs: bool = True) -> dict:
    """The semantic partition of the paper's Table 2 baseline ("semantic block-sparse
    attention"): Lloyd's k-means on the raw keys and on the raw queries (squared Euclidean
    distance, the same seeded initial points, limits and stop rule as the response-coupled
    partition), then the same routing, probes and (if cfg.repair) correction.
    Reading: "semantic" groups tokens by their own feature vectors, with no response coupling."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N = q.shape[0]
    Ck, Cq = cfg.n_kgroups, cfg.n_qgroups
    seed = getattr(cfg, "seed", 0)
    tol = float(np.float32(cfg.km_tol))
    ids = kmeans_init_ids(N, Ck, stream_seed(seed, bh, 0))
    kk = lloyd(k, k[ids], cfg.km_iters, tol)
    ids = kmeans_init_ids(N, Cq, stream_seed(seed, bh, 1))
    qq = lloyd(q, q[ids], cfg.km_iters, tol)
    out = dict(klabels=kk.labels, kcent=kk.centroids, kmeans_k=kk, qlabels=qq.labels, qcent=qq.centroids,
               kmeans_q=qq)
    out.update(route_and_probe(q, kk.labels, qq.labels, kk.centroids, cfg, bh))
    if compute_outputs:
        out.update(outputs_given_partition(q, k, v, qq.labels, kk.labels, out["route"], out["probes"],
                                           out["weights"], cfg.lam, repair=getattr(cfg, "repair", 1),
                                           correction=getattr(cfg, "correction", 0),
                                           trunc_rank=getattr(cfg, "trunc_rank", 0)))
    return out


def mean_error(O: np.ndarray, Oref: np.ndarray, rows: np.ndarray) -> float:
    """Mean normalised attention-output error over the given rows (Table 2's metric)."""
    return float(row_errors(O[rows], Oref[rows]).mean())


def error_reduction(err_method: float, err_baseline: float) -> float:
    """Relative error reduction of a method over a baseline, as in the abstract's 61.6-90.5%:
    1 - err_method / err_baseline."""
    return 1.0 - err_method / err_baseline


def call(Q, K, V, cfg, warm: Optional[Sequence[WarmState]] = None, heads=None, **kw) -> List[dict]:
    """All (b, h) of one call; Q, K, V are float64-convertible arrays [B, H, N, d]."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, H = Q.shape[:2]
    res = []
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for (b, h) in todo:
        bh = b * H + h
        ws = None if warm is None else warm[bh]
        res.append(call_head(Q[b, h], K[b, h], V[b, h], cfg, bh, warm=ws, **kw))
    return res


def warm_state(head_result: dict) -> WarmState:
    return WarmState(key_centroids=head_result["kcent"], query_centroids=head_result["qcent"])
