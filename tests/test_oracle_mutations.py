"""Planted mistakes in the oracle (CPU only): the pins must catch them.

Each mutant below changes one spot of one oracle function the way a slip would: a dropped
term, a wrong sign, scale or axis, a transposed or swapped operand, an off-by-one in a sampling
formula, a wrong tie rule or comparison. The changed source is compiled into a stand-in for
that function. The stand-in replaces the function in this process's copy of the oracle module
for one test only. The pins of test_oracle_pins.py named beside the mutant must then fail.

A control runs every listed pin against an unchanged recompiled copy of the same function. This
shows that a failure comes from the planted change and not from the recompilation.

Left out on purpose are mutants that change no result the method defines. Two examples: the
order of the sampled query rows, since a permutation of the response columns keeps every
distance; and a shift of the softmax by the global instead of the row maximum.
"""
import __future__
import inspect
import textwrap
import warnings

import pytest

from oracle import sparsepr_oracle as O

import test_oracle_pins as pins

# (id, oracle function or class, text to change (must occur once), replacement, pins that must fail)
MUTANTS = [
    # random draws
    ("splitmix-shift", "SplitMix64", "z ^ (z >> 30)", "z ^ (z >> 31)", ["splitmix64_published_vectors"]),
    ("splitmix-constant", "SplitMix64", "0xBF58476D1CE4E5B9", "0xBF58476D1CE4E5B8",
     ["splitmix64_published_vectors"]),
    ("fisher-yates-no-offset", "kmeans_init_ids", "j = i + rng.next() % (n_points - i)",
     "j = rng.next() % (n_points - i)", ["kmeans_init_ids_is_a_partial_fisher_yates"]),
    ("fisher-yates-no-swap", "kmeans_init_ids", "slots[i], slots[j] = vj, vi", "slots[i], slots[j] = vi, vj",
     ["kmeans_init_ids_is_a_partial_fisher_yates"]),
    ("stream-seed-stride", "stream_seed", "seed + 2 * bh + stage", "seed + bh + stage",
     ["stream_seeds_differ_per_head_and_stage"]),
    ("probe-seed-no-offset", "probe_stream_seed", "seed + (1 << 63) + 2 * bh", "seed + 2 * bh",
     ["random_probes_are_the_seeded_fisher_yates_draw"]),
    # sampled query rows
    ("sample-rows-left-edge", "sample_query_rows", "((2 * i + 1) * N) // (2 * s)", "(i * N) // s",
     ["sample_query_rows_formula"]),
    # k-means
    ("distance-sign", "squared_distances", "- 2.0 * (X @ C.T)", "+ 2.0 * (X @ C.T)",
     ["lloyd_matches_scikit_learn"]),
    ("distance-dropped-norm", "squared_distances", " + cc[None, :]", "", ["lloyd_matches_scikit_learn"]),
    ("ties-to-highest", "assign", "labels = np.argmin(D, axis=1)",
     "labels = D.shape[1] - 1 - np.argmin(D[:, ::-1], axis=1)", ["near_tie_margin_flags_equidistant_point"]),
    ("empty-group-averaged", "lloyd", "if counts[j] > 0:", "if counts[j] >= 0:",
     ["lloyd_empty_group_keeps_centroid_and_shadow"]),
    ("stop-rule-sign", "lloyd", "if J_hist[-2] - J <= tol * J_hist[-2]:", "if J - J_hist[-2] <= tol * J_hist[-2]:",
     ["lloyd_tolerance_stop_rule", "lloyd_objective_non_increasing_and_fixed_point"]),
    ("stop-rule-strict", "lloyd", "if J_hist[-2] - J <= tol * J_hist[-2]:", "if J_hist[-2] - J < tol * J_hist[-2]:",
     ["lloyd_tolerance_stop_rule"]),
    ("first-stop-at-two", "lloyd", "if tol >= 0 and it >= 1:", "if tol >= 0 and it >= 2:",
     ["lloyd_tolerance_stop_rule"]),
    ("objective-after-update", "lloyd", "        if tol >= 0 and it >= 1:",
     "        J_hist[-1] = float(((X - C[labels]) ** 2).sum())\n        if tol >= 0 and it >= 1:",
     ["lloyd_objective_non_increasing_and_fixed_point", "lloyd_tolerance_stop_rule"]),
    ("near-tie-mask-last-only", "lloyd", "tie_mask |= nt", "tie_mask = nt", ["near_tie_margin_flags_equidistant_point"]),
    ("margin-absolute", "assign", "(d2 - d1) / np.where(d1 > 0, d1, 1.0)", "(d2 - d1)",
     ["near_tie_margin_flags_equidistant_point"]),
    ("shadow-sum", "lloyd", "S[j] = shadow[members].mean(axis=0)", "S[j] = shadow[members].sum(axis=0)",
     ["lloyd_empty_group_keeps_centroid_and_shadow"]),
    ("key-basis-trailing", "key_response_basis", "return Vt[:rank].T", "return Vt[-rank:].T",
     ["key_response_basis_is_the_best_rank_r_approximation", "key_rank_equals_metric_kmeans_in_key_space"]),
    ("key-basis-full-rank-kept", "key_response_basis", "rank >= min(F.shape)", "rank > min(F.shape)",
     ["key_response_basis_is_the_best_rank_r_approximation"]),
    # responses
    ("response-unscaled", "query_responses", "(q @ key_centroids.T) / math.sqrt(d)", "(q @ key_centroids.T)",
     ["query_responses_and_rms"]),
    ("rms-sum", "rms_normalize", "np.mean(R * R, axis=1, keepdims=True)", "np.sum(R * R, axis=1, keepdims=True)",
     ["query_responses_and_rms"]),
    ("rms-axis", "rms_normalize", "np.mean(R * R, axis=1, keepdims=True)", "np.mean(R * R, axis=0, keepdims=True)",
     ["query_responses_and_rms"]),
    ("rms-no-epsilon", "rms_normalize", "np.sqrt(ms + RMS_EPS)", "np.sqrt(ms)", ["query_responses_and_rms"]),
    ("rms-centred", "rms_normalize", "return R / np.sqrt(ms + RMS_EPS)",
     "return (R - R.mean(axis=1, keepdims=True)) / np.sqrt(ms + RMS_EPS)", ["query_responses_and_rms"]),
    # routing
    ("score-no-log-mass", "routing_scores", "S[g] = R[rows].mean(axis=0) + logm", "S[g] = R[rows].mean(axis=0)",
     ["routing_scores_hand_case", "routing_scores_pool_by_linearity"]),
    ("score-sum", "routing_scores", "S[g] = R[rows].mean(axis=0) + logm", "S[g] = R[rows].sum(axis=0) + logm",
     ["routing_scores_hand_case"]),
    ("score-empty-kept", "routing_scores", "np.where(ksizes > 0,", "np.where(ksizes >= 0,",
     ["routing_scores_pool_by_linearity"]),
    ("score-log2", "routing_scores", "np.log(np.maximum", "np.log2(np.maximum", ["routing_scores_hand_case"]),
    ("budget-dropped-centroids", "per_row_key_budget", "(s + n_kgroups + P)", "(s + P)", ["per_row_key_budget"]),
    ("budget-density-fp64", "per_row_key_budget", "float(np.float32(density))", "float(density)",
     ["per_row_key_budget"]),
    ("route-ties-to-higher", "route_group", "key=lambda j: (-S_row[j], j)", "key=lambda j: (-S_row[j], -j)",
     ["route_group_hand_cases"]),
    ("route-ascending", "route_group", "key=lambda j: (-S_row[j], j)", "key=lambda j: (S_row[j], j)",
     ["route_group_hand_cases"]),
    ("route-non-strict", "route_group", "abs(cum + m - kappa) < abs(cum - kappa)",
     "abs(cum + m - kappa) <= abs(cum - kappa)", ["route_group_hand_cases"]),
    ("route-top-not-forced", "route_group", "if not chosen or abs(", "if abs(", ["route_group_hand_cases"]),
    ("route-empty-visited", "route_group", "if ksizes[j] > 0", "if ksizes[j] >= 0", ["route_group_hand_cases"]),
    ("route-fixed-k-off-by-one", "route_group", "chosen = order[:fixed_k]", "chosen = order[:fixed_k - 1]",
     ["route_group_hand_cases"]),
    # attention
    ("softmax-unscaled", "attention", "s = (q @ k.T) / math.sqrt(q.shape[1])", "s = (q @ k.T)",
     ["dense_attention_matches_torch_sdpa"]),
    ("softmax-scale-by-keys", "attention", "/ math.sqrt(q.shape[1])", "/ math.sqrt(k.shape[0])",
     ["dense_attention_matches_torch_sdpa"]),
    ("softmax-axis", "attention", "p /= p.sum(axis=1, keepdims=True)", "p /= p.sum(axis=0, keepdims=True)",
     ["dense_attention_matches_torch_sdpa"]),
    ("no-keys-nan", "attention", "return np.zeros((q.shape[0], v.shape[1]))",
     "return np.full((q.shape[0], v.shape[1]), np.nan)", ["sparse_attention_matches_masked_sdpa"]),
    ("sparse-query-labels", "sparse_attention", "route[g][klabels]", "route[g][qlabels]",
     ["sparse_attention_matches_masked_sdpa"]),
    ("sparse-mask-after-softmax", "sparse_attention", "out[rows] = attention(q[rows], k[keys], v[keys])",
     "out[rows] = attention(q[rows], k, v * route[g][klabels][:, None])", ["sparse_attention_matches_masked_sdpa"]),
    # probes
    ("uniform-left-edge", "probes_uniform", "((2 * i + 1) * N) // (2 * P)", "(i * N) // P",
     ["probes_uniform_formula"]),
    ("random-unsorted", "probes_random", "np.sort(np.array(", "(np.array(",
     ["random_probes_are_the_seeded_fisher_yates_draw"]),
    ("random-kmeans-stream", "probes_random", "probe_stream_seed(seed, bh)", "stream_seed(seed, bh, 0)",
     ["random_probes_are_the_seeded_fisher_yates_draw"]),
    ("stratified-smallest-remainders", "probes_stratified", "key=lambda g: (-int(rem[g]), g)",
     "key=lambda g: (int(rem[g]), g)", ["probes_stratified_hand_cases", "probes_stratified_invariants"]),
    ("stratified-ties-to-higher", "probes_stratified", "key=lambda g: (-int(rem[g]), g)",
     "key=lambda g: (-int(rem[g]), -g)", ["probes_stratified_hand_cases"]),
    ("stratified-left-edge", "probes_stratified", "((2 * i + 1) * int(n[g])) // (2 * int(m[g]))",
     "(i * int(n[g])) // int(m[g])", ["probes_stratified_hand_cases"]),
    ("stratified-weights-unscaled", "probes_stratified", "wts = wts * (P / wts.sum())", "wts = wts",
     ["probes_stratified_hand_cases", "probes_stratified_invariants"]),
    ("stratified-weights-inverted", "probes_stratified", "wts.append(float(n[g]) / float(m[g]))",
     "wts.append(float(m[g]) / float(n[g]))", ["probes_stratified_hand_cases"]),
    ("stratified-unsorted", "probes_stratified", "toks, wts = toks[o], wts[o]", "pass",
     ["probes_stratified_invariants"]),
    ("uniform-weights", "probes_uniform", "np.ones(P)", "np.full(P, 2.0)", ["probes_uniform_formula"]),
    ("stratified-rounded-share", "probes_stratified", "base = (P * n) // N", "base = (P * n + N // 2) // N",
     ["probes_stratified_hand_cases"]),
    # ridge fit, span, correction
    ("lambda-not-averaged", "ridge_lambda", "/ G.shape[0]", "", ["ridge_matches_augmented_lstsq"]),
    ("lambda-zero-means-auto", "ridge_lambda", "if lam_cfg >= 0 else", "if lam_cfg > 0 else",
     ["ridge_exact_when_residual_is_affine"]),
    ("fit-dense-not-residual", "ridge_fit", "odense_p - osp_p", "odense_p", ["ridge_exact_when_residual_is_affine"]),
    ("fit-no-intercept", "ridge_fit", "np.hstack([osp_p, np.ones((P, 1))])", "np.hstack([osp_p, np.zeros((P, 1))])",
     ["ridge_exact_when_residual_is_affine"]),
    ("fit-intercept-first", "ridge_fit", "np.hstack([osp_p, np.ones((P, 1))])", "np.hstack([np.ones((P, 1)), osp_p])",
     ["ridge_exact_when_residual_is_affine"]),
    ("ridge-unweighted-gram", "weighted_ridge", "WX = w[:, None] * X", "WX = X", ["ridge_matches_augmented_lstsq"]),
    ("ridge-unweighted-cross", "weighted_ridge", "WX.T @ R", "X.T @ R", ["ridge_matches_augmented_lstsq"]),
    ("ridge-no-lambda", "weighted_ridge", "G + lam * np.eye(X.shape[1])", "G",
     ["ridge_matches_augmented_lstsq", "ridge_mean_only_special_case"]),
    ("ridge-intercept-unpenalised", "weighted_ridge", "G + lam * np.eye(X.shape[1])",
     "G + lam * np.diag(np.r_[np.ones(X.shape[1] - 1), 0.0])",
     ["ridge_matches_augmented_lstsq", "ridge_mean_only_special_case"]),
    ("span-unweighted", "residual_span_basis", "Sg = R.T @ (w[:, None] * R)", "Sg = R.T @ R",
     ["truncated_span_is_the_leading_right_singular_subspace"]),
    ("span-trailing", "residual_span_basis", "np.argsort(-ev, kind=\"stable\")", "np.argsort(ev, kind=\"stable\")",
     ["truncated_span_is_the_leading_right_singular_subspace"]),
    ("truncation-off-by-one", "residual_span_basis", "if rank > 0 and U.shape[1] > rank:",
     "if rank > 0 and U.shape[1] > rank + 1:", ["truncated_span_is_the_leading_right_singular_subspace"]),
    ("span-not-applied", "restrict_to_residual_span", "return A @ U @ U.T", "return A", ["residual_span_projection"]),
    ("apply-intercept-first", "apply_correction", "osp @ A[:-1] + A[-1][None, :]", "osp @ A[1:] + A[0][None, :]",
     ["apply_correction_and_row_errors"]),
    ("apply-no-sparse-term", "apply_correction", "return osp + osp @ A[:-1]", "return osp @ A[:-1]",
     ["apply_correction_and_row_errors"]),
    ("error-normalised-by-output", "row_errors", "(np.linalg.norm(Oref, axis=1) + ERR_EPS)",
     "(np.linalg.norm(O, axis=1) + ERR_EPS)", ["apply_correction_and_row_errors", "mean_error_is_the_row_error_mean"]),
    ("mean-fit-first-row", "mean_fit", "A[-1] = Am[0]", "A[0] = Am[0]",
     ["mean_only_correction_is_the_weighted_mean_residual"]),
    ("probe-rows-not-exact", "outputs_given_partition", "O[probes] = odense", "O[probes] = O[probes]",
     ["call_partition_is_consistent", "repair_off_keeps_sparse_rows_and_exact_probes"]),
    ("probe-dense-on-probe-keys", "outputs_given_partition", "odense = attention(q[probes], k, v)",
     "odense = attention(q[probes], k[probes], v[probes])", ["call_with_every_group_kept_is_dense"]),
    ("sparse-labels-swapped", "outputs_given_partition", "sparse_attention(q, k, v, qlabels, klabels, route)",
     "sparse_attention(q, k, v, klabels, qlabels, route)", ["call_routes_and_sparse_rows_follow_its_partition"]),
    ("fit-unweighted-in-call", "outputs_given_partition", "fit(osp[probes], odense, weights, lam_cfg)",
     "fit(osp[probes], odense, np.ones_like(weights), lam_cfg)",
     ["call_fit_is_the_weighted_ridge_of_its_probe_residuals"]),
    ("span-of-dense-rows", "outputs_given_partition", "restrict_to_residual_span(A, odense - osp[probes],",
     "restrict_to_residual_span(A, odense,", ["call_fit_is_the_weighted_ridge_of_its_probe_residuals"]),
    ("truncation-ignored", "outputs_given_partition", "weights, trunc_rank)", "weights, 0)",
     ["call_fit_is_the_weighted_ridge_of_its_probe_residuals"]),
    ("mean-only-ignored", "outputs_given_partition", "fit = mean_fit if correction == 1 else ridge_fit",
     "fit = ridge_fit", ["call_fit_is_the_weighted_ridge_of_its_probe_residuals"]),
    ("probe-mode-swapped", "select_probes", "if cfg.probe_mode == 0:", "if cfg.probe_mode == 1:",
     ["call_fit_is_the_weighted_ridge_of_its_probe_residuals", "repair_reduces_error_on_smooth_field_inputs"]),
    # the whole call
    ("call-key-sizes-from-queries", "call_head", "m = np.bincount(klabels, minlength=Ck)",
     "m = np.bincount(qlabels, minlength=Ck)", ["call_partition_is_consistent"]),
    ("call-density-drops-centroid-pairs", "call_head", "density = (cfg.s * N + Ck * N + cfg.P * N + sparse_pairs)",
     "density = (cfg.s * N + cfg.P * N + sparse_pairs)",
     ["call_with_every_group_kept_is_dense", "call_routes_and_sparse_rows_follow_its_partition"]),
    ("call-pairs-without-group-sizes", "call_head", "sparse_pairs = int(sum(int(n[g]) * int(m[route[g]].sum())",
     "sparse_pairs = int(sum(int(m[route[g]].sum())",
     ["call_with_every_group_kept_is_dense", "call_routes_and_sparse_rows_follow_its_partition"]),
    ("warm-runs-cold-limit", "call_head", "S0, iters = warm.key_centroids, cfg.km_iters_warm",
     "S0, iters = warm.key_centroids, cfg.km_iters", ["warm_start_key_step_uses_the_current_calls_metric"]),
    ("call-routes-on-normalised-responses", "call_head", "S = routing_scores(R, qlabels, Cq, m)",
     "S = routing_scores(Rt, qlabels, Cq, m)", ["call_routes_and_sparse_rows_follow_its_partition"]),
    ("call-budget-with-query-groups", "call_head", "per_row_key_budget(cfg.density, N, cfg.s, Ck, cfg.P)",
     "per_row_key_budget(cfg.density, N, cfg.s, Cq, cfg.P)", ["call_routes_and_sparse_rows_follow_its_partition"]),
    ("call-probes-from-key-groups", "call_head", "select_probes(cfg, qlabels, Cq, N, bh)",
     "select_probes(cfg, klabels, Cq, N, bh)", ["call_routes_and_sparse_rows_follow_its_partition"]),
    ("call-responses-not-normalised", "call_head", "Rt = rms_normalize(R)", "Rt = R",
     ["warm_start_restarts_lloyd_where_the_previous_call_stopped"]),
    ("call-key-responses-of-queries", "call_head", "F = (k @ Qs.T) * scale", "F = (q @ Qs.T) * scale",
     ["key_rank_equals_metric_kmeans_in_key_space", "warm_start_key_step_uses_the_current_calls_metric"]),
    ("call-key-rank-ignored", "call_head", "Vr = key_response_basis(F, getattr(cfg, \"key_rank\", 0))", "Vr = None",
     ["key_rank_equals_metric_kmeans_in_key_space"]),
    ("warm-query-start-renormalised", "call_head", "C0q, iters = warm.query_centroids,",
     "C0q, iters = rms_normalize(warm.query_centroids),",
     ["warm_start_restarts_lloyd_where_the_previous_call_stopped"]),
    ("semantic-keys-from-queries", "semantic_call_head", "kk = lloyd(k, k[ids], cfg.km_iters, tol)",
     "kk = lloyd(q, q[ids], cfg.km_iters, tol)", ["semantic_partition_is_kmeans_on_the_raw_inputs"]),
    ("semantic-density-drops-centroid-pairs", "route_and_probe",
     "density = (cfg.s * N + Ck * N + cfg.P * N + sparse_pairs)", "density = (cfg.s * N + cfg.P * N + sparse_pairs)",
     ["call_routes_and_sparse_rows_follow_its_partition"]),
    ("semantic-routes-on-scaled-responses", "route_and_probe", "routing_scores(query_responses(q, kcent),",
     "routing_scores(2.0 * query_responses(q, kcent),", ["call_routes_and_sparse_rows_follow_its_partition"]),
    ("error-reduction-inverted", "error_reduction", "1.0 - err_method / err_baseline",
     "1.0 - err_baseline / err_method", ["table2_error_reduction_arithmetic"]),
    ("warm-key-start-unscaled", "call_head", "C0 = (warm.key_centroids @ Qs.T) * scale",
     "C0 = (warm.key_centroids @ Qs.T)", ["warm_start_restarts_lloyd_where_the_previous_call_stopped"]),
]


def _recompile(name, old=None, new=None):
    """The oracle function (or class) `name`, recompiled from its source with `old` replaced by
    `new` (or unchanged), resolving its globals in a copy of the oracle module's namespace."""
    src = textwrap.dedent(inspect.getsource(getattr(O, name)))
    if old is not None:
        assert src.count(old) == 1, f"{name}: {old!r} occurs {src.count(old)} times"
        src = src.replace(old, new)
    ns = dict(vars(O))
    code = compile(src, f"<mutant of {name}>", "exec", flags=__future__.annotations.compiler_flag,
                   dont_inherit=True)
    exec(code, ns)
    return ns[name]


def _failing(pin_names):
    """The pins among `pin_names` that fail (raise) as the oracle stands now."""
    out = []
    for p in pin_names:
        try:
            with warnings.catch_warnings():
                warnings.simplefilter("ignore")
                getattr(pins, "test_" + p)()
        except Exception:
            out.append(p)
    return out


@pytest.mark.parametrize("mid,fn,old,new,catchers", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(monkeypatch, mid, fn, old, new, catchers):
    monkeypatch.setattr(O, fn, _recompile(fn, old, new))
    missed = [p for p in catchers if p not in _failing(catchers)]
    assert not missed, f"mutant {mid} of {fn} passes the pins {missed}"


@pytest.mark.parametrize("fn", sorted({m[1] for m in MUTANTS}))
def test_unchanged_recompiled_oracle_passes_the_same_pins(monkeypatch, fn):
    catchers = sorted({p for m in MUTANTS if m[1] == fn for p in m[4]})
    monkeypatch.setattr(O, fn, _recompile(fn))
    assert _failing(catchers) == []


def test_every_mutant_names_existing_pins_and_is_unique():
    ids = [m[0] for m in MUTANTS]
    assert len(ids) == len(set(ids))
    for m in MUTANTS:
        assert m[4] and all(callable(getattr(pins, "test_" + p, None)) for p in m[4]), m[0]
        assert m[2] != m[3], m[0]
