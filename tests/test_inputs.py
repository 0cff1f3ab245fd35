"""The synthetic inputs follow the recipe stated for them (CPU only).

The generator holds none of the method's arithmetic. These tests lock its stated recipe:
- the draws and scales of the clustered-tile recipe, and the tile ids by their block coordinates;
- the 3D rotary embedding by its defining properties: norms kept, dot products that depend
  only on the displacement, the (t, y, x) split of the dimensions, and base 10000;
- the streaming recurrence, which keeps the variance;
- the smooth-field recipe's unit variance and logit contrast;
- one stream per head and per rank variant, and a single cast to the workload dtype.
"""
import numpy as np
import torch

from free_block_sparse_02_b200 import configs, gen


def _tiny_tiles():
    # bf16, tiles (4, 4, 4), no rotary embedding, two heads
    return configs.scaled_down(configs.workload(1), heads=2, grid=(4, 8, 12))


def test_tile_ids_follow_the_block_coordinates():
    w = _tiny_tiles()
    ids = gen.token_tiles(w)
    pos = gen.grid_positions(w).astype(int)
    blocks = pos // np.array(w.tile)
    # two tokens share a tile exactly when they share block coordinates
    _, first = np.unique(blocks, axis=0, return_inverse=True)
    assert len(np.unique(ids)) == w.n_tiles == len(np.unique(first))
    same_id = ids[:, None] == ids[None, :]
    same_block = (blocks[:, None, :] == blocks[None, :, :]).all(-1)
    assert np.array_equal(same_id, same_block)


def test_tile_recipe_draws_centres_then_query_and_key_noise_then_values():
    """Each head's stream is PCG64 on SeedSequence(20261202 + workload index, spawn key
    (variant,)), child bh; it draws the tile centres 2 N(0, I), the query noise, the key noise
    (0.5 N(0, I) each) and the values N(0, I), in that order."""
    w = _tiny_tiles()
    tiles = gen.token_tiles(w)
    for variant in (0, 1):
        for h in range(w.H):
            child = np.random.SeedSequence(entropy=20261202 + w.index, spawn_key=(variant,)).spawn(w.B * w.H)[h]
            rng = np.random.Generator(np.random.PCG64(child))
            mu = 2.0 * rng.standard_normal((w.n_tiles, w.d))
            q = mu[tiles] + 0.5 * rng.standard_normal((w.N, w.d))
            k = mu[tiles] + 0.5 * rng.standard_normal((w.N, w.d))
            v = rng.standard_normal((w.N, w.d))
            gq, gk, gv = next(gen.head_calls_f64(w, 0, h, variant))
            assert np.array_equal(gq, q) and np.array_equal(gk, k) and np.array_equal(gv, v)
            Q, K, V = gen.make_qkv(w, variant=variant)
            # cast once to the workload dtype
            assert Q.dtype == torch.bfloat16
            assert torch.equal(Q[0, h], torch.from_numpy(q).to(torch.bfloat16))
            assert torch.equal(V[0, h], torch.from_numpy(v).to(torch.bfloat16))


def test_heads_and_rank_variants_draw_different_inputs():
    w = _tiny_tiles()
    Q0, _, _ = gen.make_qkv(w, variant=0)
    Q1, _, _ = gen.make_qkv(w, variant=1)
    assert not torch.equal(Q0[0, 0], Q0[0, 1])
    assert not torch.equal(Q0, Q1)


def _rope_workload():
    return configs.scaled_down(configs.workload(2), heads=1, grid=(3, 5, 10))


def _token(w, t, y, x):
    T, Y, X = w.grid
    return (t * Y + y) * X + x


def test_rotary_embedding_keeps_norms_and_depends_only_on_displacement():
    w = _rope_workload()
    cos, sin = gen._rope_angles(w)
    rng = np.random.default_rng(0)
    a, b = rng.standard_normal(w.d), rng.standard_normal(w.d)
    A = gen._apply_rope(np.tile(a, (w.N, 1)), cos, sin)
    Bm = gen._apply_rope(np.tile(b, (w.N, 1)), cos, sin)
    np.testing.assert_allclose(np.linalg.norm(A, axis=1), np.linalg.norm(a), rtol=1e-13)
    # <R(p) a, R(p') b> depends on p - p' only
    pairs = [((0, 0, 0), (1, 2, 3)), ((1, 1, 1), (2, 3, 4)), ((1, 2, 5), (2, 4, 8))]
    dots = [A[_token(w, *p)] @ Bm[_token(w, *q)] for p, q in pairs]
    np.testing.assert_allclose(dots, dots[0], rtol=1e-12)
    assert abs((A[_token(w, 0, 0, 0)] @ Bm[_token(w, 0, 0, 1)]) - dots[0]) > 1e-6


def test_rotary_embedding_splits_the_dimensions_over_t_y_x_with_base_10000():
    """The d dimensions split (d/4, 3d/8, 3d/8) over (t, y, x): a move along one axis rotates
    only that axis's dimensions.  Adjacent pairs rotate by pos * 10000^(-2i/d_axis)."""
    w = _rope_workload()
    d = w.d
    cos, sin = gen._rope_angles(w)
    x = np.random.default_rng(1).standard_normal((w.N, d))
    x[:] = x[0]
    R = gen._apply_rope(x, cos, sin)
    o = R[_token(w, 0, 0, 0)]
    bounds = {"t": (0, d // 4), "y": (d // 4, d // 4 + 3 * d // 8), "x": (d // 4 + 3 * d // 8, d)}
    for axis, tok in (("t", _token(w, 1, 0, 0)), ("y", _token(w, 0, 1, 0)), ("x", _token(w, 0, 0, 1))):
        lo, hi = bounds[axis]
        changed = np.flatnonzero(np.abs(R[tok] - o) > 1e-12)
        assert changed.min() >= lo and changed.max() < hi, axis
    # pair i of the t dimensions at t = 1 turns by 10000^(-2i/(d/4)) radians
    e = np.zeros((w.N, d))
    e[:, 0::2] = 1.0
    Re = gen._apply_rope(e, cos, sin)[_token(w, 1, 0, 0)]
    dt = d // 4
    i = np.arange(dt // 2)
    np.testing.assert_allclose(Re[0:dt:2], np.cos(10000.0 ** (-2.0 * i / dt)), rtol=1e-13)
    np.testing.assert_allclose(Re[1:dt:2], np.sin(10000.0 ** (-2.0 * i / dt)), rtol=1e-13)


def test_streaming_recurrence_keeps_the_variance():
    """x_c = 0.95 x_(c-1) + 0.31 N(0, I): 0.95^2 + 0.31^2 = 0.9986, so the values stay near unit
    variance over the 8 calls and consecutive calls correlate at about 0.95."""
    assert abs(0.95 ** 2 + 0.31 ** 2 - 1.0) < 2e-3
    w = configs.scaled_down(configs.workload(4), heads=1, grid=(3, 8, 10))
    calls = list(gen.head_calls_f64(w, 0, 0))
    assert len(calls) == 8
    for c, (_, _, v) in enumerate(calls):
        assert 0.95 < v.var() < 1.05, (c, v.var())
    for (_, _, v0), (_, _, v1) in zip(calls, calls[1:]):
        r = np.corrcoef(v0.ravel(), v1.ravel())[0, 1]
        assert 0.93 < r < 0.97


def test_field_recipe_has_unit_variance_and_the_stated_logit_contrast():
    """f has unit variance per dimension; q = a f + 0.5 N(0, I) and k likewise with
    a^2 = tau / sqrt(d) (tau = 4), so a token's own query-key logit is about tau above that of
    two distant tokens, whose fields are uncorrelated."""
    w = configs.workload(1, recipe="field")
    w = configs.scaled_down(w, heads=1)
    rng = np.random.default_rng(5)
    f = gen._random_field(rng, gen.grid_positions(w), w.d, w.field_ell)
    assert abs(f.var(axis=0).mean() - 1.0) < 0.1
    q, k, _ = next(gen.head_calls_f64(w, 0, 0))
    own = np.einsum("nd,nd->n", q, k).mean() / np.sqrt(w.d)
    far = np.einsum("nd,nd->n", q[: w.N // 2], k[w.N // 2:]).mean() / np.sqrt(w.d)  # half a grid apart in t
    assert abs(own - w.field_tau) < 0.6 and abs(far) < 0.6, (own, far)
