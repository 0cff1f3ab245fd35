"""Seeded synthetic video-latent Q/K/V for the SparsePR attention operator.

The paper evaluates on activations of video models driven by VBench / PBench prompts; neither
the models nor the prompts exist here, so every input is synthetic with the same structure:
tokens on a (T, Y, X) raster grid, grouped into spatio-temporal tiles, each tile with a random
centre so that queries and keys of one tile attend mostly to each other (the locality that
block-sparse video attention exploits).

Recipe (per head, one independent PCG64 stream per (b, h)):
  * centre of tile c:   mu_c ~ 2 * N(0, I_d)
  * query of token n:   q_n = mu_tile(n) + noise * N(0, I_d)
  * key of token n:     k_n = mu_tile(n) + noise * N(0, I_d)   (independent draw)
  * value:              v_n ~ N(0, I_d)
  draws in the order centres, q-noise, k-noise, v.
  * optional 3D rotary embedding of q and k (the d dims split (t, y, x) = d/4, 3d/8, 3d/8,
    base 10000, adjacent pairs rotated by pos * 10000^(-2i/d_axis)); this is a choice of the
    generator, not of the method.
  * streaming workloads: call c > 0 is x_c = 0.95 x_{c-1} + 0.31 N(0, I) for each of q, k, v
    (q-noise, k-noise, v-noise drawn in that order per call).

Second recipe, "field" (opt-in; smooth activations whose sparse residual an affine map of the
sparse output can predict, the regime of the paper's model activations):
  * f(p) = sqrt(2/F) sum_j W_j cos(omega_j . p + b_j) over the token's (t, y, x) grid position p,
    F = 256 random Fourier features, omega_j ~ N(0, diag(1/ell^2)), b_j ~ U[0, 2 pi),
    W_j ~ N(0, I_d): a Gaussian random field, unit variance per dimension, correlation
    exp(-|dp / ell|^2 / 2) between tokens
  * q = a f(p) + noise N(0, I),  k = a f(p) + noise N(0, I),  a^2 = tau / sqrt(d), so that the
    logit q.k / sqrt(d) of two nearby tokens is about tau above that of two distant ones
  * v = g(p) + noise N(0, I) + c u, g a second independent field, u ~ N(0, I_d) one offset
    shared by every token of the head
  draws in the order (omega, b, W) of f, q-noise, k-noise, (omega, b, W) of g, v-noise, u.
Values are produced in float64 and cast once to the workload dtype; the CUDA path and the
oracle both consume the cast tensors.

This module holds no arithmetic of the method itself.
"""
from __future__ import annotations

from typing import Iterator, List, Optional, Sequence, Tuple

import numpy as np
import torch

from .configs import BF16, F32, Workload

SEED_BASE = 20261202


def _torch_dtype(code: int) -> torch.dtype:
    return torch.float32 if code == F32 else torch.bfloat16


def token_tiles(w: Workload) -> np.ndarray:
    """Tile id of every token in raster (t, y, x) order."""
    T, Y, X = w.grid
    a, b, c = w.tile
    t, y, x = np.meshgrid(np.arange(T), np.arange(Y), np.arange(X), indexing="ij")
    ny, nx = -(-Y // b), -(-X // c)          # tiles per axis (a ragged last tile is allowed)
    tid = ((t // a) * ny + (y // b)) * nx + (x // c)
    return tid.reshape(-1)


def _rope_angles(w: Workload) -> Tuple[np.ndarray, np.ndarray]:
    T, Y, X = w.grid
    d = w.d
    dt = d // 4
    dy = (d - dt) // 2
    dx = d - dt - dy
    t, y, x = np.meshgrid(np.arange(T), np.arange(Y), np.arange(X), indexing="ij")
    pos = [t.reshape(-1), y.reshape(-1), x.reshape(-1)]
    angles = []
    for p, da in zip(pos, (dt, dy, dx)):
        i = np.arange(da // 2)
        freq = 10000.0 ** (-2.0 * i / da)
        angles.append(p[:, None].astype(np.float64) * freq[None, :])
    ang = np.concatenate(angles, axis=1)  # (N, d/2)
    return np.cos(ang), np.sin(ang)


def _apply_rope(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    x0 = x[:, 0::2]
    x1 = x[:, 1::2]
    out = np.empty_like(x)
    out[:, 0::2] = x0 * cos - x1 * sin
    out[:, 1::2] = x0 * sin + x1 * cos
    return out


N_FEATURES = 256


def grid_positions(w: Workload) -> np.ndarray:
    """(N, 3) float64 (t, y, x) grid coordinates of the tokens in raster order."""
    T, Y, X = w.grid
    t, y, x = np.meshgrid(np.arange(T), np.arange(Y), np.arange(X), indexing="ij")
    return np.stack([t.reshape(-1), y.reshape(-1), x.reshape(-1)], axis=1).astype(np.float64)


def _random_field(rng: np.random.Generator, pos: np.ndarray, d: int, ell) -> np.ndarray:
    """Random-Fourier-feature Gaussian field over the grid: (N, d), unit variance per dim."""
    omega = rng.standard_normal((N_FEATURES, 3)) / np.asarray(ell, dtype=np.float64)[None, :]
    phase = rng.uniform(0.0, 2.0 * np.pi, N_FEATURES)
    W = rng.standard_normal((N_FEATURES, d))
    out = np.empty((pos.shape[0], d))
    for s in range(0, pos.shape[0], 16384):      # bounded temporaries on the large grids
        out[s:s + 16384] = np.cos(pos[s:s + 16384] @ omega.T + phase) @ W
    return out * np.sqrt(2.0 / N_FEATURES)


def _field_qkv(w: Workload, rng: np.random.Generator):
    pos = grid_positions(w)
    f = _random_field(rng, pos, w.d, w.field_ell)
    a = np.sqrt(w.field_tau / np.sqrt(w.d))
    q = a * f + w.noise * rng.standard_normal((w.N, w.d))
    k = a * f + w.noise * rng.standard_normal((w.N, w.d))
    g = _random_field(rng, pos, w.d, w.field_ell)
    v = g + w.noise * rng.standard_normal((w.N, w.d))
    v += w.value_offset * rng.standard_normal((1, w.d))
    return q, k, v


def _head_stream(w: Workload, variant: int, bh: int) -> np.random.Generator:
    ss = np.random.SeedSequence(entropy=SEED_BASE + w.index, spawn_key=(variant,))
    child = ss.spawn(w.B * w.H)[bh]
    return np.random.Generator(np.random.PCG64(child))


def head_calls_f64(w: Workload, b: int, h: int, variant: int = 0,
                   calls: Optional[int] = None) -> Iterator[Tuple[np.ndarray, np.ndarray, np.ndarray]]:
    """Yield float64 (q, k, v), each (N, d), for consecutive calls of head (b, h)."""
    calls = w.calls if calls is None else calls
    rng = _head_stream(w, variant, b * w.H + h)
    if w.recipe == "field":
        q, k, v = _field_qkv(w, rng)
    elif w.recipe == "tiles":
        tiles = token_tiles(w)
        assert tiles.shape[0] == w.N
        mu = 2.0 * rng.standard_normal((w.n_tiles, w.d))
        q = mu[tiles] + w.noise * rng.standard_normal((w.N, w.d))
        k = mu[tiles] + w.noise * rng.standard_normal((w.N, w.d))
        v = rng.standard_normal((w.N, w.d))
    else:
        raise ValueError(f"unknown input recipe {w.recipe!r}")
    if w.rope:
        cos, sin = _rope_angles(w)
        q = _apply_rope(q, cos, sin)
        k = _apply_rope(k, cos, sin)
    yield q, k, v
    for _ in range(1, calls):
        q = 0.95 * q + 0.31 * rng.standard_normal((w.N, w.d))
        k = 0.95 * k + 0.31 * rng.standard_normal((w.N, w.d))
        v = 0.95 * v + 0.31 * rng.standard_normal((w.N, w.d))
        yield q, k, v


def make_qkv(w: Workload, variant: int = 0, call: int = 0,
             heads: Optional[Sequence[Tuple[int, int]]] = None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """CPU tensors Q, K, V of shape [B, H, N, d] in the workload dtype, for one call.

    heads: optional list of (b, h) to generate; the others are left zero (for sampled checks).
    """
    dt = _torch_dtype(w.dtype)
    Q = torch.zeros((w.B, w.H, w.N, w.d), dtype=dt)
    K = torch.zeros_like(Q)
    V = torch.zeros_like(Q)
    todo = heads if heads is not None else [(b, h) for b in range(w.B) for h in range(w.H)]
    for (b, h) in todo:
        for c, (q, k, v) in enumerate(head_calls_f64(w, b, h, variant, calls=call + 1)):
            if c == call:
                Q[b, h] = torch.from_numpy(q).to(dt)
                K[b, h] = torch.from_numpy(k).to(dt)
                V[b, h] = torch.from_numpy(v).to(dt)
    return Q, K, V


def make_stream(w: Workload, variant: int = 0) -> List[Tuple[torch.Tensor, torch.Tensor, torch.Tensor]]:
    """All calls of a streaming workload: a list of (Q, K, V) CPU tensors."""
    dt = _torch_dtype(w.dtype)
    out = [tuple(torch.zeros((w.B, w.H, w.N, w.d), dtype=dt) for _ in range(3)) for _ in range(w.calls)]
    for b in range(w.B):
        for h in range(w.H):
            for c, (q, k, v) in enumerate(head_calls_f64(w, b, h, variant)):
                out[c][0][b, h] = torch.from_numpy(q).to(dt)
                out[c][1][b, h] = torch.from_numpy(k).to(dt)
                out[c][2][b, h] = torch.from_numpy(v).to(dt)
    return out


def as_f64(x: torch.Tensor) -> np.ndarray:
    """The exact values of a (bf16 or fp32) tensor as a float64 numpy array."""
    return x.detach().to("cpu").to(torch.float64).numpy()
