"""The five synthetic workloads of the SparsePR per-call attention operator.

Each workload is a video-latent-shaped attention call: B batches, H heads, N tokens on a
(T, Y, X) raster grid, head dimension d.  Sizes follow the evaluated sequence lengths of
"Partition the Support, Reconstruct the Residual" (Table C.2: 118,800 / 75,600 / 44,160-class
token counts) plus a tiny and a mid-size case.  The method parameters (sampled queries s,
key/query group counts, density target, probe budget P, ridge lambda, k-means limits) are
the operator's arguments; the 25-initial / 2-warm k-means iteration limits and the 1e-4
tolerance are those of Table C.1 of the paper.

This module only describes shapes and parameters; it holds none of the method's arithmetic.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Tuple

F32 = 0
BF16 = 1

PROBE_UNIFORM = 0
PROBE_STRATIFIED = 1
PROBE_RANDOM = 2
# correction families (Table 4): the affine map of [O_sp, 1] (SparsePR) or the mean-only one
CORRECTION_AFFINE = 0
CORRECTION_MEAN = 1
# partitions: response-coupled (SparsePR: keys by their responses to sampled queries, queries
# by their normalised responses to the key-group centroids) or semantic (k-means on the raw
# keys and the raw queries; the baseline of the paper's Table 2)
PARTITION_RESPONSE = 0
PARTITION_SEMANTIC = 1


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    B: int
    H: int
    N: int
    d: int
    grid: Tuple[int, int, int]        # (T, Y, X) latent grid, raster token order
    tile: Tuple[int, int, int]        # generator cluster tile (Tt, Ty, Tx)
    dtype: int                        # F32 or BF16 for Q/K/V
    s: int                            # sampled queries per head
    n_kgroups: int                    # C_k
    n_qgroups: int                    # C_q
    density: float                    # target executed-pair density (incl. routing + probes)
    fixed_k: int                      # >0: keep exactly this many key groups per query group
    P: int                            # probe rows per head
    probe_mode: int
    lam: float                        # <0: automatic 1e-3 * tr(X^T W X) / (d+1)
    km_iters: int
    km_iters_warm: int
    km_tol: float                     # <0: never stop early
    rope: bool = False                # 3D rotary embedding applied to q and k by the generator
    calls: int = 1                    # consecutive calls (streaming workload)
    noise: float = 0.5
    seed: int = 20261202              # k-means initial-point draw (SplitMix64 streams)
    partition: int = 0                # PARTITION_RESPONSE (SparsePR) or PARTITION_SEMANTIC
    repair: int = 1                   # 1: fit and add the probe-residual correction; 0: none
    correction: int = 0               # CORRECTION_AFFINE (SparsePR) or CORRECTION_MEAN
    trunc_rank: int = 0               # 0: whole residual span; r: its r leading directions
    key_rank: int = 0                 # 0: full key responses; r: their r leading directions (r_K)
    recipe: str = "tiles"             # input generator: "tiles" (clustered Gaussian) or "field"
    field_tau: float = 4.0            # "field": peak logit contrast of the smooth field
    field_ell: Tuple[float, float, float] = (2.0, 6.0, 6.0)  # "field": length scales (t, y, x)
    value_offset: float = 1.0         # "field": scale of the value offset shared by all tokens

    @property
    def n_tiles(self) -> int:
        T, Y, X = self.grid
        a, b, c = self.tile
        return (-(-T // a)) * (-(-Y // b)) * (-(-X // c))

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def dense_flops(self) -> float:
        """Dense-equivalent attention flops of one call: 4 * B * H * N^2 * d."""
        return 4.0 * self.B * self.H * float(self.N) ** 2 * self.d


WORKLOADS = [
    Workload(name="tiny-f32-1x1024x64", index=0, B=1, H=1, N=1024, d=64,
             grid=(4, 16, 16), tile=(2, 4, 4), dtype=F32, s=64, n_kgroups=16,
             n_qgroups=16, density=0.25, fixed_k=4, P=32, probe_mode=PROBE_UNIFORM,
             lam=-1.0, km_iters=10, km_iters_warm=0, km_tol=-1.0),
    Workload(name="mid-bf16-8x16384x64", index=1, B=1, H=8, N=16384, d=64,
             grid=(16, 32, 32), tile=(4, 4, 4), dtype=BF16, s=256, n_kgroups=64,
             n_qgroups=64, density=0.22, fixed_k=0, P=128, probe_mode=PROBE_STRATIFIED,
             lam=-1.0, km_iters=25, km_iters_warm=0, km_tol=1e-4),
    Workload(name="dit13b-720p-24x118800x128", index=2, B=1, H=24, N=118800, d=128,
             grid=(33, 45, 80), tile=(3, 5, 5), dtype=BF16, s=1024, n_kgroups=128,
             n_qgroups=128, density=0.22, fixed_k=0, P=512, probe_mode=PROBE_STRATIFIED,
             lam=-1.0, km_iters=25, km_iters_warm=0, km_tol=1e-4, rope=True),
    Workload(name="dit14b-720p-40x75600x128", index=3, B=1, H=40, N=75600, d=128,
             grid=(21, 45, 80), tile=(3, 5, 5), dtype=BF16, s=768, n_kgroups=96,
             n_qgroups=96, density=0.22, fixed_k=0, P=384, probe_mode=PROBE_STRATIFIED,
             lam=-1.0, km_iters=25, km_iters_warm=0, km_tol=1e-4, rope=True),
    Workload(name="worldmodel-stream-16x42240x128", index=4, B=1, H=16, N=42240, d=128,
             grid=(12, 44, 80), tile=(3, 4, 5), dtype=BF16, s=768, n_kgroups=96,
             n_qgroups=96, density=0.22, fixed_k=0, P=512, probe_mode=PROBE_STRATIFIED,
             lam=-1.0, km_iters=25, km_iters_warm=2, km_tol=1e-4, calls=8),
]

# Sweep points of the larger workloads (each is a separate parity case).
DENSITY_SWEEP_3 = (0.15, 0.22, 0.30)
PROBE_SWEEP_4 = (128, 512, 2048)


def workload(i: int, **overrides) -> Workload:
    w = WORKLOADS[i]
    return w.replace(**overrides) if overrides else w


def scaled_down(w: Workload, heads: Optional[int] = None, grid: Optional[Tuple[int, int, int]] = None,
                **overrides) -> Workload:
    """Same generator and parameters on fewer heads and/or a smaller grid (for tests)."""
    kw = dict(overrides)
    if heads is not None:
        kw["H"] = heads
    if grid is not None:
        kw["grid"] = grid
        kw["N"] = grid[0] * grid[1] * grid[2]
    return w.replace(**kw)
