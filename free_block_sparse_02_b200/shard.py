"""Head-sharded split of one SparsePR call over the GPUs of one node.

Every (batch, head) of the operator is independent: its partition, routes, probe rows and
fitted correction use that head's Q, K, V only.  One call over B x H heads therefore splits
without any exchange: rank r of G takes the flattened heads bh in [bh0, bh1) (a contiguous,
balanced range of b * H + h), which is a contiguous slice of the [B, H, N, d] tensors, and runs
the operator on it as a call of B = 1 and H = bh1 - bh0 heads.

The operator draws its k-means initial points (and random probe rows) from SplitMix64 streams
seeded seed + 2 * bh + stage, where bh is the head's index within the call.  A rank's call
numbers its heads from 0, so it passes seed + 2 * bh0: every head then draws exactly the
stream it draws in the single-GPU call, and the assembled per-rank outputs equal that call's.

This module holds only index arithmetic; no step of the method runs here.
"""
from __future__ import annotations

from typing import Tuple

_MASK64 = (1 << 64) - 1


def head_range(n_heads: int, world: int, rank: int) -> Tuple[int, int]:
    """[bh0, bh1) of rank `rank` out of `world`: floor(r * BH / G) .. floor((r + 1) * BH / G).
    Ranges are contiguous, disjoint, cover every head and differ in size by at most one; a rank
    gets an empty range when there are fewer heads than ranks."""
    if world < 1 or not (0 <= rank < world) or n_heads < 0:
        raise ValueError("head_range: need world >= 1, 0 <= rank < world, n_heads >= 0")
    return (rank * n_heads) // world, ((rank + 1) * n_heads) // world


def shard_workload(w, world: int, rank: int):
    """The rank's part of workload `w`: (local workload, bh0, bh1).  The local workload has
    B = 1, H = bh1 - bh0 and its seed advanced by 2 * bh0 (64-bit wrap-around), everything else
    as in `w`; None when the rank has no head."""
    bh0, bh1 = head_range(w.B * w.H, world, rank)
    if bh1 == bh0:
        return None, bh0, bh1
    return w.replace(B=1, H=bh1 - bh0, seed=(w.seed + 2 * bh0) & _MASK64), bh0, bh1


def local_slice(x, bh0: int, bh1: int):
    """Heads [bh0, bh1) of a [B, H, N, d] tensor as a [1, bh1 - bh0, N, d] view (no copy when
    `x` is contiguous)."""
    B, H, N, d = x.shape
    return x.reshape(B * H, N, d)[bh0:bh1].reshape(1, bh1 - bh0, N, d)
