"""The rounding bound behind the exact k-means labels, checked by emulation on the CPU.

The assignment scores s_j = b_j - 2 sigma (x . w_j) in fp32: x is bf16 (exact), w_j is split into
three bf16 terms (hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid)), the 3d products
(exact in fp32) are summed in fp32 -- in one chain, or as the stacked form's two chains
(hi and lo products interleaved, mid products apart) added once -- and the epilogue takes
fmaf(-2 sigma, dot, b32).  The claim: every fp32 score is within
    delta = 4 (3d + 8) 2^-23 ||sigma x|| max_j ||w_j|| + 4 2^-23 max_j |b_j|
of the exact score, so the fp64 argmin is among the groups whose fp32 score is within 2.5 delta
of the fp32 best.  Also: the running fp64 group sums of bf16 keys, moved by label changes,
equal fresh sums exactly.  This emulation shares nothing with the CUDA code; it restates the
arithmetic."""
import numpy as np


def bf16(a):
    """Round float64/float32 values to bf16 (round to nearest even), returned as float32."""
    f = np.asarray(a, dtype=np.float64).astype(np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    bits = (bits + 0x7FFF + ((bits >> 16) & 1)) & 0xFFFF0000
    return bits.astype(np.uint32).view(np.float32)


def split3(w):
    h = bf16(w)
    m = bf16(w - h.astype(np.float64))
    l = bf16(w - h.astype(np.float64) - m.astype(np.float64))
    return h, m, l


def fp32_chain(terms):
    """Sequential fp32 sum of a list of fp32 arrays."""
    acc = np.zeros_like(terms[0], dtype=np.float32)
    for t in terms:
        acc = (acc + t).astype(np.float32)
    return acc


def fmaf(a, b, c):
    return (np.float64(a) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def check(d, C, n, wscale, bscale, sigma, seed, terms=3):
    rng = np.random.default_rng(seed)
    x = bf16(rng.standard_normal((n, d)) * rng.uniform(0.5, 3.0))           # bf16 points
    W = rng.standard_normal((C, d)) * wscale * rng.uniform(0.2, 1.0, (C, 1))  # fp64 weights
    b = rng.uniform(0.0, 1.0, C) * bscale                                     # fp64 biases
    h, m, l = split3(W)
    xf = x.astype(np.float32)
    prod = lambda T, k: (xf[:, None, k] * T[None, :, k]).astype(np.float32)  # exact in fp32
    if terms == 3:
        chain = fp32_chain([prod(T, k) for T in (h, m, l) for k in range(d)])
        stacked = (fp32_chain([p for k in range(d) for p in (prod(h, k), prod(l, k))])
                   + fp32_chain([prod(m, k) for k in range(d)])).astype(np.float32)
    else:  # hi and mid only: the split leaves |w - hi - mid| <= 2^-18 |w|
        chain = fp32_chain([prod(T, k) for T in (h, m) for k in range(d)])
        stacked = (fp32_chain([prod(h, k) for k in range(d)]) + fp32_chain([prod(m, k) for k in range(d)])).astype(np.float32)
    b32 = b.astype(np.float32)
    m2s = np.float32(-2.0 * sigma)
    exact = b[None, :] - 2.0 * np.float64(np.float32(sigma)) * (x.astype(np.float64) @ W.T)
    u = 2.0 ** -23
    xn = np.linalg.norm(x.astype(np.float64) * np.float32(sigma), axis=1)
    wmax = np.linalg.norm(W, axis=1).max()
    if terms == 3:
        delta = 4 * (3 * d + 8) * u * xn * wmax + 4 * u * np.abs(b).max()
    else:
        delta = (4 * (2 * d + 8) * u + 4 * 2.0 ** -18) * xn * wmax + 4 * u * np.abs(b).max()
    for dot in (chain, stacked):
        sc = fmaf(m2s, dot, np.broadcast_to(b32, dot.shape))
        err = np.abs(sc.astype(np.float64) - exact)
        assert np.all(err <= delta[:, None]), (err / delta[:, None]).max()
        # the fp64 argmin is among the candidates within 2.5 delta of the fp32 best
        best = sc.min(axis=1).astype(np.float64)
        cand = sc.astype(np.float64) <= best[:, None] + 2.5 * delta[:, None]
        assert np.all(cand[np.arange(n), exact.argmin(axis=1)])
    return float((np.abs(fmaf(m2s, chain, np.broadcast_to(b32, chain.shape)).astype(np.float64) - exact)
                  / delta[:, None]).max())


def test_bound_covers_keys_at_d128():
    assert check(d=128, C=64, n=96, wscale=1.0, bscale=50.0, sigma=1.0, seed=1) < 1.0


def test_bound_covers_queries_with_a_scale_at_d64():
    assert check(d=64, C=48, n=128, wscale=0.3, bscale=5.0, sigma=0.37, seed=2) < 1.0


def test_bound_covers_large_magnitude_spread():
    assert check(d=64, C=32, n=64, wscale=100.0, bscale=1e5, sigma=1.0, seed=3) < 1.0


def test_two_term_split_bound_covers_keys_and_queries():
    """With hi and mid only, the split error (2^-18 of sum |x_k w_k|) is a few percent of the
    accumulation bound, so delta_2 = (4 (2d + 8) 2^-23 + 4 2^-18) ||sigma x|| max ||w|| +
    4 2^-23 max |b| -- smaller than the three-term delta -- still covers every score."""
    assert check(d=128, C=64, n=96, wscale=1.0, bscale=50.0, sigma=1.0, seed=4, terms=2) < 1.0
    assert check(d=64, C=48, n=128, wscale=0.3, bscale=5.0, sigma=0.37, seed=5, terms=2) < 1.0
    assert check(d=64, C=32, n=64, wscale=100.0, bscale=1e5, sigma=1.0, seed=6, terms=2) < 1.0


def _bf16(x):
    """Round float32 values to bf16 (round to nearest even) and return them as float64."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16 << 16
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


def test_running_group_sums_of_bf16_keys_equal_fresh_sums():
    """The k-means update keeps each group's fp64 sum of member keys as a running total, moved
    by -x under a point's old label and +x under its new one, in whatever order the atomics
    land.  For bf16 keys of the workloads' scale every partial sum is exactly representable in
    fp64 (8-bit significands, an exponent spread of a few tens of bits, at most 2^17 terms), so
    the running totals equal the sums formed afresh, bit for bit."""
    rng = np.random.default_rng(7)
    n, d, C = 4096, 16, 32
    x = _bf16(rng.standard_normal((n, d)).astype(np.float32) * 2.0)
    lab = rng.integers(0, C, n)
    run = np.zeros((C, d))
    for p in rng.permutation(n):  # the first iteration: every point, in a shuffled order
        run[lab[p]] += x[p]
    for _ in range(6):  # later iterations: about a tenth of the points change group
        new = lab.copy()
        ch = rng.random(n) < 0.1
        new[ch] = rng.integers(0, C, ch.sum())
        for p in rng.permutation(np.flatnonzero(new != lab)):
            run[lab[p]] -= x[p]
            run[new[p]] += x[p]
        lab = new
        fresh = np.zeros((C, d))
        np.add.at(fresh, lab, x)
        assert np.array_equal(run, fresh)
