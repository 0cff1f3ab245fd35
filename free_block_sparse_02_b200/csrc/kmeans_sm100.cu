// k-means assignment, update and per-row quadratic forms of the partition on the tensor cores
// (tcgen05, results in TMEM, operands by TMA).
//
// "Partition the Support, Reconstruct the Residual" (arXiv 2608.18484), abstract: keys are
// grouped by their responses to sampled queries, queries by how they respond to the key-group
// centroids; both groupings are k-means (Table C.1: 25 / 2 iterations, tolerance 1e-4).
//
// Both k-means run on the d-dimensional inputs (see partition.cu): the score of point x against
// group j is  s_j = b_j - 2 sigma_x (x . w_j)  with (keys) w = M c, b = c^T M c, sigma = 1, or
// (queries) w = u = C^T nu / sqrt(d), b = ||nu||^2, sigma = 1/rms_q; the label is argmin_j s_j,
// lowest j on ties.
//
// One Lloyd iteration on the tensor-core path is two kernels over the same static split of the
// BH * ceil(N/128) point tiles into G contiguous ranges (one per CTA, ranges may cross heads),
// after the prep kernel of partition.cu:
//
//  assignment  Persistent and warp-specialised (384 threads): warp 0 streams 128-point tiles of
//              X by TMA through a ring of shared-memory stages (and the head's two-term W when
//              the head changes), warp 1 issues the MMA chain X (128 x d, bf16, exact) times W^T
//              (d x C; W = hi + mid in bf16, fp32 accumulation) into one of two TMEM
//              accumulators, and two epilogue warpgroups take alternate tiles: one thread per
//              point (its TMEM lane) scans every group's score, keeps the best two, writes the
//              label and adds the best score to the objective.  A point whose two best are within
//              a rigorous rounding bound goes to the CTA's re-decision list.  More than 256
//              groups: one launch per chunk of 256, the best two carried between launches.
//  update      First re-decides the points its range's assignment CTA listed, in fp64 (one warp
//              each; label and objective corrected); then, for chunks of up to 12288 points of
//              one head, counting-sorts the points by label in shared memory and sums each
//              group's run: one thread per (group, 8 dimensions) gathers the run's rows
//              (consecutive threads read consecutive 16-byte pieces of a row), accumulates
//              sigma x in fp64 registers and adds the result with one atomic per (group,
//              dimension) per chunk.  From the second iteration on only the points whose label
//              changed are summed, as -x under the old label and +x under the new one: the
//              group sums are running totals, not recomputed.
//
// Labels therefore equal the argmin of an fp64 evaluation, and the group sums are fp64 sums of
// the exact inputs (keys) or of the inputs times their fp64 scale 1/rms (queries).
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"
#include "kmeans.cuh"
#include "sm100.cuh"

namespace sparsepr {

using namespace sm100;

constexpr int kKmTile = 128;
// bf16 terms of W in the assignment's products: hi + mid leaves |w - hi - mid| <= 2^-18 |w|, an
// error the rounding bound below covers (the split error is a few percent of the bound)
constexpr int kKmWTerms = 2;
constexpr int kKmThreads = 384;   // warp 0 TMA, warp 1 MMA, warps 4..11 epilogue
constexpr int kKmUpdThreads = 512;
constexpr int kKmMaxStages = 3;  // 3 measured 2% faster than 4 at the 13B-DiT shape
constexpr int kKmUpdChunk = 12288;  // entries of one head sorted and summed at a time by the update
                                    // (points, or two per label change)
constexpr size_t kKmUpdStaticSmem = 17 * 1024;  // bound of the update kernel's static shared memory
constexpr int kKmUpdItemRows = 64;   // rows of one accumulation item: a group's run is split into
                                     // pieces of at most this many rows, summed by different warps
__host__ __device__ constexpr int km_upd_max_items(int C) { return kKmUpdChunk / kKmUpdItemRows + C; }


// Shared memory of the assignment kernel: the kKmWTerms-term W, `stages` X tiles, barriers,
// per-warp bias copies.
__host__ inline size_t km_assign_smem(int D, int Np, int stages) {
  return (size_t)kKmWTerms * Np * D * 2 + (size_t)stages * kKmTile * D * 2 + 1024 /*align*/ + 256 /*barriers*/ +
         (size_t)8 * 256 * 4 /*bias*/;
}

// Shared memory of the update kernel: labels and sorted order of a chunk of points, per-group
// offsets and cursors.
__host__ inline size_t km_update_smem(int D, int C) {
  const size_t chunk = (size_t)3 * kKmUpdChunk * 4 /*labels, order, entries*/ +
                       (size_t)(4 * C + 2) * 4 /*offs, cursor, ioff, signed counts*/ +
                       (size_t)2 * km_upd_max_items(C) * 4 /*item group, item start*/;
  return std::max(chunk, (size_t)D * D * sizeof(double) /*Gc during the re-decision*/);
}

__device__ __forceinline__ int km_tiles_per_head(const Layout& L) { return (L.N + kKmTile - 1) / kKmTile; }

// Tile range [t0, t1) of CTA c of G over T = BH * tiles_per_head tiles.
__device__ __forceinline__ void km_range(long long T, int G, int c, int& t0, int& t1) {
  t0 = (int)(T * c / G);
  t1 = (int)(T * (c + 1) / G);
}

// Groups are scored in chunks of at most kKmChunk (all of W of a chunk sits in shared memory
// and a chunk's scores in one TMEM accumulator).  With more groups than that, one launch per
// chunk: chunk ci covers groups [c0, c0 + cn); every launch but the last merges its best two
// scores into each point's running best two (ktop / qtop), and the last one writes the label.
constexpr int kKmChunk = kKmChunkGroups;

template <bool kKeys>
__global__ void __launch_bounds__(kKmThreads, 1)
    kmeans_assign_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                            Layout L, int it, int G, int S, int c0g, int cn, int ci, int nci) {
  pdl_entry();
  const int which = kKeys ? 0 : 1;
  const int D = L.d, KB = D / 64;
  const int C = kKeys ? L.Ck : L.Cq;
  const int NpAll = kKeys ? L.Ckp : L.Cqp;      // padded groups of the head's W rows
  const int Np = nci == 1 ? NpAll : (cn + 15) / 16 * 16;  // padded groups of this chunk
  const int Npr = (Np + 31) & ~31;  // score columns: the epilogue reads 32 at a time
  const bool first = ci == 0, last = ci == nci - 1;
  int4* top = kKeys ? L.ktop : L.qtop;  // running best two of every point across chunks
  // With at most 128 (padded) groups, a multiple of 32, the hi and mid terms of W form one B
  // operand of 2 Np rows (one N = 2 Np MMA per K step writes X W_hi and X W_mid side by side)
  // and the lo term adds into the hi half (N = Np): 16 MMAs per tile instead of 24, measured
  // faster per flop.  The epilogue adds the two halves.
  const bool stack = Np <= 128 && (Np & 31) == 0;
  const int A = stack ? 2 * Np : Npr;  // columns per TMEM accumulator
  const int tph = km_tiles_per_head(L);
  int t0, t1;
  km_range((long long)L.BH * tph, G, blockIdx.x, t0, t1);
  if (t0 >= t1) return;  // uniform, before any barrier or TMEM use

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sW = sm;                                   // [KB][kKmWTerms terms][Np rows][128 B]
  uint8_t* sX = sW + (size_t)kKmWTerms * Np * D * 2;  // [S][KB][128 rows][128 B]
  uint64_t* bars = (uint64_t*)(sX + (size_t)S * kKmTile * D * 2);
  uint64_t* x_full = bars;                            // [S]
  uint64_t* x_empty = bars + kKmMaxStages;            // [S]
  uint64_t* acc_full = bars + 2 * kKmMaxStages;       // [2]
  uint64_t* acc_empty = acc_full + 2;                 // [2]
  uint64_t* w_full = acc_empty + 2;
  uint64_t* w_empty = w_full + 1;
  uint64_t* mma_done = w_empty + 1;
  uint32_t* tmem_slot = (uint32_t*)(mma_done + 1);
  float* sBias = (float*)(bars + 32);                 // [8 epilogue warps][256]
  __shared__ volatile int s_abort;
  __shared__ int s_rcnt;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t tcols = km_tc_tmem_cols(2 * A);  // two accumulators of A columns
  if (tid == 0) {
    s_abort = 0;
    s_rcnt = 0;
    for (int s = 0; s < S; ++s) {
      mbar_init(x_full + s, 1);
      mbar_init(x_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full + b, 1);
      mbar_init(acc_empty + b, 128);
    }
    mbar_init(w_full, 1);
    mbar_init(w_empty, 1);
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // every role walks the same tiles: those of heads whose loop has not stopped
  auto active = [&](int t) { return it < L.stop_at[(t / tph) * 2 + which]; };

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmX);
      prefetch_tmap(&tmW);
      int i = 0, wloads = 0, cur = -1;
      for (int t = t0; t < t1; ++t) {
        if (!active(t)) continue;
        const int bh = t / tph;
        if (bh != cur) {  // the head's W, once the MMAs on the previous head's W have completed
          if (wloads > 0 && !mbar_wait(w_empty, (wloads - 1) & 1, &s_abort)) break;
          mbar_arrive_expect_tx(w_full, (uint32_t)(kKmWTerms * Np * D * 2));
          for (int term = 0; term < kKmWTerms; ++term)
            for (int kb = 0; kb < KB; ++kb)
              tma_load_2d(sW + ((size_t)kb * kKmWTerms + term) * Np * 128, &tmW, w_full, kb * 64,
                          term * L.BH * NpAll + bh * NpAll + c0g);
          ++wloads;
          cur = bh;
        }
        const int s = i % S;
        if (i >= S && !mbar_wait(x_empty + s, ((i / S) - 1) & 1, &s_abort)) break;
        mbar_arrive_expect_tx(x_full + s, (uint32_t)(kKmTile * D * 2));
        for (int kb = 0; kb < KB; ++kb)
          tma_load_2d(sX + ((size_t)s * KB + kb) * kKmTile * 128, &tmX, x_full + s, kb * 64,
                      bh * L.N + (t % tph) * kKmTile);
        ++i;
      }
      // never leave with copies in flight into this CTA's shared memory
      for (int j = max(0, i - S); j < i; ++j) mbar_wait_drain(x_full + (j % S), (j / S) & 1);
      if (wloads > 0) mbar_wait_drain(w_full, (wloads - 1) & 1);
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kKmTile, Np, 0, 0);
      const uint32_t idesc2 = idesc_bf16_f32(kKmTile, stack ? 2 * Np : Np, 0, 0);
      int i = 0, wl = 0, cur = -1;
      for (int t = t0; t < t1; ++t) {
        if (!active(t)) continue;
        const int bh = t / tph;
        if (bh != cur) {
          if (wl > 0) mma_commit(w_empty);  // the previous head's W is free once these complete
          if (!mbar_wait(w_full, wl & 1, &s_abort)) break;
          ++wl;
          cur = bh;
        }
        const int s = i % S, b = i & 1;
        if (!mbar_wait(x_full + s, (i / S) & 1, &s_abort)) break;
        if (i >= 2 && !mbar_wait(acc_empty + b, ((i >> 1) - 1) & 1, &s_abort)) break;
        tc_fence_after();
        auto wdesc = [&](int term, int ks) {  // K step ks of W term `term` (rows contiguous per kb)
          return sdesc_sw128(smem_u32(sW + ((size_t)(ks >> 2) * kKmWTerms + term) * Np * 128) + (ks & 3) * 32, 16,
                             1024);
        };
        auto xdesc = [&](int ks) {
          return sdesc_sw128(smem_u32(sX + ((size_t)s * KB + (ks >> 2)) * kKmTile * 128) + (ks & 3) * 32, 16, 1024);
        };
        if (stack) {
          for (int ks = 0; ks < D / 16; ++ks) {
            mma_ss(tmem + b * A, xdesc(ks), wdesc(0, ks), idesc2, ks > 0 ? 1u : 0u);  // [X W_hi | X W_mid]
            if (kKmWTerms == 3) mma_ss(tmem + b * A, xdesc(ks), wdesc(2, ks), idesc, 1u);  // X W_lo into hi
          }
        } else {
          uint32_t acc = 0;
          for (int term = 0; term < kKmWTerms; ++term)
            for (int ks = 0; ks < D / 16; ++ks) {
              mma_ss(tmem + b * A, xdesc(ks), wdesc(term, ks), idesc, acc);
              acc = 1;
            }
        }
        mma_commit(x_empty + s);
        mma_commit(acc_full + b);
        ++i;
      }
      // every MMA issued by this thread has completed before TMEM is released
      mma_commit(mma_done);
      mbar_wait_drain(mma_done, 0);
    }
  } else if (warp >= 4) {
    // ================================================================ epilogue
    const int e = (warp - 4) >> 2;          // warpgroup: the CTA's active tiles k with k % 2 == e
    const int q = tid - 128 - 128 * e;      // point of the tile = TMEM lane
    const int ew = warp - 4;
    float* bias = sBias + ew * 256;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    int* labels = kKeys ? L.klabel : L.qlabel;
    double* Jarr = kKeys ? L.kJ : L.qJ;
    int* refined = kKeys ? L.krefined : L.qrefined;
    const float u = 1.1920929e-7f;  // 2^-23
    double jsum = 0.0;
    int nref = 0, cur = -1;
    float wmax = 0.f, bmax = 0.f;
    auto flush = [&](int bh) {  // this warp's objective and re-decision count of head bh
      const double js = warp_sum(jsum);
      const int nr = (int)warp_sum((double)nref);
      if (lane == 0) {
        atomicAdd(Jarr + (size_t)bh * L.iters_cap + it, js);
        if (nr) atomicAdd(refined + bh, nr);
      }
      jsum = 0.0;
      nref = 0;
    };
    auto next_active = [&](int t) {
      while (t < t1 && !active(t)) ++t;
      return t;
    };
    // per-point scalars of a tile: 1/rms (queries) and the norm in the rounding bound
    auto scalars = [&](int t, float& sq, float& xn) {
      sq = 0.f;
      xn = 0.f;
      if (t >= t1) return;
      const int bh = t / tph, p0 = (t % tph) * kKmTile;
      if (q < L.N - p0) {
        const size_t row = (size_t)bh * L.N + p0 + q;
        sq = kKeys ? 1.f : L.inv_rms[row];
        xn = kKeys ? L.knorm[row] : L.qxnorm[row];
      }
    };
    // x . w_j for groups j = c0 .. c0 + 31 from accumulator b: one TMEM read, or with the stacked
    // terms two (columns c0 and Np + c0 of the accumulator, both inside its 2 Np columns) added
    auto load_dots = [&](int b, int c0, float (&r)[32]) {
      uint32_t u[32];
      tmem_ld32(tmem + lane_base + b * A + c0, u);
      if (stack) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + b * A + Np + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int kk = 0; kk < 32; ++kk) r[kk] = __uint_as_float(u[kk]) + __uint_as_float(v[kk]);
      } else {
        tmem_wait_ld();
#pragma unroll
        for (int kk = 0; kk < 32; ++kk) r[kk] = __uint_as_float(u[kk]);
      }
    };
    int t = next_active(t0), k = 0;
    if (e == 1 && t < t1) {
      t = next_active(t + 1);
      k = 1;
    }
    float sq, xn;
    scalars(t, sq, xn);
    while (t < t1) {
      int tn = next_active(t + 1);
      if (tn < t1) tn = next_active(tn + 1);  // this warpgroup's next tile
      float nsq, nxn;
      scalars(tn, nsq, nxn);                  // in flight while this tile is scanned
      const int bh = t / tph;
      if (bh != cur) {
        if (cur >= 0 && last) flush(cur);
        cur = bh;
        // the head's biases (this warp's copy) and the maxima of the bound.  Columns C .. Npr-1
        // (padded groups, and columns the MMA does not write) get +inf: their score is +inf or
        // nan, which never wins.
        const float* B32 = (kKeys ? L.kbias32 : L.qbias32) + (size_t)bh * C;
        const float* WN = (kKeys ? L.kwnorm : L.qwnorm) + (size_t)bh * C;
        __syncwarp();  // every lane is done with the previous head's copy
        float wm = 0.f, bm = 0.f;
        for (int j = lane; j < kKmChunk; j += 32) bias[j] = j < cn ? B32[c0g + j] : INFINITY;
        for (int j = lane; j < C; j += 32) {  // the bound takes the maxima over all groups
          bm = fmaxf(bm, fabsf(B32[j]));
          wm = fmaxf(wm, WN[j]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          wm = fmaxf(wm, __shfl_xor_sync(0xffffffffu, wm, o));
          bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
        }
        wmax = wm;
        bmax = bm;
        __syncwarp();
      }
      const int p0 = (t % tph) * kKmTile;
      const bool valid = q < L.N - p0;
      const size_t row = (size_t)bh * L.N + p0 + q;
      const int b = k & 1;
      // warp-uniform: the tcgen05.ld below needs every lane of the warp
      const bool okw = mbar_wait(acc_full + b, (k >> 1) & 1, &s_abort);
      if (!__all_sync(0xffffffffu, okw)) break;
      tc_fence_after();
      const float m2s = -2.f * sq;
      float b1 = INFINITY, b2 = INFINITY;
      int i1 = -1;
      for (int c0 = 0; c0 < Npr; c0 += 32) {
        // columns C .. Npr-1 (padded groups) have bias +inf and never win
        float r[32];
        load_dots(b, c0, r);
        float bq[8][4];
#pragma unroll
        for (int k4 = 0; k4 < 8; ++k4) {
          const float4 v4 = reinterpret_cast<const float4*>(bias + c0)[k4];
          bq[k4][0] = v4.x;
          bq[k4][1] = v4.y;
          bq[k4][2] = v4.z;
          bq[k4][3] = v4.w;
        }
#pragma unroll
        for (int kk = 0; kk < 32; ++kk) {
          // ascending j and strict <: the lowest index of equal scores wins (the biases are read
          // four at a time: 16-byte shared-memory loads, a quarter of the load instructions)
          const float sc = fmaf(m2s, r[kk], bq[kk >> 2][kk & 3]);
          const bool lt = sc < b1;
          b2 = lt ? b1 : fminf(b2, sc);
          i1 = lt ? c0 + kk : i1;
          b1 = lt ? sc : b1;
        }
      }
      if (!first && valid) {  // merge with the best two of the earlier chunks (lower indices win ties)
        const int4 pv = top[row];
        const float pb1 = __int_as_float(pv.x), pb2 = __int_as_float(pv.y);
        if (b1 < pb1) {
          b2 = fminf(pb1, b2);
          i1 += c0g;
        } else {
          b2 = fminf(pb2, b1);
          b1 = pb1;
          i1 = pv.z;
        }
      } else if (i1 >= 0) {
        i1 += c0g;
      }
      if (!last) {  // not the last chunk: keep the running best two for the next launch
        tc_fence_before();
        mbar_arrive(acc_empty + b);
        if (valid) top[row] = make_int4(__float_as_int(b1), __float_as_int(b2), i1, 0);
        t = tn;
        k += 2;
        sq = nsq;
        xn = nxn;
        continue;
      }
      // rounding bound of the fp32 scores: kKmWTerms * D products in one fp32 chain, plus the
      // epilogue's operations (the stacked form sums the terms in two chains and adds them once,
      // which the same bound covers), plus, with two terms, the split error 2^-18 |x| |w|
      const float delta = kKmWTerms == 3
                              ? 4.f * (3 * D + 8) * u * xn * wmax + 4.f * u * bmax
                              : (4.f * (2 * D + 8) * u + 4.f * 3.81469727e-6f) * xn * wmax + 4.f * u * bmax;
      const bool ref = valid && !(b2 - b1 > 2.f * delta);
      // candidates of a flagged point: every group whose fp32 score is within the bound of the
      // best (the fp64 argmin is among them).  With at most 128 groups the warp reads its scores
      // once more (warp-uniform branch, before the accumulator is released).
      int nc = 255;
      uint32_t cpk = 0;  // up to four candidate groups, 8 bits each
      if (nci == 1 && Npr <= 128 && __any_sync(0xffffffffu, ref)) {
        const float thr = b1 + 2.5f * delta;
        int cnt = 0;
#pragma unroll 1
        for (int c0 = 0; c0 < Npr; c0 += 32) {
          float r[32];
          load_dots(b, c0, r);
          if (ref) {
#pragma unroll
            for (int kk = 0; kk < 32; ++kk) {
              const float sc = fmaf(m2s, r[kk], bias[c0 + kk]);
              if (sc <= thr) {
                if (cnt < 4) cpk |= (uint32_t)(c0 + kk) << (8 * cnt);
                ++cnt;
              }
            }
          }
        }
        if (ref) nc = (cnt > 4 || cnt == 0) ? 255 : cnt;
      }
      tc_fence_before();
      mbar_arrive(acc_empty + b);
      if (valid) {
        labels[row] = (i1 >= 0 && i1 < C) ? i1 : 0;  // non-finite scores never yield a bad label
        jsum += (double)b1;
        if (ref) {
          const int c0 = cpk & 0xFF, c1 = (cpk >> 8) & 0xFF, c2 = (cpk >> 16) & 0xFF, c3 = cpk >> 24;
          const int slot = atomicAdd(&s_rcnt, 1);
          L.rlist[(size_t)t0 * kKmTile + slot] =
              make_int4((int)row, __float_as_int(b1), nc | (c0 << 8) | (c1 << 18), c2 | (c3 << 16));
          ++nref;
        }
      }
      t = tn;
      k += 2;
      sq = nsq;
      xn = nxn;
    }
    if (cur >= 0 && last) flush(cur);
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    if (last) L.rcnt[blockIdx.x] = s_rcnt;
    if (s_abort) atomicCAS(L.status, kDevOk, kDevTimeout);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}

// fp64 re-decision of the points the assignment listed for CTA range c, run by the update
// kernel's CTA c before it reads the labels (the ranges of the two kernels are the same): the
// CTA's warps take every kKmUpdWarps-th entry, one warp per point; the label and the objective
// (its fp64 score minus the tentative fp32 one) are corrected in place.  Points with a short
// candidate list evaluate only those groups; queries stage Gc in shared memory (gcs: d * d
// doubles, free until the update's chunk loop) for the exact scale.  Every thread of the CTA
// calls this (it has block barriers).
constexpr int kKmUpdWarps = kKmUpdThreads / 32;

template <bool kKeys>
__device__ __forceinline__ void redecide_range(const __nv_bfloat16* __restrict__ X, const Layout& L, int it, int t0,
                                               int t1, double* gcs) {
  __shared__ double xs_all[kKmUpdWarps][128];
  __shared__ int s_need[kKmUpdWarps];
  const int D = L.d, C = kKeys ? L.Ck : L.Cq;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nlist = min(max(L.rcnt[blockIdx.x], 0), max(t1 - t0, 0) * kKmTile);  // never past the segment
  const int4* list = L.rlist + (size_t)t0 * kKmTile;
  int* labels = kKeys ? L.klabel : L.qlabel;
  double* Jarr = kKeys ? L.kJ : L.qJ;
  double* xs = xs_all[warp];
  int gc_head = -1;  // head whose Gc is staged (the range spans few heads; stage per change)
  for (int li0 = 0; li0 < nlist; li0 += kKmUpdWarps) {  // the same trip count in every thread
    const int li = li0 + warp;
    int bh = -1;
    int4 en = make_int4(0, 0, 0, 0);
    if (li < nlist) {
      en = list[li];
      bh = en.x / L.N;
    }
    if constexpr (!kKeys) {  // the CTA's warps agree on the heads they need: stage on change
      const int need = __shfl_sync(0xffffffffu, bh, 0);
      if (lane == 0) s_need[warp] = need;
      __syncthreads();
      int first = -1;
      bool mixed = false;
      for (int w = 0; w < kKmUpdWarps; ++w)
        if (s_need[w] >= 0) {
          if (first < 0) first = s_need[w];
          else if (s_need[w] != first) mixed = true;
        }
      if (!mixed && first >= 0 && first != gc_head) {
        const double* src = L.Gc + (size_t)first * D * D;
        for (int e = threadIdx.x; e < D * D / 2; e += blockDim.x)
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(gcs + 2 * e)),
                       "l"(src + 2 * e)
                       : "memory");
        asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
        gc_head = first;
      } else if (mixed) {
        gc_head = -1;  // heads differ inside this round: read Gc from global memory
      }
      __syncthreads();
    }
    if (li >= nlist) continue;
    const int row = en.x;
    for (int a = lane; a < D; a += 32) xs[a] = (double)__bfloat162float(X[(size_t)row * D + a]);
    __syncwarp();
    int best;
    double bv;
    const double* W64 = (kKeys ? L.kW64 : L.qU64) + (size_t)bh * C * D;
    const double* B64 = (kKeys ? L.kbias64 : L.qbias64) + (size_t)bh * C;
    const double* Gc = (!kKeys && gc_head == bh) ? gcs : L.Gc + (size_t)bh * D * D;
    const int nc = en.z & 0xFF;
    if (nc <= 4) {
      int cand[4] = {(en.z >> 8) & 0x3FF, (en.z >> 18) & 0x3FF, en.w & 0xFFFF, (en.w >> 16) & 0xFFFF};
      double scale = 1.0;
      if (!kKeys && !L.semantic) {
        double xl[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) xl[k] = lane + 32 * k < D ? xs[lane + 32 * k] : 0.0;
        scale = query_scale_fp64(Gc, xs, xl, D);
      }
      redecide_candidates(xs, D, W64, B64, scale, cand, nc, best, bv);
    } else {
      redecide_fp64<kKeys>(L, bh, xs, D, C, W64, B64, best, bv, Gc);
    }
    if (lane == 0) {
      labels[row] = best;
      atomicAdd(Jarr + (size_t)bh * L.iters_cap + it, bv - (double)__int_as_float(en.y));
    }
    __syncwarp();
  }
  __syncthreads();  // final labels are visible to the whole CTA; gcs is free again
}

template <bool kKeys>
__global__ void __launch_bounds__(kKmUpdThreads, 1)
    kmeans_update_kernel(const __nv_bfloat16* __restrict__ X, Layout L, int it, int G) {
  pdl_entry();
  const int which = kKeys ? 0 : 1;
  const int D = L.d;
  const int C = kKeys ? L.Ck : L.Cq;
  const int tph = km_tiles_per_head(L);
  int t0, t1;
  km_range((long long)L.BH * tph, G, blockIdx.x, t0, t1);
  if (t0 >= t1) return;

  extern __shared__ uint8_t smem_raw[];
  // the re-decision of the points the assignment flagged in this range comes first; it may
  // use the start of the dynamic shared memory for Gc (d * d doubles <= the two chunk arrays)
  redecide_range<kKeys>(X, L, it, t0, t1, (double*)smem_raw);
  int* lab = (int*)smem_raw;                   // [kKmUpdChunk] label (key) of each entry of the chunk
  int* order = lab + kKmUpdChunk;              // [kKmUpdChunk] entries sorted by label
  int* ent = order + kKmUpdChunk;              // [kKmUpdChunk] entry codes (label changes only)
  int* offs = ent + kKmUpdChunk;               // [C + 1] start of each label's run
  int* cursor = offs + (C + 1);                // [C] histogram, then next slot per label
  int* ioff = cursor + C;                      // [C + 1] first accumulation item of each label
  int* sdc = ioff + (C + 1);                   // [C] signed count changes (label changes only)
  int* item_g = sdc + C;                       // [km_upd_max_items] group of each item
  int* item_s = item_g + km_upd_max_items(C);  // [km_upd_max_items] first slot of `order` of each item
  __shared__ int s_next, s_nent;
  // From the second iteration on (tensor-core path), the sums and counts move only by the
  // points whose label changed since the iteration before: each such point is two entries, -x
  // under its old label and +x under its new one (code 2 i + 1 and 2 i), summed through the same
  // sort and items as a full pass.  Key sums of bf16 inputs are exact in fp64, so this equals a
  // full pass; query sums (scaled by 1/rms) agree to rounding.  The first iteration sums every
  // point and records the labels in prev.
  const bool delta = it > 0;
  int* prev = kKeys ? L.kprev : L.qprev;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int* labels = kKeys ? L.klabel : L.qlabel;
  double* sums_all = kKeys ? L.ksum : L.qsum;
  int* counts_all = kKeys ? L.kcount : L.qcount;
  const int octs = D / 8;  // threads per row: eight dimensions (16 bytes) each
  int t = t0;
  while (t < t1) {
    const int bh = t / tph;
    if (it >= L.stop_at[bh * 2 + which]) {  // this head's loop has stopped: skip its tiles
      t = (bh + 1) * tph;
      continue;
    }
    // chunk: tiles [t, te) of head bh, at most kKmUpdChunk points (half as many with label
    // changes: two entries each).  With label changes, the changed points of the head's whole
    // segment of the range are counted first: when their entries fit, the segment is one chunk
    // (after the first iterations few points change, and one sort serves the whole segment).
    const int te_seg = min(t1, (bh + 1) * tph);
    int te = min(te_seg, t + (delta ? kKmUpdChunk / 2 : kKmUpdChunk) / kKmTile);
    auto changed = [&](size_t row) {  // the comparison of the entry pass below
      int gn = labels[row], go = prev[row];
      gn = (gn >= 0 && gn < C) ? gn : 0;
      go = (go >= 0 && go < C) ? go : 0;
      return gn != go;
    };
    if (delta && te < te_seg) {
      const int q_lo = (t % tph) * kKmTile, q_hi = min(L.N, (te_seg - 1) % tph * kKmTile + kKmTile);
      const size_t r0 = (size_t)bh * L.N + q_lo;
      if (tid == 0) s_nent = 0;
      __syncthreads();
      int c = 0;
      const int nq = q_hi - q_lo;
      for (int i0 = tid; i0 < nq; i0 += 8 * kKmUpdThreads) {  // eight points per thread in flight
        bool chg[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = i0 + u * kKmUpdThreads;
          chg[u] = i < nq && changed(r0 + i);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) c += chg[u] ? 1 : 0;
      }
      c = __reduce_add_sync(0xffffffffu, c);
      if (lane == 0 && c) atomicAdd(&s_nent, c);
      __syncthreads();
      if (2 * s_nent <= kKmUpdChunk) te = te_seg;
      __syncthreads();  // s_nent is reset below
    }
    const int p_lo = (t % tph) * kKmTile;
    const int p_hi = min(L.N, (te - 1) % tph * kKmTile + kKmTile);
    const int np = p_hi - p_lo;
    const size_t row0 = (size_t)bh * L.N + p_lo;
    for (int j = tid; j < C; j += kKmUpdThreads) {
      cursor[j] = 0;
      sdc[j] = 0;
    }
    if (tid == 0) s_nent = 0;
    __syncthreads();
    if (delta) {  // the entries of the points whose label changed (eight rounds' loads in flight)
      for (int i00 = 0; i00 < np; i00 += 8 * kKmUpdThreads) {
        int gnv[8], gov[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = i00 + u * kKmUpdThreads + tid;
          gnv[u] = i < np ? labels[row0 + i] : 0;
          gov[u] = i < np ? prev[row0 + i] : 0;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = i00 + u * kKmUpdThreads + tid;
          const int gn = (gnv[u] >= 0 && gnv[u] < C) ? gnv[u] : 0;
          const int go = (gov[u] >= 0 && gov[u] < C) ? gov[u] : 0;
          const bool ch = i < np && gn != go;  // (the same test as `changed`)
          const unsigned m = __ballot_sync(0xffffffffu, ch);
          int base = 0;
          if (lane == 0 && m) base = atomicAdd(&s_nent, 2 * __popc(m));
          base = __shfl_sync(0xffffffffu, base, 0);
          if (ch) {
            const int k = base + 2 * __popc(m & ((1u << lane) - 1));
            lab[k] = go;
            ent[k] = 2 * i + 1;
            lab[k + 1] = gn;
            ent[k + 1] = 2 * i;
            prev[row0 + i] = gn;
            atomicAdd(&sdc[go], -1);
            atomicAdd(&sdc[gn], 1);
          }
        }
      }
      __syncthreads();
    }
    const int n = delta ? s_nent : np;  // entries of the chunk
    // histogram: lanes holding the same label add once (labels are spatially coherent)
    for (int i0 = 0; i0 < n; i0 += kKmUpdThreads) {
      const int i = i0 + tid;
      int g = -1;
      if (i < n) {
        if (delta) {
          g = lab[i];
        } else {
          g = labels[row0 + i];
          g = (g >= 0 && g < C) ? g : 0;
          lab[i] = g;
          prev[row0 + i] = g;
        }
      }
      const unsigned act = __ballot_sync(0xffffffffu, i < n);
      if (i < n) {
        const unsigned same = __match_any_sync(act, g);
        if (lane == __ffs(same) - 1) atomicAdd(&cursor[g], __popc(same));
      }
    }
    __syncthreads();
    if (warp == 0) {  // exclusive prefixes over the groups (slots and items), and the counts
      int run = 0, irun = 0;
      for (int c0 = 0; c0 < C; c0 += 32) {
        const int j = c0 + lane;
        const int v = j < C ? cursor[j] : 0;
        const int nv = (v + kKmUpdItemRows - 1) / kKmUpdItemRows;
        int x = v, y = nv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int a = __shfl_up_sync(0xffffffffu, x, o);
          const int b = __shfl_up_sync(0xffffffffu, y, o);
          if (lane >= o) {
            x += a;
            y += b;
          }
        }
        if (j < C) {
          offs[j] = run + x - v;
          cursor[j] = run + x - v;
          ioff[j] = irun + y - nv;
          const int dc = delta ? sdc[j] : v;  // count change of the group
          if (dc) atomicAdd(counts_all + (size_t)bh * C + j, dc);
        }
        run += __shfl_sync(0xffffffffu, x, 31);
        irun += __shfl_sync(0xffffffffu, y, 31);
      }
      if (lane == 0) {
        offs[C] = run;
        ioff[C] = irun;
      }
    }
    __syncthreads();
    // scatter: lanes with the same label take consecutive slots from one atomic
    for (int i0 = 0; i0 < n; i0 += kKmUpdThreads) {
      const int i = i0 + tid;
      const unsigned act = __ballot_sync(0xffffffffu, i < n);
      if (i < n) {
        const int g = lab[i];
        const unsigned same = __match_any_sync(act, g);
        const int leader = __ffs(same) - 1;
        int base = 0;
        if (lane == leader) base = atomicAdd(&cursor[g], __popc(same));
        base = __shfl_sync(same, base, leader);
        order[base + __popc(same & ((1u << lane) - 1))] = i;
      }
    }
    // the item table: group g's run is cut into pieces of at most kKmUpdItemRows rows
    for (int g = tid; g < C; g += kKmUpdThreads) {
      const int q0 = offs[g], q1 = offs[g + 1];
      for (int i = ioff[g], q = q0; q < q1; ++i, q += kKmUpdItemRows) {
        item_g[i] = g;
        item_s[i] = q;
      }
    }
    if (tid == 0) s_next = 0;
    __syncthreads();
    // accumulation: a warp takes the next 32 / octs items; within it, consecutive lanes read
    // consecutive 16-byte pieces (eight dimensions) of the same rows; each item's rows are summed
    // in fp64 registers and added to the group's sums with one atomic per dimension
    const __nv_bfloat16* Xc = X + row0 * D;
    const double* sig = L.inv_rms64 + row0;
    double* sums = sums_all + (size_t)bh * C * D;
    const int gpw = 32 / octs;
    const int nitems = ioff[C];
    while (true) {
      int k = 0;
      if (lane == 0) k = atomicAdd(&s_next, 1);
      k = __shfl_sync(0xffffffffu, k, 0);
      if (k * gpw >= nitems) break;  // the same for the whole warp
      const int ii = k * gpw + lane / octs;
      if (ii >= nitems) continue;
      const int g = item_g[ii], oc = lane % octs;
      const int q0 = item_s[ii], q1 = min(q0 + kKmUpdItemRows, offs[g + 1]);
      double r[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) r[k] = 0.0;
      int q = q0;
      // entry at sorted slot q: its point and its factor (+1 or -1 for a label change; times the
      // point's 1/rms for queries)
      auto entry = [&](int q, int& p, double& f) {
        const int e = order[q];
        if (delta) {
          const int code = ent[e];
          p = code >> 1;
          f = (code & 1) ? -1.0 : 1.0;
        } else {
          p = e;
          f = 1.0;
        }
        if constexpr (!kKeys) f *= sig[p];
      };
      for (; q + 8 <= q1; q += 8) {  // eight rows in flight per lane
        int pidx[8];
        double fac[8];
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) entry(q + u, pidx[u], fac[u]);
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = *(const uint4*)(Xc + (size_t)pidx[u] * D + 8 * oc);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // (with factor 1 an exact addition)
            r[2 * k] = fma(bf16_bits_to_f64(w[k] & 0xFFFFu), fac[u], r[2 * k]);
            r[2 * k + 1] = fma(bf16_bits_to_f64(w[k] >> 16), fac[u], r[2 * k + 1]);
          }
        }
      }
      for (; q < q1; ++q) {
        int p;
        double sg;
        entry(q, p, sg);
        const uint4 v = *(const uint4*)(Xc + (size_t)p * D + 8 * oc);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          r[2 * k] = fma(bf16_bits_to_f64(w[k] & 0xFFFFu), sg, r[2 * k]);
          r[2 * k + 1] = fma(bf16_bits_to_f64(w[k] >> 16), sg, r[2 * k + 1]);
        }
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) atomicAdd(sums + (size_t)g * D + 8 * oc + k, r[k]);
    }
    __syncthreads();  // lab / order / offs are rewritten by the next chunk
    t = te;
  }
}

// Per-row quadratic forms x^T G x (G = M for keys, Gc for queries) and norms, 128 rows per
// tile: U = X G on the tensor cores (G symmetric, split into three bf16 terms), then each
// thread dots its row of U (TMEM lane) with its row of X (shared memory).
//   keys    (which 0): T0k += sum x^T M x;  knorm = ||x||
//   queries (which 1): ms = x^T Gc x;  inv_rms = 1/sqrt(ms + 1e-12);  qxnorm = ||x|| inv_rms;
//                      T0q += C_k ms / (ms + 1e-12)   (= ||r~||^2)
// Two X stages and two TMEM accumulators: the products of tile i + 1 run while the threads
// read tile i, and the copy of tile i + 2 is issued as soon as tile i's stage is read.
__global__ void __launch_bounds__(128, 1)
    rowqf_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmG, Layout L,
                    int which, int tiles_per_cta) {
  pdl_entry();
  const int bh = blockIdx.y, D = L.d, KB = D / 64;
  const int tile0 = blockIdx.x * tiles_per_cta;
  const int ntiles_head = (L.N + kKmTile - 1) / kKmTile;
  const int ntile = min(tiles_per_cta, ntiles_head - tile0);
  if (ntile <= 0) return;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const size_t xbytes = (size_t)kKmTile * D * 2;
  uint8_t* sG = sm;                              // [3][KB][D rows][128 B]
  uint8_t* sX = sG + (size_t)3 * D * D * 2;      // [2 stages][KB][128 rows][128 B]
  uint64_t* g_full = (uint64_t*)(sX + 2 * xbytes);
  uint64_t* x_full = g_full + 1;                 // [2]
  uint64_t* mma_done = x_full + 2;               // [2]
  uint64_t* mma_all = mma_done + 2;              // every product of the CTA (before TMEM is freed)
  uint32_t* tmem_slot = (uint32_t*)(mma_all + 1);
  __shared__ volatile int s_abort;
  __shared__ double red[4];
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t tcols = km_tc_tmem_cols(2 * D);
  if (tid == 0) {
    s_abort = 0;
    mbar_init(g_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(x_full + b, 1);
      mbar_init(mma_done + b, 1);
    }
    mbar_init(mma_all, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t idesc = idesc_bf16_f32(kKmTile, D, 0, 0);
  int issued = 0;  // X copies issued (thread 0)
  auto load_x = [&](int ti) {  // thread 0: tile ti into stage ti & 1
    const int b = ti & 1;
    mbar_arrive_expect_tx(x_full + b, (uint32_t)xbytes);
    for (int kb = 0; kb < KB; ++kb)
      tma_load_2d(sX + b * xbytes + (size_t)kb * kKmTile * 128, &tmX, x_full + b, kb * 64,
                  bh * L.N + (tile0 + ti) * kKmTile);
    ++issued;
  };
  auto issue_mma = [&](int ti) -> bool {  // thread 0: U_ti = X_ti G into accumulator ti & 1
    const int b = ti & 1;
    if (!mbar_wait(x_full + b, (ti >> 1) & 1, &s_abort)) return false;
    tc_fence_after();
    uint32_t acc = 0;
    for (int gt = 0; gt < 3; ++gt)
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t xa = smem_u32(sX + b * xbytes + (size_t)(ks >> 2) * kKmTile * 128) + (ks & 3) * 32;
        const uint32_t ga = smem_u32(sG + ((size_t)gt * KB + (ks >> 2)) * D * 128) + (ks & 3) * 32;
        mma_ss(tmem + b * D, sdesc_sw128(xa, 16, 1024), sdesc_sw128(ga, 16, 1024), idesc, acc);
        acc = 1;
      }
    mma_commit(mma_done + b);
    return true;
  };
  if (tid == 0) {
    mbar_arrive_expect_tx(g_full, (uint32_t)(3 * D * D * 2));
    for (int t = 0; t < 3; ++t)
      for (int kb = 0; kb < KB; ++kb)
        tma_load_2d(sG + ((size_t)t * KB + kb) * D * 128, &tmG, g_full, kb * 64, t * L.BH * D + bh * D);
    load_x(0);
    if (ntile > 1) load_x(1);
    if (mbar_wait(g_full, 0, &s_abort)) issue_mma(0);
  }
  double tot = 0.0;
  for (int ti = 0; ti < ntile; ++ti) {
    const int b = ti & 1;
    if (tid == 0 && ti + 1 < ntile && !s_abort) issue_mma(ti + 1);  // runs while tile ti is read
    const bool waited = !s_abort && mbar_wait(mma_done + b, (ti >> 1) & 1, &s_abort);
    if (__syncthreads_or(!waited)) break;  // uniform: every thread leaves or none does
    tc_fence_after();
    const int p0 = (tile0 + ti) * kKmTile;
    const int np = min(kKmTile, L.N - p0);
    const int p = tid;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint8_t* xs = sX + b * xbytes;
    float qf = 0.f, nn = 0.f;
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + lane_base + b * D + c0, r);
      tmem_wait_ld();
      // the row's elements eight at a time (16-byte shared-memory loads of the swizzled tile),
      // in the same order: element a = c0 + k, k ascending
#pragma unroll
      for (int k8 = 0; k8 < 4; ++k8) {
        const int a = c0 + 8 * k8, kb = a >> 6, w = a & 63;
        const uint32_t off = (uint32_t)p * 128 + (((w >> 3) ^ (p & 7)) << 4);
        const uint4 v = *(const uint4*)(xs + (size_t)kb * kKmTile * 128 + off);
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float x0 = __uint_as_float(wv[u] << 16), x1 = __uint_as_float(wv[u] & 0xFFFF0000u);
          qf = fmaf(x0, __uint_as_float(r[8 * k8 + 2 * u]), qf);
          nn = fmaf(x0, x0, nn);
          qf = fmaf(x1, __uint_as_float(r[8 * k8 + 2 * u + 1]), qf);
          nn = fmaf(x1, x1, nn);
        }
      }
    }
    if (p < np) {
      const size_t row = (size_t)bh * L.N + p0 + p;
      if (which == 0) {
        L.knorm[row] = sqrtf(nn);
        tot += (double)qf;
      } else {
        const double ms = (double)qf;
        if (L.semantic) {  // raw queries: scale 1, objective constant ||q||^2
          L.inv_rms[row] = 1.f;
          L.inv_rms64[row] = 1.0;
          L.qxnorm[row] = sqrtf(nn);
          tot += ms;
        } else {
          const float inv = (float)(1.0 / sqrt(ms + 1e-12));
          L.inv_rms[row] = inv;
          L.inv_rms64[row] = 1.0 / sqrt(ms + 1e-12);
          L.qxnorm[row] = sqrtf(nn) * inv;
          tot += (double)L.Ck * ms / (ms + 1e-12);
        }
      }
    }
    tc_fence_before();
    __syncthreads();  // stage b and accumulator b are read: the copy of tile ti + 2 may land in b
    if (tid == 0 && ti + 2 < ntile && !s_abort) load_x(ti + 2);
  }
  tot = block_sum(tot, red);
  if (tid == 0) {
    atomicAdd((which == 0 ? L.T0k : L.T0q) + bh, tot);
    if (s_abort) {
      atomicCAS(L.status, kDevOk, kDevTimeout);
      // never leave with copies or products in flight: the last copies issued into each stage,
      // and every product committed so far
      mbar_wait_drain(g_full, 0);
      for (int ti = max(0, issued - 2); ti < issued; ++ti) mbar_wait_drain(x_full + (ti & 1), (ti >> 1) & 1);
    }
    mma_commit(mma_all);  // arrives once every MMA this thread issued has completed
    mbar_wait_drain(mma_all, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}

// ----------------------------------------------------------------------------------- host
static int km_stages(const Layout& L, int Np) {
  const size_t budget = 227 * 1024;
  const size_t fixed = km_assign_smem(L.d, Np, 0);
  if (fixed >= budget) return 0;
  const size_t per = (size_t)kKmTile * L.d * 2;
  return (int)std::min<size_t>(kKmMaxStages, (budget - fixed) / per);
}

// Padded groups of one assignment launch: all of them, or a chunk of kKmChunk.
static int km_chunk_rows(const Layout& L, bool keys) {
  const int Np = keys ? L.Ckp : L.Cqp;
  return Np <= kKmChunk ? Np : kKmChunk;
}

bool km_tc_supported(const Layout& L, bool keys) {
  if (L.dtype != SPARSEPR_BF16) return false;
  const int C = keys ? L.Ck : L.Cq;
  const bool chunked = (keys ? L.Ckp : L.Cqp) > kKmChunk;
  if (chunked && !(keys ? L.ktop : L.qtop)) return false;
  return km_stages(L, km_chunk_rows(L, keys)) >= 2 && km_update_smem(L.d, C) + kKmUpdStaticSmem <= 227 * 1024;
}

// CTAs of both k-means kernels: as many as fit the device at once (so the static ranges run in
// one wave), at most one per tile.
int km_tc_grid(const Layout& L, bool keys) {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  const int Np = km_chunk_rows(L, keys);
  const int S = km_stages(L, Np);
  const size_t smem = km_assign_smem(L.d, Np, S);
  int occ = 1;
  if (keys) {
    cudaFuncSetAttribute(kmeans_assign_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kmeans_assign_tc_kernel<true>, kKmThreads, smem);
  } else {
    cudaFuncSetAttribute(kmeans_assign_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kmeans_assign_tc_kernel<false>, kKmThreads, smem);
  }
  occ = std::max(1, std::min(occ, 2));
  const long long T = (long long)L.BH * ((L.N + kKmTile - 1) / kKmTile);
  return (int)std::min<long long>(T, (long long)sms * occ);
}

sparsepr_status launch_kmeans_iteration_tc(const Layout& L, bool keys, const void* X, int it, int G,
                                           cudaStream_t st, const KernelEvents* ev) {
  auto mark = [&](int id, bool stop) {
    const cudaEvent_t e = ev ? (stop ? ev->stop[id] : ev->start[id]) : nullptr;
    if (e) cudaEventRecord(e, st);
  };
  CUtensorMap mX, mW;
  const int D = L.d;
  const int NpAll = keys ? L.Ckp : L.Cqp;
  const int C = keys ? L.Ck : L.Cq;
  const void* wbase = keys ? (const void*)L.kWb : (const void*)L.qWb;
  if (!make_tmap_bf16(&mX, X, (long long)L.BH * L.N, D, kKmTile)) return SPARSEPR_ERR_CUDA;
  const int nci = NpAll <= kKmChunk ? 1 : (C + kKmChunk - 1) / kKmChunk;
  const int S = km_stages(L, km_chunk_rows(L, keys));
  const size_t smem_a = km_assign_smem(D, km_chunk_rows(L, keys), S);
  const size_t smem_u = km_update_smem(D, C);
  const __nv_bfloat16* Xb = (const __nv_bfloat16*)X;
  auto assign = keys ? kmeans_assign_tc_kernel<true> : kmeans_assign_tc_kernel<false>;
  auto update = keys ? kmeans_update_kernel<true> : kmeans_update_kernel<false>;
  cudaFuncSetAttribute(assign, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_a);
  cudaFuncSetAttribute(update, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_u);
  if (keys) mark(SPARSEPR_KERNEL_KMEANS_ASSIGN, false);
  for (int ci = 0; ci < nci; ++ci) {
    // chunk ci: groups [c0, c0 + cn), W rows [c0, c0 + round16(cn)) of each head and term
    const int c0 = ci * kKmChunk, cn = nci == 1 ? C : std::min(kKmChunk, C - c0);
    const int rows = nci == 1 ? NpAll : (cn + 15) / 16 * 16;
    if (!make_tmap_bf16(&mW, wbase, 3LL * L.BH * NpAll, D, rows)) return SPARSEPR_ERR_CUDA;
    launch(assign, G, kKmThreads, smem_a, st, mX, mW, L, it, G, S, c0, cn, ci, nci);
  }
  if (keys) mark(SPARSEPR_KERNEL_KMEANS_ASSIGN, true);
  if (keys) mark(SPARSEPR_KERNEL_KMEANS_UPDATE, false);
  launch(update, G, kKmUpdThreads, smem_u, st, Xb, L, it, G);
  if (keys) mark(SPARSEPR_KERNEL_KMEANS_UPDATE, true);
  SPR_LAUNCH_CHECK();
  return SPARSEPR_OK;
}

// Tiles per CTA of the row quadratic forms: enough CTAs for about four per SM.
static int tiles_per_cta(const Layout& L) {
  const int ntiles = (L.N + kKmTile - 1) / kKmTile;
  int tpc = (int)(((long long)ntiles * L.BH + 148 * 4 - 1) / (148 * 4));
  return tpc < 1 ? 1 : (tpc > 16 ? 16 : tpc);
}

sparsepr_status launch_rowqf_tc(const Layout& L, int which, const void* X, cudaStream_t st) {
  CUtensorMap mX, mG;
  const int D = L.d;
  const void* gbase = which == 0 ? (const void*)L.Mb : (const void*)L.Gcb;
  if (!make_tmap_bf16(&mX, X, (long long)L.BH * L.N, D, kKmTile) ||
      !make_tmap_bf16(&mG, gbase, 3LL * L.BH * D, D, D))
    return SPARSEPR_ERR_CUDA;
  const size_t smem = (size_t)3 * D * D * 2 + (size_t)2 * kKmTile * D * 2 + 1024 + 64;
  const int tpc = tiles_per_cta(L);
  const int ntiles = (L.N + kKmTile - 1) / kKmTile;
  cudaFuncSetAttribute(rowqf_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  launch(rowqf_tc_kernel, dim3((ntiles + tpc - 1) / tpc, L.BH), dim3(128), smem, st, mX, mG, L, which, tpc);
  SPR_LAUNCH_CHECK();
  return SPARSEPR_OK;
}

}  // namespace sparsepr
