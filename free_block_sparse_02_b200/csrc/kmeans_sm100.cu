// k-means assignment and per-row quadratic forms of the partition on the tensor cores
// (tcgen05, results in TMEM, operands by TMA).
//
// "Partition the Support, Reconstruct the Residual" (arXiv 2608.18484), abstract: keys are
// grouped by their responses to sampled queries, queries by their responses to the key-group
// centroids; both groupings are k-means (Table C.1: 25 / 2 iterations, tolerance 1e-4).
//
// Both k-means run on the d-dimensional inputs (see partition.cu): the score of point x against
// group j is  s_j = b_j - 2 sigma_x (x . w_j)  with (keys) w = M c, b = c^T M c, sigma = 1, or
// (queries) w = u = C^T nu / sqrt(d), b = ||nu||^2, sigma = 1/rms_q; the label is argmin_j s_j,
// lowest j on ties.  The dot products of a 128-point tile against every group are one MMA chain:
// X (128 x d, bf16, exact) times W^T (d x C), W split into three bf16 terms (hi + mid + lo)
// accumulated in fp32 in TMEM, which gives fp32-grade dots.  The epilogue (two threads per
// point, its TMEM lane) keeps the best two scores; a point whose two best are within a
// rigorous rounding bound is re-decided over all groups in fp64 by one warp, so labels agree
// with an fp64 evaluation.  The objective takes the chosen group's score; the group sums
// (fp64, of sigma x) are accumulated per run of equal labels after a counting sort of the
// tile and flushed with one atomic per (run, dim).
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"
#include "kmeans.cuh"
#include "sm100.cuh"

namespace sparsepr {

using namespace sm100;

constexpr int kKmTile = 128;

__host__ __device__ inline int km_tc_tmem_cols(int n) {
  int c = 32;
  while (c < n) c <<= 1;
  return c;
}

__host__ inline size_t km_tc_smem(int D, int Np) {
  const size_t w = (size_t)3 * Np * D * 2;
  const size_t x = (size_t)kKmTile * D * 2;
  return w + x + 1024 /*align*/ + 24576 /*bias, scale, labels, order, list, histogram, merge, scores, rows*/;
}

// Tiles per CTA: enough CTAs for about four per SM; each loads the weights once for its tiles.
static int tiles_per_cta(const Layout& L) {
  const int ntiles = (L.N + kKmTile - 1) / kKmTile;
  int tpc = (int)(((long long)ntiles * L.BH + 148 * 4 - 1) / (148 * 4));
  return tpc < 1 ? 1 : (tpc > 16 ? 16 : tpc);
}

template <bool kKeys>
__global__ void __launch_bounds__(256, 1)
    kmeans_assign_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                            Layout L, int it, int tiles_per_cta) {
  const int bh = blockIdx.y;
  const int which = kKeys ? 0 : 1;
  if (it >= L.stop_at[bh * 2 + which]) return;
  const int D = L.d;
  const int C = kKeys ? L.Ck : L.Cq;
  const int Np = kKeys ? L.Ckp : L.Cqp;
  const int KB = D / 64;
  const int tile0 = blockIdx.x * tiles_per_cta;
  const int ntiles_head = (L.N + kKmTile - 1) / kKmTile;
  const int ntile = min(tiles_per_cta, ntiles_head - tile0);
  if (ntile <= 0) return;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sW = sm;                                   // [3 terms][KB][Np rows][128 B]
  uint8_t* sX = sW + (size_t)3 * Np * D * 2;          // [KB][128 rows][128 B]
  float* sB = (float*)(sX + (size_t)kKmTile * D * 2);  // [256] bias
  float* scl = sB + 256;                             // [128] sigma of each point
  int* lab = (int*)(scl + kKmTile);                  // [128]
  int* order = lab + kKmTile;                        // [128]
  int* rlist = order + kKmTile;                      // [128] points to re-decide
  int* hist = rlist + kKmTile;                       // [256] points per label in the tile
  int* cursor = hist + 256;                          // [256] next slot per label
  float* mb1 = (float*)(cursor + 256);               // [128] partial best / second / index
  float* mb2 = mb1 + kKmTile;
  int* mi1 = (int*)(mb2 + kKmTile);
  double* bval = (double*)(mi1 + kKmTile);           // [128] score of the chosen group
  double* xs64 = bval + kKmTile;                     // [8 warps][128] fp64 features
  uint64_t* bars = (uint64_t*)(xs64 + 8 * 128);      // w_full, x_full, mma_done
  uint32_t* tmem_slot = (uint32_t*)(bars + 3);
  __shared__ volatile int s_abort;
  __shared__ float s_wmax, s_bmax;
  __shared__ int s_nlist;
  __shared__ double red[8];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* B32 = (kKeys ? L.kbias32 : L.qbias32) + (size_t)bh * C;
  const float* WN = (kKeys ? L.kwnorm : L.qwnorm) + (size_t)bh * C;
  const double* W64 = (kKeys ? L.kW64 : L.qU64) + (size_t)bh * C * D;
  const double* B64 = (kKeys ? L.kbias64 : L.qbias64) + (size_t)bh * C;
  const uint32_t tcols = km_tc_tmem_cols(Np);

  if (tid == 0) {
    s_abort = 0;
    s_nlist = 0;
    mbar_init(bars + 0, 1);
    mbar_init(bars + 1, 1);
    mbar_init(bars + 2, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, tcols);
    tmem_relinquish();
  }
  for (int j = tid; j < 256; j += blockDim.x) sB[j] = j < C ? B32[j] : INFINITY;
  {
    float wm = 0.f, bm = 0.f;
    for (int j = tid; j < C; j += blockDim.x) {
      wm = fmaxf(wm, WN[j]);
      bm = fmaxf(bm, fabsf(B32[j]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      wm = fmaxf(wm, __shfl_xor_sync(0xffffffffu, wm, o));
      bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
    }
    __shared__ float pw[8], pb[8];
    if (lane == 0) {
      pw[warp] = wm;
      pb[warp] = bm;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      float a = 0.f, b = 0.f;
      for (int w = 0; w < 8; ++w) {
        a = fmaxf(a, pw[w]);
        b = fmaxf(b, pb[w]);
      }
      s_wmax = a;
      s_bmax = b;
    }
  }
  const uint32_t tmem = *tmem_slot;
  if (tid == 0) {  // weights: 3 terms x KB column blocks, one TMA box of Np rows each
    mbar_arrive_expect_tx(bars + 0, (uint32_t)(3 * Np * D * 2));
    for (int t = 0; t < 3; ++t)
      for (int kb = 0; kb < KB; ++kb)
        tma_load_2d(sW + ((size_t)t * KB + kb) * Np * 128, &tmW, bars + 0, kb * 64, t * L.BH * Np + bh * Np);
  }
  __syncthreads();

  const uint32_t idesc = idesc_bf16_f32(kKmTile, Np, 0, 0);
  // |error of b - 2 sigma x.w| <= 2 sigma ||x|| ||w|| (3D + 8) 2^-23 (three-term split, fp32
  // accumulation) + 2^-23 |b|; a factor-2 margin on top
  const float u = 1.1920929e-7f;  // 2^-23
  double jsum = 0.0;
  int nref = 0;
  for (int ti = 0; ti < ntile && !s_abort; ++ti) {
    const int p0 = (tile0 + ti) * kKmTile;
    const int np = min(kKmTile, L.N - p0);
    if (tid == 0) {
      mbar_arrive_expect_tx(bars + 1, (uint32_t)(kKmTile * D * 2));
      for (int kb = 0; kb < KB; ++kb)
        tma_load_2d(sX + (size_t)kb * kKmTile * 128, &tmX, bars + 1, kb * 64, bh * L.N + p0);
      const bool ok = (ti > 0 || mbar_wait(bars + 0, 0, &s_abort)) && mbar_wait(bars + 1, ti & 1, &s_abort);
      if (ok) {
        tc_fence_after();
        uint32_t acc = 0;
        for (int wt = 0; wt < 3; ++wt)
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t xa = smem_u32(sX + (size_t)(ks >> 2) * kKmTile * 128) + (ks & 3) * 32;
            const uint32_t wa = smem_u32(sW + ((size_t)wt * KB + (ks >> 2)) * Np * 128) + (ks & 3) * 32;
            mma_ss(tmem, sdesc_sw128(xa, 16, 1024), sdesc_sw128(wa, 16, 1024), idesc, acc);
            acc = 1;
          }
      }
      mma_commit(bars + 2);
    }
    if (tid < kKmTile) scl[tid] = kKeys ? 1.f : (tid < np ? L.inv_rms[(size_t)bh * L.N + p0 + tid] : 0.f);
    // epilogue: point q = tid % 128 (TMEM lane q); warps w and w+4 read alternate 32-column
    // chunks of that lane's scores, then merge
    const bool waited = mbar_wait(bars + 2, ti & 1, &s_abort);
    if (__syncthreads_or(!waited)) break;  // uniform: every thread leaves or none does
    tc_fence_after();
    const int q = tid & 127, half = tid >> 7;
    const float sq = scl[q];
    float b1 = INFINITY, b2 = INFINITY;
    int i1 = 0x7fffffff;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    for (int c0 = half * 32; c0 < Np; c0 += 64) {
      uint32_t r[32];
      tmem_ld32(tmem + lane_base + c0, r);  // c0 + 32 <= tcols: tcols is a power of two >= 32, >= Np
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const int j = c0 + k;
        if (j >= C) break;
        const float sc = sB[j] - 2.f * sq * __uint_as_float(r[k]);
        if (sc < b1 || (sc == b1 && j < i1)) {
          b2 = b1;
          b1 = sc;
          i1 = j;
        } else if (sc < b2) {
          b2 = sc;
        }
      }
    }
    if (half == 1) {
      mb1[q] = b1;
      mb2[q] = b2;
      mi1[q] = i1;
    }
    __syncthreads();
    if (half == 0) {
      const float ob1 = mb1[q], ob2 = mb2[q];
      const int oi1 = mi1[q];
      if (ob1 < b1 || (ob1 == b1 && oi1 < i1)) {
        b2 = fminf(b1, ob2);
        b1 = ob1;
        i1 = oi1;
      } else {
        b2 = fminf(b2, ob1);
      }
      const bool valid = q < np;
      const size_t row = (size_t)bh * L.N + p0 + q;
      const float xn = valid ? (kKeys ? L.knorm[row] : L.qxnorm[row]) : 0.f;
      const float delta = 4.f * (3 * D + 8) * u * xn * s_wmax + 4.f * u * s_bmax;
      const bool ref = valid && !(b2 - b1 > 2.f * delta);
      lab[q] = (i1 >= 0 && i1 < C) ? i1 : 0;  // non-finite scores never yield a bad label
      bval[q] = valid ? (double)b1 : 0.0;
      if (ref) rlist[atomicAdd(&s_nlist, 1)] = q;
      nref += ref ? 1 : 0;
    }
    for (int j = tid; j < C; j += blockDim.x) hist[j] = 0;
    __syncthreads();
    // fp64 re-decision over every group: one warp per listed point
    const int nlist = s_nlist;
    for (int li = warp; li < nlist; li += 8) {
      const int p = rlist[li];
      double* xs = xs64 + warp * 128;
      for (int a = lane; a < D; a += 32) {
        const int kb = a >> 6, w = a & 63;
        const uint32_t off = (uint32_t)p * 128 + ((((w >> 3) ^ (p & 7)) << 4) | ((w & 7) << 1));
        xs[a] = (double)__bfloat162float(*(const __nv_bfloat16*)(sX + (size_t)kb * kKmTile * 128 + off));
      }
      __syncwarp();
      int best;
      double bv;
      redecide_fp64<kKeys>(L, bh, xs, D, C, W64, B64, best, bv);
      if (lane == 0) {
        lab[p] = best;
        bval[p] = bv;
      }
      __syncwarp();
    }
    __syncthreads();
    if (tid < np) {
      ((kKeys ? L.klabel : L.qlabel) + (size_t)bh * L.N)[p0 + tid] = lab[tid];
      jsum += bval[tid];
      atomicAdd(&hist[lab[tid]], 1);
    }
    tc_fence_before();
    __syncthreads();
    // counting sort of the tile's points by label (the order inside a label is irrelevant:
    // each run's fp64 partial sums of exact products are exact)
    if (warp == 0) {
      int run = 0;
      for (int c0 = 0; c0 < C; c0 += 32) {
        const int j = c0 + lane;
        const int v = j < C ? hist[j] : 0;
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        if (j < C) cursor[j] = run + x - v;
        run += __shfl_sync(0xffffffffu, x, 31);
      }
    }
    __syncthreads();
    int* counts = (kKeys ? L.kcount : L.qcount) + (size_t)bh * C;
    for (int j = tid; j < C; j += blockDim.x)
      if (hist[j]) atomicAdd(counts + j, hist[j]);
    if (tid < np) order[atomicAdd(&cursor[lab[tid]], 1)] = tid;
    __syncthreads();
    double* sums = (kKeys ? L.ksum : L.qsum) + (size_t)bh * C * D;
    const int nparts = 256 / D;
    {
      const int a = tid % D, part = tid / D;
      const int q0 = part * np / nparts, q1 = (part + 1) * np / nparts;
      const int kb = a >> 6, w = a & 63;
      const uint8_t* colbase = sX + (size_t)kb * kKmTile * 128;
      double acc = 0.0;
      for (int qq = q0; qq < q1; ++qq) {
        const int p = order[qq];
        const uint32_t off = (uint32_t)p * 128 + ((((w >> 3) ^ (p & 7)) << 4) | ((w & 7) << 1));
        acc += (double)__bfloat162float(*(const __nv_bfloat16*)(colbase + off)) * (double)scl[p];
        if (qq == q1 - 1 || lab[order[qq + 1]] != lab[p]) {
          atomicAdd(sums + (size_t)lab[p] * D + a, acc);
          acc = 0.0;
        }
      }
    }
    if (tid == 0) s_nlist = 0;
    tc_fence_before();
    __syncthreads();
  }
  const double js = block_sum(jsum, red);
  const double nr = block_sum((double)nref, red);
  if (tid == 0) {
    atomicAdd((kKeys ? L.kJ : L.qJ) + (size_t)bh * L.iters_cap + it, js);
    if (nr > 0.0) atomicAdd((kKeys ? L.krefined : L.qrefined) + bh, (int)nr);
    if (s_abort) {
      atomicCAS(L.status, kDevOk, kDevTimeout);
      // never leave with copies in flight into this CTA's shared memory
      mbar_wait_drain(bars + 0, 0);
      for (int ti = 0; ti < ntile; ++ti) mbar_wait_drain(bars + 1, ti & 1);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}

// Per-row quadratic forms x^T G x (G = M for keys, Gc for queries) and norms, 128 rows per
// tile: U = X G on the tensor cores (G symmetric, split into three bf16 terms), then each
// thread dots its row of U (TMEM lane) with its row of X (shared memory).
//   keys    (which 0): T0k += sum x^T M x;  knorm = ||x||
//   queries (which 1): ms = x^T Gc x;  inv_rms = 1/sqrt(ms + 1e-12);  qxnorm = ||x|| inv_rms;
//                      T0q += C_k ms / (ms + 1e-12)   (= ||r~||^2)
__global__ void __launch_bounds__(128, 1)
    rowqf_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmG, Layout L,
                    int which, int tiles_per_cta) {
  const int bh = blockIdx.y, D = L.d, KB = D / 64;
  const int tile0 = blockIdx.x * tiles_per_cta;
  const int ntiles_head = (L.N + kKmTile - 1) / kKmTile;
  const int ntile = min(tiles_per_cta, ntiles_head - tile0);
  if (ntile <= 0) return;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sG = sm;                              // [3][KB][D rows][128 B]
  uint8_t* sX = sG + (size_t)3 * D * D * 2;      // [KB][128 rows][128 B]
  uint64_t* bars = (uint64_t*)(sX + (size_t)kKmTile * D * 2);
  uint32_t* tmem_slot = (uint32_t*)(bars + 3);
  __shared__ volatile int s_abort;
  __shared__ double red[4];
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t tcols = km_tc_tmem_cols(D);
  if (tid == 0) {
    s_abort = 0;
    mbar_init(bars + 0, 1);
    mbar_init(bars + 1, 1);
    mbar_init(bars + 2, 1);
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
  if (tid == 0) {
    mbar_arrive_expect_tx(bars + 0, (uint32_t)(3 * D * D * 2));
    for (int t = 0; t < 3; ++t)
      for (int kb = 0; kb < KB; ++kb)
        tma_load_2d(sG + ((size_t)t * KB + kb) * D * 128, &tmG, bars + 0, kb * 64, t * L.BH * D + bh * D);
  }
  const uint32_t idesc = idesc_bf16_f32(kKmTile, D, 0, 0);
  double tot = 0.0;
  for (int ti = 0; ti < ntile && !s_abort; ++ti) {
    const int p0 = (tile0 + ti) * kKmTile;
    const int np = min(kKmTile, L.N - p0);
    if (tid == 0) {
      mbar_arrive_expect_tx(bars + 1, (uint32_t)(kKmTile * D * 2));
      for (int kb = 0; kb < KB; ++kb)
        tma_load_2d(sX + (size_t)kb * kKmTile * 128, &tmX, bars + 1, kb * 64, bh * L.N + p0);
      const bool ok = (ti > 0 || mbar_wait(bars + 0, 0, &s_abort)) && mbar_wait(bars + 1, ti & 1, &s_abort);
      if (ok) {
        tc_fence_after();
        uint32_t acc = 0;
        for (int gt = 0; gt < 3; ++gt)
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t xa = smem_u32(sX + (size_t)(ks >> 2) * kKmTile * 128) + (ks & 3) * 32;
            const uint32_t ga = smem_u32(sG + ((size_t)gt * KB + (ks >> 2)) * D * 128) + (ks & 3) * 32;
            mma_ss(tmem, sdesc_sw128(xa, 16, 1024), sdesc_sw128(ga, 16, 1024), idesc, acc);
            acc = 1;
          }
      }
      mma_commit(bars + 2);
    }
    const bool waited = mbar_wait(bars + 2, ti & 1, &s_abort);
    if (__syncthreads_or(!waited)) break;
    tc_fence_after();
    const int p = tid;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float qf = 0.f, nn = 0.f;
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + lane_base + c0, r);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const int a = c0 + k, kb = a >> 6, w = a & 63;
        const uint32_t off = (uint32_t)p * 128 + ((((w >> 3) ^ (p & 7)) << 4) | ((w & 7) << 1));
        const float x = __bfloat162float(*(const __nv_bfloat16*)(sX + (size_t)kb * kKmTile * 128 + off));
        qf = fmaf(x, __uint_as_float(r[k]), qf);
        nn = fmaf(x, x, nn);
      }
    }
    if (p < np) {
      const size_t row = (size_t)bh * L.N + p0 + p;
      if (which == 0) {
        L.knorm[row] = sqrtf(nn);
        tot += (double)qf;
      } else {
        const double ms = (double)qf;
        const float inv = (float)(1.0 / sqrt(ms + 1e-12));
        L.inv_rms[row] = inv;
        L.qxnorm[row] = sqrtf(nn) * inv;
        tot += (double)L.Ck * ms / (ms + 1e-12);
      }
    }
    tc_fence_before();
    __syncthreads();
  }
  tot = block_sum(tot, red);
  if (tid == 0) {
    atomicAdd((which == 0 ? L.T0k : L.T0q) + bh, tot);
    if (s_abort) {
      atomicCAS(L.status, kDevOk, kDevTimeout);
      mbar_wait_drain(bars + 0, 0);
      for (int ti = 0; ti < ntile; ++ti) mbar_wait_drain(bars + 1, ti & 1);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}

// ----------------------------------------------------------------------------------- host
bool km_tc_supported(const Layout& L, bool keys) {
  if (L.dtype != SPARSEPR_BF16) return false;
  const int Np = keys ? L.Ckp : L.Cqp;
  return Np <= 256 && km_tc_smem(L.d, Np) <= 227 * 1024;
}

sparsepr_status launch_kmeans_assign_tc(const Layout& L, bool keys, const void* X, int it, cudaStream_t st) {
  CUtensorMap mX, mW;
  const int D = L.d;
  const int Np = keys ? L.Ckp : L.Cqp;
  const void* wbase = keys ? (const void*)L.kWb : (const void*)L.qWb;
  if (!make_tmap_bf16(&mX, X, (long long)L.BH * L.N, D, kKmTile) ||
      !make_tmap_bf16(&mW, wbase, 3LL * L.BH * Np, D, Np))
    return SPARSEPR_ERR_CUDA;
  const size_t smem = km_tc_smem(D, Np);
  const int tpc = tiles_per_cta(L);
  const int ntiles = (L.N + kKmTile - 1) / kKmTile;
  const dim3 grid((ntiles + tpc - 1) / tpc, L.BH);
  if (keys) {
    cudaFuncSetAttribute(kmeans_assign_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    launch(kmeans_assign_tc_kernel<true>, grid, dim3(256), smem, st, mX, mW, L, it, tpc);
  } else {
    cudaFuncSetAttribute(kmeans_assign_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    launch(kmeans_assign_tc_kernel<false>, grid, dim3(256), smem, st, mX, mW, L, it, tpc);
  }
  SPR_LAUNCH_CHECK();
  return SPARSEPR_OK;
}

sparsepr_status launch_rowqf_tc(const Layout& L, int which, const void* X, cudaStream_t st) {
  CUtensorMap mX, mG;
  const int D = L.d;
  const void* gbase = which == 0 ? (const void*)L.Mb : (const void*)L.Gcb;
  if (!make_tmap_bf16(&mX, X, (long long)L.BH * L.N, D, kKmTile) ||
      !make_tmap_bf16(&mG, gbase, 3LL * L.BH * D, D, D))
    return SPARSEPR_ERR_CUDA;
  const size_t smem = (size_t)3 * D * D * 2 + (size_t)kKmTile * D * 2 + 1024 + 64;
  const int tpc = tiles_per_cta(L);
  const int ntiles = (L.N + kKmTile - 1) / kKmTile;
  cudaFuncSetAttribute(rowqf_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  launch(rowqf_tc_kernel, dim3((ntiles + tpc - 1) / tpc, L.BH), dim3(128), smem, st, mX, mG, L, which, tpc);
  SPR_LAUNCH_CHECK();
  return SPARSEPR_OK;
}

}  // namespace sparsepr
