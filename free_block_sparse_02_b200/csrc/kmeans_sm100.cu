// Lloyd assignment step of the partition on the tensor cores (tcgen05, scores in TMEM).
//
// "Partition the Support, Reconstruct the Residual" (arXiv 2608.18484), abstract: keys are
// grouped by their responses to sampled queries, queries by their responses to the key-group
// centroids; both groupings are k-means (Table C.1: 25 / 2 iterations, tolerance 1e-4).
//
// Score of point x against group j: s_j = b_j - 2 x . w_j (keys: w = M c, b = c^T M c;
// queries: w = nu, b = ||nu||^2); the label is argmin_j s_j, lowest j on ties.  The dot
// products of a 128-point tile against every group are one MMA chain: X (128 x D) times W^T
// (D x C) with bf16 operands -- a key tile is exact in bf16, a response tile and every weight
// matrix are split into three bf16 terms (hi + mid + lo), and the products of combined order
// up to 2^-16 are accumulated in fp32 in TMEM (3 MMA chains for keys, 6 for queries), giving
// fp32-grade scores.  The epilogue (one thread per point, its TMEM lane) keeps the best two
// scores; a point whose two best are within a rigorous rounding bound is re-decided over all
// groups in fp64, so labels agree with an fp64 evaluation.  Then, as in the CUDA-core
// version: the chosen group's exact fp64 score (objective), and fp64 group sums per run of
// equal labels (block-sorted), flushed with one atomic per (run, dim).
//
// CTA = 128 threads, one head, kTilesPerCta consecutive 128-point tiles; the weights are
// loaded once per CTA by TMA.
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace sparsepr {

using namespace sm100;

constexpr int kKmTile = 128;

struct KmTcCfg {
  int D;        // feature dims (multiple of 64)
  int Np;       // groups padded to 16 (MMA N)
  int C;        // real groups
  int xterms;   // 1 (keys) or 3 (responses)
};

__host__ __device__ inline int km_tc_tmem_cols(int Np) {
  int c = 32;
  while (c < Np) c <<= 1;
  return c;
}

__host__ inline size_t km_tc_smem(int D, int Np, int xterms) {
  const size_t w = (size_t)3 * Np * D * 2;
  const size_t x = (size_t)xterms * kKmTile * D * 2;
  return w + x + 1024 /*align*/ + 24576 /*bias, labels, order, list, histogram, merge, scores, fp64 rows, barriers*/;
}

template <bool kKeys>
__global__ void __launch_bounds__(256, 1)
    kmeans_assign_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                            Layout L, const __nv_bfloat16* __restrict__ K, int it, int tiles_per_cta) {
  const int bh = blockIdx.y;
  const int which = kKeys ? 0 : 1;
  if (it >= L.stop_at[bh * 2 + which]) return;
  const int D = kKeys ? L.d : L.Dq;
  const int Dreal = kKeys ? L.d : L.Ck;
  const int C = kKeys ? L.Ck : L.Cq;
  const int Np = kKeys ? L.Ckp : L.Cqp;
  const int xterms = kKeys ? 1 : 3;
  const int KB = D / 64;
  const int tile0 = blockIdx.x * tiles_per_cta;
  const int ntiles_head = (L.N + kKmTile - 1) / kKmTile;
  const int ntile = min(tiles_per_cta, ntiles_head - tile0);
  if (ntile <= 0) return;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sW = sm;                                   // [3 terms][KB][Np rows][128 B]
  uint8_t* sX = sW + (size_t)3 * Np * D * 2;          // [xterms][KB][128 rows][128 B]
  float* sB = (float*)(sX + (size_t)xterms * kKmTile * D * 2);  // [256] bias
  int* lab = (int*)(sB + 256);                       // [128]
  int* order = lab + kKmTile;                        // [128]
  int* rlist = order + kKmTile;                      // [128] points to re-decide
  int* hist = rlist + kKmTile;                       // [256] points per label in the tile
  int* cursor = hist + 256;                          // [256] next slot per label
  float* mb1 = (float*)(cursor + 256);               // [128] partial best / second / index
  float* mb2 = mb1 + kKmTile;
  int* mi1 = (int*)(mb2 + kKmTile);
  double* bval = (double*)(mi1 + kKmTile);           // [128] score of the chosen group
  double* xs64 = bval + kKmTile;                     // [8 warps][256] fp64 features
  uint64_t* bars = (uint64_t*)(xs64 + 8 * 256);      // w_full, x_full, mma_done
  uint32_t* tmem_slot = (uint32_t*)(bars + 3);
  __shared__ volatile int s_abort;
  __shared__ float s_wmax, s_bmax;
  __shared__ double red[8];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* B32 = kKeys ? L.kbias32 + (size_t)bh * C : L.qbias32 + (size_t)bh * C;
  const float* WN = kKeys ? L.kwnorm + (size_t)bh * C : L.qwnorm + (size_t)bh * C;
  const double* W64 = kKeys ? L.kW64 + (size_t)bh * C * Dreal : L.qcent + (size_t)bh * C * Dreal;
  const double* B64 = kKeys ? L.kbias64 + (size_t)bh * C : L.qbias64 + (size_t)bh * C;
  const uint32_t tcols = km_tc_tmem_cols(Np);

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
  // weights: 3 terms x KB column blocks, one TMA box of Np rows each
  if (tid == 0) {
    mbar_arrive_expect_tx(bars + 0, (uint32_t)(3 * Np * D * 2));
    for (int t = 0; t < 3; ++t)
      for (int kb = 0; kb < KB; ++kb)
        tma_load_2d(sW + ((size_t)t * KB + kb) * Np * 128, &tmW, bars + 0, kb * 64,
                    t * L.BH * Np + bh * Np);
  }
  __syncthreads();

  const uint32_t idesc = idesc_bf16_f32(kKmTile, Np, 0, 0);
  const float u = 4.76837158e-7f;  // 2^-21: covers the three-term split and fp32 accumulation
  double jsum = 0.0;
  int nref = 0;
  __shared__ int s_nlist;
  if (tid == 0) s_nlist = 0;
  __syncthreads();
  for (int ti = 0; ti < ntile && !s_abort; ++ti) {
    const int p0 = (tile0 + ti) * kKmTile;
    const int np = min(kKmTile, L.N - p0);
    if (tid == 0) {
      mbar_arrive_expect_tx(bars + 1, (uint32_t)(xterms * kKmTile * D * 2));
      const long long plane_rows = (long long)L.BH * L.N;
      for (int t = 0; t < xterms; ++t)
        for (int kb = 0; kb < KB; ++kb)
          tma_load_2d(sX + ((size_t)t * KB + kb) * kKmTile * 128, &tmX, bars + 1, kb * 64,
                      (int)(t * plane_rows + (long long)bh * L.N + p0));
      bool ok = (ti > 0 || mbar_wait(bars + 0, 0, &s_abort)) && mbar_wait(bars + 1, ti & 1, &s_abort);
      if (ok) {
        tc_fence_after();
        // products (x term, w term) of combined order <= 2^-16
        const int pairs_k[3][2] = {{0, 0}, {0, 1}, {0, 2}};
        const int pairs_q[6][2] = {{0, 0}, {0, 1}, {1, 0}, {0, 2}, {1, 1}, {2, 0}};
        const int npairs = kKeys ? 3 : 6;
        uint32_t acc = 0;
        for (int pi = 0; pi < npairs; ++pi) {
          const int xt = kKeys ? pairs_k[pi][0] : pairs_q[pi][0];
          const int wt = kKeys ? pairs_k[pi][1] : pairs_q[pi][1];
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t xa = smem_u32(sX + ((size_t)xt * KB + (ks >> 2)) * kKmTile * 128) + (ks & 3) * 32;
            const uint32_t wa = smem_u32(sW + ((size_t)wt * KB + (ks >> 2)) * Np * 128) + (ks & 3) * 32;
            mma_ss(tmem, sdesc_sw128(xa, 16, 1024), sdesc_sw128(wa, 16, 1024), idesc, acc);
            acc = 1;
          }
        }
      }
      mma_commit(bars + 2);
    }
    __syncwarp();
    // epilogue: point q = tid % 128 (TMEM lane q); warps w and w+4 read alternate 32-column
    // chunks of that lane's scores, then merge
    const bool waited = mbar_wait(bars + 2, ti & 1, &s_abort);
    if (__syncthreads_or(!waited)) break;  // uniform: every thread leaves or none does
    tc_fence_after();
    const int q = tid & 127, half = tid >> 7;
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
        const float sc = sB[j] - 2.f * __uint_as_float(r[k]);
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
    const int np_ = np;
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
      const bool valid = q < np_;
      const size_t row = (size_t)bh * L.N + p0 + q;
      const float xn = valid ? (kKeys ? L.knorm[row] : L.rnorm[row]) : 0.f;
      const float delta = 4.f * (Dreal + 8) * u * xn * s_wmax + 2.f * u * s_bmax;
      const bool ref = valid && !(b2 - b1 > 2.f * delta);
      lab[q] = (i1 >= 0 && i1 < C) ? i1 : 0;
      bval[q] = valid ? (double)b1 : 0.0;  // fp32-grade score of the chosen group (objective)
      if (ref) rlist[atomicAdd(&s_nlist, 1)] = q;
      nref += ref ? 1 : 0;
    }
    for (int j = tid; j < C; j += blockDim.x) hist[j] = 0;
    __syncthreads();
    // fp64 re-decision over every group (lowest index on exact ties): one warp per listed
    // point, its features staged in shared memory, lanes over groups
    const int nlist = s_nlist;
    for (int li = warp; li < nlist; li += 8) {
      const int p = rlist[li];
      const size_t rr = (size_t)bh * L.N + p0 + p;
      double* xs = xs64 + warp * 256;
      for (int a = lane; a < Dreal; a += 32) {
        if constexpr (kKeys) xs[a] = (double)__bfloat162float(K[rr * Dreal + a]);
        else xs[a] = L.r64[rr * Dreal + a];
      }
      __syncwarp();
      double bv = INFINITY;
      int bj = 0x7fffffff;
      for (int j = lane; j < C; j += 32) {
        const double* w = W64 + (size_t)j * Dreal;
        double d0 = 0.0, d1 = 0.0, d2 = 0.0, d3 = 0.0;
        int a = 0;
        for (; a + 4 <= Dreal; a += 4) {
          d0 += xs[a] * w[a];
          d1 += xs[a + 1] * w[a + 1];
          d2 += xs[a + 2] * w[a + 2];
          d3 += xs[a + 3] * w[a + 3];
        }
        for (; a < Dreal; ++a) d0 += xs[a] * w[a];
        const double sc = B64[j] - 2.0 * ((d0 + d1) + (d2 + d3));
        if (sc < bv) {
          bv = sc;
          bj = j;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
        if (ov < bv || (ov == bv && oj < bj)) {
          bv = ov;
          bj = oj;
        }
      }
      if (lane == 0) {
        lab[p] = (bj >= 0 && bj < C) ? bj : 0;
        bval[p] = bv;
      }
      __syncwarp();
    }
    __syncthreads();
    if (tid < np_) {
      ((kKeys ? L.klabel : L.qlabel) + (size_t)bh * L.N)[p0 + tid] = lab[tid];
      jsum += bval[tid];
      atomicAdd(&hist[lab[tid]], 1);
    }
    tc_fence_before();
    __syncthreads();
    // counting sort of the tile's points by label (order inside a label is irrelevant: each
    // run's fp64 partial sums are exact for keys and fp32-grade values for responses)
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
    if (tid < np_) order[atomicAdd(&cursor[lab[tid]], 1)] = tid;
    __syncthreads();
    double* sums = (kKeys ? L.ksum : L.qsum) + (size_t)bh * C * Dreal;
    // feature (p, a) from the swizzled tile(s) in shared memory: keys exactly, responses as
    // hi + mid + lo (fp32-grade)
    auto feat = [&](int p, int a) -> double {
      const int kb = a >> 6, w = a & 63;
      const uint32_t off = (uint32_t)p * 128 + ((((w >> 3) ^ (p & 7)) << 4) | ((w & 7) << 1));
      double v = 0.0;
      for (int t = 0; t < xterms; ++t) {
        const __nv_bfloat16 h = *(const __nv_bfloat16*)(sX + ((size_t)t * KB + kb) * kKmTile * 128 + off);
        v += (double)__bfloat162float(h);
      }
      return v;
    };
    const int nparts = Dreal >= 256 ? 1 : 256 / Dreal;
    if (tid < nparts * Dreal || Dreal > 256) {
      for (int a = tid % Dreal; a < Dreal; a += (Dreal > 256 ? 256 : Dreal)) {
        const int part = Dreal > 256 ? 0 : tid / Dreal;
        const int q0 = part * np_ / nparts, q1 = (part + 1) * np_ / nparts;
        double acc = 0.0;
        for (int qq = q0; qq < q1; ++qq) {
          const int p = order[qq];
          acc += feat(p, a);
          if (qq == q1 - 1 || lab[order[qq + 1]] != lab[p]) {
            atomicAdd(sums + (size_t)lab[p] * Dreal + a, acc);
            acc = 0.0;
          }
        }
        if (Dreal <= 256) break;
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

// ----------------------------------------------------------------------------------- host
bool km_tc_supported(const Layout& L, bool keys) {
  if (L.dtype != SPARSEPR_BF16) return false;
  const int Np = keys ? L.Ckp : L.Cqp;
  const int D = keys ? L.d : L.Dq;
  return Np <= 256 && km_tc_smem(D, Np, keys ? 1 : 3) <= 227 * 1024;
}

sparsepr_status launch_kmeans_assign_tc(const Layout& L, bool keys, const void* K, int it, cudaStream_t st) {
  CUtensorMap mX, mW;
  const int D = keys ? L.d : L.Dq;
  const int Np = keys ? L.Ckp : L.Cqp;
  const long long xrows = keys ? (long long)L.BH * L.N : 3LL * L.BH * L.N;
  const void* xbase = keys ? K : (const void*)L.rb;
  const void* wbase = keys ? (const void*)L.kWb : (const void*)L.qWb;
  if (!make_tmap_bf16(&mX, xbase, xrows, D, kKmTile) || !make_tmap_bf16(&mW, wbase, 3LL * L.BH * Np, D, Np))
    return SPARSEPR_ERR_CUDA;
  const size_t smem = km_tc_smem(D, Np, keys ? 1 : 3);
  const int ntiles = (L.N + kKmTile - 1) / kKmTile;
  // enough CTAs for about four per SM; each loads the weights once for its tiles
  int tpc = (int)(((long long)ntiles * L.BH + 148 * 4 - 1) / (148 * 4));
  tpc = tpc < 1 ? 1 : (tpc > 16 ? 16 : tpc);
  const dim3 grid((ntiles + tpc - 1) / tpc, L.BH);
  if (keys) {
    cudaFuncSetAttribute(kmeans_assign_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    launch(kmeans_assign_tc_kernel<true>, grid, dim3(256), smem, st, mX, mW, L, (const __nv_bfloat16*)K, it, tpc);
  } else {
    cudaFuncSetAttribute(kmeans_assign_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    launch(kmeans_assign_tc_kernel<false>, grid, dim3(256), smem, st, mX, mW, L, (const __nv_bfloat16*)K, it, tpc);
  }
  SPR_LAUNCH_CHECK();
  return SPARSEPR_OK;
}

}  // namespace sparsepr
