// The residual correction of the unprobed rows on the tensor cores (tcgen05, TMEM accumulator).
//
// "Partition the Support, Reconstruct the Residual" (arXiv 2608.18484), abstract: each unprobed
// query's sparse output is corrected by the residual the fitted map predicts for it; probe rows
// keep their exact dense output.  Per head, with A the (d+1) x d fitted map:
//   O_i = O_sp,i + O_sp,i A[0:d] + A[d]   (unprobed rows),   O_p = O_dense,p   (probe rows),
// written back in token order.
//
// O_sp . A[0:d] is a dense (rows x d) by (d x d) product: 128-row tiles of O_sp (fp32, in query-
// group order) are split into bf16 hi + lo in shared memory, A into bf16 hi + lo once per head,
// and the MMA chain Xhi Ahi + Xhi Alo + Xlo Ahi accumulates in fp32 in TMEM (the dropped
// Xlo Alo term and the splits leave a relative error of about 2^-16 of the correction).  The
// epilogue adds O_sp itself (fp32, exact) and A[d], and writes each row to its token.
// Persistent: CTA c of G takes tiles [c T / G, (c+1) T / G) of the T = BH * ceil(N/128) tiles.
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace sparsepr {

using namespace sm100;

constexpr int kApTile = 128;
constexpr int kApThreads = 256;

template <int D>
struct ApCfg {
  static constexpr int kKB = D / 64;
  static constexpr int kATerm = D * D * 2;           // one bf16 term of A^T: [KB][D rows][128 B]
  static constexpr int kXTerm = kApTile * D * 2;     // one bf16 term of X:   [KB][128 rows][128 B]
  static constexpr int kXStage = 2 * kXTerm;         // hi and lo of one X tile
  static constexpr int kSmem = 2 * kATerm + 2 * kXStage + 64 /*barriers, slot*/ + 1024;
  static constexpr uint32_t kTmemCols = 2 * D;       // two accumulators
  static constexpr int kVecPerThread = kApTile * D / 4 / kApThreads;  // float4 of a tile per thread
};

// Byte offset of bf16 element (row, k) in a K-major tile of `rows` rows stored as KB blocks of
// [rows][128 B] with the 128-byte swizzle (16-byte chunk index XOR row % 8).
__device__ __forceinline__ uint32_t sw128_off(int rows, int row, int k) {
  const int kb = k >> 6, w = k & 63;
  return (uint32_t)(kb * rows * 128 + row * 128 + ((((w >> 3) ^ (row & 7)) << 4) | ((w & 7) << 1)));
}

__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

// Two X stages and two TMEM accumulators: while the tensor core forms tile i's product, the
// threads load and split tile i + 1 (every float4 of a thread's share in flight at once), then
// write tile i's rows.
template <typename To, int D>
__global__ void __launch_bounds__(kApThreads, 1) apply_tc_kernel(Layout L, To* __restrict__ O, int G) {
  pdl_entry();
  using C = ApCfg<D>;
  const int tph = (L.N + kApTile - 1) / kApTile;
  const long long T = (long long)L.BH * tph;
  const int t0 = (int)(T * blockIdx.x / G), t1 = (int)(T * (blockIdx.x + 1) / G);
  if (t0 >= t1) return;  // uniform, before any barrier or TMEM use

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sA = sm;                             // [hi, lo] A^T: row n = output dim, K = input dim
  uint8_t* sX = sA + 2 * C::kATerm;             // [2 stages][hi, lo] X tile
  uint64_t* mma_done = (uint64_t*)(sX + 2 * C::kXStage);  // [2]
  uint64_t* mma_all = mma_done + 2;
  uint32_t* tmem_slot = (uint32_t*)(mma_all + 1);
  __shared__ volatile int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    s_abort = 0;
    mbar_init(mma_done + 0, 1);
    mbar_init(mma_done + 1, 1);
    mbar_init(mma_all, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t idesc = idesc_bf16_f32(kApTile, D, 0, 0);
  int cur = -1;
  // the head's map: A^T split into two bf16 terms (every thread; the caller makes sure that no
  // product still reads sA)
  auto load_map = [&](int bh) {
    const float* A = L.A32 + (size_t)bh * (D + 1) * D;
    for (int e = tid; e < D * D; e += kApThreads) {
      const int k = e / D, nn = e % D;  // A[k][nn] -> B operand row nn, column k
      __nv_bfloat16 hi, lo;
      split_bf16(A[e], hi, lo);
      const uint32_t off = sw128_off(D, nn, k);
      *(__nv_bfloat16*)(sA + off) = hi;
      *(__nv_bfloat16*)(sA + C::kATerm + off) = lo;
    }
  };
  // X tile t: rows of O_sp (fp32), split into bf16 hi + lo in stage b; rows past the head are zero
  auto load_x = [&](int t, int b) {
    const int bh = t / tph, r0 = (t % tph) * kApTile, np = min(kApTile, L.N - r0);
    const float* osp = L.Osp + ((size_t)bh * L.N + r0) * D;
    constexpr int kVecPerRow = D / 4;
    float4 v[C::kVecPerThread];
#pragma unroll
    for (int i = 0; i < C::kVecPerThread; ++i) {
      const int e = tid + i * kApThreads, row = e / kVecPerRow, k = (e % kVecPerRow) * 4;
      v[i] = row < np ? *(const float4*)(osp + (size_t)row * D + k) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    uint8_t* xs = sX + b * C::kXStage;
#pragma unroll
    for (int i = 0; i < C::kVecPerThread; ++i) {
      const int e = tid + i * kApThreads, row = e / kVecPerRow, k = (e % kVecPerRow) * 4;
      __nv_bfloat16 h[4], l[4];
      split_bf16(v[i].x, h[0], l[0]);
      split_bf16(v[i].y, h[1], l[1]);
      split_bf16(v[i].z, h[2], l[2]);
      split_bf16(v[i].w, h[3], l[3]);
      const uint32_t off = sw128_off(kApTile, row, k);  // 4 elements = 8 bytes inside one chunk
      *(uint2*)(xs + off) = *(const uint2*)h;
      *(uint2*)(xs + C::kXTerm + off) = *(const uint2*)l;
    }
  };
  auto issue = [&](int b) {  // thread 0: the products of stage b into accumulator b
    tc_fence_after();
    uint32_t acc = 0;
    // (X hi, A hi), (X hi, A lo), (X lo, A hi)
    for (int term = 0; term < 3; ++term) {
      const uint8_t* xa = sX + b * C::kXStage + (term == 2 ? C::kXTerm : 0);
      const uint8_t* wa = sA + (term == 1 ? C::kATerm : 0);
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t xo = (ks >> 2) * (kApTile * 128) + (ks & 3) * 32;
        const uint32_t wo = (ks >> 2) * (D * 128) + (ks & 3) * 32;
        mma_ss(tmem + b * D, sdesc_sw128(smem_u32(xa) + xo, 16, 1024), sdesc_sw128(smem_u32(wa) + wo, 16, 1024),
               idesc, acc);
        acc = 1;
      }
    }
    mma_commit(mma_done + b);
  };
  cur = t0 / tph;
  load_map(cur);
  load_x(t0, 0);
  // shared-memory writes of the threads become visible to the tensor core (async proxy)
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  if (tid == 0) issue(0);
  int n = 0;
  for (int t = t0; t < t1; ++t, ++n) {
    const int b = n & 1, bh = t / tph, r0 = (t % tph) * kApTile, np = min(kApTile, L.N - r0);
    bool waited = false;  // tile t's products have been waited for
    if (t + 1 < t1) {
      const int nbh = (t + 1) / tph;
      if (nbh != cur) {  // the next tile starts a new head: tile t's products read sA until done
        waited = !s_abort && mbar_wait(mma_done + b, (n >> 1) & 1, &s_abort);
        if (__syncthreads_or(!waited)) break;
        load_map(nbh);
        cur = nbh;
      }
      load_x(t + 1, b ^ 1);  // stage b ^ 1 was read by tile t - 1's products, already complete
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      __syncthreads();
      if (tid == 0 && !s_abort) issue(b ^ 1);
    }
    if (!waited) {
      waited = !s_abort && mbar_wait(mma_done + b, (n >> 1) & 1, &s_abort);
      if (__syncthreads_or(!waited)) break;  // uniform: every thread leaves or none does
    }
    tc_fence_after();
    // epilogue: row = TMEM lane; warps w and w + 4 take the two halves of the columns
    {
      const int row = (warp & 3) * 32 + lane, half = warp >> 2;
      const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
      const bool valid = row < np;
      const int pos = r0 + row;
      const int tok = valid ? L.qperm[(size_t)bh * L.N + pos] : 0;
      const int p = valid ? L.probe_of[(size_t)bh * L.N + tok] : -1;
      To* orow = O + ((size_t)bh * L.N + tok) * D;
      const float* xrow = L.Osp + ((size_t)bh * L.N + r0 + row) * D;
      const float* drow = L.Odense + ((size_t)bh * L.P + (p < 0 ? 0 : p)) * D;
      const float* bias = L.A32 + (size_t)bh * (D + 1) * D + (size_t)D * D;  // A[d]
#pragma unroll
      for (int c0 = half * (D / 2); c0 < (half + 1) * (D / 2); c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + b * D + c0, r);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int k = 0; k < 32; k += 4) {
            float4 y;
            if (p >= 0) {
              y = *(const float4*)(drow + c0 + k);
            } else {
              const float4 x = *(const float4*)(xrow + c0 + k);
              const float4 a = *(const float4*)(bias + c0 + k);
              y.x = x.x + (__uint_as_float(r[k]) + a.x);
              y.y = x.y + (__uint_as_float(r[k + 1]) + a.y);
              y.z = x.z + (__uint_as_float(r[k + 2]) + a.z);
              y.w = x.w + (__uint_as_float(r[k + 3]) + a.w);
            }
            if constexpr (std::is_same<To, float>::value) {
              *(float4*)(orow + c0 + k) = y;
            } else {
              __nv_bfloat162 a2 = __floats2bfloat162_rn(y.x, y.y), b2 = __floats2bfloat162_rn(y.z, y.w);
              uint2 u;
              u.x = *(const uint32_t*)&a2;
              u.y = *(const uint32_t*)&b2;
              *(uint2*)(orow + c0 + k) = u;
            }
          }
        }
      }
    }
    tc_fence_before();
    __syncthreads();  // accumulator b is read: tile t + 2's products may use it
  }
  if (tid == 0) {
    if (s_abort) atomicCAS(L.status, kDevOk, kDevTimeout);
    mma_commit(mma_all);  // arrives once every product this thread issued has completed
    mbar_wait_drain(mma_all, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <typename To, int D>
static sparsepr_status launch_apply_tc_t(const Layout& L, void* O, cudaStream_t st) {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  const long long T = (long long)L.BH * ((L.N + kApTile - 1) / kApTile);
  const int G = (int)std::min<long long>(T, sms);
  cudaFuncSetAttribute(apply_tc_kernel<To, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, ApCfg<D>::kSmem);
  launch(apply_tc_kernel<To, D>, G, kApThreads, (size_t)ApCfg<D>::kSmem, st, L, (To*)O, G);
  SPR_LAUNCH_CHECK();
  return SPARSEPR_OK;
}

sparsepr_status launch_apply_tc(const Layout& L, void* O, int out_dtype, cudaStream_t st) {
  if (out_dtype == SPARSEPR_F32)
    return L.d == 64 ? launch_apply_tc_t<float, 64>(L, O, st) : launch_apply_tc_t<float, 128>(L, O, st);
  return L.d == 64 ? launch_apply_tc_t<__nv_bfloat16, 64>(L, O, st) : launch_apply_tc_t<__nv_bfloat16, 128>(L, O, st);
}

}  // namespace sparsepr
