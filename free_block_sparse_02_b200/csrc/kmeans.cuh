// Device helpers shared by the CUDA-core and tensor-core k-means assignment kernels.
#pragma once

#include "common.cuh"

namespace sparsepr {

// TMEM columns to allocate for n accumulator columns: a power of two, at least 32.
__host__ __device__ inline int km_tc_tmem_cols(int n) {
  int c = 32;
  while (c < n) c <<= 1;
  return c;
}

// A load of data that other CTAs of the same launch may have rewritten (kCg: served by L2, never
// by a stale L1 line), or a plain load.
template <bool kCg, typename T>
__device__ __forceinline__ T ld_w(const T* p) {
  if constexpr (kCg) return __ldcg(p);
  else return *p;
}

// x = hi + mid + lo in bf16 (each term the bf16 rounding of what the previous ones left),
// written at index i of three planes `plane` elements apart.
__device__ __forceinline__ void split3(double x, __nv_bfloat16* base, size_t plane, size_t i) {
  const __nv_bfloat16 h = __double2bfloat16(x);
  const double r1 = x - (double)__bfloat162float(h);
  const __nv_bfloat16 m = __double2bfloat16(r1);
  const double r2 = r1 - (double)__bfloat162float(m);
  base[i] = h;
  base[plane + i] = m;
  base[2 * plane + i] = __double2bfloat16(r2);
}

__device__ __forceinline__ bool km_should_stop(const double* J, int it, int iters, float tol) {
  if (it >= iters) return true;
  if (it >= 2 && tol >= 0.f) {
    const double Jp = J[it - 2], Jc = J[it - 1];
    return Jp - Jc <= (double)tol * Jp;
  }
  return false;
}

// Exact fp64 value of a bf16 given by its 16 bits (through its exact fp32 value).
__device__ __forceinline__ double bf16_bits_to_f64(uint32_t b) { return (double)__uint_as_float(b << 16); }

// Sum over the 32 lanes of each of 32 values: afterwards lane l holds the total of v[l]
// (recursive halving: 16 + 8 + 4 + 2 + 1 shuffles instead of 32 full warp sums).
__device__ __forceinline__ double warp_transpose_sum32(double (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool up = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const double send = up ? v[i] : v[i + s];
      const double keep = up ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return v[0];
}

// The exact query scale 1/rms = 1/sqrt(x^T Gc x + 1e-12) (Gc in global or shared memory), one
// warp: each lane sums over its columns, one warp sum at the end.
__device__ __forceinline__ double query_scale_fp64(const double* Gc, const double* xs, const double (&xl)[4], int D) {
  const int lane = threadIdx.x & 31;
  double part = 0.0;
#pragma unroll 16
  for (int a = 0; a < D; ++a) {
    double row = 0.0;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (lane + 32 * k < D) row += Gc[(size_t)a * D + lane + 32 * k] * xl[k];
    part += row * xs[a];
  }
  return 1.0 / sqrt(warp_sum(part) + 1e-12);
}

// fp64 argmin over a short candidate list (ascending group ids; the lowest id wins exact ties),
// one warp; `scale` is 1 for keys.
template <bool kCg = false>
__device__ __forceinline__ void redecide_candidates(const double* xs, int D, const double* W64, const double* B64,
                                                    double scale, const int* cand, int ncand, int& best_out,
                                                    double& bestv_out) {
  const int lane = threadIdx.x & 31;
  // every candidate's W row piece and bias first (all loads in flight), then the scores
  double wv[4][4], bb[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int j = c < ncand ? cand[c] : 0;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      wv[c][k] = (c < ncand && lane + 32 * k < D) ? ld_w<kCg>(W64 + (size_t)j * D + lane + 32 * k) : 0.0;
    bb[c] = c < ncand ? ld_w<kCg>(B64 + j) : 0.0;
  }
  double bv = INFINITY;
  int bj = 0;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    if (c >= ncand) break;
    double part = 0.0;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (lane + 32 * k < D) part += wv[c][k] * xs[lane + 32 * k];
    const double sc = bb[c] - 2.0 * scale * warp_sum(part);
    if (sc < bv) {
      bv = sc;
      bj = cand[c];
    }
  }
  best_out = bj;
  bestv_out = bv;
}

// fp64 score of every group for one point (one warp), lowest index on exact ties; x staged in
// xs (fp64, shared memory).  Lanes run over the dimensions, so every row of W and Gc is read
// coalesced.  Queries need the exact scale 1/rms: ms = x^T Gc x, each lane summing over its
// columns and one warp sum at the end.  Group dots are formed 32 groups at a time and
// transposed across the lanes (lane l gets group 32 c + l), then the lowest score wins.
template <bool kKeys, bool kCg = false>
__device__ void redecide_fp64(const Layout& L, int bh, const double* xs, int D, int C, const double* W64,
                              const double* B64, int& best_out, double& bestv_out, const double* Gc_in = nullptr) {
  const int lane = threadIdx.x & 31;
  double xl[4];  // this lane's dimensions lane, lane + 32, ... (D <= 128)
#pragma unroll
  for (int k = 0; k < 4; ++k) xl[k] = lane + 32 * k < D ? xs[lane + 32 * k] : 0.0;
  double scale = 1.0;
  if (!kKeys && !L.semantic) {  // the semantic partition clusters the raw queries (scale 1)
    const double* Gc = Gc_in ? Gc_in : L.Gc + (size_t)bh * D * D;
    double part = 0.0;
#pragma unroll 4
    for (int a = 0; a < D; ++a) {
      double row = 0.0;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (lane + 32 * k < D) row += Gc[(size_t)a * D + lane + 32 * k] * xl[k];
      part += row * xs[a];
    }
    const double ms = warp_sum(part);
    scale = 1.0 / sqrt(ms + 1e-12);
  }
  double bv = INFINITY;
  int bj = 0x7fffffff;
  for (int j0 = 0; j0 < C; j0 += 32) {
    double part[32];
#pragma unroll
    for (int g = 0; g < 32; ++g) {
      part[g] = 0.0;
      if (j0 + g < C) {
        const double* w = W64 + (size_t)(j0 + g) * D;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (lane + 32 * k < D) part[g] += ld_w<kCg>(w + lane + 32 * k) * xl[k];
      }
    }
    const double dot = warp_transpose_sum32(part);  // group j0 + lane
    const int j = j0 + lane;
    if (j < C) {
      const double sc = ld_w<kCg>(B64 + j) - 2.0 * scale * dot;
      if (sc < bv) {  // ascending j per lane: strict < keeps the lower index
        bv = sc;
        bj = j;
      }
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
  best_out = (bj >= 0 && bj < C) ? bj : 0;
  bestv_out = bv;
}

}  // namespace sparsepr
