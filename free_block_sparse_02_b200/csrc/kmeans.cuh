// Device helpers shared by the CUDA-core and tensor-core k-means assignment kernels.
#pragma once

#include "common.cuh"

namespace sparsepr {

// fp64 score of every group for one point (one warp), lowest index on exact ties; x staged in
// xs (fp64).  Queries need the exact 1/rms: ms = x^T Gc x.
template <bool kKeys>
__device__ void redecide_fp64(const Layout& L, int bh, const double* xs, int D, int C, const double* W64,
                              const double* B64, int& best_out, double& bestv_out) {
  const int lane = threadIdx.x & 31;
  double scale = 1.0;
  if constexpr (!kKeys) {
    const double* Gc = L.Gc + (size_t)bh * D * D;
    double ms = 0.0;
    for (int a = lane; a < D; a += 32) {
      double u = 0.0;
      for (int b = 0; b < D; ++b) u += Gc[(size_t)a * D + b] * xs[b];
      ms += u * xs[a];
    }
    ms = warp_sum(ms);
    scale = 1.0 / sqrt(ms + 1e-12);
  }
  double bv = INFINITY;
  int bj = 0x7fffffff;
  for (int j = lane; j < C; j += 32) {
    const double* w = W64 + (size_t)j * D;
    double d0 = 0.0, d1 = 0.0, d2 = 0.0, d3 = 0.0;
    int a = 0;
    for (; a + 4 <= D; a += 4) {
      d0 += xs[a] * w[a];
      d1 += xs[a + 1] * w[a + 1];
      d2 += xs[a + 2] * w[a + 2];
      d3 += xs[a + 3] * w[a + 3];
    }
    for (; a < D; ++a) d0 += xs[a] * w[a];
    const double sc = B64[j] - 2.0 * scale * ((d0 + d1) + (d2 + d3));
    if (sc < bv) {  // ascending j per lane: strict < keeps the lower index
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
  best_out = (bj >= 0 && bj < C) ? bj : 0;
  bestv_out = bv;
}

}  // namespace sparsepr
