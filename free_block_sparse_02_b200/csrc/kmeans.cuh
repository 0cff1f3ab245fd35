// Device helpers shared by the CUDA-core and tensor-core k-means assignment kernels.
#pragma once

#include "common.cuh"

namespace sparsepr {

// fp64 score of every group for one point (one warp), lowest index on exact ties; x staged in
// xs (fp64, shared memory).  Lanes run over the dimensions, so every row of W (and of Gc) is
// read coalesced; each dot is completed by a warp sum, identical in every lane.  Queries need
// the exact scale 1/rms: ms = x^T Gc x.  Eight groups per step keep eight rows of loads in flight.
template <bool kKeys>
__device__ void redecide_fp64(const Layout& L, int bh, const double* xs, int D, int C, const double* W64,
                              const double* B64, int& best_out, double& bestv_out) {
  const int lane = threadIdx.x & 31;
  double xl[4];  // this lane's dimensions lane, lane + 32, ... (D <= 128)
#pragma unroll
  for (int k = 0; k < 4; ++k) xl[k] = lane + 32 * k < D ? xs[lane + 32 * k] : 0.0;
  double scale = 1.0;
  if constexpr (!kKeys) {
    const double* Gc = L.Gc + (size_t)bh * D * D;
    double ms = 0.0;
    for (int a = 0; a < D; ++a) {
      double part = 0.0;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (lane + 32 * k < D) part += Gc[(size_t)a * D + lane + 32 * k] * xl[k];
      ms += warp_sum(part) * xs[a];
    }
    scale = 1.0 / sqrt(ms + 1e-12);
  }
  double bv = INFINITY;
  int bj = 0x7fffffff;
  for (int j0 = 0; j0 < C; j0 += 8) {
    double part[8];
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      part[g] = 0.0;
      if (j0 + g < C) {
        const double* w = W64 + (size_t)(j0 + g) * D;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (lane + 32 * k < D) part[g] += w[lane + 32 * k] * xl[k];
      }
    }
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      const double dot = warp_sum(part[g]);
      if (j0 + g < C) {
        const double sc = B64[j0 + g] - 2.0 * scale * dot;
        if (sc < bv) {  // ascending j: strict < keeps the lower index
          bv = sc;
          bj = j0 + g;
        }
      }
    }
  }
  best_out = (bj >= 0 && bj < C) ? bj : 0;
  bestv_out = bv;
}

}  // namespace sparsepr
