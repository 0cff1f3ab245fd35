// Key-response rank of the partition (listing page, Table C.1: "Key response rank r_K", 48 in
// the paper's runs).
//
// Reading: the N x s key responses F = K Q_s^T / sqrt(d) are taken in the basis of their r_K
// leading right singular vectors before the key k-means (the best rank-r_K approximation of the
// response matrix, not centred).  The key k-means runs on the keys themselves with the metric M
// (distances ||f_t - mu_j||^2 = (k_t - c_j)^T M (k_t - c_j), M = Q_s^T Q_s / d), so the rank-r_K
// projection becomes a rank-r_K metric.  With M = L L^T, the response rows are an isometric image
// of the rows of K L, whose right singular vectors are the eigenvectors Z of
// H = L^T (K^T K) L; projecting on the r_K leading ones gives
//     M_r = (L Z_r)(L Z_r)^T,
// which replaces M before the k-means starts (W = M_r c, biases c^T M_r c, the objective).  When
// M is singular (fewer sampled queries than d), L = E D^(1/2) from the eigen-decomposition
// M = E D E^T instead of the Cholesky factor; the identity is the same.
//
// Kernels: fp64 partial Grams K^T K over chunks of keys (sums in a fixed order, so the result
// is reproducible), their in-order reduction, and one CTA per head for the factor, H, its
// eigen-decomposition (parallel cyclic Jacobi) and M_r.
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"
#include "linalg.cuh"

namespace sparsepr {

constexpr int kGramRows = 16;    // rows of K^T K per block
constexpr int kGramStage = 64;   // keys staged in shared memory at a time

// Block (bh, y, c): rows [16 y, 16 y + 16) of the Gram of keys [c kGramChunk, (c+1) kGramChunk)
// of head bh, products of the exact input values summed in fp64 in key order.
template <typename T>
__global__ void __launch_bounds__(256) key_gram_partial_kernel(Layout L, const T* __restrict__ K) {
  pdl_entry();
  __shared__ float ks[kGramStage][128];
  const int bh = blockIdx.x, a0 = blockIdx.y * kGramRows, c = blockIdx.z, d = L.d, tid = threadIdx.x;
  const int b = tid % d, lanes_per_b = 256 / d, r0 = tid / d;
  const int nout = kGramRows / lanes_per_b;  // d = 128: 8 rows per thread; d = 64: 4
  const T* k = K + (size_t)bh * L.N * d;
  const int t0 = c * kGramChunk, t1 = min(L.N, t0 + kGramChunk);
  double acc[kGramRows / 2];
#pragma unroll
  for (int r = 0; r < kGramRows / 2; ++r) acc[r] = 0.0;
  for (int i0 = t0; i0 < t1; i0 += kGramStage) {
    const int ni = min(kGramStage, t1 - i0);
    __syncthreads();
    for (int e = tid; e < ni * d; e += 256) ks[e / d][e % d] = to_f32(k[(size_t)(i0 + e / d) * d + e % d]);
    __syncthreads();
    for (int i = 0; i < ni; ++i) {
      const double xb = (double)ks[i][b];
#pragma unroll
      for (int r = 0; r < kGramRows / 2; ++r)
        if (r < nout) acc[r] += (double)ks[i][a0 + r0 + r * lanes_per_b] * xb;
    }
  }
#pragma unroll
  for (int r = 0; r < kGramRows / 2; ++r)
    if (r < nout)
      L.kgram_part[(((size_t)bh * gridDim.z + c) * d + a0 + r0 + r * lanes_per_b) * d + b] = acc[r];
}

// K^T K of head bh = sum of its chunks' partial Grams, chunk 0 first.
__global__ void key_gram_reduce_kernel(Layout L, int nchunk) {
  pdl_entry();
  const int bh = blockIdx.x, a = blockIdx.y, d = L.d;
  for (int b = threadIdx.x; b < d; b += blockDim.x) {
    double s = 0.0;
    for (int c = 0; c < nchunk; ++c) s += L.kgram_part[(((size_t)bh * nchunk + c) * d + a) * d + b];
    L.kgram[((size_t)bh * d + a) * d + b] = s;
  }
}

// One CTA per head: M <- M_r (see the file comment).  Dynamic shared memory: d x d doubles.
__global__ void __launch_bounds__(256) key_rank_kernel(Layout L) {
  pdl_entry();
  extern __shared__ double sS[];  // [d][d]
  __shared__ double diag[128];
  __shared__ double ev[128];
  __shared__ int order[128];
  const int bh = blockIdx.x, d = L.d, tid = threadIdx.x, nt = blockDim.x;
  const size_t dd = (size_t)d * d;
  double* M = L.M + bh * dd;
  const double* G = L.kgram + bh * dd;
  double* Lf = L.kr_L + bh * dd;  // the factor L (d x d, row-major)
  double* V = L.kr_V + bh * dd;   // eigenvectors (rows, as jacobi_eig leaves them)
  double* T = L.kr_T + bh * dd;   // G L, later Y = L Z_r (d x r)
  // factor of M: Cholesky when M is positive definite, else E D^(1/2)
  for (size_t e = tid; e < dd; e += nt) sS[e] = M[e];
  __syncthreads();
  double mx = 0.0;
  for (int i = 0; i < d; ++i) mx = fmax(mx, sS[i * d + i]);
  const bool chol = mx > 0.0 && chol_smem_tol(sS, d, d, 1e-13 * mx, diag);  // the same in every thread
  if (chol) {
    for (size_t e = tid; e < dd; e += nt) {
      const int i = (int)(e / d), k = (int)(e % d);
      Lf[e] = i > k ? sS[k * d + i] : (i == k ? diag[k] : 0.0);  // L_ik sits at [k][i], i > k
    }
  } else {
    for (size_t e = tid; e < dd; e += nt) sS[e] = M[e];
    __syncthreads();
    jacobi_eig(sS, V, d);
    for (size_t e = tid; e < dd; e += nt) {
      const int i = (int)(e / d), k = (int)(e % d);  // L = E D^(1/2): E[i][k] = row k of V, entry i
      Lf[e] = V[(size_t)k * d + i] * sqrt(fmax(sS[k * d + k], 0.0));
    }
  }
  __syncthreads();
  // H = L^T (G L): T = G L in global memory, then H into shared memory
  for (size_t e = tid; e < dd; e += nt) {
    const int i = (int)(e / d), j = (int)(e % d);
    double s = 0.0;
    for (int m = 0; m < d; ++m) s += G[(size_t)i * d + m] * Lf[(size_t)m * d + j];
    T[e] = s;
  }
  __syncthreads();
  for (size_t e = tid; e < dd; e += nt) {
    const int i = (int)(e / d), j = (int)(e % d);
    double s = 0.0;
    for (int m = 0; m < d; ++m) s += Lf[(size_t)m * d + i] * T[(size_t)m * d + j];
    sS[e] = s;
  }
  __syncthreads();
  jacobi_eig(sS, V, d);
  // the r leading eigenvalues (descending, ties to the lower index)
  for (int i = tid; i < d; i += nt) {
    const double e = sS[i * d + i];
    ev[i] = isnan(e) ? -INFINITY : e;  // NaN (from non-finite inputs) ranks last: order[] stays a permutation
  }
  __syncthreads();
  for (int i = tid; i < d; i += nt) {
    int rk = 0;
    for (int j = 0; j < d; ++j) rk += ev[j] > ev[i] || (ev[j] == ev[i] && j < i);
    order[rk] = i;
  }
  __syncthreads();
  const int r = min(L.key_rank, d);
  // Y = L Z_r (d x r) into T, then M_r = Y Y^T
  for (int e = tid; e < d * r; e += nt) {
    const int i = e / r, q = e % r, col = order[q];
    double s = 0.0;
    for (int m = 0; m < d; ++m) s += Lf[(size_t)i * d + m] * V[(size_t)col * d + m];
    T[e] = s;
  }
  __syncthreads();
  for (size_t e = tid; e < dd; e += nt) {
    const int i = (int)(e / d), j = (int)(e % d);
    double s = 0.0;
    for (int q = 0; q < r; ++q) s += T[(size_t)i * r + q] * T[(size_t)j * r + q];
    M[e] = s;
  }
}

template <typename T>
sparsepr_status launch_key_rank_t(const Layout& L, const T* K, cudaStream_t st) {
  const int nchunk = (L.N + kGramChunk - 1) / kGramChunk;
  launch(key_gram_partial_kernel<T>, dim3(L.BH, L.d / kGramRows, nchunk), 256, 0, st, L, K);
  launch(key_gram_reduce_kernel, dim3(L.BH, L.d), 128, 0, st, L, nchunk);
  const size_t smem = (size_t)L.d * L.d * sizeof(double);
  cudaFuncSetAttribute(key_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  launch(key_rank_kernel, L.BH, 256, smem, st, L);
  SPR_LAUNCH_CHECK();
  return SPARSEPR_OK;
}

sparsepr_status launch_key_rank(const Layout& L, const void* K, cudaStream_t st) {
  if (L.dtype == SPARSEPR_F32) return launch_key_rank_t(L, (const float*)K, st);
  return launch_key_rank_t(L, (const __nv_bfloat16*)K, st);
}

}  // namespace sparsepr
