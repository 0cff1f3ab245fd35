// Probe-Fitted Residual Reconstruction of the SparsePR operator.
//
// "Partition the Support, Reconstruct the Residual" (arXiv 2608.18484), abstract: an affine
// map from the sparse output to the probe rows' dense-minus-sparse differences is fitted by
// weighted ridge regression and the residual it predicts is added to every unprobed row; the
// arXiv abstract page confines the correction to the subspace the probe residuals span; the
// project page's method column names the step Probe-Fitted Residual Reconstruction.
//
// Per head, with X_p = [O_sp(p), 1], R_p = O_dense(p) - O_sp(p), W = diag(w):
//   A = (X^T W X + lam I)^-1 X^T W R,   lam = 1e-3 tr(X^T W X)/(d+1) unless given,
//   A <- A U U^T with U an orthonormal basis of span{R_p},
//   O_i = O_sp,i + [O_sp,i, 1] A for unprobed rows, O_dense for probe rows.
// The normal equations and the span basis are solved in fp64 by one CTA per head.
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"
#include "linalg.cuh"

namespace sparsepr {

constexpr int kRidgeRows = 8;    // rows of G/B/S per block
constexpr int kRidgeChunk = 32;  // probes staged per step
// threads of a solve CTA: every step of the Gauss-Jordan inverse, the Cholesky test, the
// Gram-Schmidt and the Jacobi rotations is one barrier-separated pass over a (d+1)^2 or d^2
// matrix, so more threads shorten each step (1024 measured 30 us faster per mid-size call than 256)
constexpr int kRidgeSolveThreads = 1024;

// G = X^T W X ((d+1)^2), B = X^T W R ((d+1) x d), S = R^T W R (d x d): rows
// [8 y, 8 y + 8) of each, summed over the probes in a fixed order.
__global__ void __launch_bounds__(256) ridge_gram_kernel(Layout L) {
  pdl_entry();
  extern __shared__ double shr[];
  const int bh = blockIdx.x, d = L.d, n1 = d + 1, P = L.P, tid = threadIdx.x;
  double* X = shr;                       // [32][n1]
  double* R = X + kRidgeChunk * n1;      // [32][d]
  double* w = R + kRidgeChunk * d;       // [32]
  const int a0 = blockIdx.y * kRidgeRows;
  // outputs owned by this thread: index o over [8 rows] x [n1 (G) + d (B) + d (S)]
  const int per_row = n1 + 2 * d;
  const int n_out = kRidgeRows * per_row;
  double acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.0;
  const int* tok = L.probe_tok + (size_t)bh * P;
  const int* qinv = L.qinv + (size_t)bh * L.N;
  const float* osp = L.Osp + (size_t)bh * L.N * d;
  const float* od = L.Odense + (size_t)bh * P * d;
  for (int p0 = 0; p0 < P; p0 += kRidgeChunk) {
    const int np = min(kRidgeChunk, P - p0);
    __syncthreads();
    for (int e = tid; e < kRidgeChunk * n1; e += 256) {
      const int p = e / n1, a = e % n1;
      double v = 0.0;
      if (p < np) v = a < d ? (double)osp[(size_t)qinv[tok[p0 + p]] * d + a] : 1.0;
      X[e] = v;
    }
    for (int e = tid; e < kRidgeChunk * d; e += 256) {
      const int p = e / d, a = e % d;
      R[e] = p < np ? (double)od[(size_t)(p0 + p) * d + a] - (double)osp[(size_t)qinv[tok[p0 + p]] * d + a] : 0.0;
    }
    if (tid < kRidgeChunk) w[tid] = tid < np ? L.probe_w[(size_t)bh * P + p0 + tid] : 0.0;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int o = tid + i * 256;
      if (o >= n_out) break;
      const int rr = o / per_row, c = o % per_row, a = a0 + rr;
      if (a >= n1) continue;
      double s = 0.0;
      if (c < n1) {
        for (int p = 0; p < np; ++p) s += w[p] * X[p * n1 + a] * X[p * n1 + c];
      } else if (c < n1 + d) {
        const int cc = c - n1;
        for (int p = 0; p < np; ++p) s += w[p] * X[p * n1 + a] * R[p * d + cc];
      } else {
        const int cc = c - n1 - d;
        if (a < d)
          for (int p = 0; p < np; ++p) s += w[p] * R[p * d + a] * R[p * d + cc];
      }
      acc[i] += s;
    }
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int o = tid + i * 256;
    if (o >= n_out) break;
    const int rr = o / per_row, c = o % per_row, a = a0 + rr;
    if (a >= n1) continue;
    if (c < n1) L.ridgeG[((size_t)bh * n1 + a) * n1 + c] = acc[i];
    else if (c < n1 + d) L.ridgeB[((size_t)bh * n1 + a) * d + (c - n1)] = acc[i];
    else if (a < d) L.spanS[((size_t)bh * d + a) * d + (c - n1 - d)] = acc[i];
  }
}

// Shared memory of the solve: the (d+1)^2 system and a (d+1) x 33 block of right-hand sides.
// Dynamic shared memory of ridge_solve_kernel: G + lam I and 32 staged columns of B (role 0),
// S (role 1); at d <= 64 also room for the Jacobi rotations next to S (2 d^2 doubles).
__host__ __device__ inline size_t ridge_solve_smem(int d) {
  const size_t base = (size_t)((d + 1) * (d + 1) + (d + 1) * 33) * sizeof(double);
  const size_t jac = d <= 64 ? (size_t)2 * d * d * sizeof(double) : 0;
  return base > jac ? base : jac;
}

// In-place Gauss-Jordan inverse of the symmetric positive definite n x n matrix in shared
// memory (no pivoting: the pivots of an SPD matrix are the Cholesky pivots squared and stay
// positive), two barriers per step.  False if a pivot is not positive (or not finite).
__device__ bool gj_inverse_spd(double* G, int n, int ld) {
  const int nthr = blockDim.x;
  __syncthreads();
  for (int k = 0; k < n; ++k) {
    const double p = G[k * ld + k];
    if (!(p > 0.0) || !isfinite(p)) return false;  // the same value in every thread
    const double inv = 1.0 / p;
    // every (i, j) off row and column k: reads row k and column k, which this phase leaves alone
    // (warps over rows, lanes over columns)
    const int nw = nthr >> 5, w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = w; i < n; i += nw) {
      if (i == k) continue;
      const double f = G[i * ld + k] * inv;
      for (int j = lane; j < n; j += 32)
        if (j != k) G[i * ld + j] -= f * G[k * ld + j];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < n; e += nthr) {
      if (e != k) {
        G[k * ld + e] *= inv;
        G[e * ld + k] *= -inv;
      }
    }
    if (threadIdx.x == 0) G[k * ld + k] = inv;
    __syncthreads();
  }
  return true;
}

// The r leading eigenvectors of S = R^T W R (Table D.2's output truncation), by the parallel
// cyclic Jacobi method (jacobi_eig): S in shared memory, the accumulated rotations V next to it
// when both fit (d = 64), else in the head's spanS (global, where S came from).  The
// eigenvectors of eigenvalue above 1e-10 of the largest are ranked by eigenvalue (ties: lower
// index) and the first min(r, count) become the basis; the count goes to span_rank.

__device__ __noinline__ void span_basis_truncated(const Layout& L, int bh, double* S) {
  const int d = L.d, tid = threadIdx.x, nt = blockDim.x;
  double* Ug = L.spanS + (size_t)bh * d * d;
  // the rotations accumulate in shared memory next to S when both fit (d = 64), else in L2
  double* V = (size_t)2 * d * d * sizeof(double) <= ridge_solve_smem(d) ? S + d * d : Ug;
  __shared__ double ev[128];
  __shared__ int order[128];
  __shared__ int s_kept;
  for (int e = tid; e < d * d; e += nt) S[e] = Ug[e];
  __syncthreads();
  jacobi_eig(S, V, d);
  // eigenvalues, the kept ones ranked by size, the leading min(r, kept) columns of V
  for (int i = tid; i < d; i += nt) ev[i] = S[i * d + i];
  __syncthreads();
  double top = 0.0;
  for (int i = 0; i < d; ++i) top = fmax(top, ev[i]);
  const double thr = 1e-10 * top;
  if (tid == 0) s_kept = 0;
  __syncthreads();
  for (int i = tid; i < d; i += nt) {
    if (top > 0.0 && ev[i] > thr) {
      int rk = 0;
      for (int j = 0; j < d; ++j) rk += ev[j] > thr && (ev[j] > ev[i] || (ev[j] == ev[i] && j < i));
      order[rk] = i;
      atomicAdd(&s_kept, 1);
    }
  }
  __syncthreads();
  const int rank = min(L.trunc_rank, s_kept);
  for (int e = tid; e < d * rank; e += nt) S[e] = V[order[e % rank] * d + e / rank];  // [d][rank] (V: rows)
  __syncthreads();
  for (int e = tid; e < d * rank; e += nt) Ug[(e / rank) * d + e % rank] = S[e];  // U[i*d + r]
  if (tid == 0) L.stats[bh].span_rank = rank;
}

// The residual-span basis of head bh (role 1 of ridge_solve_kernel): span of the residual rows
// = range(S), S = R^T W R, whose rank goes to the head's statistics and whose basis (when the
// rank is below d) goes to spanS for the projection kernel.
__device__ __noinline__ void ridge_span_basis(const Layout& L, int bh, double* G, double* ldiag) {
  const int d = L.d, tid = threadIdx.x;
  sparsepr_head_stats& st = L.stats[bh];
  // span of the residual rows = range(S), S = R^T W R.  Full rank is the common case: a
  // Cholesky of S whose pivots all stay above 1e-10 of the largest diagonal entry proves it,
  // and then the projector is the identity.  Otherwise an orthonormal basis U of range(S) comes
  // from column-pivoted Gram-Schmidt on the columns of S (column norms scale like
  // eigenvalue^2, so the cut is 1e-20 of the largest squared norm).
  double* S = G;
  const double* Sg = L.spanS + (size_t)bh * d * d;
  __shared__ double s_dmax;
  for (int e = tid; e < d * d; e += blockDim.x) S[e] = Sg[e];
  __syncthreads();
  if (tid == 0) {
    double mx = 0.0;
    for (int i = 0; i < d; ++i) mx = fmax(mx, S[i * d + i]);
    s_dmax = mx;
  }
  __syncthreads();
  int rank = 0;
  __shared__ int bcol[128];  // pivot columns in basis order
  bool full = s_dmax > 0.0 && chol_smem_tol(S, d, d, 1e-10 * s_dmax, ldiag);
  if (full) {
    rank = d;
  } else if (s_dmax > 0.0) {
    // Column-pivoted Gram-Schmidt with one barrier per step: every warp finds the same pivot
    // (largest remaining squared norm cn, lowest index on ties); the unused columns remove
    // their component along the pivot column v_p (v_c -= (v_p . v_c / |v_p|^2) v_p, the pivot
    // column itself is normalised once at the end), tpc threads per column.
    // S[i*ld + c]: column c, entry i; rows padded to d + 1 so the tpc threads of a column,
    // on rows i, i + 1, ..., read different banks
    const int ld = d + 1;
    for (int e = tid; e < d * d; e += blockDim.x) S[(e / d) * ld + (e % d)] = Sg[e];
    __shared__ double cn[128];
    __shared__ int used[128];
    __shared__ double binv[128];
    const int tpc = blockDim.x / d, sub = tid % tpc;  // 4 (d = 64) or 2 (d = 128)
    __syncthreads();
    for (int c = tid / tpc; c < d; c += blockDim.x / tpc) {
      double sacc = 0.0;
      for (int i = sub; i < d; i += tpc) sacc += S[i * ld + c] * S[i * ld + c];
      for (int o = 1; o < tpc; o <<= 1) sacc += __shfl_xor_sync(0xffffffffu, sacc, o);
      if (sub == 0) {
        cn[c] = sacc;
        used[c] = 0;
      }
    }
    __syncthreads();
    const int lane = tid & 31;
    double mx = 0.0;
    for (int c = lane; c < d; c += 32) mx = fmax(mx, cn[c]);
    for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const double tol = mx * 1e-20;
    for (int step = 0; step < d; ++step) {
      double bv = -1.0;
      int bi = -1;
      for (int c = lane; c < d; c += 32)
        if (!used[c] && cn[c] > bv) {
          bv = cn[c];
          bi = c;
        }
      for (int o = 16; o > 0; o >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi >= 0 && (bi < 0 || oi < bi))) {
          bv = ov;
          bi = oi;
        }
      }
      if (!(bi >= 0 && bv > tol && bv > 0.0)) break;  // the same in every thread
      const double inv2 = 1.0 / bv;
      for (int c = tid / tpc; c < d; c += blockDim.x / tpc) {
        const bool act = !used[c] && c != bi;
        double dot = 0.0;
        if (act)
          for (int i = sub; i < d; i += tpc) dot += S[i * ld + bi] * S[i * ld + c];
        for (int o = 1; o < tpc; o <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        dot *= inv2;
        double sacc = 0.0;
        if (act)
          for (int i = sub; i < d; i += tpc) {
            const double v = S[i * ld + c] - dot * S[i * ld + bi];
            S[i * ld + c] = v;
            sacc += v * v;
          }
        for (int o = 1; o < tpc; o <<= 1) sacc += __shfl_xor_sync(0xffffffffu, sacc, o);
        if (act && sub == 0) cn[c] = sacc;
      }
      if (tid == 0) {
        used[bi] = 1;
        bcol[rank] = bi;
        binv[rank] = sqrt(inv2);
      }
      ++rank;
      __syncthreads();
    }
    for (int e = tid; e < d * rank; e += blockDim.x) {  // normalise the basis columns
      const int i = e / rank, r = e % rank;
      S[i * ld + bcol[r]] *= binv[r];
    }
    __syncthreads();
  }
  // hand the basis to the projection kernel: columns r < rank of spanS are U's columns
  __syncthreads();
  if (rank < d) {
    double* U = L.spanS + (size_t)bh * d * d;
    for (int e = tid; e < d * rank; e += blockDim.x) {
      const int i = e / rank, r = e % rank;
      U[i * d + r] = S[i * (d + 1) + bcol[r]];  // the Gram-Schmidt rows are padded to d + 1
    }
  }
  if (tid == 0) st.span_rank = rank;
}

// Two CTAs per head, which run at the same time: role 0 takes lam, the inverse of G + lam I
// with up to three x10 jitter retries and the d right-hand sides; role 1 takes the residual-span
// basis (a full-rank test, else column-pivoted Gram-Schmidt on S = R^T W R).  The projection
// A <- A U U^T follows in ridge_project_kernel.
__global__ void __launch_bounds__(kRidgeSolveThreads) ridge_solve_kernel(Layout L) {
  pdl_entry();
  extern __shared__ double shs[];
  const int bh = blockIdx.x >> 1, role = blockIdx.x & 1, d = L.d, n1 = d + 1, tid = threadIdx.x;
  double* G = shs;  // [n1][n1], later S [d][d]
  __shared__ double red[kRidgeSolveThreads / 32];
  __shared__ double ldiag[129];  // diagonal of the Cholesky factor
  const double* Gg = L.ridgeG + (size_t)bh * n1 * n1;
  double* A = L.A64 + (size_t)bh * n1 * d;
  sparsepr_head_stats& st = L.stats[bh];

  if (L.P == 0) {
    if (role == 0) {
      for (int e = tid; e < n1 * d; e += blockDim.x) {
        A[e] = 0.0;
        L.A32[(size_t)bh * n1 * d + e] = 0.f;
      }
      if (tid == 0) {
        st.lambda = 0.0;
        st.fit_retries = 0;
      }
    } else if (tid == 0) {
      st.span_rank = 0;
    }
    return;
  }
  if (role == 1) {
    if (L.trunc_rank > 0 && L.trunc_rank < d)
      span_basis_truncated(L, bh, shs);
    else
      ridge_span_basis(L, bh, shs, ldiag);
    return;
  }
  if (L.correction == SPARSEPR_CORRECTION_MEAN) {
    // Table 4 "Mean-only": the constant feature alone, A_lin = 0 and intercept
    // (sum w + lam)^-1 sum w R, i.e. row d of B over G[d][d] (+ lam; lam < 0 selects
    // 1e-3 * sum w, the rule of the 1 x 1 Gram)
    const double sw = Gg[(size_t)d * n1 + d];
    const double lam = L.lambda >= 0.0 ? L.lambda : 1e-3 * sw;
    const double* Bg = L.ridgeB + (size_t)bh * n1 * d;
    const double den = sw + lam;
    for (int e = tid; e < n1 * d; e += blockDim.x) A[e] = (e >= d * d && den > 0.0) ? Bg[e] / den : 0.0;
    if (tid == 0) {
      st.lambda = lam;
      st.fit_retries = 0;
    }
    return;
  }
  double tr = 0.0;
  for (int i = tid; i < n1; i += blockDim.x) tr += Gg[i * n1 + i];
  tr = block_sum(tr, red);
  double lam = L.lambda >= 0.0 ? L.lambda : 1e-3 * tr / n1;
  int retries = 0;
  bool ok = false;
  for (; retries <= 3; ++retries) {
    for (int e = tid; e < n1 * n1; e += blockDim.x) G[e] = Gg[e] + ((e / n1) == (e % n1) ? lam : 0.0);
    __syncthreads();
    ok = gj_inverse_spd(G, n1, n1);
    if (ok) break;
    lam = lam > 0.0 ? lam * 10.0 : (tr > 0.0 ? 1e-12 * tr / n1 : 1e-30);
  }
  if (!ok) {
    if (tid == 0) {
      atomicCAS(L.status, kDevOk, kDevNumeric);
      st.fit_retries = retries - 1;  // the three jitter retries all failed; A is zero
    }
    for (int e = tid; e < n1 * d; e += blockDim.x) {
      A[e] = 0.0;
      L.A32[(size_t)bh * n1 * d + e] = 0.f;
    }
    return;
  }
  // A = (G + lam I)^-1 B, 32 columns of B at a time staged in shared memory (all loads in
  // flight together); thread = (row, column) of the chunk
  {
    const double* Bg = L.ridgeB + (size_t)bh * n1 * d;
    double* Y = G + n1 * n1;  // [n1][33]
    for (int c0 = 0; c0 < d; c0 += 32) {
      __syncthreads();
      for (int e = tid; e < n1 * 32; e += blockDim.x) Y[(e >> 5) * 33 + (e & 31)] = Bg[(size_t)(e >> 5) * d + c0 + (e & 31)];
      __syncthreads();
      for (int e = tid; e < n1 * 32; e += blockDim.x) {
        const int a = e >> 5, j = e & 31;
        const double* gr = G + a * n1;
        double acc0 = 0.0, acc1 = 0.0;
        int k = 0;
        for (; k + 1 < n1; k += 2) {
          acc0 += gr[k] * Y[k * 33 + j];
          acc1 += gr[k + 1] * Y[(k + 1) * 33 + j];
        }
        if (k < n1) acc0 += gr[k] * Y[k * 33 + j];
        A[(size_t)a * d + c0 + j] = acc0 + acc1;
      }
    }
  }
  if (tid == 0) {
    st.lambda = lam;
    st.fit_retries = retries;
  }
}

// A <- (A U) U^T with U (d x rank) the residual-span basis; 8 rows of A per block.  A
// full-rank span is all of R^d: the projector is the identity and A is only copied to fp32.
__global__ void __launch_bounds__(256) ridge_project_kernel(Layout L) {
  pdl_entry();
  extern __shared__ double shp2[];
  const int bh = blockIdx.x, d = L.d, n1 = d + 1, tid = threadIdx.x;
  const int rank = L.P > 0 ? L.stats[bh].span_rank : d;
  const int a0 = blockIdx.y * 8, na = min(8, n1 - a0);
  double* A = L.A64 + (size_t)bh * n1 * d;
  float* A32 = L.A32 + (size_t)bh * n1 * d;
  if (rank >= d) {
    for (int e = tid; e < na * d; e += blockDim.x) A32[(size_t)a0 * d + e] = (float)A[(size_t)a0 * d + e];
    return;
  }
  double* U = shp2;                 // [d][rank]
  double* Ar = U + d * rank;        // [8][d]
  double* T = Ar + 8 * d;           // [8][rank]
  const double* Ug = L.spanS + (size_t)bh * d * d;
  for (int e = tid; e < d * rank; e += blockDim.x) U[e] = Ug[(e / rank) * d + (e % rank)];
  for (int e = tid; e < na * d; e += blockDim.x) Ar[e] = A[(size_t)a0 * d + e];
  __syncthreads();
  for (int e = tid; e < na * rank; e += blockDim.x) {
    const int r8 = e / rank, k = e % rank;
    double acc = 0.0;
    for (int i = 0; i < d; ++i) acc += Ar[r8 * d + i] * U[i * rank + k];
    T[r8 * rank + k] = acc;
  }
  __syncthreads();
  for (int e = tid; e < na * d; e += blockDim.x) {
    const int r8 = e / d, i = e % d;
    double acc = 0.0;
    for (int k = 0; k < rank; ++k) acc += T[r8 * rank + k] * U[i * rank + k];
    A[(size_t)a0 * d + e] = acc;
    A32[(size_t)a0 * d + e] = (float)acc;
  }
}

// a10: O[token] = O_sp + [O_sp, 1] A for unprobed rows, O_dense for probe rows; 64 permuted
// rows per block, written back to original token order.
template <typename To, int D>
__global__ void __launch_bounds__(256) apply_kernel(Layout L, To* __restrict__ O) {
  pdl_entry();
  extern __shared__ float sha[];
  float* As = sha;                  // [(D+1)][D]
  float* Xs = As + (D + 1) * D;     // [64][D]
  const int bh = blockIdx.y, tid = threadIdx.x;
  const int r0 = blockIdx.x * 64, nr = min(64, L.N - r0);
  const float* A = L.A32 + (size_t)bh * (D + 1) * D;
  for (int e = tid; e < (D + 1) * D; e += 256) As[e] = A[e];
  const float* osp = L.Osp + ((size_t)bh * L.N + r0) * D;
  for (int e = tid; e < 64 * D; e += 256) Xs[e] = e / D < nr ? osp[e] : 0.f;
  __syncthreads();
  const int* perm = L.qperm + (size_t)bh * L.N;
  const int* pof = L.probe_of + (size_t)bh * L.N;
  const float* od = L.Odense + (size_t)bh * L.P * D;
  for (int e = tid; e < nr * D; e += 256) {
    const int r = e / D, c = e % D;
    const int t = perm[r0 + r];
    const int p = pof[t];
    float v;
    if (p >= 0) {
      v = od[(size_t)p * D + c];
    } else {
      float acc = As[D * D + c];
      const float* x = Xs + r * D;
#pragma unroll 8
      for (int a = 0; a < D; ++a) acc = fmaf(x[a], As[a * D + c], acc);
      v = x[c] + acc;
    }
    To* orow = O + ((size_t)bh * L.N + t) * D;
    if constexpr (std::is_same<To, float>::value) orow[c] = v;
    else orow[c] = __float2bfloat16_rn(v);
  }
}

template <typename To, int D>
static sparsepr_status launch_apply(const Layout& L, void* O, cudaStream_t st) {
  const size_t smem = (size_t)((D + 1) * D + 64 * D) * 4;
  cudaFuncSetAttribute(apply_kernel<To, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  launch(apply_kernel<To, D>, dim3((L.N + 63) / 64, L.BH), 256, smem, st, L, (To*)O);
  SPR_LAUNCH_CHECK();
  return SPARSEPR_OK;
}

// No correction (repair off): A = 0, so unprobed rows keep O_sp and probe rows take O_dense.
__global__ void zero_fit_kernel(Layout L) {
  pdl_entry();
  const int bh = blockIdx.x, n = (L.d + 1) * L.d;
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    L.A64[(size_t)bh * n + e] = 0.0;
    L.A32[(size_t)bh * n + e] = 0.f;
  }
  if (threadIdx.x == 0) {
    L.stats[bh].lambda = 0.0;
    L.stats[bh].fit_retries = 0;
    L.stats[bh].span_rank = 0;
  }
}

sparsepr_status launch_fit_apply(const Layout& L, void* O, int out_dtype, cudaStream_t st) {
  const int d = L.d, n1 = d + 1;
  if (!L.repair) {
    launch(zero_fit_kernel, L.BH, 256, 0, st, L);
    SPR_LAUNCH_CHECK();
  } else if (L.P > 0) {
    const size_t gsm = (size_t)(kRidgeChunk * n1 + kRidgeChunk * d + kRidgeChunk) * sizeof(double);
    cudaFuncSetAttribute(ridge_gram_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gsm);
    launch(ridge_gram_kernel, dim3(L.BH, (n1 + kRidgeRows - 1) / kRidgeRows), 256, gsm, st, L);
  }
  if (L.repair) {
    const sparsepr_status s = launch_ridge_solve(L, st);
    if (s != SPARSEPR_OK) return s;
  }
  if (L.dtype == SPARSEPR_BF16) return launch_apply_tc(L, O, out_dtype, st);
  if (out_dtype == SPARSEPR_F32)
    return d == 64 ? launch_apply<float, 64>(L, O, st) : launch_apply<float, 128>(L, O, st);
  return d == 64 ? launch_apply<__nv_bfloat16, 64>(L, O, st) : launch_apply<__nv_bfloat16, 128>(L, O, st);
}

}  // namespace sparsepr

namespace sparsepr {

// The solve (two CTAs per head) and the projection on ridge matrices that are already in
// L.ridgeG / ridgeB / spanS.
sparsepr_status launch_ridge_solve(const Layout& L, cudaStream_t st) {
  const size_t ssm = ridge_solve_smem(L.d);
  cudaFuncSetAttribute(ridge_solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssm);
  launch(ridge_solve_kernel, 2 * L.BH, kRidgeSolveThreads, ssm, st, L);  // two roles per head
  const size_t psm = (size_t)(L.d * L.d + 8 * L.d + 8 * L.d) * sizeof(double);
  cudaFuncSetAttribute(ridge_project_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)psm);
  launch(ridge_project_kernel, dim3(L.BH, (L.d + 1 + 7) / 8), 256, psm, st, L);
  SPR_LAUNCH_CHECK();
  return SPARSEPR_OK;
}

}  // namespace sparsepr
