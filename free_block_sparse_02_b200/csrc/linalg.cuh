// Dense fp64 linear algebra on small (d x d, d <= 128) matrices held in shared memory, run by
// one CTA (every thread of the block calls these; they contain block barriers): a Cholesky
// factorisation with a pivot test, and a parallel cyclic Jacobi eigensolver.  Used by the ridge
// fit (residual span, output truncation) and by the key-response rank projection.
#pragma once

#include <math.h>

#include "common.cuh"

namespace sparsepr {

// Cholesky G = L L^T of the n x n matrix in shared memory with one barrier per step: step k
// reads column k of the (lower) trailing matrix, writes L's column k below the diagonal into
// row k of the upper triangle (L_ik at G[k][i], i > k) and L_kk into diag[k], and updates the
// trailing lower part G[i][j] -= G[i][k] G[j][k] / G[k][k] (k < j <= i) without touching
// column k.  False if a pivot is not above `tol` (or not finite).
static __device__ bool chol_smem_tol(double* G, int n, int ld, double tol, double* diag) {
  const int nthr = blockDim.x;
  __syncthreads();
  for (int k = 0; k < n; ++k) {
    const double piv = G[k * ld + k];
    if (!(piv > tol) || !isfinite(piv)) return false;  // the same value in every thread
    const double lkk = sqrt(piv), inv = 1.0 / lkk, ipiv = 1.0 / piv;
    if (threadIdx.x == 0) diag[k] = lkk;
    for (int i = k + 1 + threadIdx.x; i < n; i += nthr) G[k * ld + i] = G[i * ld + k] * inv;
    // trailing pairs (i, j), k < j <= i < n: warp-strided rows, lanes over columns
    const int nw = nthr >> 5, w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = k + 1 + w; i < n; i += nw) {
      const double lik = G[i * ld + k] * ipiv;
      for (int j = k + 1 + lane; j <= i; j += 32) G[i * ld + j] -= lik * G[j * ld + k];
    }
    __syncthreads();
  }
  return true;
}

constexpr int kJacobiSweeps = 30;

// Eigen-decomposition of the symmetric d x d matrix S (shared memory, d even, d <= 128) by the
// parallel cyclic Jacobi method in fp64 (Golub & Van Loan, "Matrix Computations": the symmetric
// Schur rotation and the round-robin ordering).  A round applies d/2 disjoint rotations, chosen
// by the circle method so that every (p, q) pair meets once per sweep; sweeps run until the
// off-diagonal Frobenius norm is below 1e-13 of the matrix's, or kJacobiSweeps.  On return S is
// diagonal up to that tolerance (the eigenvalues) and Vt (d x d, shared or global memory,
// initialised here to I) holds the eigenvectors as ROWS: row p is the eigenvector of S[p][p].
// Rows, so that a rotation of the pair (p, q) reads and writes two contiguous rows.
static __device__ __noinline__ void jacobi_eig(double* S, double* Vt, int d) {
  const int tid = threadIdx.x, nt = blockDim.x, half = d / 2;
  __shared__ double rc[64], rs[64];
  __shared__ int rp[64], rq[64];
  __shared__ double red2[2][32];
  for (int e = tid; e < d * d; e += nt) Vt[e] = (e / d == e % d) ? 1.0 : 0.0;
  __syncthreads();
  for (int sweep = 0; sweep < kJacobiSweeps; ++sweep) {
    double off = 0.0, tot = 0.0;
    for (int e = tid; e < d * d; e += nt) {
      const double x = S[e] * S[e];
      tot += x;
      if (e / d != e % d) off += x;
    }
    for (int o = 16; o > 0; o >>= 1) {
      off += __shfl_xor_sync(0xffffffffu, off, o);
      tot += __shfl_xor_sync(0xffffffffu, tot, o);
    }
    if ((tid & 31) == 0) {
      red2[0][tid >> 5] = off;
      red2[1][tid >> 5] = tot;
    }
    __syncthreads();
    off = 0.0;
    tot = 0.0;
    for (int w = 0; w < nt / 32; ++w) {
      off += red2[0][w];
      tot += red2[1][w];
    }
    __syncthreads();
    // converged when the off-diagonal Frobenius norm is below 1e-13 of the whole: fp64 rounding
    // keeps it near d * 1e-16 relative, so a tighter test would never stop before the sweep limit
    if (!(off > 1e-26 * tot)) break;  // the same in every thread (also for a zero S)
    for (int round = 0; round < d - 1; ++round) {
      if (tid < half) {
        const int k = tid;
        const int a = k == 0 ? 0 : 1 + (k - 1 + round) % (d - 1);
        const int b = 1 + (d - 2 - k + round) % (d - 1);
        const int p = min(a, b), q = max(a, b);
        const double apq = S[p * d + q];
        double c = 1.0, sn = 0.0;
        if (apq != 0.0) {
          const double tau = (S[q * d + q] - S[p * d + p]) / (2.0 * apq);
          const double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
          c = 1.0 / sqrt(1.0 + t * t);
          sn = t * c;
        }
        rp[k] = p;
        rq[k] = q;
        rc[k] = c;
        rs[k] = sn;
      }
      __syncthreads();
      // S <- S J (columns p, q of every row); consecutive threads take different pairs of the
      // same row, so their shared-memory words fall in different banks
      for (int e = tid; e < half * d; e += nt) {
        const int k = e % half, i = e / half, p = rp[k], q = rq[k];
        const double c = rc[k], sn = rs[k], x = S[i * d + p], y = S[i * d + q];
        S[i * d + p] = c * x - sn * y;
        S[i * d + q] = sn * x + c * y;
      }
      __syncthreads();
      for (int e = tid; e < half * d; e += nt) {  // S <- J^T S (rows p, q), V <- V J (rows of Vt)
        const int k = e / d, j = e % d, p = rp[k], q = rq[k];
        const double c = rc[k], sn = rs[k];
        const double x = S[p * d + j], y = S[q * d + j];
        S[p * d + j] = c * x - sn * y;
        S[q * d + j] = sn * x + c * y;
        const double u = Vt[p * d + j], v = Vt[q * d + j];
        Vt[p * d + j] = c * u - sn * v;
        Vt[q * d + j] = sn * u + c * v;
      }
      __syncthreads();
    }
  }
  __syncthreads();
}

}  // namespace sparsepr
