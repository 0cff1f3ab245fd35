// Response-Coupled Partitioning, routing and probe choice of the SparsePR operator.
//
// "Partition the Support, Reconstruct the Residual" (arXiv 2608.18484), abstract: keys are
// grouped by their responses to sampled queries (paired K/V groups), queries by how they
// respond to the key-group centroids (shared sparse routing); project page "SparsePR:
// Training-Free Sparse Attention for Video Generation", method pipeline steps 01-03.
//
// Neither response matrix is materialised; both k-means run on the d-dimensional inputs.
// Keys: f_t = Q_s k_t / sqrt(d) (s dims).  For a group mean mu_j = Q_s c_j / sqrt(d) (c_j the
// mean of the member keys), ||f_t - mu_j||^2 = (k_t - c_j)^T M (k_t - c_j) with
// M = Q_s^T Q_s / d, so the label is argmin_j (c_j^T M c_j - 2 k_t . (M c_j)).
// Queries: the per-query RMS-normalised responses (Table D.1, "Per query RMS") are
// r~_q = C q / (sqrt(d) rms_q) with rms_q^2 = q^T Gc q + 1e-12, Gc = C^T C / (d C_k); for a group
// mean nu_g of r~, ||r~_q - nu_g||^2 = ||r~_q||^2 + ||nu_g||^2 - 2 (q . u_g) / rms_q with
// u_g = C^T nu_g / sqrt(d), and nu_g = C S_g / (sqrt(d) n_g) with S_g the sum of q / rms_q.
//
// Exactness: scores carry a rigorous rounding bound; a point whose best two scores are within
// it is re-decided over all groups in fp64, so labels agree with an fp64 evaluation except at
// ties far below the fp32 resolution.  Group sums are fp64.
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"
#include "kmeans.cuh"

namespace sparsepr {

// ------------------------------------------------------------------------------------------
// a1 + a2 prologue: M = Q_s^T Q_s / d (fp64, exact products, summed over the samples in order)
// per head.  Block (bh, y) computes rows [16 y, 16 y + 16) of M; the sampled rows are staged in
// shared memory (fp32, exact for bf16 and fp32 inputs) 64 at a time.
// ------------------------------------------------------------------------------------------
constexpr int kMetricRows = 16;
constexpr int kMetricChunk = 64;

template <typename T>
__global__ void __launch_bounds__(256) metric_kernel(Layout L, const T* __restrict__ Q) {
  pdl_entry();
  __shared__ float qs[kMetricChunk][128];
  __shared__ long long rowi[kMetricChunk];
  const int bh = blockIdx.x, a0 = blockIdx.y * kMetricRows, d = L.d, tid = threadIdx.x;
  const int b = tid % d, lanes_per_b = 256 / d, r0 = tid / d;
  constexpr int kMaxOut = kMetricRows / 2;  // d = 128: 8 rows per thread; d = 64: 4
  const int nout = kMetricRows / lanes_per_b;
  if (L.semantic) {  // the semantic partition clusters the raw keys: Euclidean metric M = I
    for (int k = 0; k < nout; ++k) {
      const int a = a0 + r0 + k * lanes_per_b;
      L.M[((size_t)bh * d + a) * d + b] = a == b ? 1.0 : 0.0;
    }
    return;
  }
  const T* q = Q + (size_t)bh * L.N * d;
  double acc[kMaxOut];
#pragma unroll
  for (int k = 0; k < kMaxOut; ++k) acc[k] = 0.0;
  for (int i0 = 0; i0 < L.s; i0 += kMetricChunk) {
    const int ni = min(kMetricChunk, L.s - i0);
    __syncthreads();
    if (tid < ni) rowi[tid] = ((2LL * (i0 + tid) + 1) * L.N) / (2LL * L.s);
    __syncthreads();
    for (int e = tid; e < ni * d; e += 256) {
      const int i = e / d, c = e % d;
      qs[i][c] = to_f32(q[rowi[i] * d + c]);
    }
    __syncthreads();
    for (int i = 0; i < ni; ++i) {
      const double xb = (double)qs[i][b];
#pragma unroll
      for (int k = 0; k < kMaxOut; ++k)
        if (k < nout) acc[k] += (double)qs[i][a0 + r0 + k * lanes_per_b] * xb;
    }
  }
#pragma unroll
  for (int k = 0; k < kMaxOut; ++k)
    if (k < nout) L.M[((size_t)bh * d + a0 + r0 + k * lanes_per_b) * d + b] = acc[k] / d;
}

// fp64 [BH, d, d] matrices split into three bf16 planes (tensor-core operands).
__global__ void split_mat_kernel(const double* __restrict__ src, __nv_bfloat16* __restrict__ dst, size_t n) {
  pdl_entry();
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const double x = src[i];
    const __nv_bfloat16 h = __double2bfloat16(x);
    const double r1 = x - (double)__bfloat162float(h);
    const __nv_bfloat16 m = __double2bfloat16(r1);
    dst[i] = h;
    dst[n + i] = m;
    dst[2 * n + i] = __double2bfloat16(r1 - (double)__bfloat162float(m));
  }
}

// Gc = C^T C / (d C_k) from the key-group centroids (fp64): rms_q^2 = q^T Gc q + 1e-12 is the
// mean square of the query's responses to every key group.
__global__ void gc_kernel(Layout L) {
  pdl_entry();
  const int bh = blockIdx.x, a = blockIdx.y, b = threadIdx.x, d = L.d;
  if (b >= d) return;
  if (L.semantic) {  // raw queries: the row quadratic form is ||q||^2
    L.Gc[((size_t)bh * d + a) * d + b] = a == b ? 1.0 : 0.0;
    return;
  }
  const double* C = L.kcent + (size_t)bh * L.Ck * d;
  double acc = 0.0;
  for (int j = 0; j < L.Ck; ++j) acc += C[(size_t)j * d + a] * C[(size_t)j * d + b];
  L.Gc[((size_t)bh * d + a) * d + b] = acc / ((double)d * L.Ck);
}

// Per-row quadratic forms on CUDA cores (the tensor-core version serves bf16 inputs).
//   keys    (which 0): x^T M x summed into T0k (the constant of the key objective); ||x||.
//   queries (which 1): ms = x^T Gc x; 1/rms, ||x||/rms, and C_k ms/(ms + 1e-12) = ||r~||^2
//                      summed into T0q.
// 64 rows per block; G staged in shared memory as fp32; thread (row p = tid/4, quarter q).
template <typename T>
__global__ void __launch_bounds__(256) rowqf_simt_kernel(Layout L, const T* __restrict__ X, int which) {
  pdl_entry();
  extern __shared__ float shm[];
  const int d = L.d, bh = blockIdx.y, tid = threadIdx.x;
  const int DP = d + 1;
  float* Gs = shm;              // [d][DP]
  float* Xs = Gs + d * DP;      // [64][DP]
  __shared__ double red[8];
  const int p0 = blockIdx.x * 64, np = min(64, L.N - p0);
  const double* G = (which == 0 ? L.M : L.Gc) + (size_t)bh * d * d;
  for (int e = tid; e < d * d; e += 256) Gs[(e / d) * DP + (e % d)] = (float)G[e];
  for (int e = tid; e < 64 * d; e += 256) {
    const int p = e / d, a = e % d;
    Xs[p * DP + a] = p < np ? to_f32(X[((size_t)bh * L.N + p0 + p) * d + a]) : 0.f;
  }
  __syncthreads();
  const int p = tid >> 2, q = tid & 3, dq = d >> 2;
  const float* xp = Xs + p * DP;
  float part = 0.f, nn = 0.f;
  for (int a = q * dq; a < (q + 1) * dq; ++a) {
    const float* Gr = Gs + a * DP;
    float u = 0.f;
    for (int b = 0; b < d; ++b) u = fmaf(Gr[b], xp[b], u);
    part = fmaf(u, xp[a], part);
    nn = fmaf(xp[a], xp[a], nn);
  }
  part += __shfl_xor_sync(0xffffffffu, part, 1);
  part += __shfl_xor_sync(0xffffffffu, part, 2);
  nn += __shfl_xor_sync(0xffffffffu, nn, 1);
  nn += __shfl_xor_sync(0xffffffffu, nn, 2);
  double contrib = 0.0;
  if (q == 0 && p < np) {
    const size_t row = (size_t)bh * L.N + p0 + p;
    if (which == 0) {
      L.knorm[row] = sqrtf(nn);
      contrib = part;
    } else {
      const double ms = (double)part;
      if (L.semantic) {  // raw queries: scale 1, objective constant ||q||^2
        L.inv_rms[row] = 1.f;
        L.inv_rms64[row] = 1.0;
        L.qxnorm[row] = sqrtf(nn);
        contrib = ms;
      } else {
        const float inv = (float)(1.0 / sqrt(ms + 1e-12));
        L.inv_rms[row] = inv;
        L.inv_rms64[row] = 1.0 / sqrt(ms + 1e-12);
        L.qxnorm[row] = sqrtf(nn) * inv;
        contrib = (double)L.Ck * ms / (ms + 1e-12);
      }
    }
  }
  const double tot = block_sum(contrib, red);
  if (tid == 0) atomicAdd((which == 0 ? L.T0k : L.T0q) + bh, tot);
}

// ------------------------------------------------------------------------------------------
// k-means initial points: SplitMix64 (Steele, Lea & Flood 2014) partial Fisher-Yates.
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ uint64_t splitmix64_next(uint64_t& state) {
  state += 0x9E3779B97F4A7C15ULL;
  uint64_t z = state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

// One thread per (head, side): block (bh, stage) draws the key (stage 0) or query (stage 1)
// initial points of head bh.  The draws depend on the seed alone, so both sides run in one
// launch.  The slots touched by C swaps live in a shared-memory hash map (slot -> value), so the
// identity array of N slots is never written.
__global__ void km_draw_kernel(Layout L) {
  pdl_entry();
  constexpr int kTab = 4096;  // >= 2 * 2 * kMaxGroups
  __shared__ int keys[kTab];
  __shared__ int vals[kTab];
  const int bh = blockIdx.x, stage = blockIdx.y, C = stage == 0 ? L.Ck : L.Cq;
  for (int i = threadIdx.x; i < kTab; i += blockDim.x) keys[i] = -1;
  __syncthreads();
  if (threadIdx.x != 0) return;
  auto slot_ref = [&](int slot) -> int* {
    unsigned h = ((unsigned)slot * 2654435761u) >> 20;  // 12 bits
    while (true) {
      if (keys[h] == slot) return &vals[h];
      if (keys[h] == -1) {
        keys[h] = slot;
        vals[h] = slot;
        return &vals[h];
      }
      h = (h + 1) & (kTab - 1);
    }
  };
  uint64_t state = L.seed + 2ULL * (uint64_t)bh + (uint64_t)stage;
  const uint64_t n = (uint64_t)L.N;
  int* out = L.init_ids + (size_t)bh * (L.Ck + L.Cq) + (stage == 0 ? 0 : L.Ck);
  for (int i = 0; i < C; ++i) {
    const uint64_t r = splitmix64_next(state);
    const int j = i + (int)(r % (n - (uint64_t)i));
    int* pi = slot_ref(i);
    int* pj = slot_ref(j);
    const int vi = *pi, vj = *pj;
    *pi = vj;
    *pj = vi;
    out[i] = vj;
  }
}

template <typename T>
__global__ void kcent_init_kernel(Layout L, const T* __restrict__ K) {
  pdl_entry();
  const int bh = blockIdx.x, j = blockIdx.y, a = threadIdx.x;
  if (a >= L.d) return;
  const int t = L.init_ids[(size_t)bh * (L.Ck + L.Cq) + j];
  L.kcent[((size_t)bh * L.Ck + j) * L.d + a] = (double)to_f32(K[((size_t)bh * L.N + t) * L.d + a]);
}

// Cold start of the query groups: nu_g = r~ of the drawn query, in fp64.
template <typename T>
__global__ void __launch_bounds__(128) qcent_init_kernel(Layout L, const T* __restrict__ Q) {
  pdl_entry();
  __shared__ double qv[128];
  __shared__ double red[4];
  const int bh = blockIdx.x, g = blockIdx.y, d = L.d, Ck = L.Ck, tid = threadIdx.x;
  const int t = L.init_ids[(size_t)bh * (L.Ck + L.Cq) + L.Ck + g];
  if (L.semantic) {  // raw queries: the drawn query itself is the centroid
    if (tid < d) L.qU64[((size_t)bh * L.Cq + g) * d + tid] = (double)to_f32(Q[((size_t)bh * L.N + t) * d + tid]);
    return;
  }
  if (tid < d) qv[tid] = (double)to_f32(Q[((size_t)bh * L.N + t) * d + tid]);
  __syncthreads();
  const double rsd = 1.0 / sqrt((double)d);
  double* nu = L.qcent + ((size_t)bh * L.Cq + g) * Ck;
  double ms = 0.0;
  for (int j = tid; j < Ck; j += blockDim.x) {
    const double* c = L.kcent + ((size_t)bh * Ck + j) * d;
    double r = 0.0;
    for (int a = 0; a < d; ++a) r += qv[a] * c[a];
    r *= rsd;
    nu[j] = r;
    ms += r * r;
  }
  ms = block_sum(ms, red) / Ck;
  const double inv = 1.0 / sqrt(ms + 1e-12);
  __syncthreads();
  for (int j = tid; j < Ck; j += blockDim.x) nu[j] *= inv;
}

// J arrays start at the objective constant; the stop marker starts at the iteration limit.
__global__ void km_reset_kernel(Layout L, int which, int iters) {
  pdl_entry();
  const int bh = blockIdx.x;
  double* J = (which == 0 ? L.kJ : L.qJ) + (size_t)bh * L.iters_cap;
  const double c = which == 0 ? L.T0k[bh] : L.T0q[bh];
  for (int i = threadIdx.x; i < L.iters_cap; i += blockDim.x) J[i] = c;
  if (threadIdx.x == 0) {
    L.stop_at[bh * 2 + which] = iters;
    (which == 0 ? L.krefined : L.qrefined)[bh] = 0;
  }
}

// ------------------------------------------------------------------------------------------
// Lloyd step 1 of iteration `it`: centroid update from the sums of assignment it-1, the stop
// test, then the score weights of the next assignment.  Grid (BH, C), one block per group.
//   keys:    c_j (key space), W_j = M c_j, bias_j = c_j^T M c_j
//   queries: nu_g (response space), W_g = nu_g, bias_g = ||nu_g||^2
// ------------------------------------------------------------------------------------------
constexpr int kPrepGroups = 8;  // groups per block of the centroid-update kernels

// Sums of kPrepGroups values per thread over the block (128 threads): out[g] for g < n.
__device__ __forceinline__ void block_sums8(const double (&v)[kPrepGroups], double* red /*[8][4]*/, double* out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int g = 0; g < kPrepGroups; ++g) {
    const double x = warp_sum(v[g]);
    if (lane == 0) red[g * 4 + warp] = x;
  }
  __syncthreads();
  if (threadIdx.x < kPrepGroups) {
    const double* r = red + threadIdx.x * 4;
    out[threadIdx.x] = (r[0] + r[1]) + (r[2] + r[3]);
  }
  __syncthreads();
}

constexpr int kPrepRows = 32;  // rows of M or C staged in shared memory at a time (fp64): 32 rows keep
                               // a block at 32 KB at d = 128, so several blocks share an SM and their
                               // staging overlaps (128 rows held one block per SM)

// Rows [r0, r0 + nr) of a row-major fp64 matrix with `cols` (even) columns into shared memory
// by 16-byte asynchronous copies, all issued before one wait (many in flight).  Both addresses
// are 16-byte aligned: workspace regions are 256-byte aligned and rows hold an even count of
// doubles.  The caller synchronises the block afterwards.
__device__ __forceinline__ void stage_rows(double* dst, const double* __restrict__ src, int r0, int nr, int cols) {
  const int n16 = nr * cols / 2;
  const double* s = src + (size_t)r0 * cols;
  for (int e = threadIdx.x; e < n16; e += blockDim.x)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst + 2 * e)),
                 "l"(s + 2 * e)
                 : "memory");
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Keys, kPrepGroups groups per block (grid BH x ceil(C_k / 8), thread a = dimension):
// c_j <- sum_j / n_j (groups that received points), the stop test, then W_j = M c_j (M staged in
// shared memory, symmetric: thread a reads column a), bias_j = c_j^T W_j, ||W_j||, and the sums
// zeroed for a pass over every point: always before the first assignment, and before each one
// when `keep` is 0 (the CUDA-core path sums every point each iteration; the tensor-core path
// only moves the sums by label changes after the first).  Dynamic shared memory:
// min(d, kPrepRows) rows of M.
__global__ void __launch_bounds__(128) kprep_kernel(Layout L, int it, int iters, int keep) {
  pdl_entry();
  extern __shared__ double Ms[];
  __shared__ double c[kPrepGroups][128];
  __shared__ double red[kPrepGroups * 4], bias_s[kPrepGroups], wn_s[kPrepGroups];
  const int bh = blockIdx.x, j0 = blockIdx.y * kPrepGroups, a = threadIdx.x, d = L.d;
  if (it > L.stop_at[bh * 2 + 0]) return;
  const int ng = min(kPrepGroups, L.Ck - j0);
  const size_t g0 = (size_t)bh * L.Ck + j0;
  for (int g = 0; g < ng; ++g) {
    double* cj = L.kcent + (g0 + g) * d;
    if (it > 0) {
      const int cnt = L.kcount[g0 + g];
      if (cnt > 0 && a < d) cj[a] = L.ksum[(g0 + g) * d + a] / (double)cnt;
    }
    if (a < d) c[g][a] = cj[a];
  }
  if (km_should_stop(L.kJ + (size_t)bh * L.iters_cap, it, iters, L.km_tol)) {
    if (a == 0 && blockIdx.y == 0) L.stop_at[bh * 2 + 0] = it;
    return;
  }
  double w[kPrepGroups];
#pragma unroll
  for (int g = 0; g < kPrepGroups; ++g) w[g] = 0.0;
  const double* M = L.M + (size_t)bh * d * d;
  for (int b0 = 0; b0 < d; b0 += kPrepRows) {
    const int nb = min(kPrepRows, d - b0);
    __syncthreads();
    stage_rows(Ms, M, b0, nb, d);
    __syncthreads();
    if (a < d)
      for (int bb = 0; bb < nb; ++bb) {
        const double m = Ms[bb * d + a];  // M[b][a] = M[a][b]
#pragma unroll
        for (int g = 0; g < kPrepGroups; ++g) w[g] += m * c[g][b0 + bb];
      }
  }
  double cb[kPrepGroups], wn[kPrepGroups];
#pragma unroll
  for (int g = 0; g < kPrepGroups; ++g) {
    const bool on = a < d && g < ng;
    cb[g] = on ? c[g][a] * w[g] : 0.0;
    wn[g] = on ? w[g] * w[g] : 0.0;
    if (on) {
      const size_t gj = g0 + g;
      L.kW64[gj * d + a] = w[g];
      L.kW32[gj * d + a] = (float)w[g];
      if (!keep || it == 0) L.ksum[gj * d + a] = 0.0;
      split3(w[g], L.kWb, (size_t)L.BH * L.Ckp * d, ((size_t)bh * L.Ckp + j0 + g) * d + a);
    }
  }
  block_sums8(cb, red, bias_s);
  block_sums8(wn, red, wn_s);
  if (a < ng) {
    const size_t gj = g0 + a;
    L.kbias64[gj] = bias_s[a];
    L.kbias32[gj] = (float)bias_s[a];
    if (!keep || it == 0) L.kcount[gj] = 0;
    L.kwnorm[gj] = (float)sqrt(wn_s[a]);
  }
}

// Queries, kPrepGroups groups per block (grid BH x ceil(C_q / 8)):
// nu_g <- C S_g / (sqrt(d) n_g) (the mean normalised response of the members), the stop test,
// then u_g = C^T nu_g / sqrt(d), bias ||nu_g||^2, ||u_g||, and the sums zeroed as in
// kprep_kernel.  The key-group centroids C are staged in shared memory kPrepRows rows at a time.
// Dynamic shared memory: kPrepGroups * C_k doubles (nu of the block's groups), then
// min(C_k, kPrepRows) rows of C.
__global__ void __launch_bounds__(128) qprep_kernel(Layout L, int it, int iters, int keep) {
  pdl_entry();
  extern __shared__ double qsm[];
  __shared__ double Sv[kPrepGroups][128];
  __shared__ double red[kPrepGroups * 4], nn_s[kPrepGroups], un_s[kPrepGroups];
  __shared__ int cnt_s[kPrepGroups];
  const int bh = blockIdx.x, g0i = blockIdx.y * kPrepGroups, d = L.d, Ck = L.Ck, tid = threadIdx.x;
  if (it > L.stop_at[bh * 2 + 1]) return;
  double* nus = qsm;                             // [kPrepGroups][Ck]
  double* Cs = qsm + (size_t)kPrepGroups * Ck;   // [kPrepRows][d]
  const int ng = min(kPrepGroups, L.Cq - g0i);
  const size_t g0 = (size_t)bh * L.Cq + g0i;
  const double* C = L.kcent + (size_t)bh * Ck * d;
  const double rsd = 1.0 / sqrt((double)d);
  if (tid < kPrepGroups) cnt_s[tid] = (it > 0 && tid < ng) ? L.qcount[g0 + tid] : 0;
  __syncthreads();
  if (L.semantic) {  // raw queries: u_g = c_g = S_g / n_g (groups that received points), bias ||c_g||^2
    if (it > 0 && tid < d)
      for (int g = 0; g < ng; ++g)
        if (cnt_s[g] > 0) L.qU64[(g0 + g) * d + tid] = L.qsum[(g0 + g) * d + tid] / (double)cnt_s[g];
    if (km_should_stop(L.qJ + (size_t)bh * L.iters_cap, it, iters, L.km_tol)) {
      if (tid == 0 && blockIdx.y == 0) L.stop_at[bh * 2 + 1] = it;
      return;
    }
    double cc[kPrepGroups];
#pragma unroll
    for (int g = 0; g < kPrepGroups; ++g) {
      const bool on = tid < d && g < ng;
      const double u = on ? L.qU64[(g0 + g) * d + tid] : 0.0;
      cc[g] = u * u;
      if (on) {
        const size_t gg = g0 + g;
        L.qU32[gg * d + tid] = (float)u;
        split3(u, L.qWb, (size_t)L.BH * L.Cqp * d, ((size_t)bh * L.Cqp + g0i + g) * d + tid);
        if (!keep || it == 0) L.qsum[gg * d + tid] = 0.0;
      }
    }
    block_sums8(cc, red, nn_s);
    if (tid < ng) {
      const size_t gg = g0 + tid;
      L.qbias64[gg] = nn_s[tid];
      L.qbias32[gg] = (float)nn_s[tid];
      if (!keep || it == 0) L.qcount[gg] = 0;
      L.qwnorm[gg] = (float)sqrt(nn_s[tid]);
    }
    return;
  }
  if (it > 0) {  // nu_g = C S_g / (sqrt(d) n_g) for the groups that received points
#pragma unroll
    for (int g = 0; g < kPrepGroups; ++g)
      if (tid < d) Sv[g][tid] = cnt_s[g] > 0 ? L.qsum[(g0 + g) * d + tid] / (double)cnt_s[g] : 0.0;
    for (int jc = 0; jc < Ck; jc += kPrepRows) {
      const int nj = min(kPrepRows, Ck - jc);
      __syncthreads();
      stage_rows(Cs, C, jc, nj, d);
      __syncthreads();
      for (int jj = tid; jj < nj; jj += blockDim.x) {
        double acc[kPrepGroups];
#pragma unroll
        for (int g = 0; g < kPrepGroups; ++g) acc[g] = 0.0;
        const double* cj = Cs + (size_t)jj * d;
        int aa = jj % d;  // rotated start: the lanes of a warp read different banks
        for (int a = 0; a < d; ++a) {
          const double x = cj[aa];
#pragma unroll
          for (int g = 0; g < kPrepGroups; ++g) acc[g] += x * Sv[g][aa];
          aa = aa + 1 == d ? 0 : aa + 1;
        }
#pragma unroll
        for (int g = 0; g < kPrepGroups; ++g)
          if (g < ng && cnt_s[g] > 0) L.qcent[(g0 + g) * Ck + jc + jj] = acc[g] * rsd;
      }
    }
  }
  if (km_should_stop(L.qJ + (size_t)bh * L.iters_cap, it, iters, L.km_tol)) {
    if (tid == 0 && blockIdx.y == 0) L.stop_at[bh * 2 + 1] = it;
    return;
  }
  __syncthreads();
  double nn[kPrepGroups];
#pragma unroll
  for (int g = 0; g < kPrepGroups; ++g) nn[g] = 0.0;
  for (int j = tid; j < Ck; j += blockDim.x)
#pragma unroll
    for (int g = 0; g < kPrepGroups; ++g) {
      const double v = g < ng ? L.qcent[(g0 + g) * Ck + j] : 0.0;
      nus[g * Ck + j] = v;
      nn[g] += v * v;
    }
  block_sums8(nn, red, nn_s);  // (its barriers also publish nus)
  // u_g = C^T nu_g / sqrt(d): thread = dimension, rows of C from shared memory
  double uu[kPrepGroups], un[kPrepGroups];
#pragma unroll
  for (int g = 0; g < kPrepGroups; ++g) uu[g] = 0.0;
  for (int jc = 0; jc < Ck; jc += kPrepRows) {
    const int nj = min(kPrepRows, Ck - jc);
    __syncthreads();
    stage_rows(Cs, C, jc, nj, d);
    __syncthreads();
    if (tid < d)
      for (int jj = 0; jj < nj; ++jj) {
        const double x = Cs[(size_t)jj * d + tid];
#pragma unroll
        for (int g = 0; g < kPrepGroups; ++g) uu[g] += x * nus[g * Ck + jc + jj];
      }
  }
#pragma unroll
  for (int g = 0; g < kPrepGroups; ++g) {
    const bool on = tid < d && g < ng;
    const double u = uu[g] * rsd;
    un[g] = on ? u * u : 0.0;
    if (on) {
      const size_t gg = g0 + g;
      L.qU64[gg * d + tid] = u;
      L.qU32[gg * d + tid] = (float)u;
      split3(u, L.qWb, (size_t)L.BH * L.Cqp * d, ((size_t)bh * L.Cqp + g0i + g) * d + tid);
      if (!keep || it == 0) L.qsum[gg * d + tid] = 0.0;
    }
  }
  block_sums8(un, red, un_s);
  if (tid < ng) {
    const size_t gg = g0 + tid;
    L.qbias64[gg] = nn_s[tid];
    L.qbias32[gg] = (float)nn_s[tid];
    if (!keep || it == 0) L.qcount[gg] = 0;
    L.qwnorm[gg] = (float)sqrt(un_s[tid]);
  }
}

// ------------------------------------------------------------------------------------------
// Lloyd step 2 on CUDA cores (fp32 inputs, or more groups than the tensor-core kernel holds):
// 128 points per block against all groups, register tile 8 points x 4 groups per thread
// (pg = tid / 16, cg = tid % 16), groups in chunks of 64.  Feature rows are the inputs
// themselves (keys, or queries scaled by 1/rms_q in the score); every bf16/fp32 input is exact
// in fp32 and fp64.  A point whose two best fp32 scores are within the rounding bound is
// re-decided over all groups in fp64.
// ------------------------------------------------------------------------------------------
struct KeyFeat {};
struct QueryFeat {};

constexpr int kAsgPts = 128;
constexpr int kAsgChunk = 64;

inline size_t assign_smem_bytes(int D) {
  return (size_t)(kAsgPts + kAsgChunk) * (D + 1) * 4 + kAsgChunk * 4 + kAsgPts * 4 /*scale*/ +
         3 * kAsgPts * 4 /*lab, order, refine*/ + kAsgPts * 8 /*score*/ + 8 * 128 * 8 /*fp64 rows*/;
}

template <typename T, typename Feat>
__global__ void __launch_bounds__(256) kmeans_assign_kernel(Layout L, const T* __restrict__ X, int it) {
  pdl_entry();
  constexpr bool kKeys = std::is_same<Feat, KeyFeat>::value;
  const int bh = blockIdx.y;
  const int which = kKeys ? 0 : 1;
  if (it >= L.stop_at[bh * 2 + which]) return;
  const int D = L.d;
  const int C = kKeys ? L.Ck : L.Cq;
  const int DP = D + 1;
  const int p0 = blockIdx.x * kAsgPts;
  const int np = min(kAsgPts, L.N - p0);
  if (np <= 0) return;

  const float* W32 = (kKeys ? L.kW32 : L.qU32) + (size_t)bh * C * D;
  const float* B32 = (kKeys ? L.kbias32 : L.qbias32) + (size_t)bh * C;
  const double* W64 = (kKeys ? L.kW64 : L.qU64) + (size_t)bh * C * D;
  const double* B64 = (kKeys ? L.kbias64 : L.qbias64) + (size_t)bh * C;
  const float* WN = (kKeys ? L.kwnorm : L.qwnorm) + (size_t)bh * C;

  extern __shared__ float smem[];
  float* Xs = smem;                          // [128][DP]
  float* Ws = Xs + kAsgPts * DP;             // [64][DP]
  float* Bs = Ws + kAsgChunk * DP;           // [64]
  float* scl = Bs + kAsgChunk;               // [128] per-point score scale
  int* lab = (int*)(scl + kAsgPts);          // [128]
  int* order = lab + kAsgPts;                // [128]
  int* refine = order + kAsgPts;             // [128]
  double* bval = (double*)(refine + kAsgPts);  // [128]
  double* xs64 = bval + kAsgPts;             // [8 warps][128]
  __shared__ float s_red[2][8];
  __shared__ double red[8];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  {
    const int p = tid >> 1, h = tid & 1;
    const size_t row = (size_t)bh * L.N + p0 + p;
    for (int a = h; a < D; a += 2) Xs[p * DP + a] = p < np ? to_f32(X[row * D + a]) : 0.f;
  }
  if (tid < kAsgPts) scl[tid] = kKeys ? 1.f : (tid < np ? L.inv_rms[(size_t)bh * L.N + p0 + tid] : 0.f);
  {
    float wm = 0.f, bm = 0.f;
    for (int j = tid; j < C; j += 256) {
      wm = fmaxf(wm, WN[j]);
      bm = fmaxf(bm, fabsf(B32[j]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      wm = fmaxf(wm, __shfl_xor_sync(0xffffffffu, wm, o));
      bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
    }
    if (lane == 0) {
      s_red[0][warp] = wm;
      s_red[1][warp] = bm;
    }
  }
  __syncthreads();
  float s_wmax = 0.f, s_bmax = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    s_wmax = fmaxf(s_wmax, s_red[0][w]);
    s_bmax = fmaxf(s_bmax, s_red[1][w]);
  }

  const int pg = tid >> 4, cg = tid & 15;
  float b1[8], b2[8];
  int i1[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    b1[r] = INFINITY;
    b2[r] = INFINITY;
    i1[r] = 0x7fffffff;
  }
  for (int c0 = 0; c0 < C; c0 += kAsgChunk) {
    const int nc = min(kAsgChunk, C - c0);
    __syncthreads();
    {
      const int j = tid >> 2, q = tid & 3;
      for (int a = q; a < D; a += 4) Ws[j * DP + a] = j < nc ? W32[(size_t)(c0 + j) * D + a] : 0.f;
      if (tid < kAsgChunk) Bs[tid] = tid < nc ? B32[c0 + tid] : 0.f;
    }
    __syncthreads();
    float acc[8][4];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[r][i] = 0.f;
#pragma unroll 2
    for (int a = 0; a < D; ++a) {
      float x[8], w[4];
#pragma unroll
      for (int r = 0; r < 8; ++r) x[r] = Xs[(pg + 16 * r) * DP + a];
#pragma unroll
      for (int i = 0; i < 4; ++i) w[i] = Ws[(cg + 16 * i) * DP + a];
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[r][i] = fmaf(x[r], w[i], acc[r][i]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int j = cg + 16 * i;
      if (j >= nc) continue;
      const int gj = c0 + j;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const float sc = Bs[j] - 2.f * acc[r][i] * scl[pg + 16 * r];
        if (sc < b1[r] || (sc == b1[r] && gj < i1[r])) {
          b2[r] = b1[r];
          b1[r] = sc;
          i1[r] = gj;
        } else if (sc < b2[r]) {
          b2[r] = sc;
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < 8; ++r) {
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) {
      const float ob1 = __shfl_xor_sync(0xffffffffu, b1[r], o);
      const float ob2 = __shfl_xor_sync(0xffffffffu, b2[r], o);
      const int oi1 = __shfl_xor_sync(0xffffffffu, i1[r], o);
      if (ob1 < b1[r] || (ob1 == b1[r] && oi1 < i1[r])) {
        b2[r] = fminf(b1[r], ob2);
        b1[r] = ob1;
        i1[r] = oi1;
      } else {
        b2[r] = fminf(b2[r], ob1);
      }
    }
  }
  const float u = 5.9604645e-8f;  // 2^-24
  if (cg == 0) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int p = pg + 16 * r;
      const size_t row = (size_t)bh * L.N + p0 + p;
      const float xn = p < np ? (kKeys ? L.knorm[row] : L.qxnorm[row]) : 0.f;
      // |error of b - 2 s x.w| <= 2 (D+2) u ||x|| s ||w|| + u |b| (+ the scale's rounding); x4 margin
      const float delta = 4.f * (D + 4) * u * xn * s_wmax + 2.f * u * s_bmax;
      lab[p] = (i1[r] >= 0 && i1[r] < C) ? i1[r] : 0;  // non-finite scores never yield a bad label
      bval[p] = (double)b1[r];
      refine[p] = (p < np) && !(b2[r] - b1[r] > 2.f * delta);
    }
  }
  __syncthreads();
  for (int p = warp; p < np; p += 8) {
    if (!refine[p]) continue;
    double* xs = xs64 + warp * 128;
    for (int a = lane; a < D; a += 32) xs[a] = (double)Xs[p * DP + a];
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
  int* labels = (kKeys ? L.klabel : L.qlabel) + (size_t)bh * L.N;
  if (tid < np) labels[p0 + tid] = lab[tid];
  const double jsum = block_sum(tid < np ? bval[tid] : 0.0, red);
  const int nref = __syncthreads_count(tid < np ? refine[tid] : 0);
  if (tid == 0) {
    atomicAdd((kKeys ? L.kJ : L.qJ) + (size_t)bh * L.iters_cap + it, jsum);
    if (nref) atomicAdd((kKeys ? L.krefined : L.qrefined) + bh, nref);
  }
  if (tid < np) {
    const int l = lab[tid];
    int rk = 0;
    for (int q = 0; q < np; ++q) {
      const int lq = lab[q];
      rk += (lq < l) || (lq == l && q < tid);
    }
    order[rk] = tid;
  }
  __syncthreads();
  // group sums (fp64): keys x, queries x / rms with the fp64 scale
  double* sums = (kKeys ? L.ksum : L.qsum) + (size_t)bh * C * D;
  int* counts = (kKeys ? L.kcount : L.qcount) + (size_t)bh * C;
  const int nparts = 256 / D;
  if (tid < nparts * D) {
    const int a = tid % D, part = tid / D;
    const int q0 = part * np / nparts, q1 = (part + 1) * np / nparts;
    double acc = 0.0;
    for (int q = q0; q < q1; ++q) {
      const int p = order[q];
      acc += (double)Xs[p * DP + a] * (kKeys ? 1.0 : L.inv_rms64[(size_t)bh * L.N + p0 + p]);
      if (q == q1 - 1 || lab[order[q + 1]] != lab[p]) {
        atomicAdd(sums + (size_t)lab[p] * D + a, acc);
        acc = 0.0;
      }
    }
  }
  if (tid < np && (tid == 0 || lab[order[tid - 1]] != lab[order[tid]])) {
    const int l = lab[order[tid]];
    int q = tid + 1;
    while (q < np && lab[order[q]] == l) ++q;
    atomicAdd(counts + l, q - tid);
  }
}

// ------------------------------------------------------------------------------------------
// a6 prologue: stable counting sort of the labels, in parallel over chunks of kSortChunk
// tokens.  Members of a group keep ascending token order.  perm[pos] = token,
// inv[token] = pos, off = group starts.
//   1. group_hist_kernel    per (chunk, head, side): label histogram of the chunk
//   2. group_scan_kernel    per (head, side): group starts, and each chunk's start inside every
//                           group (chunks in token order), in place of the histogram
//   3. group_scatter_kernel per (chunk, head, side): one warp places the chunk's tokens in
//                           token order from those starts
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ int* sort_hist(const Layout& L, int bh, int side, int chunk) {
  const int nch = (L.N + kSortChunk - 1) / kSortChunk, Cm = max(L.Ck, L.Cq);
  return L.sort_hist + (((size_t)bh * 2 + side) * nch + chunk) * Cm;
}

__global__ void __launch_bounds__(256) group_hist_kernel(Layout L) {
  pdl_entry();
  __shared__ int h[kMaxGroups];
  const int chunk = blockIdx.x, bh = blockIdx.y, side = blockIdx.z, tid = threadIdx.x, lane = tid & 31;
  const int C = side == 0 ? L.Ck : L.Cq;
  const int* labels = (side == 0 ? L.klabel : L.qlabel) + (size_t)bh * L.N;
  for (int c = tid; c < C; c += blockDim.x) h[c] = 0;
  __syncthreads();
  const int t_lo = chunk * kSortChunk, t_hi = min(L.N, t_lo + kSortChunk);
  for (int t0 = t_lo; t0 < t_hi; t0 += blockDim.x) {
    const int t = t0 + tid;
    const unsigned act = __ballot_sync(0xffffffffu, t < t_hi);
    if (t < t_hi) {
      const int l = labels[t];
      const unsigned same = __match_any_sync(act, l);
      if (lane == __ffs(same) - 1) atomicAdd(&h[l], __popc(same));
    }
  }
  __syncthreads();
  int* out = sort_hist(L, bh, side, chunk);
  for (int c = tid; c < C; c += blockDim.x) out[c] = h[c];
}

__global__ void __launch_bounds__(1024) group_scan_kernel(Layout L) {
  pdl_entry();
  __shared__ int wsum[32];
  const int bh = blockIdx.x, side = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int C = side == 0 ? L.Ck : L.Cq;
  const int nch = (L.N + kSortChunk - 1) / kSortChunk;
  int* off = (side == 0 ? L.koff : L.qoff) + (size_t)bh * (C + 1);
  // totals per group (thread g walks the chunks)
  int v = 0;
  if (tid < C)
    for (int ch = 0; ch < nch; ++ch) v += sort_hist(L, bh, side, ch)[tid];
  // exclusive scan over the groups (C <= 1024 = blockDim)
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    wsum[lane] = w;
  }
  __syncthreads();
  const int excl = x - v + (warp > 0 ? wsum[warp - 1] : 0);
  if (tid < C) {
    off[tid] = excl;
    int run = excl;  // each chunk's start inside group tid, chunks in token order
    for (int ch = 0; ch < nch; ++ch) {
      int* hc = sort_hist(L, bh, side, ch);
      const int n = hc[tid];
      hc[tid] = run;
      run += n;
    }
  }
  if (tid == 0) off[C] = L.N;
}

__global__ void __launch_bounds__(32) group_scatter_kernel(Layout L) {
  pdl_entry();
  __shared__ int cursor[kMaxGroups];
  __shared__ int lab[kSortChunk];
  const int chunk = blockIdx.x, bh = blockIdx.y, side = blockIdx.z, lane = threadIdx.x;
  const int C = side == 0 ? L.Ck : L.Cq;
  const int* labels = (side == 0 ? L.klabel : L.qlabel) + (size_t)bh * L.N;
  int* perm = (side == 0 ? L.kperm : L.qperm) + (size_t)bh * L.N;
  int* inv = (side == 0 ? L.kinv : L.qinv) + (size_t)bh * L.N;
  const int* start = sort_hist(L, bh, side, chunk);
  for (int c = lane; c < C; c += 32) cursor[c] = start[c];
  const int t_lo = chunk * kSortChunk, t_hi = min(L.N, t_lo + kSortChunk);
#pragma unroll 8
  for (int t = t_lo + lane; t < t_hi; t += 32) lab[t - t_lo] = labels[t];  // loads in flight together
  __syncwarp();
  const unsigned lt = (1u << lane) - 1u;
  for (int base = t_lo; base < t_hi; base += 32) {
    const int t = base + lane;
    const bool valid = t < t_hi;
    const int l = valid ? lab[t - t_lo] : -1;
    const unsigned m = __match_any_sync(0xffffffffu, l);
    const int pos = valid ? cursor[l] + __popc(m & lt) : 0;
    __syncwarp();
    if (valid && (m & lt) == 0) cursor[l] += __popc(m);
    __syncwarp();
    if (valid) {
      perm[pos] = t;
      inv[t] = pos;
    }
  }
}

static void launch_group_sort(const Layout& L, cudaStream_t st) {
  const int nch = (L.N + kSortChunk - 1) / kSortChunk;
  launch(group_hist_kernel, dim3(nch, L.BH, 2), 256, 0, st, L);
  launch(group_scan_kernel, dim3(L.BH, 2), 1024, 0, st, L);
  launch(group_scatter_kernel, dim3(nch, L.BH, 2), 32, 0, st, L);
}

// ------------------------------------------------------------------------------------------
// a5: routing.  S[g,j] = (mean query of group g) . c_j / sqrt(d) + ln m_j over non-empty key
// groups, visited by score (ties: lower j).  fixed_k > 0 keeps the first fixed_k; otherwise
// the top one is kept and every later one iff it brings the running key count strictly
// closer to kappa = density*N - (s + C_k + P).
// ------------------------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) route_select_kernel(Layout L, const T* __restrict__ Q) {
  pdl_entry();
  __shared__ double qbar[128];
  __shared__ double qpart[4][128];
  __shared__ double S[kMaxGroups];
  __shared__ int ord[kMaxGroups];
  const int bh = blockIdx.x, g = blockIdx.y, d = L.d, Ck = L.Ck, tid = threadIdx.x;
  const int* qoff = L.qoff + (size_t)bh * (L.Cq + 1);
  const int* koff = L.koff + (size_t)bh * (Ck + 1);
  unsigned char* route = L.route + ((size_t)bh * L.Cq + g) * Ck;
  const int r0 = qoff[g], n = qoff[g + 1] - r0;
  for (int j = tid; j < Ck; j += blockDim.x) route[j] = 0;
  if (n == 0) return;
  {  // mean query of the group: thread (dimension, part) sums every parts-th member
    const int parts = blockDim.x / d, a = tid % d, part = tid / d;
    const int* perm = L.qperm + (size_t)bh * L.N + r0;
    const T* Qh = Q + (size_t)bh * L.N * d + a;
    double acc = 0.0;
    int i = part;
    for (; i + 3 * parts < n; i += 4 * parts) {
      const int t0 = perm[i], t1 = perm[i + parts], t2 = perm[i + 2 * parts], t3 = perm[i + 3 * parts];
      const float x0 = to_f32(Qh[(size_t)t0 * d]), x1 = to_f32(Qh[(size_t)t1 * d]);
      const float x2 = to_f32(Qh[(size_t)t2 * d]), x3 = to_f32(Qh[(size_t)t3 * d]);
      acc += (double)x0;
      acc += (double)x1;
      acc += (double)x2;
      acc += (double)x3;
    }
    for (; i < n; i += parts) acc += (double)to_f32(Qh[(size_t)perm[i] * d]);
    qpart[part][a] = acc;
    __syncthreads();
    if (tid < d) {
      double t = 0.0;
      for (int q = 0; q < parts; ++q) t += qpart[q][tid];
      qbar[tid] = t / (double)n;
    }
  }
  __syncthreads();
  const double rsd = 1.0 / sqrt((double)d);
  for (int j = tid; j < Ck; j += blockDim.x) {
    const int m = koff[j + 1] - koff[j];
    double v = -INFINITY;
    if (m > 0) {
      const double* c = L.kcent + ((size_t)bh * Ck + j) * d;
      double dot = 0.0;
      for (int a = 0; a < d; ++a) dot += qbar[a] * c[a];
      v = dot * rsd + log((double)m);
      // a non-finite input can make a score NaN; ranking it as -inf keeps the rank count below
      // a strict total order, so ord[] is a permutation and every index written from it is valid
      if (isnan(v)) v = -INFINITY;
    }
    S[j] = v;
  }
  __syncthreads();
  for (int j = tid; j < Ck; j += blockDim.x) {
    if (koff[j + 1] - koff[j] == 0) continue;
    const double sj = S[j];
    int rk = 0;
    for (int i = 0; i < Ck; ++i) {
      if (koff[i + 1] - koff[i] == 0) continue;
      rk += (S[i] > sj) || (S[i] == sj && i < j);
    }
    ord[rk] = j;
  }
  __syncthreads();
  if (tid == 0) {
    int nne = 0;
    for (int j = 0; j < Ck; ++j) nne += koff[j + 1] - koff[j] > 0;
    if (L.fixed_k > 0) {
      for (int r = 0; r < min(L.fixed_k, nne); ++r) route[ord[r]] = 1;
    } else {
      const double kappa = (double)L.density * (double)L.N - (double)(L.s + Ck + L.P);
      double cum = 0.0;
      for (int r = 0; r < nne; ++r) {
        const int j = ord[r];
        const double m = (double)(koff[j + 1] - koff[j]);
        if (r == 0 || fabs((cum + m) - kappa) < fabs(cum - kappa)) {
          route[j] = 1;
          cum += m;
        }
      }
    }
  }
}

// Route lists (ascending key-group ids), visible keys per group, query-tile prefix and the
// realised density.  One block per head.
__global__ void __launch_bounds__(256) route_build_kernel(Layout L, int tile_m) {
  pdl_entry();
  __shared__ int tiles[kMaxGroups + 1];
  __shared__ long long pairs[kMaxGroups];
  const int bh = blockIdx.x, Ck = L.Ck, Cq = L.Cq;
  const int* koff = L.koff + (size_t)bh * (Ck + 1);
  const int* qoff = L.qoff + (size_t)bh * (Cq + 1);
  for (int g = threadIdx.x; g < Cq; g += blockDim.x) {
    const unsigned char* route = L.route + ((size_t)bh * Cq + g) * Ck;
    int* list = L.route_list + ((size_t)bh * Cq + g) * Ck;
    int cnt = 0, keys = 0;
    for (int j = 0; j < Ck; ++j)
      if (route[j]) {
        list[cnt++] = j;
        keys += koff[j + 1] - koff[j];
      }
    const int n = qoff[g + 1] - qoff[g];
    L.route_cnt[(size_t)bh * Cq + g] = cnt;
    L.route_keys[(size_t)bh * Cq + g] = keys;
    tiles[g] = (n + tile_m - 1) / tile_m;
    pairs[g] = (long long)n * keys;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int* toff = L.tile_off + (size_t)bh * (Cq + 1);
    int run = 0;
    long long tot = 0;
    for (int g = 0; g < Cq; ++g) {
      toff[g] = run;
      run += tiles[g];
      tot += pairs[g];
    }
    toff[Cq] = run;
    const double N = (double)L.N;
    L.stats[bh].sparse_pairs = tot;
    L.stats[bh].density = ((double)L.s * N + (double)Ck * N + (double)L.P * N + (double)tot) / (N * N);
  }
}

// ------------------------------------------------------------------------------------------
// Probe rows (Table 4).  Uniform spatiotemporal: rows floor((2i+1)N/(2P)), weight 1.
// Query-group stratified: m_g = floor(P n_g / N) plus one for the largest remainders
// (P n_g mod N, ties to the lower g); member floor((2i+1) n_g / (2 m_g)) of group g in token
// order; weight n_g / m_g scaled to sum P.  Output in ascending token order.
// ------------------------------------------------------------------------------------------
constexpr int kProbeTab = 4 * kMaxProbes;  // random mode: open-addressing table of the swapped slots
constexpr size_t kProbeSmem = kMaxProbes * (sizeof(double) + sizeof(int)) + kMaxGroups * sizeof(long long) +
                              (2 * kMaxGroups + 1) * sizeof(int) + 2 * kProbeTab * sizeof(int);

__global__ void __launch_bounds__(1024) probe_select_kernel(Layout L) {
  pdl_entry();
  extern __shared__ double shp[];
  double* cw = shp;                                  // [kMaxProbes]
  long long* rem = (long long*)(cw + kMaxProbes);    // [kMaxGroups]
  int* ctok = (int*)(rem + kMaxGroups);              // [kMaxProbes]
  int* mg = ctok + kMaxProbes;                       // [kMaxGroups]
  int* slot = mg + kMaxGroups;                       // [kMaxGroups + 1]
  __shared__ double s_sum;
  const int bh = blockIdx.x, P = L.P, Cq = L.Cq, N = L.N, tid = threadIdx.x;
  int* pof = L.probe_of + (size_t)bh * N;
  for (int t = tid; t < N; t += blockDim.x) pof[t] = -1;
  if (P == 0) return;
  if (L.probe_mode == SPARSEPR_PROBE_UNIFORM) {
    for (int i = tid; i < P; i += blockDim.x) {
      ctok[i] = (int)(((2LL * i + 1) * N) / (2LL * P));
      cw[i] = 1.0;
    }
    if (tid == 0) s_sum = (double)P;
  } else if (L.probe_mode == SPARSEPR_PROBE_RANDOM) {
    // P distinct rows: partial Fisher-Yates over [0, N) driven by SplitMix64 on the head's
    // probe stream (seed + 2^63 + 2 bh); the few slots a draw touches (at most 2P) live in an
    // open-addressing table (load <= 1/2)
    int* hk = slot + kMaxGroups + 1;  // [kProbeTab] slot index, -1 = empty
    int* hv = hk + kProbeTab;         // [kProbeTab] value now in that slot
    for (int i = tid; i < kProbeTab; i += blockDim.x) hk[i] = -1;
    for (int i = tid; i < P; i += blockDim.x) cw[i] = 1.0;
    __syncthreads();
    if (tid == 0) {
      auto slot_ref = [&](int sl) -> int* {
        unsigned h = ((unsigned)sl * 2654435761u) >> 18;  // 14 bits: kProbeTab = 16384
        while (true) {
          if (hk[h] == sl) return &hv[h];
          if (hk[h] == -1) {
            hk[h] = sl;
            hv[h] = sl;
            return &hv[h];
          }
          h = (h + 1) & (kProbeTab - 1);
        }
      };
      uint64_t state = L.seed + (1ULL << 63) + 2ULL * (uint64_t)bh;
      const uint64_t n = (uint64_t)N;
      for (int i = 0; i < P; ++i) {
        const uint64_t r = splitmix64_next(state);
        const int j = i + (int)(r % (n - (uint64_t)i));
        int* pi = slot_ref(i);
        int* pj = slot_ref(j);
        const int vi = *pi, vj = *pj;
        *pi = vj;
        *pj = vi;
        ctok[i] = vj;
      }
      s_sum = (double)P;
    }
  } else {
    const int* qoff = L.qoff + (size_t)bh * (Cq + 1);
    const int* qperm = L.qperm + (size_t)bh * N;
    for (int g = tid; g < Cq; g += blockDim.x) {
      const long long n = qoff[g + 1] - qoff[g];
      mg[g] = (int)((P * n) / N);
      rem[g] = (P * n) % N;
    }
    __syncthreads();
    __shared__ int s_extra;
    if (tid == 0) {
      int tot = 0;
      for (int g = 0; g < Cq; ++g) tot += mg[g];
      s_extra = P - tot;
    }
    __syncthreads();
    for (int g = tid; g < Cq; g += blockDim.x) {
      int rk = 0;
      for (int h = 0; h < Cq; ++h) rk += (rem[h] > rem[g]) || (rem[h] == rem[g] && h < g);
      if (rk < s_extra) mg[g] += 1;  // each g is written by its own thread only
    }
    __syncthreads();
    if (tid == 0) {
      int run = 0;
      for (int g = 0; g < Cq; ++g) {
        slot[g] = run;
        run += mg[g];
      }
      slot[Cq] = run;
    }
    __syncthreads();
    for (int g = tid; g < Cq; g += blockDim.x) {
      const int n = qoff[g + 1] - qoff[g], m = mg[g];
      for (int i = 0; i < m; ++i) {
        ctok[slot[g] + i] = qperm[qoff[g] + (int)(((2LL * i + 1) * n) / (2LL * m))];
        cw[slot[g] + i] = (double)n / (double)m;
      }
    }
    __syncthreads();
    if (tid == 0) {
      double s = 0.0;
      for (int i = 0; i < P; ++i) s += cw[i];
      s_sum = s;
    }
  }
  __syncthreads();
  int* tok = L.probe_tok + (size_t)bh * P;
  double* w = L.probe_w + (size_t)bh * P;
  const double scale = (double)P / s_sum;
  for (int i = tid; i < P; i += blockDim.x) {
    const int t = ctok[i];
    int rk = 0;
    for (int k = 0; k < P; ++k) rk += ctok[k] < t;
    tok[rk] = t;
    w[rk] = cw[i] * scale;
    pof[t] = rk;
  }
}

// probe_of from an installed probe list (sparsepr_set_partition).
__global__ void probe_index_kernel(Layout L) {
  pdl_entry();
  const int bh = blockIdx.x;
  int* pof = L.probe_of + (size_t)bh * L.N;
  for (int t = threadIdx.x; t < L.N; t += blockDim.x) pof[t] = -1;
  __syncthreads();
  for (int i = threadIdx.x; i < L.P; i += blockDim.x) pof[L.probe_tok[(size_t)bh * L.P + i]] = i;
}

// Per-head k-means statistics after both loops.
__global__ void plan_stats_kernel(Layout L) {
  pdl_entry();
  const int bh = blockIdx.x * blockDim.x + threadIdx.x;
  if (bh >= L.BH) return;
  sparsepr_head_stats& st = L.stats[bh];
  const int ki = L.stop_at[bh * 2 + 0], qi = L.stop_at[bh * 2 + 1];
  st.k_iters = ki;
  st.q_iters = qi;
  st.k_refined = L.krefined[bh];
  st.q_refined = L.qrefined[bh];
  st.k_objective = ki > 0 ? L.kJ[(size_t)bh * L.iters_cap + ki - 1] : 0.0;
  st.q_objective = qi > 0 ? L.qJ[(size_t)bh * L.iters_cap + qi - 1] : 0.0;
}

// ------------------------------------------------------------------------------------------
// a6: gather rows into group-contiguous order (one warp per row, 16-byte chunks).
// ------------------------------------------------------------------------------------------
__global__ void permute_rows_kernel(Layout L, const void* __restrict__ src, void* __restrict__ dst,
                                    const int* __restrict__ perm, int rows_per_head, int src_rows_per_head) {
  pdl_entry();
  const int bh = blockIdx.y;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= rows_per_head) return;
  const size_t rb = (size_t)L.d * elt_size(L.dtype);
  const int chunks = (int)(rb / 16);
  const int t = perm[(size_t)bh * rows_per_head + warp];
  const uint4* s = (const uint4*)((const char*)src + ((size_t)bh * src_rows_per_head + t) * rb);
  uint4* o = (uint4*)((char*)dst + ((size_t)bh * rows_per_head + warp) * rb);
  for (int c = lane; c < chunks; c += 32) o[c] = s[c];
}

// Q by the query-group order, K and V by the key-group order, in one pass: thread = one
// 16-byte piece of a row of each (three independent loads in flight per piece).
__global__ void __launch_bounds__(256) permute_qkv_kernel(Layout L, const void* __restrict__ Q,
                                                          const void* __restrict__ K, const void* __restrict__ V) {
  pdl_entry();
  const int bh = blockIdx.y;
  const size_t rb = (size_t)L.d * elt_size(L.dtype);
  const int chunks = (int)(rb / 16);
  const long long total = (long long)L.N * chunks;
  const int* qp = L.qperm + (size_t)bh * L.N;
  const int* kp = L.kperm + (size_t)bh * L.N;
  const char* q = (const char*)Q + (size_t)bh * L.N * rb;
  const char* k = (const char*)K + (size_t)bh * L.N * rb;
  const char* v = (const char*)V + (size_t)bh * L.N * rb;
  char* qo = (char*)L.Qp + (size_t)bh * L.N * rb;
  char* ko = (char*)L.Kp + (size_t)bh * L.N * rb;
  char* vo = (char*)L.Vp + (size_t)bh * L.N * rb;
  for (long long p = (long long)blockIdx.x * blockDim.x + threadIdx.x; p < total; p += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(p / chunks), c = (int)(p % chunks);
    const size_t so = (size_t)c * 16, dofs = (size_t)r * rb + so;
    const int tq = qp[r], tk = kp[r];
    const uint4 a = *(const uint4*)(q + (size_t)tq * rb + so);
    const uint4 b = *(const uint4*)(k + (size_t)tk * rb + so);
    const uint4 e = *(const uint4*)(v + (size_t)tk * rb + so);
    *(uint4*)(qo + dofs) = a;
    *(uint4*)(ko + dofs) = b;
    *(uint4*)(vo + dofs) = e;
  }
}

// ------------------------------------------------------------------------------------------
// Host launchers.
// ------------------------------------------------------------------------------------------
template <typename T>
static sparsepr_status plan_typed(const Layout& L, const T* Q, const T* K, bool warm, int iters,
                                  cudaStream_t st, const KernelEvents& ev) {
  const int d = L.d;
  const bool tc = L.dtype == SPARSEPR_BF16;  // bf16 inputs: tensor-core quadratic forms
  const size_t dd = (size_t)L.BH * d * d;
  const int split_blocks = (int)((dd + 255) / 256 < 4096 ? (dd + 255) / 256 : 4096);
  const size_t qf_smem = (size_t)(d + 64) * (d + 1) * sizeof(float);
  cudaFuncSetAttribute(rowqf_simt_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)qf_smem);
  // keys: metric M = Qs^T Qs / d, objective constant sum_t k_t^T M k_t, key norms
  launch(metric_kernel<T>, dim3(L.BH, d / kMetricRows), 256, 0, st, L, Q);
  if (L.kgram) {  // key-response rank r_K: M <- M_r before anything uses M
    const sparsepr_status s = launch_key_rank(L, K, st);
    if (s != SPARSEPR_OK) return s;
  }
  cudaMemsetAsync(L.T0k, 0, sizeof(double) * L.BH, st);
  cudaMemsetAsync(L.T0q, 0, sizeof(double) * L.BH, st);
  if (tc) {
    launch(split_mat_kernel, split_blocks, 256, 0, st, (const double*)L.M, L.Mb, dd);
    const sparsepr_status s = launch_rowqf_tc(L, 0, K, st);
    if (s != SPARSEPR_OK) return s;
  } else {
    launch(rowqf_simt_kernel<T>, dim3((L.N + 63) / 64, L.BH), 256, qf_smem, st, L, K, 0);
  }
  if (!warm) {
    launch(km_draw_kernel, dim3(L.BH, 2), 128, 0, st, L);  // both sides' initial points
    launch(kcent_init_kernel<T>, dim3(L.BH, L.Ck), 128, 0, st, L, K);
  }
  SPR_LAUNCH_CHECK();
  launch(km_reset_kernel, L.BH, 128, 0, st, L, 0, iters);
  // bf16 inputs with at most 256 groups score on the tensor cores; otherwise on CUDA cores
  const bool tc_keys = km_tc_supported(L, true), tc_queries = km_tc_supported(L, false);
  const int Gk = tc_keys ? km_tc_grid(L, true) : 0, Gq = tc_queries ? km_tc_grid(L, false) : 0;
  cudaMemsetAsync(L.kWb, 0, (size_t)3 * L.BH * L.Ckp * d * 2, st);
  cudaMemsetAsync(L.qWb, 0, (size_t)3 * L.BH * L.Cqp * d * 2, st);
  const size_t asg_smem = assign_smem_bytes(d);
  const int nblk = (L.N + kAsgPts - 1) / kAsgPts;
  cudaFuncSetAttribute(kmeans_assign_kernel<T, KeyFeat>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)asg_smem);
  cudaFuncSetAttribute(kmeans_assign_kernel<T, QueryFeat>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)asg_smem);
  const size_t kprep_smem = (size_t)std::min(d, kPrepRows) * d * sizeof(double);
  cudaFuncSetAttribute(kprep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kprep_smem);
  if (km_loop_supported(L, true)) {  // mid-size calls: the whole loop in one launch
    const cudaEvent_t e0 = ev.start[SPARSEPR_KERNEL_KMEANS_LOOP], e1 = ev.stop[SPARSEPR_KERNEL_KMEANS_LOOP];
    if (e0) cudaEventRecord(e0, st);
    const sparsepr_status s = launch_kmeans_loop(L, true, K, iters, st);
    if (s != SPARSEPR_OK) return s;
    if (e1) cudaEventRecord(e1, st);
  } else {
    for (int it = 0; it <= iters; ++it) {
      launch(kprep_kernel, dim3(L.BH, (L.Ck + kPrepGroups - 1) / kPrepGroups), 128, kprep_smem, st, L, it, iters,
             tc_keys ? 1 : 0);
      if (it < iters) {
        if (tc_keys) {
          const sparsepr_status s = launch_kmeans_iteration_tc(L, true, K, it, Gk, st, it == 0 ? &ev : nullptr);
          if (s != SPARSEPR_OK) return s;
        } else {
          launch(kmeans_assign_kernel<T, KeyFeat>, dim3(nblk, L.BH), 256, asg_smem, st, L, K, it);
        }
      }
    }
  }
  SPR_LAUNCH_CHECK();
  // queries: Gc from the key-group centroids, 1/rms_q, ||r~_q||, objective constant
  launch(gc_kernel, dim3(L.BH, d), 128, 0, st, L);
  if (tc) {
    launch(split_mat_kernel, split_blocks, 256, 0, st, (const double*)L.Gc, L.Gcb, dd);
    const sparsepr_status s = launch_rowqf_tc(L, 1, Q, st);
    if (s != SPARSEPR_OK) return s;
  } else {
    launch(rowqf_simt_kernel<T>, dim3((L.N + 63) / 64, L.BH), 256, qf_smem, st, L, Q, 1);
  }
  if (!warm) {
    launch(qcent_init_kernel<T>, dim3(L.BH, L.Cq), 128, 0, st, L, Q);
  }
  launch(km_reset_kernel, L.BH, 128, 0, st, L, 1, iters);
  SPR_LAUNCH_CHECK();
  const size_t qprep_smem = ((size_t)kPrepGroups * L.Ck + (size_t)std::min(L.Ck, kPrepRows) * d) * sizeof(double);
  cudaFuncSetAttribute(qprep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)qprep_smem);
  if (km_loop_supported(L, false)) {
    const sparsepr_status s = launch_kmeans_loop(L, false, Q, iters, st);
    if (s != SPARSEPR_OK) return s;
  } else {
    for (int it = 0; it <= iters; ++it) {
      launch(qprep_kernel, dim3(L.BH, (L.Cq + kPrepGroups - 1) / kPrepGroups), 128, qprep_smem, st, L, it, iters,
             tc_queries ? 1 : 0);
      if (it < iters) {
        if (tc_queries) {
          const sparsepr_status s = launch_kmeans_iteration_tc(L, false, Q, it, Gq, st);
          if (s != SPARSEPR_OK) return s;
        } else {
          launch(kmeans_assign_kernel<T, QueryFeat>, dim3(nblk, L.BH), 256, asg_smem, st, L, Q, it);
        }
      }
    }
  }
  SPR_LAUNCH_CHECK();
  launch_group_sort(L, st);
  launch(route_select_kernel<T>, dim3(L.BH, L.Cq), 256, 0, st, L, Q);
  launch(route_build_kernel, L.BH, 256, 0, st, L, attn_tile_m(L));
  cudaFuncSetAttribute(probe_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kProbeSmem);
  launch(probe_select_kernel, L.BH, 1024, kProbeSmem, st, L);
  launch(plan_stats_kernel, (L.BH + 127) / 128, 128, 0, st, L);
  SPR_LAUNCH_CHECK();
  return SPARSEPR_OK;
}

sparsepr_status launch_plan(const Layout& L, const void* Q, const void* K, bool warm, int iters,
                            cudaStream_t st, const KernelEvents& ev) {
  if (L.dtype == SPARSEPR_F32) return plan_typed<float>(L, (const float*)Q, (const float*)K, warm, iters, st, ev);
  return plan_typed<__nv_bfloat16>(L, (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K, warm, iters, st, ev);
}

sparsepr_status launch_installed_partition(const Layout& L, cudaStream_t st) {
  launch_group_sort(L, st);
  launch(route_build_kernel, L.BH, 256, 0, st, L, attn_tile_m(L));
  launch(probe_index_kernel, L.BH, 1024, 0, st, L);
  SPR_LAUNCH_CHECK();
  return SPARSEPR_OK;
}

sparsepr_status launch_permute(const Layout& L, const void* Q, const void* K, const void* V,
                               cudaStream_t st) {
  {
    const long long pieces = (long long)L.N * (L.d * (long long)elt_size(L.dtype) / 16);
    const int gx = (int)std::min<long long>((pieces + 1023) / 1024, 65535);  // about four pieces per thread
    launch(permute_qkv_kernel, dim3(gx, L.BH), 256, 0, st, L, Q, K, V);
  }
  if (L.P > 0)
    launch(permute_rows_kernel, dim3((L.P * 32 + 255) / 256, L.BH), 256, 0, st, L, Q, L.Qprobe, L.probe_tok, L.P, L.N);
  SPR_LAUNCH_CHECK();
  return SPARSEPR_OK;
}

}  // namespace sparsepr
