// Shared definitions of the SparsePR CUDA library: the workspace layout every kernel receives
// by value, element conversions, warp reductions and launch checking.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <type_traits>
#include <utility>

#include "../../include/sparsepr.h"

namespace sparsepr {

constexpr int kMaxGroups = 1024;  // C_k, C_q upper bound (route rows fit one CTA's smem)
constexpr int kMaxProbes = 4096;
constexpr int kSortChunk = 4096;   // tokens per chunk of the parallel stable group sort
constexpr int kKmChunkGroups = 256;  // groups per launch of the tensor-core k-means assignment
constexpr int kGramChunk = 4096;     // keys per partial Gram of the key-response rank projection
constexpr int kKmLoopMaxCtas = 160;  // CTAs of one whole-loop k-means launch at most (>= the SMs)

// Device status word values (a subset of sparsepr_status).
constexpr int kDevOk = 0;
constexpr int kDevNumeric = SPARSEPR_ERR_NUMERIC;
constexpr int kDevTimeout = SPARSEPR_ERR_TIMEOUT;

// Everything a kernel needs to find its data: sizes and device pointers carved from the
// caller's workspace.  Arrays are head-major: head bh = b*H + h owns one contiguous slice.
struct Layout {
  int BH, H, N, d, s, Ck, Cq, P;
  int dtype;            // SPARSEPR_F32 / SPARSEPR_BF16 of Q, K, V
  int fixed_k;
  int iters_cap;        // length of the per-iteration objective arrays
  int probe_mode;
  float density;
  float km_tol;
  double lambda;
  uint64_t seed;
  int semantic;         // 1: k-means on the raw keys and queries (M = I, Gc = I, scale 1)
  int repair;           // 1: fit and add the probe-residual correction
  int correction;       // SPARSEPR_CORRECTION_AFFINE / _MEAN
  int trunc_rank;       // 0: whole residual span; r: its r leading eigenvectors
  long long attn_wait_limit;  // > 0: the attention kernel's bounded waits give up after this
                              // many cycles (test hook of the timeout path); 0: the default
  int key_rank;         // 0 < r < d: the key k-means metric restricted to the r leading
                        // directions of the key responses (r_K); else the full metric
  int km_steps;         // 1: k-means one launch per step of every iteration even where the
                        // whole loop fits one launch (test hook); 0: the faster path
  long long km_wait_limit;  // > 0: the whole-loop k-means head barriers give up after this many
                            // cycles (test hook of its timeout path); 0: the default

  // status + per-head statistics
  int* status;                    // [1]
  sparsepr_head_stats* stats;     // [BH]

  // key responses: metric M = Qs^T Qs / d and the objective constants
  double* M;                      // [BH, d, d]
  double* T0k;                    // [BH]  sum_t ||f_t||^2
  double* T0q;                    // [BH]  sum_q ||r~_q||^2

  // key-response rank projection (key_rank in (0, d)): partial and total K^T K, the factor of
  // M, the eigenvectors of L^T K^T K L and a product scratch
  double* kgram_part;             // [BH, ceil(N / kGramChunk), d, d]
  double* kgram;                  // [BH, d, d]
  double* kr_L;                   // [BH, d, d]
  double* kr_V;                   // [BH, d, d]
  double* kr_T;                   // [BH, d, d]

  // k-means shared scratch
  int* init_ids;                  // [BH, Ck + Cq] initial points: keys, then queries
  int* fy;                        // [BH, N] Fisher-Yates slots
  int* iters_run;                 // [BH, 2] iterations for keys / queries (run-time state)
  int* stop_at;                   // [BH, 2] iteration at which the loop stopped
  int* warm;                      // [1] 1 = warm start from stored centroids

  // key k-means (features: keys with metric M)
  double* kcent;                  // [BH, Ck, d]   key-space centroids
  double* kW64;                   // [BH, Ck, d]   M c_j
  float* kW32;                    // [BH, Ck, d]
  double* kbias64;                // [BH, Ck]      c_j^T M c_j
  float* kbias32;                 // [BH, Ck]
  float* kwnorm;                  // [BH, Ck]      ||W_j||_2
  double* ksum;                   // [BH, Ck, d]
  int* kcount;                    // [BH, Ck]
  int* klabel;                    // [BH, N]
  double* kJ;                     // [BH, iters_cap]
  int* krefined;                  // [BH]

  // query k-means.  The normalised responses are linear in the query,
  //   r~_q = C q / (sqrt(d) rms_q),   rms_q^2 = q^T Gc q + 1e-12,   Gc = C^T C / (d C_k),
  // (C = key-group centroids, rows c_j), so the iteration runs on the d-dim queries: the score
  // of group g is ||nu_g||^2 - 2 (q . u_g) / rms_q with u_g = C^T nu_g / sqrt(d), and the group
  // sums are sums of q / rms_q, projected back as nu_g = C S_g / (sqrt(d) n_g).
  double* Gc;                     // [BH, d, d]
  float* inv_rms;                 // [BH, N]   1 / rms_q (scores)
  double* inv_rms64;              // [BH, N]   1 / rms_q (group sums)
  float* qxnorm;                  // [BH, N]   ||q|| / rms_q  (= ||r~_q|| bound for the score error)
  double* qcent;                  // [BH, Cq, Ck] nu_g (response space)
  double* qU64;                   // [BH, Cq, d]  u_g
  float* qU32;                    // [BH, Cq, d]
  double* qbias64;                // [BH, Cq]     ||nu_g||^2
  float* qbias32;                 // [BH, Cq]
  float* qwnorm;                  // [BH, Cq]     ||u_g||_2
  double* qsum;                   // [BH, Cq, d]  sums of q / rms_q
  int* qcount;                    // [BH, Cq]
  int* qlabel;                    // [BH, N]
  double* qJ;                     // [BH, iters_cap]
  int* qrefined;                  // [BH]

  // bf16 operands of the tensor-core kernels: fp64 matrices split into three bf16 terms
  // (hi + mid + lo reproduces the value to ~2^-24 relative; the k-means assignment reads hi and
  // mid, the row quadratic forms all three); group rows padded to 16
  int Ckp, Cqp;
  __nv_bfloat16* kWb;             // [3][BH, Ckp, d]   W_j = M c_j
  __nv_bfloat16* qWb;             // [3][BH, Cqp, d]   u_g
  __nv_bfloat16* Mb;              // [3][BH, d, d]     M
  __nv_bfloat16* Gcb;             // [3][BH, d, d]     Gc
  float* knorm;                   // [BH, N] ||k_t||_2 (rounding bound of the key scores)
  // running best two scores of every point across the group chunks of one assignment (more
  // than kKmChunkGroups groups): {best bits, second bits, best group, 0}; null when unused
  int4* ktop;                     // [BH, N]
  int4* qtop;                     // [BH, N]
  // each point's label in the iteration before (the per-iteration update moves the group sums
  // by the points whose label changed)
  int* kprev;                     // [BH, N]
  int* qprev;                     // [BH, N]
  // whole-loop k-means (mid-size calls: every Lloyd iteration of a side in one launch, G CTAs
  // per head): each CTA's partial group sums, counts and objective, the head barrier counters
  // and the abort flag; null when no side qualifies
  int klp_G;                      // CTAs per head the partial arrays hold
  double* klp_sum;                // [BH, klp_G, max C, d]
  int* klp_cnt;                   // [BH, klp_G, max C]
  double* klp_J;                  // [BH, klp_G]
  unsigned* klp_bar;              // [BH + 1]: head counters, then the abort flag

  // points of the tensor-core assignment whose two best scores were within the rounding bound,
  // re-decided in fp64: CTA c of the assignment grid appends to its own segment starting at
  // (first tile of c) * 128 and leaves the segment length in rcnt[c].  Entry: x = row bh*N + p,
  // y = float bits of the tentative score, z = candidate count (bits 0..7; 255 = all groups) |
  // candidate 0 << 8 | candidate 1 << 18, w = candidate 2 | candidate 3 << 16 (candidates: the
  // groups whose fp32 score is within the bound of the best, ascending)
  int4* rlist;                    // [BH * ceil(N/128) * 128]
  int* rcnt;                      // [BH * ceil(N/128)]

  // group-contiguous order (stable counting sort)
  int* sort_hist;                 // [BH, 2, ceil(N / kSortChunk), max(Ck, Cq)] chunk histograms
  int* kperm;                     // [BH, N]   position -> token
  int* kinv;                      // [BH, N]   token -> position
  int* koff;                      // [BH, Ck+1]
  int* qperm;
  int* qinv;
  int* qoff;                      // [BH, Cq+1]

  // routing
  unsigned char* route;           // [BH, Cq, Ck]
  int* route_list;                // [BH, Cq, Ck]  kept key groups, ascending
  int* route_cnt;                 // [BH, Cq]
  int* route_keys;                // [BH, Cq]      keys visible to the group (sum of m_j)
  int* tile_off;                  // [BH, Cq+1]    prefix of query tiles per group

  // probes
  int* probe_tok;                 // [BH, P]
  double* probe_w;                // [BH, P]
  int* probe_of;                  // [BH, N]  token -> probe index or -1

  // permuted operands (input dtype) and outputs
  void* Qp;                       // [BH, N, d]
  void* Kp;
  void* Vp;
  void* Qprobe;                   // [BH, P, d]
  float* Osp;                     // [BH, N, d]  permuted (query-group) order
  float* Odense;                  // [BH, P, d]

  // ridge
  double* ridgeG;                 // [BH, d+1, d+1]
  double* ridgeB;                 // [BH, d+1, d]
  double* spanS;                  // [BH, d, d]   R^T W R
  double* A64;                    // [BH, d+1, d]
  float* A32;                     // [BH, d+1, d]
};

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide sum of a double; every thread gets the result.  `red` needs blockDim/32 doubles.
__device__ __forceinline__ double block_sum(double v, double* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  double t = 0.0;
  for (int i = 0; i < nw; ++i) t += red[i];
  return t;
}

__host__ __device__ inline size_t elt_size(int dtype) { return dtype == SPARSEPR_F32 ? 4 : 2; }

// Kernels launched by this library since it was loaded (read by sparsepr_launch_count).
extern std::atomic<long long> g_launches;

// Programmatic dependent launch.  Every kernel of the library starts with pdl_entry(): it waits
// until the kernels before it in the stream have completed and their memory is visible (the
// same ordering as a plain launch), then allows the next kernel's CTAs to be launched.  The
// launch work and CTA start of kernel n+1 so overlap the tail of kernel n.
__device__ __forceinline__ void pdl_entry() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Every kernel of the library is launched through this helper, which counts the launch and
// marks it as programmatically dependent on the previous kernel in the stream.
template <typename... KArgs, typename... Args>
inline void launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                   Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  g_launches.fetch_add(1, std::memory_order_relaxed);
}

}  // namespace sparsepr

#define SPR_LAUNCH_CHECK()                                   \
  do {                                                       \
    cudaError_t e_ = cudaGetLastError();                     \
    if (e_ != cudaSuccess) return SPARSEPR_ERR_CUDA;         \
  } while (0)
