// Host-side entry points of the kernel files, called by the C ABI in sparsepr_api.cu.
#pragma once

#include "common.cuh"

namespace sparsepr {

// Query rows per attention work item (the block-sparse pass tiles each query group by this):
// 64 for the fp32 CUDA-core kernel, 256 (two 128-row MMA tiles) for the bf16 tensor-core kernel.
constexpr int kAttnTileM = 64;
constexpr int kAttnTileMTc = 256;
inline int attn_tile_m(const Layout& L) { return L.dtype == SPARSEPR_BF16 ? kAttnTileMTc : kAttnTileM; }

// Optional events recorded around single launches (ids: SPARSEPR_KERNEL_*).
struct KernelEvents {
  static constexpr int kCount = 4;
  cudaEvent_t start[kCount] = {};
  cudaEvent_t stop[kCount] = {};
};

sparsepr_status launch_plan(const Layout& L, const void* Q, const void* K, bool warm, int iters,
                            cudaStream_t st, const KernelEvents& ev);
sparsepr_status launch_installed_partition(const Layout& L, cudaStream_t st);
sparsepr_status launch_permute(const Layout& L, const void* Q, const void* K, const void* V,
                               cudaStream_t st);
sparsepr_status launch_attention(const Layout& L, cudaStream_t st, cudaEvent_t ev_start, cudaEvent_t ev_stop);
sparsepr_status launch_attention_tc(const Layout& L, cudaStream_t st, cudaEvent_t ev_start, cudaEvent_t ev_stop);
sparsepr_status launch_fit_apply(const Layout& L, void* O, int out_dtype, cudaStream_t st);
// O = O_sp + [O_sp, 1] A on unprobed rows, O_dense on probe rows, in token order (tensor cores).
sparsepr_status launch_apply_tc(const Layout& L, void* O, int out_dtype, cudaStream_t st);
sparsepr_status launch_ridge_solve(const Layout& L, cudaStream_t st);
bool km_tc_supported(const Layout& L, bool keys);
int km_tc_grid(const Layout& L, bool keys);
// One Lloyd iteration after the centroid update: tensor-core assignment, then the fp64
// re-decisions, group sums and counts (both kernels over the same G tile ranges).
sparsepr_status launch_kmeans_iteration_tc(const Layout& L, bool keys, const void* X, int it, int G,
                                           cudaStream_t st, const KernelEvents* ev = nullptr);
// Whole-loop k-means (kmeans_loop.cu): CTAs per head and resident tiles per CTA when `ctas`
// CTAs can be co-resident, 0 when the side does not qualify; whether the plan's workspace and
// the device allow it; the launch (every Lloyd iteration of one side, the stop test included).
int km_loop_ctas_per_head(int BH, int N, int d, int dtype, int C, int Ck, bool keys, int ctas, int* cap_out);
bool km_loop_supported(const Layout& L, bool keys);
sparsepr_status launch_kmeans_loop(const Layout& L, bool keys, const void* X, int iters, cudaStream_t st);
sparsepr_status launch_rowqf_tc(const Layout& L, int which, const void* X, cudaStream_t st);
// M <- its rank-r_K restriction to the leading key-response directions (key_rank in (0, d)).
sparsepr_status launch_key_rank(const Layout& L, const void* K, cudaStream_t st);

// Upper bound of the number of query tiles of one head: sum_g ceil(n_g / tile) <= N/tile + C_q.
inline int max_query_tiles(const Layout& L, int tile) { return (L.N + tile - 1) / tile + L.Cq; }

}  // namespace sparsepr
