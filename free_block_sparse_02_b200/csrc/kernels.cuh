// Host-side entry points of the kernel files, called by the C ABI in sparsepr_api.cu.
#pragma once

#include "common.cuh"

namespace sparsepr {

// Query rows per attention work item (the block-sparse pass tiles each query group by this).
constexpr int kAttnTileM = 64;

sparsepr_status launch_plan(const Layout& L, const void* Q, const void* K, bool warm, int iters,
                            cudaStream_t st);
sparsepr_status launch_installed_partition(const Layout& L, cudaStream_t st);
sparsepr_status launch_permute(const Layout& L, const void* Q, const void* K, const void* V,
                               cudaStream_t st);
sparsepr_status launch_attention(const Layout& L, cudaStream_t st, cudaEvent_t ev_start, cudaEvent_t ev_stop);
sparsepr_status launch_fit_apply(const Layout& L, void* O, int out_dtype, cudaStream_t st);
sparsepr_status launch_ridge_solve(const Layout& L, cudaStream_t st);

// Upper bound of the number of query tiles of one head: sum_g ceil(n_g / tile) <= N/tile + C_q.
inline int max_query_tiles(const Layout& L, int tile) { return (L.N + tile - 1) / tile + L.Cq; }

}  // namespace sparsepr
