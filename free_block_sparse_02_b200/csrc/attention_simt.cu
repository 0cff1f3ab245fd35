// Block-sparse attention and dense probe-row attention on CUDA cores (fp32 arithmetic).
//
// "Partition the Support, Reconstruct the Residual" (arXiv 2608.18484), abstract: block-sparse
// attention evaluates only the selected (query group, key group) cells; queries of one query
// group attend to the keys of its kept key groups, softmax over the retained keys only (hard
// drop); the few probe rows get exact attention over every key.
//
// Operands are the group-permuted Q/K/V: query group g is rows [qoff_g, qoff_{g+1}) of Qp and
// key group j is rows [koff_j, koff_{j+1}) of Kp/Vp.  A work item is one 64-row query tile of
// one group; it streams the concatenation of its kept key groups in 64-key tiles with an
// online softmax (running max and sum per row).  This is the fp32 path of the operator (fp32
// inputs need fp32 products for the 1e-4 output tolerance); bf16 inputs run on the
// tensor-core kernel.
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"

namespace sparsepr {

constexpr int kSimtTileN = 64;

// Virtual key position v (0-based in the concatenation of the kept segments) -> Kp row.
__device__ __forceinline__ int virt_to_row(int v, const int* segpre, const int* segstart, int nseg) {
  int lo = 0, hi = nseg - 1;
  while (lo < hi) {  // last segment with segpre <= v
    const int mid = (lo + hi + 1) >> 1;
    if (segpre[mid] <= v) lo = mid;
    else hi = mid - 1;
  }
  return segstart[lo] + (v - segpre[lo]);
}

// mode 0: block-sparse pass, blockIdx.x = query tile of the head (mapped to its group).
// mode 1: probe rows, blockIdx.x = 64-row tile of the head's probe rows, all keys.
template <typename T, int D>
__global__ void __launch_bounds__(256) attn_simt_kernel(Layout L, int mode) {
  pdl_entry();
  constexpr int DP = D + 1;
  extern __shared__ float sm[];
  float* Qs = sm;                              // [64][DP]
  float* Ks = Qs + kAttnTileM * DP;            // [64][DP]
  float* Vs = Ks + kSimtTileN * DP;            // [64][DP]
  float* Ps = Vs + kSimtTileN * DP;            // [64][65]
  int* segpre = (int*)(Ps + kAttnTileM * 65);  // [kMaxGroups + 1]
  int* segstart = segpre + kMaxGroups + 1;     // [kMaxGroups]
  __shared__ int s_info[4];

  const int bh = blockIdx.y, tid = threadIdx.x;
  const T* Qsrc;
  int qrow0, nrows, nseg, nkeys;
  float* out;
  if (mode == 0) {
    const int* toff = L.tile_off + (size_t)bh * (L.Cq + 1);
    const int x = blockIdx.x;
    if (x >= toff[L.Cq]) return;
    int lo = 0, hi = L.Cq - 1;
    while (lo < hi) {  // last group with toff <= x
      const int mid = (lo + hi + 1) >> 1;
      if (toff[mid] <= x) lo = mid;
      else hi = mid - 1;
    }
    const int g = lo;
    const int* qoff = L.qoff + (size_t)bh * (L.Cq + 1);
    qrow0 = qoff[g] + (x - toff[g]) * kAttnTileM;
    nrows = min(kAttnTileM, qoff[g + 1] - qrow0);
    Qsrc = (const T*)L.Qp + (size_t)bh * L.N * D;
    out = L.Osp + (size_t)bh * L.N * D;
    nseg = L.route_cnt[(size_t)bh * L.Cq + g];
    if (tid == 0) {
      const int* list = L.route_list + ((size_t)bh * L.Cq + g) * L.Ck;
      const int* koff = L.koff + (size_t)bh * (L.Ck + 1);
      int run = 0;
      for (int i = 0; i < nseg; ++i) {
        const int j = list[i];
        segpre[i] = run;
        segstart[i] = koff[j];
        run += koff[j + 1] - koff[j];
      }
      segpre[nseg] = run;
      s_info[0] = run;
    }
  } else {
    qrow0 = blockIdx.x * kAttnTileM;
    nrows = min(kAttnTileM, L.P - qrow0);
    if (nrows <= 0) return;
    Qsrc = (const T*)L.Qprobe + (size_t)bh * L.P * D;
    out = L.Odense + (size_t)bh * L.P * D;
    nseg = 1;
    if (tid == 0) {
      segpre[0] = 0;
      segstart[0] = 0;
      segpre[1] = L.N;
      s_info[0] = L.N;
    }
  }
  const T* Kg = (const T*)L.Kp + (size_t)bh * L.N * D;
  const T* Vg = (const T*)L.Vp + (size_t)bh * L.N * D;
  for (int e = tid; e < kAttnTileM * D; e += 256) {
    const int r = e / D, a = e % D;
    Qs[r * DP + a] = r < nrows ? to_f32(Qsrc[(size_t)(qrow0 + r) * D + a]) : 0.f;
  }
  __syncthreads();
  nkeys = s_info[0];

  const int r = tid >> 2, qd = tid & 3;
  constexpr int DQ = D / 4;
  float o[DQ];
#pragma unroll
  for (int i = 0; i < DQ; ++i) o[i] = 0.f;
  float mrun = -INFINITY, lpart = 0.f;
  const float scale = 1.0f / sqrtf((float)D);

  for (int v0 = 0; v0 < nkeys; v0 += kSimtTileN) {
    const int nv = min(kSimtTileN, nkeys - v0);
    __syncthreads();
    {
      const int kk = tid >> 2;  // key row of the tile this thread loads a quarter of
      const int row = kk < nv ? virt_to_row(v0 + kk, segpre, segstart, nseg) : 0;
      for (int a = qd * DQ; a < (qd + 1) * DQ; ++a) {
        Ks[kk * DP + a] = kk < nv ? to_f32(Kg[(size_t)row * D + a]) : 0.f;
        Vs[kk * DP + a] = kk < nv ? to_f32(Vg[(size_t)row * D + a]) : 0.f;
      }
    }
    __syncthreads();
    float s[16];
    float tmax = -INFINITY;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int c = qd + 4 * i;
      float acc = 0.f;
#pragma unroll 8
      for (int a = 0; a < D; ++a) acc = fmaf(Qs[r * DP + a], Ks[c * DP + a], acc);
      s[i] = c < nv ? acc * scale : -INFINITY;
      tmax = fmaxf(tmax, s[i]);
    }
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
    const float mnew = fmaxf(mrun, tmax);
    const float corr = expf(mrun - mnew);  // exp(-inf) = 0 on the first tile
    mrun = mnew;
    lpart *= corr;
#pragma unroll
    for (int i = 0; i < DQ; ++i) o[i] *= corr;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float p = expf(s[i] - mnew);
      lpart += p;
      Ps[r * 65 + qd + 4 * i] = p;
    }
    __syncthreads();
    for (int c = 0; c < nv; ++c) {
      const float p = Ps[r * 65 + c];
#pragma unroll
      for (int i = 0; i < DQ; ++i) o[i] = fmaf(p, Vs[c * DP + qd * DQ + i], o[i]);
    }
  }
  float l = lpart;
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);
  if (r < nrows) {
    const float inv = l > 0.f ? 1.0f / l : 0.f;
    float* orow = out + (size_t)(qrow0 + r) * D + qd * DQ;
#pragma unroll
    for (int i = 0; i < DQ; ++i) orow[i] = o[i] * inv;
  }
}

template <typename T, int D>
static sparsepr_status launch_simt(const Layout& L, cudaStream_t st, cudaEvent_t ev0, cudaEvent_t ev1) {
  const size_t smem = (size_t)(kAttnTileM + 2 * kSimtTileN) * (D + 1) * 4 + kAttnTileM * 65 * 4 +
                      (2 * kMaxGroups + 1) * 4;
  cudaFuncSetAttribute(attn_simt_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (ev0) cudaEventRecord(ev0, st);
  launch(attn_simt_kernel<T, D>, dim3(max_query_tiles(L, kAttnTileM), L.BH), 256, smem, st, L, 0);
  if (ev1) cudaEventRecord(ev1, st);
  if (L.P > 0)
    launch(attn_simt_kernel<T, D>, dim3((L.P + kAttnTileM - 1) / kAttnTileM, L.BH), 256, smem, st, L, 1);
  SPR_LAUNCH_CHECK();
  return SPARSEPR_OK;
}

// fp32 inputs run here; bf16 inputs run on the tensor-core kernel (attention_sm100.cu).
sparsepr_status launch_attention(const Layout& L, cudaStream_t st, cudaEvent_t e0, cudaEvent_t e1) {
  if (L.dtype == SPARSEPR_F32)
    return L.d == 64 ? launch_simt<float, 64>(L, st, e0, e1) : launch_simt<float, 128>(L, st, e0, e1);
  return launch_attention_tc(L, st, e0, e1);
}

}  // namespace sparsepr
