// Allocation-free entry point: the weighted ridge fit of the probe correction with its scratch
// in a fixed device array instead of a caller-provided workspace.
//
// Who needs it: callers that cannot call cudaMalloc themselves, or hand this library device
// memory for scratch, at the point where they fit the correction -- for example code running
// under a memory pool or allocator that must not grow during a step, or a host runtime that
// only passes the tensors it already owns (inputs and outputs).  This entry point allocates
// nothing: its scratch lives in one file-scope __device__ array that every GPU which loads the
// library reserves until the process exits.
//
// Scratch layout (doubles): ridge Gram G [H][129][129], cross term B [H][129][128], residual
// Gram S [H][128][128], the float copy of A, per-head statistics and a status word, for at
// most kStaticMaxHeads heads of head dimension <= 128 (about 7.4 MB).
#include <math.h>
#include <string.h>

#include <mutex>

#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"

namespace sparsepr {

constexpr int kStaticMaxHeads = 16;
constexpr int kStaticMaxDim = 128;
constexpr int kStaticMaxProbes = kMaxProbes;
constexpr size_t kStaticN1 = kStaticMaxDim + 1;
constexpr size_t kStaticG = kStaticMaxHeads * kStaticN1 * kStaticN1;
constexpr size_t kStaticB = kStaticMaxHeads * kStaticN1 * kStaticMaxDim;
constexpr size_t kStaticS = kStaticMaxHeads * (size_t)kStaticMaxDim * kStaticMaxDim;
constexpr size_t kStaticA32 = (kStaticMaxHeads * kStaticN1 * kStaticMaxDim + 1) / 2;  // floats, in doubles
constexpr size_t kStaticStats = (kStaticMaxHeads * sizeof(sparsepr_head_stats) + 7) / 8;
constexpr size_t kStaticStatus = 32;  // one int, padded to 256 bytes
constexpr size_t kStaticDoubles = kStaticG + kStaticB + kStaticS + kStaticA32 + kStaticStats + kStaticStatus;

static __device__ __align__(256) double g_ridge_scratch[kStaticDoubles];

constexpr int kMaxDevices = 64;
static std::mutex g_scratch_mu;
struct ScratchAddr {
  unsigned long long ctx_id;  // the context the address belongs to (0 = not looked up yet)
  double* addr;
};
static ScratchAddr g_scratch_addr[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (cuCtxGetId: never reused within a
// process), or 0 when there is none or the driver does not provide it.
static unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = (CtxGetCurrentFn)p;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = (CtxGetIdFn)p;
    looked_up = true;
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array on the current device.  In host code the array's name is
// only a host-side stand-in, so the address is looked up with cudaGetSymbolAddress, with the
// device current, the first time a device is used, and cached together with the id of the
// context it was taken in.  A later call under another context of that device (after a
// cudaDeviceReset the module is loaded again, possibly at another address) looks it up again.
static sparsepr_status scratch_address(double** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SPARSEPR_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SPARSEPR_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchAddr& e = g_scratch_addr[dev];
  const unsigned long long id = current_context_id();
  if (!e.addr || id == 0 || id != e.ctx_id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ridge_scratch) != cudaSuccess || p == nullptr) return SPARSEPR_ERR_CUDA;
    e.addr = (double*)p;
    e.ctx_id = current_context_id();  // the lookup itself makes the primary context current
  }
  *out = e.addr;
  return SPARSEPR_OK;
}

// G = X^T W X, B = X^T W R, S = R^T W R with X_p = [osp_p, 1], R_p = odense_p - osp_p, for
// probe rows given directly (rows [8 y, 8 y + 8) of each; probes summed in a fixed order).
__global__ void __launch_bounds__(256) ridge_gram_rows_kernel(const float* __restrict__ osp,
                                                              const float* __restrict__ od,
                                                              const double* __restrict__ pw, int P, int d,
                                                              double* __restrict__ G, double* __restrict__ B,
                                                              double* __restrict__ S) {
  pdl_entry();
  extern __shared__ double shx[];
  constexpr int kRows = 8, kChunk = 32;
  const int bh = blockIdx.x, n1 = d + 1, tid = threadIdx.x;
  double* X = shx;                  // [32][n1]
  double* R = X + kChunk * n1;      // [32][d]
  double* w = R + kChunk * d;       // [32]
  const int a0 = blockIdx.y * kRows;
  const int per_row = n1 + 2 * d;
  const int n_out = kRows * per_row;
  double acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.0;
  const float* xs = osp + (size_t)bh * P * d;
  const float* ys = od + (size_t)bh * P * d;
  for (int p0 = 0; p0 < P; p0 += kChunk) {
    const int np = min(kChunk, P - p0);
    __syncthreads();
    for (int e = tid; e < kChunk * n1; e += 256) {
      const int p = e / n1, a = e % n1;
      X[e] = p < np ? (a < d ? (double)xs[(size_t)(p0 + p) * d + a] : 1.0) : 0.0;
    }
    for (int e = tid; e < kChunk * d; e += 256) {
      const int p = e / d, a = e % d;
      R[e] = p < np ? (double)ys[(size_t)(p0 + p) * d + a] - (double)xs[(size_t)(p0 + p) * d + a] : 0.0;
    }
    if (tid < kChunk) w[tid] = tid < np ? pw[(size_t)bh * P + p0 + tid] : 0.0;
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
    if (c < n1) G[((size_t)bh * n1 + a) * n1 + c] = acc[i];
    else if (c < n1 + d) B[((size_t)bh * n1 + a) * d + (c - n1)] = acc[i];
    else if (a < d) S[((size_t)bh * d + a) * d + (c - n1 - d)] = acc[i];
  }
}

}  // namespace sparsepr

using namespace sparsepr;

extern "C" sparsepr_status sparsepr_ridge_fit_static(const float* osp_probe, const float* odense_probe,
                                                     const double* probe_w, int32_t n_heads, int32_t P, int32_t d,
                                                     double lambda, double* A, int32_t* status_out,
                                                     void* stream) {
  if (!A || (P > 0 && (!osp_probe || !odense_probe || !probe_w)) || !isfinite(lambda))
    return SPARSEPR_ERR_INVALID_ARG;
  if (n_heads < 1 || P < 0) return SPARSEPR_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SPARSEPR_ERR_UNSUPPORTED;
  if (n_heads > kStaticMaxHeads || d > kStaticMaxDim || P > kStaticMaxProbes) return SPARSEPR_ERR_WORKSPACE;
  double* base = nullptr;
  sparsepr_status s = scratch_address(&base);
  if (s != SPARSEPR_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  Layout L;
  memset(&L, 0, sizeof(L));
  L.BH = n_heads;
  L.d = d;
  L.P = P;
  L.lambda = lambda;
  L.ridgeG = base;
  L.ridgeB = L.ridgeG + kStaticG;
  L.spanS = L.ridgeB + kStaticB;
  L.A32 = (float*)(L.spanS + kStaticS);
  L.stats = (sparsepr_head_stats*)((double*)L.A32 + kStaticA32);
  L.status = (int*)((double*)L.stats + kStaticStats);
  L.A64 = A;
  // the status word is the only scratch that must start at zero; every other scratch entry a
  // call reads is written by the same call first
  if (cudaMemsetAsync(L.status, 0, sizeof(int), st) != cudaSuccess) return SPARSEPR_ERR_CUDA;
  if (P > 0) {
    const int n1 = d + 1;
    const size_t smem = (size_t)(32 * n1 + 32 * d + 32) * sizeof(double);
    cudaFuncSetAttribute(ridge_gram_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    launch(ridge_gram_rows_kernel, dim3(n_heads, (n1 + 7) / 8), 256, smem, st, osp_probe, odense_probe, probe_w,
           (int)P, (int)d, L.ridgeG, L.ridgeB, L.spanS);
    SPR_LAUNCH_CHECK();
  }
  s = launch_ridge_solve(L, st);
  if (s != SPARSEPR_OK) return s;
  if (status_out &&
      cudaMemcpyAsync(status_out, L.status, sizeof(int), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return SPARSEPR_ERR_CUDA;
  return SPARSEPR_OK;
}
