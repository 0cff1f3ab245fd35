// C ABI of the SparsePR operator (declared in include/sparsepr.h): argument checking,
// workspace carving, call ordering and result queries.  All device work is in the kernel
// files; this file only enqueues it.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <new>
#include <vector>

#include "common.cuh"
#include "kernels.cuh"

using namespace sparsepr;

struct sparsepr_plan_s {
  sparsepr_config cfg;
  Layout L;
  void* ws;
  size_t ws_bytes;
  bool planned = false;     // a partition is installed (plan or set_partition)
  bool attended = false;    // attention ran on the current partition
  bool have_state = false;  // centroids of a previous plan exist (warm start)
  cudaStream_t last = nullptr;
  KernelEvents ev;  // optional timing hooks (see sparsepr_set_kernel_events)
};

std::atomic<long long> sparsepr::g_launches{0};

namespace {


sparsepr_status validate(const sparsepr_config* c) {
  if (!c) return SPARSEPR_ERR_INVALID_ARG;
  if (c->B < 1 || c->H < 1 || c->N < 1) return SPARSEPR_ERR_INVALID_ARG;
  if (c->dtype != SPARSEPR_F32 && c->dtype != SPARSEPR_BF16) return SPARSEPR_ERR_INVALID_ARG;
  if (c->s < 1 || c->s > c->N) return SPARSEPR_ERR_INVALID_ARG;
  if (c->n_kgroups < 1 || c->n_kgroups > c->N || c->n_qgroups < 1 || c->n_qgroups > c->N)
    return SPARSEPR_ERR_INVALID_ARG;
  if (c->n_kgroups > kMaxGroups || c->n_qgroups > kMaxGroups) return SPARSEPR_ERR_INVALID_ARG;
  if (c->fixed_k < 0) return SPARSEPR_ERR_INVALID_ARG;
  if (c->fixed_k == 0 && !(c->density > 0.f && c->density <= 1.f)) return SPARSEPR_ERR_INVALID_ARG;
  if (c->P < 0 || c->P > c->N || c->P > kMaxProbes) return SPARSEPR_ERR_INVALID_ARG;
  if (c->probe_mode != SPARSEPR_PROBE_UNIFORM && c->probe_mode != SPARSEPR_PROBE_STRATIFIED &&
      c->probe_mode != SPARSEPR_PROBE_RANDOM)
    return SPARSEPR_ERR_INVALID_ARG;
  if (!isfinite(c->lambda) || c->km_iters < 1 || c->km_iters_warm < 0 || !isfinite(c->km_tol))
    return SPARSEPR_ERR_INVALID_ARG;
  if (c->km_iters > 10000 || c->km_iters_warm > 10000) return SPARSEPR_ERR_INVALID_ARG;
  if (c->partition != SPARSEPR_PARTITION_RESPONSE && c->partition != SPARSEPR_PARTITION_SEMANTIC)
    return SPARSEPR_ERR_INVALID_ARG;
  if (c->repair != 0 && c->repair != 1) return SPARSEPR_ERR_INVALID_ARG;
  if (c->correction != SPARSEPR_CORRECTION_AFFINE && c->correction != SPARSEPR_CORRECTION_MEAN)
    return SPARSEPR_ERR_INVALID_ARG;
  if (c->trunc_rank < 0 || c->trunc_rank > c->d) return SPARSEPR_ERR_INVALID_ARG;
  if (c->key_rank < 0 || c->key_rank > c->d) return SPARSEPR_ERR_INVALID_ARG;
  if ((double)c->B * c->H * c->N * 256.0 > 9.0e18) return SPARSEPR_ERR_INVALID_ARG;
  if (c->d != 64 && c->d != 128) return SPARSEPR_ERR_UNSUPPORTED;
  // rows of the [B*H*N, d] views are int32 in the kernels (tiles of 128 rows)
  if ((double)c->B * c->H * (((double)c->N + 127.0) / 128.0) * 128.0 > 2147483647.0) return SPARSEPR_ERR_UNSUPPORTED;
  return SPARSEPR_OK;
}

// Assigns every workspace region (256-byte aligned) from `base`; returns the total size.
// With base == nullptr only the size is computed.
size_t carve(const sparsepr_config& c, char* base, Layout& L) {
  memset(&L, 0, sizeof(L));
  const size_t BH = (size_t)c.B * c.H, N = c.N, d = c.d, Ck = c.n_kgroups, Cq = c.n_qgroups,
               P = c.P;
  const size_t e = elt_size(c.dtype);
  L.BH = (int)BH;
  L.H = c.H;
  L.N = c.N;
  L.d = c.d;
  L.s = c.s;
  L.Ck = c.n_kgroups;
  L.Cq = c.n_qgroups;
  L.P = c.P;
  L.dtype = c.dtype;
  L.fixed_k = c.fixed_k;
  L.iters_cap = std::max(c.km_iters, c.km_iters_warm) + 1;
  L.probe_mode = c.probe_mode;
  L.density = c.density;
  L.km_tol = c.km_tol;
  L.lambda = c.lambda;
  L.seed = c.seed;
  L.semantic = c.partition == SPARSEPR_PARTITION_SEMANTIC;
  L.repair = c.repair;
  L.correction = c.correction;
  L.trunc_rank = c.trunc_rank;
  L.key_rank = c.key_rank;
  size_t off = 0;
  auto take = [&](auto*& ptr, size_t bytes) {
    using P_ = std::remove_reference_t<decltype(ptr)>;
    ptr = base ? (P_)(base + off) : nullptr;
    off += (bytes + 255) & ~(size_t)255;
  };
  const size_t cap = L.iters_cap;
  take(L.status, 4);
  take(L.stats, BH * sizeof(sparsepr_head_stats));
  take(L.M, BH * d * d * 8);
  take(L.T0k, BH * 8);
  take(L.T0q, BH * 8);
  if (c.key_rank > 0 && c.key_rank < c.d && c.partition == SPARSEPR_PARTITION_RESPONSE) {
    take(L.kgram_part, BH * ((N + kGramChunk - 1) / kGramChunk) * d * d * 8);
    take(L.kgram, BH * d * d * 8);
    take(L.kr_L, BH * d * d * 8);
    take(L.kr_V, BH * d * d * 8);
    take(L.kr_T, BH * d * d * 8);
  }
  take(L.init_ids, BH * (Ck + Cq) * 4);
  take(L.fy, 4);  // unused: the draw keeps its slots in shared memory
  take(L.iters_run, BH * 2 * 4);
  take(L.stop_at, BH * 2 * 4);
  take(L.warm, 4);
  take(L.kcent, BH * Ck * d * 8);
  take(L.kW64, BH * Ck * d * 8);
  take(L.kW32, BH * Ck * d * 4);
  take(L.kbias64, BH * Ck * 8);
  take(L.kbias32, BH * Ck * 4);
  take(L.kwnorm, BH * Ck * 4);
  take(L.ksum, BH * Ck * d * 8);
  take(L.kcount, BH * Ck * 4);
  take(L.klabel, BH * N * 4);
  take(L.kJ, BH * cap * 8);
  take(L.krefined, BH * 4);
  L.Ckp = (c.n_kgroups + 15) / 16 * 16;
  L.Cqp = (c.n_qgroups + 15) / 16 * 16;
  take(L.Gc, BH * d * d * 8);
  take(L.inv_rms, BH * N * 4);
  take(L.inv_rms64, BH * N * 8);
  take(L.qxnorm, BH * N * 4);
  take(L.qcent, BH * Cq * Ck * 8);
  take(L.qU64, BH * Cq * d * 8);
  take(L.qU32, BH * Cq * d * 4);
  take(L.qbias64, BH * Cq * 8);
  take(L.qbias32, BH * Cq * 4);
  take(L.qwnorm, BH * Cq * 4);
  take(L.qsum, BH * Cq * d * 8);
  take(L.qcount, BH * Cq * 4);
  take(L.qlabel, BH * N * 4);
  take(L.qJ, BH * cap * 8);
  take(L.qrefined, BH * 4);
  take(L.kWb, 3 * BH * (size_t)L.Ckp * d * 2);
  take(L.qWb, 3 * BH * (size_t)L.Cqp * d * 2);
  take(L.Mb, 3 * BH * d * d * 2);
  take(L.Gcb, 3 * BH * d * d * 2);
  take(L.knorm, BH * N * 4);
  if (L.Ckp > kKmChunkGroups) take(L.ktop, BH * N * 16);
  if (L.Cqp > kKmChunkGroups) take(L.qtop, BH * N * 16);
  take(L.kprev, BH * N * 4);
  take(L.qprev, BH * N * 4);
  {  // whole-loop k-means: partials for the most CTAs per head either side could use
    const int Gk = km_loop_ctas_per_head(c.B * c.H, c.N, c.d, c.dtype, c.n_kgroups, c.n_kgroups, true,
                                         kKmLoopMaxCtas, nullptr);
    const int Gq = km_loop_ctas_per_head(c.B * c.H, c.N, c.d, c.dtype, c.n_qgroups, c.n_kgroups, false,
                                         kKmLoopMaxCtas, nullptr);
    const int G = std::max(Gk, Gq);
    if (G > 0) {
      L.klp_G = G;
      const size_t Cm = std::max(Gk > 0 ? Ck : 0, Gq > 0 ? Cq : 0);
      take(L.klp_sum, BH * G * Cm * d * 8);
      take(L.klp_cnt, BH * G * Cm * 4);
      take(L.klp_J, BH * G * 8);
      take(L.klp_bar, (BH + 1) * 4);
    }
  }
  const size_t km_tiles = BH * (size_t)((N + 127) / 128);
  take(L.rlist, km_tiles * 128 * 16);
  take(L.rcnt, km_tiles * 4);
  take(L.sort_hist, BH * 2 * ((N + kSortChunk - 1) / kSortChunk) * std::max(Ck, Cq) * 4);
  take(L.kperm, BH * N * 4);
  take(L.kinv, BH * N * 4);
  take(L.koff, BH * (Ck + 1) * 4);
  take(L.qperm, BH * N * 4);
  take(L.qinv, BH * N * 4);
  take(L.qoff, BH * (Cq + 1) * 4);
  take(L.route, BH * Cq * Ck);
  take(L.route_list, BH * Cq * Ck * 4);
  take(L.route_cnt, BH * Cq * 4);
  take(L.route_keys, BH * Cq * 4);
  take(L.tile_off, BH * (Cq + 1) * 4);
  take(L.probe_tok, BH * std::max<size_t>(P, 1) * 4);
  take(L.probe_w, BH * std::max<size_t>(P, 1) * 8);
  take(L.probe_of, BH * N * 4);
  take(L.Qp, BH * N * d * e);
  take(L.Kp, BH * N * d * e);
  take(L.Vp, BH * N * d * e);
  take(L.Qprobe, BH * std::max<size_t>(P, 1) * d * e);
  take(L.Osp, BH * N * d * 4);
  take(L.Odense, BH * std::max<size_t>(P, 1) * d * 4);
  take(L.ridgeG, BH * (d + 1) * (d + 1) * 8);
  take(L.ridgeB, BH * (d + 1) * d * 8);
  take(L.spanS, BH * d * d * 8);
  take(L.A64, BH * (d + 1) * d * 8);
  take(L.A32, BH * (d + 1) * d * 4);
  return off;
}

sparsepr_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SPARSEPR_OK : SPARSEPR_ERR_CUDA; }

sparsepr_status wait_and_status(const sparsepr_plan_t* p, bool clear) {
  cudaError_t e = p->last ? cudaStreamSynchronize(p->last) : cudaDeviceSynchronize();
  if (e != cudaSuccess) return SPARSEPR_ERR_CUDA;
  int s = 0;
  if (cudaMemcpy(&s, p->L.status, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return SPARSEPR_ERR_CUDA;
  if (clear && s != 0 && cudaMemset(p->L.status, 0, 4) != cudaSuccess) return SPARSEPR_ERR_CUDA;
  return (sparsepr_status)s;
}

template <typename T>
sparsepr_status copy_out(void* dst, size_t bytes, const T* src, size_t count) {
  if (bytes != count * sizeof(T)) return SPARSEPR_ERR_INVALID_ARG;
  return cuda_status(cudaMemcpy(dst, src, bytes, cudaMemcpyDeviceToHost));
}

}  // namespace

extern "C" {

int32_t sparsepr_version(void) { return 100; }

const char* sparsepr_status_string(sparsepr_status s) {
  switch (s) {
    case SPARSEPR_OK: return "ok";
    case SPARSEPR_ERR_INVALID_ARG: return "invalid argument";
    case SPARSEPR_ERR_UNSUPPORTED: return "unsupported configuration";
    case SPARSEPR_ERR_CUDA: return "CUDA error";
    case SPARSEPR_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case SPARSEPR_ERR_NUMERIC: return "ridge system not positive definite";
    case SPARSEPR_ERR_TIMEOUT: return "device wait timed out";
    case SPARSEPR_ERR_STATE: return "call out of order";
  }
  return "unknown status";
}

sparsepr_status sparsepr_workspace_size(const sparsepr_config* cfg, size_t* bytes) {
  sparsepr_status s = validate(cfg);
  if (s != SPARSEPR_OK) return s;
  if (!bytes) return SPARSEPR_ERR_INVALID_ARG;
  Layout L;
  *bytes = carve(*cfg, nullptr, L);
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_plan_create(const sparsepr_config* cfg, void* workspace, size_t ws_bytes,
                                     sparsepr_plan_t** plan) {
  sparsepr_status s = validate(cfg);
  if (s != SPARSEPR_OK) return s;
  if (!plan) return SPARSEPR_ERR_INVALID_ARG;
  *plan = nullptr;
  if (!workspace || ((uintptr_t)workspace & 255u)) return SPARSEPR_ERR_WORKSPACE;
  Layout L;
  const size_t need = carve(*cfg, nullptr, L);
  if (ws_bytes < need) return SPARSEPR_ERR_WORKSPACE;
  sparsepr_plan_t* p = new (std::nothrow) sparsepr_plan_s();
  if (!p) return SPARSEPR_ERR_INVALID_ARG;
  p->cfg = *cfg;
  carve(*cfg, (char*)workspace, p->L);
  p->ws = workspace;
  p->ws_bytes = ws_bytes;
  if (cudaMemset(p->L.status, 0, 4) != cudaSuccess ||
      cudaMemset(p->L.stats, 0, p->L.BH * sizeof(sparsepr_head_stats)) != cudaSuccess) {
    delete p;
    return SPARSEPR_ERR_CUDA;
  }
  *plan = p;
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_plan(sparsepr_plan_t* p, const void* Q, const void* K, void* stream) {
  if (!p || !Q || !K) return SPARSEPR_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const bool warm = p->have_state && p->cfg.km_iters_warm > 0;
  const int iters = warm ? p->cfg.km_iters_warm : p->cfg.km_iters;
  p->last = st;
  p->planned = false;
  p->attended = false;
  sparsepr_status s = launch_plan(p->L, Q, K, warm, iters, st, p->ev);
  if (s != SPARSEPR_OK) return s;
  p->planned = true;
  p->have_state = true;
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_set_partition(sparsepr_plan_t* p, const int32_t* klabels, const int32_t* qlabels,
                                       const uint8_t* route, const int32_t* probes, const double* probe_w,
                                       void* stream) {
  if (!p || !klabels || !qlabels || !route) return SPARSEPR_ERR_INVALID_ARG;
  const Layout& L = p->L;
  if (L.P > 0 && (!probes || !probe_w)) return SPARSEPR_ERR_INVALID_ARG;
  const size_t BH = L.BH, N = L.N;
  for (size_t i = 0; i < BH * N; ++i)
    if (klabels[i] < 0 || klabels[i] >= L.Ck || qlabels[i] < 0 || qlabels[i] >= L.Cq)
      return SPARSEPR_ERR_INVALID_ARG;
  std::vector<unsigned char> seen(N);
  for (size_t h = 0; h < BH; ++h) {
    std::fill(seen.begin(), seen.end(), 0);
    for (int i = 0; i < L.P; ++i) {
      const int t = probes[h * L.P + i];
      if (t < 0 || (size_t)t >= N || seen[t] || !isfinite(probe_w[h * L.P + i])) return SPARSEPR_ERR_INVALID_ARG;
      seen[t] = 1;
    }
  }
  cudaStream_t st = (cudaStream_t)stream;
  p->last = st;
  p->planned = false;
  p->attended = false;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SPARSEPR_ERR_CUDA;
  const size_t nb = BH * N * 4;
  if (cudaMemcpy(L.klabel, klabels, nb, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(L.qlabel, qlabels, nb, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(L.route, route, BH * L.Cq * L.Ck, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemset(L.stats, 0, BH * sizeof(sparsepr_head_stats)) != cudaSuccess)
    return SPARSEPR_ERR_CUDA;
  if (L.P > 0 && (cudaMemcpy(L.probe_tok, probes, BH * L.P * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
                  cudaMemcpy(L.probe_w, probe_w, BH * L.P * 8, cudaMemcpyHostToDevice) != cudaSuccess))
    return SPARSEPR_ERR_CUDA;
  sparsepr_status s = launch_installed_partition(L, st);
  if (s != SPARSEPR_OK) return s;
  p->planned = true;
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_attention(sparsepr_plan_t* p, const void* Q, const void* K, const void* V,
                                   void* stream) {
  if (!p || !Q || !K || !V) return SPARSEPR_ERR_INVALID_ARG;
  if (!p->planned) return SPARSEPR_ERR_STATE;
  cudaStream_t st = (cudaStream_t)stream;
  p->last = st;
  sparsepr_status s = launch_permute(p->L, Q, K, V, st);
  if (s != SPARSEPR_OK) return s;
  s = launch_attention(p->L, st, p->ev.start[SPARSEPR_KERNEL_BLOCK_SPARSE], p->ev.stop[SPARSEPR_KERNEL_BLOCK_SPARSE]);
  if (s != SPARSEPR_OK) return s;
  p->attended = true;
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_fit_apply(sparsepr_plan_t* p, void* O, int32_t out_dtype, void* stream) {
  if (!p || !O) return SPARSEPR_ERR_INVALID_ARG;
  if (out_dtype != SPARSEPR_F32 && out_dtype != SPARSEPR_BF16) return SPARSEPR_ERR_INVALID_ARG;
  if (!p->attended) return SPARSEPR_ERR_STATE;
  cudaStream_t st = (cudaStream_t)stream;
  p->last = st;
  return launch_fit_apply(p->L, O, out_dtype, st);
}

sparsepr_status sparsepr_sync(sparsepr_plan_t* p) {
  if (!p) return SPARSEPR_ERR_INVALID_ARG;
  return wait_and_status(p, true);
}

sparsepr_status sparsepr_plan_query(const sparsepr_plan_t* p, int32_t what, void* dst, size_t bytes) {
  if (!p || !dst) return SPARSEPR_ERR_INVALID_ARG;
  sparsepr_status s = wait_and_status(p, false);
  if (s != SPARSEPR_OK) return s;
  const Layout& L = p->L;
  const size_t BH = L.BH, N = L.N, d = L.d;
  switch (what) {
    case SPARSEPR_Q_KLABELS: return copy_out(dst, bytes, L.klabel, BH * N);
    case SPARSEPR_Q_QLABELS: return copy_out(dst, bytes, L.qlabel, BH * N);
    case SPARSEPR_Q_ROUTE: return copy_out(dst, bytes, L.route, BH * L.Cq * L.Ck);
    case SPARSEPR_Q_PROBES: return copy_out(dst, bytes, L.probe_tok, BH * L.P);
    case SPARSEPR_Q_PROBE_W: return copy_out(dst, bytes, L.probe_w, BH * L.P);
    case SPARSEPR_Q_FIT: return copy_out(dst, bytes, L.A64, BH * (d + 1) * d);
    case SPARSEPR_Q_KCENT: return copy_out(dst, bytes, L.kcent, BH * L.Ck * d);
    case SPARSEPR_Q_QCENT: return copy_out(dst, bytes, L.qcent, BH * L.Cq * L.Ck);
    case SPARSEPR_Q_ODENSE: return copy_out(dst, bytes, L.Odense, BH * L.P * d);
    case SPARSEPR_Q_STATS: return copy_out(dst, bytes, L.stats, BH);
    case SPARSEPR_Q_KM_PATH: {
      const int32_t path[2] = {km_loop_supported(L, true) ? 1 : 0, km_loop_supported(L, false) ? 1 : 0};
      if (bytes != sizeof(path)) return SPARSEPR_ERR_INVALID_ARG;
      memcpy(dst, path, sizeof(path));
      return SPARSEPR_OK;
    }
    case SPARSEPR_Q_OSP: {
      if (bytes != BH * N * d * 4) return SPARSEPR_ERR_INVALID_ARG;
      std::vector<float> tmp(BH * N * d);
      std::vector<int> perm(BH * N);
      if (cudaMemcpy(tmp.data(), L.Osp, bytes, cudaMemcpyDeviceToHost) != cudaSuccess ||
          cudaMemcpy(perm.data(), L.qperm, BH * N * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
        return SPARSEPR_ERR_CUDA;
      float* out = (float*)dst;
      for (size_t h = 0; h < BH; ++h)
        for (size_t pos = 0; pos < N; ++pos)
          memcpy(out + (h * N + perm[h * N + pos]) * d, tmp.data() + (h * N + pos) * d, d * 4);
      return SPARSEPR_OK;
    }
    case SPARSEPR_Q_KOBJ:
    case SPARSEPR_Q_QOBJ: {
      const size_t it = p->cfg.km_iters;
      if (bytes != BH * it * 8) return SPARSEPR_ERR_INVALID_ARG;
      std::vector<double> J(BH * L.iters_cap);
      std::vector<sparsepr_head_stats> st(BH);
      if (cudaMemcpy(J.data(), what == SPARSEPR_Q_KOBJ ? L.kJ : L.qJ, J.size() * 8, cudaMemcpyDeviceToHost) != cudaSuccess ||
          cudaMemcpy(st.data(), L.stats, BH * sizeof(sparsepr_head_stats), cudaMemcpyDeviceToHost) != cudaSuccess)
        return SPARSEPR_ERR_CUDA;
      double* out = (double*)dst;
      for (size_t h = 0; h < BH; ++h) {
        const int run = what == SPARSEPR_Q_KOBJ ? st[h].k_iters : st[h].q_iters;
        for (size_t i = 0; i < it; ++i) out[h * it + i] = (int)i < run ? J[h * L.iters_cap + i] : 0.0;
      }
      return SPARSEPR_OK;
    }
    default: return SPARSEPR_ERR_INVALID_ARG;
  }
}

void sparsepr_plan_destroy(sparsepr_plan_t* p) { delete p; }

sparsepr_status sparsepr_set_kernel_events(sparsepr_plan_t* p, int32_t kernel, void* start_event,
                                           void* stop_event) {
  if (!p || kernel < 0 || kernel >= KernelEvents::kCount) return SPARSEPR_ERR_INVALID_ARG;
  if ((start_event == nullptr) != (stop_event == nullptr)) return SPARSEPR_ERR_INVALID_ARG;
  p->ev.start[kernel] = (cudaEvent_t)start_event;
  p->ev.stop[kernel] = (cudaEvent_t)stop_event;
  return SPARSEPR_OK;
}

int64_t sparsepr_launch_count(void) { return (int64_t)g_launches.load(); }

sparsepr_status sparsepr_set_kmeans_path(sparsepr_plan_t* p, int32_t mode) {
  if (!p || (mode != 0 && mode != 1)) return SPARSEPR_ERR_INVALID_ARG;
  p->L.km_steps = mode;
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_set_wait_limit(sparsepr_plan_t* p, int32_t kernel, int64_t cycles) {
  if (!p || cycles < 0) return SPARSEPR_ERR_INVALID_ARG;
  if (kernel == SPARSEPR_KERNEL_BLOCK_SPARSE) p->L.attn_wait_limit = (long long)cycles;
  else if (kernel == SPARSEPR_KERNEL_KMEANS_LOOP) p->L.km_wait_limit = (long long)cycles;
  else return SPARSEPR_ERR_UNSUPPORTED;
  return SPARSEPR_OK;
}

}  // extern "C"
