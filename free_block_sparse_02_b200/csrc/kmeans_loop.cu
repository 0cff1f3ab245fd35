// Every Lloyd iteration of one k-means side in a single cooperative launch, for calls whose
// points fit in the shared memory of the CTAs they are spread over (mid-size calls).
//
// "Partition the Support, Reconstruct the Residual" (arXiv 2608.18484), abstract and Table C.1:
// keys are grouped by k-means on their responses to sampled queries, queries by k-means on their
// normalised responses to the key-group centroids (25 iterations cold, 2 warm, tolerance 1e-4).
// The scores, the rounding bound, the fp64 re-decision and the centroid formulas are those of
// the per-iteration kernels (kmeans_sm100.cu, the prep kernels of partition.cu); this file only
// changes where the data lives and how the steps are ordered:
//
//  * G CTAs per head (one per SM, all co-resident: cooperative launch), CTA r holding the
//    contiguous point tiles [r T / G, (r + 1) T / G) of its head in shared memory for the whole
//    loop: X is read from HBM once, not twice per iteration.
//  * Per iteration: the head's two-term W (hi, mid) and biases are copied into shared memory;
//    the tensor cores score every resident tile (tcgen05, up to four TMEM accumulators, two
//    epilogue warpgroups); flagged points are re-decided in fp64; the CTA's partial group sums
//    are formed in fp64 (the first iteration sums every point, each warp an equal slice of the
//    points sorted by label; later iterations move the partials by the points whose label
//    changed).  A head barrier; then CTA r owns groups [r C / G, (r + 1) C / G): it adds the
//    G partials of each owned group in CTA order, updates the centroid, takes the stop test (the
//    objective is summed in the same order by every CTA of the head, so all of them decide
//    alike) and, unless the loop stops, forms the next W, bias and norm of its groups.  A second
//    head barrier publishes them.
//  * Head barriers are counters in global memory with bounded waits: a wait that runs out sets
//    a launch-wide abort flag that every other wait polls, and the call reports
//    SPARSEPR_ERR_TIMEOUT.
//
// Data produced inside the launch by other CTAs (partial sums, W, biases) is read with L2 loads
// (ld.global.cg), never through L1.
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"
#include "kmeans.cuh"
#include "sm100.cuh"

namespace sparsepr {

using namespace sm100;

constexpr int kKlThreads = 384;  // warp 1 issues the MMAs, warps 4..11 are the two epilogue warpgroups;
                                 // every warp takes part in the other phases
constexpr int kKlWarps = kKlThreads / 32;
constexpr int kKlTile = 128;
constexpr int kKlBatch = 4;          // owned groups updated together in the centroid step
constexpr int kKlMaxKGroups = 256;   // key groups the query step stages per owned group
constexpr size_t kKlStaticSmem = 10 * 1024;  // bound of the kernel's static shared memory

// Scratch doubles shared by three phases that never overlap: the per-warp fp64 copy of a point
// being re-decided (128 per warp), the run pieces of the group sums (2 D per warp) and the
// slices of the centroid step's products (kKlThreads / D slices x kKlBatch x D = 1536).
__host__ __device__ constexpr int km_loop_scratch(int D) {
  return kKlWarps * 128 > kKlWarps * 2 * D ? kKlWarps * 128 : kKlWarps * 2 * D;
}

// Shared memory of the loop kernel for `cap` resident tiles: X, the two W terms, per point
// (label, sorted order, 1/rms in fp32 and fp64, bound norm, re-decision entry), the scratch,
// biases, group offsets, barriers.  At least 120 KB, so that two CTAs never share an SM: each
// may hold all 512 TMEM columns, and a CTA blocked in the allocator would never reach the head
// barrier its partner waits at.
__host__ __device__ inline size_t km_loop_smem(int D, int Np, int C, int cap) {
  const size_t pts = (size_t)cap * kKlTile;
  const size_t need = 1024 /*align*/ + pts * D * 2 + (size_t)2 * Np * D * 2 + pts * (4 + 4 + 4 + 4 + 8 + 16) +
                      (size_t)km_loop_scratch(D) * 8 + (size_t)Np * 4 + (size_t)(2 * C + 2) * 4 + 128 /*barriers*/;
  return need > (size_t)120 * 1024 ? need : (size_t)120 * 1024;
}

struct KmLoopArgs {
  int G;        // CTAs per head
  int cap;      // resident tiles the shared memory was sized for
  int iters;    // iteration limit
};

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int ld_volatile_i32(const int* p) { return *(const volatile int*)p; }
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Barrier of the G CTAs of one head: the n-th call of every CTA of the head returns once all of
// them have made it (counter target G n): a release addition, then acquire loads.  Bounded: it
// gives up, sets the launch's abort flag and returns false after `limit` cycles, or as soon as
// another CTA has set the flag.  Called by every thread of the CTA (block barriers on both sides).
__device__ __forceinline__ bool head_barrier(unsigned* ctr, unsigned target, int* gabort, volatile int* s_abort,
                                             long long limit) {
  __syncthreads();
  if (threadIdx.x == 0 && !*s_abort) {
    // release: the CTA's writes before the block barrier above are visible to every CTA whose
    // acquire load sees this addition
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(ctr), "r"(1u) : "memory");
    const long long t0 = clock64();
    while (ld_acquire_u32(ctr) < target) {
      if (ld_volatile_i32(gabort)) {
        *s_abort = 1;
        break;
      }
      if (clock64() - t0 > limit) {
        *s_abort = 1;
        atomicExch(gabort, 1);
        break;
      }
    }
  }
  __syncthreads();  // the acquire above orders the whole CTA's later reads (block barrier)
  return !*s_abort;
}

template <bool kKeys>
__global__ void __launch_bounds__(kKlThreads, 1)
    kmeans_loop_kernel(const __grid_constant__ CUtensorMap tmX, Layout L, KmLoopArgs P) {
  pdl_entry();  // (launched without the dependent-launch attribute: the wait returns at once)
  const int D = L.d, KB = D / 64;
  const int C = kKeys ? L.Ck : L.Cq;
  const int Npg = kKeys ? L.Ckp : L.Cqp;  // W rows of a head in global memory (groups padded to 16)
  const int Np = (Npg + 31) & ~31;         // W rows in shared memory and score columns: at most 128
  const int A = 2 * Np;                    // accumulator columns: [X W_hi | X W_mid]
  const int NACC = 4 * A <= 512 ? 4 : 2;   // TMEM accumulators: the MMAs run ahead of the epilogue
  const int G = P.G, cap = P.cap;
  const int bh = blockIdx.x / G, r = blockIdx.x % G;
  const int tph = (L.N + kKlTile - 1) / kKlTile;
  const int t0 = (int)((long long)tph * r / G), t1 = (int)((long long)tph * (r + 1) / G);
  const int nt = min(t1 - t0, cap);
  const int npts = min(nt * kKlTile, L.N - t0 * kKlTile);  // valid points of this CTA
  const int j0 = (int)((long long)C * r / G), j1 = (int)((long long)C * (r + 1) / G);  // owned groups
  const size_t row0 = (size_t)bh * L.N + (size_t)t0 * kKlTile;
  const size_t hc = (size_t)bh * G;  // first (head, CTA) slot of this head

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const size_t pts = (size_t)cap * kKlTile;
  uint8_t* sX = sm;                                          // [cap][KB][128 rows][128 B]
  uint8_t* sW = sX + pts * D * 2;                            // [KB][2 terms][Np rows][128 B]
  int* lab = (int*)(sW + (size_t)2 * Np * D * 2);            // [pts]
  int* order = lab + pts;                                    // [pts] points sorted by label (first
                                                             // iteration), then the labels before
  float* sq = (float*)(order + pts);                         // [pts] 1/rms (queries), 1 (keys)
  float* xn = sq + pts;                                      // [pts] norm in the rounding bound
  double* sig = (double*)(xn + pts);                         // [pts] scale of the group sums
  int4* flags = (int4*)(sig + pts);                          // [pts] re-decision entries, then the
                                                             // points whose label changed
  double* xs_all = (double*)(flags + pts);                   // scratch: km_loop_scratch(D) doubles
  float* sbias = (float*)(xs_all + km_loop_scratch(D));      // [Np]
  int* offs = (int*)(sbias + Np);                            // [C + 1]
  int* cursor = offs + C + 1;                                // [C + 1]
  uint64_t* bars = (uint64_t*)(((uintptr_t)(cursor + C + 1) + 7) & ~(uintptr_t)7);
  uint64_t* x_full = bars;
  uint64_t* acc_full = bars + 1;   // [NACC]
  uint64_t* acc_empty = bars + 5;  // [NACC]
  uint64_t* mma_done = bars + 9;
  uint32_t* tmem_slot = (uint32_t*)(bars + 10);
  __shared__ volatile int s_abort;
  __shared__ int s_nflag, s_nchg;
  __shared__ float s_wmax, s_bmax;
  __shared__ double s_red[kKlWarps], s_redc[kKlWarps];
  __shared__ double s_red8[2 * kKlBatch][kKlWarps];
  __shared__ double s_J;
  __shared__ double cb[kKlBatch][kKlMaxKGroups];  // centroid step: owned groups' vectors
  __shared__ double s_gred[kKlBatch][2];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t tcols = km_tc_tmem_cols(NACC * A);
  int* gabort = (int*)(L.klp_bar + L.BH);
  unsigned* hbar = L.klp_bar + bh;
  unsigned nbar = 0;  // head barriers passed
  const long long blim = L.km_wait_limit > 0 ? L.km_wait_limit : kWaitLimitCycles;
  if (tid == 0) {
    s_abort = 0;
    mbar_init(x_full, 1);
    for (int b = 0; b < NACC; ++b) {
      mbar_init(acc_full + b, 1);
      mbar_init(acc_empty + b, 128);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (tid == 0) {  // the CTA's tiles, once (rows past the head's end belong to no point of it)
    prefetch_tmap(&tmX);
    mbar_arrive_expect_tx(x_full, (uint32_t)(nt * kKlTile * D * 2));
    for (int t = 0; t < nt; ++t)
      for (int kb = 0; kb < KB; ++kb)
        tma_load_2d(sX + ((size_t)t * KB + kb) * kKlTile * 128, &tmX, x_full, kb * 64,
                    bh * L.N + (t0 + t) * kKlTile);
  }
  for (int p = tid; p < nt * kKlTile; p += kKlThreads) {
    const bool v = p < npts;
    const size_t row = row0 + p;
    sq[p] = (!kKeys && v) ? L.inv_rms[row] : 1.f;
    xn[p] = v ? (kKeys ? L.knorm[row] : L.qxnorm[row]) : 0.f;
    sig[p] = (!kKeys && v) ? L.inv_rms64[row] : 1.0;
  }
  double* Jarr = (kKeys ? L.kJ : L.qJ) + (size_t)bh * L.iters_cap;
  const double T0 = kKeys ? L.T0k[bh] : L.T0q[bh];
  const double rsd = 1.0 / sqrt((double)D);
  double Jprev = 0.0;

  // ------------------------------------------------------------- centroid step of owned groups
  // update: c <- (sum of the G partial sums) / count for groups that received points (keys: c in
  // key space; queries: nu = C S / (sqrt(d) n), or the raw mean in the semantic partition);
  // weights: the score weights, bias and norm of the next assignment.  The matrix-vector
  // products are split over every thread (thread = (dimension, slice of the inner index), 16
  // loads in flight), the slices' sums staged in wpart and added in a fixed order: the operands
  // come from L2, and one thread walking a whole column would wait for each load in turn.
  double* wpart = xs_all;             // [nsplit][kKlBatch][D]: the re-decision staging, free here
  const int nsplit = kKlThreads / D;  // 6 (d = 64) or 3 (d = 128): nsplit * kKlBatch * D = 1536
  auto centroid_step = [&](bool update, bool weights) {
    const double* Cg = L.kcent + (size_t)bh * L.Ck * D;  // key-group centroids (the query side's C)
    for (int gb = j0; gb < j1; gb += kKlBatch) {
      const int nb = min(kKlBatch, j1 - gb);
      const int Vd = (kKeys || L.semantic) ? D : L.Ck;  // length of a centroid vector
      __syncthreads();  // cb and wpart are free
      if (update) {
        // counts: warp g of the batch, lanes over the head's CTAs
        if (warp < nb) {
          int c = 0;
          for (int q = lane; q < G; q += 32) c += __ldcg(L.klp_cnt + (hc + q) * C + gb + warp);
          c = __reduce_add_sync(0xffffffffu, c);
          if (lane == 0) s_gred[warp][0] = (double)c;
        }
        // sums of the G partials of (group g, dimension a), 16 CTAs' loads in flight per batch; the
        // old centroid (kept where no point joined) fetched alongside
        double tot[2] = {0.0, 0.0}, old[2] = {0.0, 0.0};
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int e = tid + i * kKlThreads;
          if (e >= nb * D) continue;
          const int g = e / D, a = e % D, j = gb + g;
          if (kKeys) old[i] = L.kcent[((size_t)bh * C + j) * D + a];
          else if (L.semantic) old[i] = L.qU64[((size_t)bh * C + j) * D + a];
          const double* src = L.klp_sum + (hc * C + j) * D + a;  // CTA q's value at src[q C D]
          for (int q0 = 0; q0 < G; q0 += 16) {
            double v[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) v[k] = q0 + k < G ? __ldcg(src + (size_t)(q0 + k) * C * D) : 0.0;
#pragma unroll
            for (int k = 0; k < 16; ++k) tot[i] += v[k];
          }
        }
        __syncthreads();  // counts in s_gred
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int e = tid + i * kKlThreads;
          if (e >= nb * D) continue;
          const int g = e / D, a = e % D;
          const double cnt = s_gred[g][0];
          const double mean = cnt > 0.0 ? tot[i] / cnt : 0.0;
          if (kKeys || L.semantic) {  // the new centroid, or the old one where no point joined
            cb[g][a] = cnt > 0.0 ? mean : old[i];
            if (cnt > 0.0) (kKeys ? L.kcent : L.qU64)[((size_t)bh * C + gb + g) * D + a] = mean;
          } else {
            cb[g][a] = mean;  // S_g / n_g, projected to nu below
          }
        }
        __syncthreads();
        if (!kKeys && !L.semantic) {
          // nu_g[j] = C[j] . S_g / sqrt(d): thread (j, slice of the dimensions), every load of the
          // slice in flight, the slices' sums staged in wpart and added in a fixed order; nu
          // replaces S_g in cb (the old nu where no point joined)
          const int nsl = kKlThreads / L.Ck;  // slices per key group (>= 1: C_k <= 256)
          {
            const int j = tid % L.Ck, sl = tid / L.Ck;
            if (sl < nsl) {
              const int a0s = 2 * (sl * (D / 2) / nsl), a1s = 2 * ((sl + 1) * (D / 2) / nsl);
              double acc[kKlBatch];
#pragma unroll
              for (int g = 0; g < kKlBatch; ++g) acc[g] = 0.0;
              const double* row = Cg + (size_t)j * D;
#pragma unroll 16
              for (int a = a0s; a < a1s; a += 2) {
                const double2 v = *(const double2*)(row + a);
#pragma unroll
                for (int g = 0; g < kKlBatch; ++g) acc[g] += v.x * cb[g][a] + v.y * cb[g][a + 1];
              }
#pragma unroll
              for (int g = 0; g < kKlBatch; ++g) wpart[((size_t)sl * kKlBatch + g) * L.Ck + j] = acc[g];
            }
          }
          __syncthreads();  // every thread has read S from cb
          for (int e = tid; e < nb * L.Ck; e += kKlThreads) {
            const int g = e / L.Ck, j = e % L.Ck;
            double nu = 0.0;
            for (int sl = 0; sl < nsl; ++sl) nu += wpart[((size_t)sl * kKlBatch + g) * L.Ck + j];
            nu *= rsd;
            const bool joined = s_gred[g][0] > 0.0;
            cb[g][j] = joined ? nu : L.qcent[((size_t)bh * C + gb + g) * L.Ck + j];
            if (joined) L.qcent[((size_t)bh * C + gb + g) * L.Ck + j] = nu;
          }
          __syncthreads();
        }
      }
      if (!weights) continue;
      if (!update) {  // the initial centroid vectors of the batch into cb
        const double* cent = kKeys ? L.kcent : (L.semantic ? L.qU64 : L.qcent);
        for (int e = tid; e < nb * Vd; e += kKlThreads) {
          const int g = e / Vd, a = e % Vd;
          cb[g][a] = cent[((size_t)bh * C + gb + g) * Vd + a];
        }
        __syncthreads();
      }
      // w[g][a] = sum_k Op[k][a] cb[g][k]: keys Op = M (symmetric, so its column a is row a read
      // down), queries Op = C (k over the key groups, then / sqrt(d)); the semantic queries take
      // w = cb.  Thread (a, slice): the slice's partial sums of every group of the batch.
      const int Kin = kKeys ? D : (L.semantic ? 0 : L.Ck);
      if (Kin > 0) {
        const int a = tid % D, part = tid / D;
        const int k0 = part * Kin / nsplit, k1 = (part + 1) * Kin / nsplit;
        const double* Op = (kKeys ? L.M + (size_t)bh * D * D : Cg) + a;  // element (k, a) at Op[k * D]
        double acc[kKlBatch];
#pragma unroll
        for (int g = 0; g < kKlBatch; ++g) acc[g] = 0.0;
#pragma unroll 16
        for (int k = k0; k < k1; ++k) {
          const double m = Op[(size_t)k * D];
#pragma unroll
          for (int g = 0; g < kKlBatch; ++g) acc[g] += m * cb[g][k];
        }
#pragma unroll
        for (int g = 0; g < kKlBatch; ++g) wpart[((size_t)part * kKlBatch + g) * D + a] = acc[g];
      }
      __syncthreads();
      double pb[kKlBatch], pn[kKlBatch];
#pragma unroll
      for (int g = 0; g < kKlBatch; ++g) pb[g] = pn[g] = 0.0;
#pragma unroll
      for (int k = 0; k < (kKlBatch * 128 + kKlThreads - 1) / kKlThreads; ++k) {
        const int e = tid + k * kKlThreads;
        if (e >= nb * D) continue;
        const int g = e / D, a = e % D;
        double w;
        if (Kin > 0) {
          w = 0.0;
          for (int q = 0; q < nsplit; ++q) w += wpart[((size_t)q * kKlBatch + g) * D + a];
          if (!kKeys) w *= rsd;
        } else {
          w = cb[g][a];
        }
        const size_t gj = (size_t)bh * C + gb + g;
        if (kKeys) {
          L.kW64[gj * D + a] = w;
          L.kW32[gj * D + a] = (float)w;
          split3(w, L.kWb, (size_t)L.BH * Npg * D, ((size_t)bh * Npg + gb + g) * D + a);
        } else {
          L.qU64[gj * D + a] = w;
          L.qU32[gj * D + a] = (float)w;
          split3(w, L.qWb, (size_t)L.BH * Npg * D, ((size_t)bh * Npg + gb + g) * D + a);
        }
#pragma unroll
        for (int gg = 0; gg < kKlBatch; ++gg)
          if (gg == g) {
            pb[gg] += kKeys ? cb[g][a] * w : (L.semantic ? w * w : 0.0);
            pn[gg] += w * w;
          }
      }
      if (!kKeys && !L.semantic)  // queries (response): bias = ||nu||^2 over the key groups
        for (int e = tid; e < nb * L.Ck; e += kKlThreads) {
          const int g = e / L.Ck, j = e % L.Ck;
#pragma unroll
          for (int gg = 0; gg < kKlBatch; ++gg)
            if (gg == g) pb[gg] += cb[g][j] * cb[g][j];
        }
      // block sums of pb, pn per group: warp sums, then the warps' partials in a fixed order
#pragma unroll
      for (int g = 0; g < kKlBatch; ++g) {
        const double s1 = warp_sum(pb[g]), s2 = warp_sum(pn[g]);
        if (lane == 0) {
          s_red8[g][warp] = s1;
          s_red8[kKlBatch + g][warp] = s2;
        }
      }
      __syncthreads();
      if (tid < 2 * kKlBatch) {
        double t = 0.0;
        for (int w2 = 0; w2 < kKlWarps; ++w2) t += s_red8[tid][w2];
        s_gred[tid % kKlBatch][tid / kKlBatch] = t;
      }
      __syncthreads();
      if (tid < nb) {
        const size_t gj = (size_t)bh * C + gb + tid;
        const double bias = s_gred[tid][0];
        (kKeys ? L.kbias64 : L.qbias64)[gj] = bias;
        (kKeys ? L.kbias32 : L.qbias32)[gj] = (float)bias;
        (kKeys ? L.kwnorm : L.qwnorm)[gj] = (float)sqrt(s_gred[tid][1]);
      }
    }
  };

  // ------------------------------------------------------------- assignment of the resident tiles
  const int epi = warp >= 4 ? (warp - 4) >> 2 : -1;  // epilogue warpgroup: accumulators b with b % 2 = epi
  auto assign = [&](int it) {
    if (warp == 1 && lane == 0) {
      const uint32_t idesc2 = idesc_bf16_f32(kKlTile, A, 0, 0);
      tc_fence_after();
      for (int k = 0; k < nt; ++k) {
        const int use = it * nt + k, b = use % NACC, n = use / NACC;
        if (n >= 1 && !mbar_wait(acc_empty + b, (n - 1) & 1, &s_abort)) break;
        tc_fence_after();
        // both W terms stacked as one operand of 2 Np rows: [X W_hi | X W_mid] side by side (one
        // chain per term, added in the epilogue; the rounding bound covers both forms).  Measured
        // faster here than one chain of both terms into Np columns.
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t xd =
              sdesc_sw128(smem_u32(sX + ((size_t)k * KB + (ks >> 2)) * kKlTile * 128) + (ks & 3) * 32, 16, 1024);
          const uint64_t wd = sdesc_sw128(smem_u32(sW + (size_t)(ks >> 2) * 2 * Np * 128) + (ks & 3) * 32, 16, 1024);
          mma_ss(tmem + b * A, xd, wd, idesc2, ks > 0 ? 1u : 0u);
        }
        mma_commit(acc_full + b);
      }
    } else if (epi >= 0) {
      const int q = tid - 128 - 128 * epi;
      const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
      const float u = 1.1920929e-7f;  // 2^-23
      const float wmax = s_wmax, bmax = s_bmax;
      double jsum = 0.0;
      for (int k = 0; k < nt; ++k) {
        const int use = it * nt + k, b = use % NACC, n = use / NACC;
        if ((b & 1) != epi) continue;
        const bool okw = mbar_wait(acc_full + b, n & 1, &s_abort);
        if (!__all_sync(0xffffffffu, okw)) break;
        tc_fence_after();
        const int p = k * kKlTile + q;
        const bool valid = p < npts;
        const float m2s = -2.f * sq[p];
        auto load_dots = [&](int c0, float (&rr)[32]) {
          uint32_t hv[32], mv[32];
          tmem_ld32(tmem + lane_base + b * A + c0, hv);
          tmem_ld32(tmem + lane_base + b * A + Np + c0, mv);
          tmem_wait_ld();
#pragma unroll
          for (int kk = 0; kk < 32; ++kk) rr[kk] = __uint_as_float(hv[kk]) + __uint_as_float(mv[kk]);
        };
        float b1 = INFINITY, b2 = INFINITY;
        int i1 = -1;
        for (int c0 = 0; c0 < Np; c0 += 32) {
          float rr[32];
          load_dots(c0, rr);
          float bq[8][4];  // the biases four at a time (16-byte shared-memory loads)
#pragma unroll
          for (int k4 = 0; k4 < 8; ++k4) {
            const float4 v4 = reinterpret_cast<const float4*>(sbias + c0)[k4];
            bq[k4][0] = v4.x;
            bq[k4][1] = v4.y;
            bq[k4][2] = v4.z;
            bq[k4][3] = v4.w;
          }
#pragma unroll
          for (int kk = 0; kk < 32; ++kk) {
            const float sc = fmaf(m2s, rr[kk], bq[kk >> 2][kk & 3]);  // padded groups: bias +inf
            const bool lt = sc < b1;
            b2 = lt ? b1 : fminf(b2, sc);
            i1 = lt ? c0 + kk : i1;
            b1 = lt ? sc : b1;
          }
        }
        // the rounding bound of the two-term scores (the same as the per-iteration assignment)
        const float delta = (4.f * (2 * D + 8) * u + 4.f * 3.81469727e-6f) * xn[p] * wmax + 4.f * u * bmax;
        const bool ref = valid && !(b2 - b1 > 2.f * delta);
        int nc = 255;
        uint32_t cpk = 0;
        if (__any_sync(0xffffffffu, ref)) {
          const float thr = b1 + 2.5f * delta;
          int cnt = 0;
#pragma unroll 1
          for (int c0 = 0; c0 < Np; c0 += 32) {
            float rr[32];
            load_dots(c0, rr);
            if (ref) {
#pragma unroll
              for (int kk = 0; kk < 32; ++kk) {
                const float sc = fmaf(m2s, rr[kk], sbias[c0 + kk]);
                if (sc <= thr && c0 + kk < C) {  // padded groups are never candidates
                  if (cnt < 4) cpk |= (uint32_t)(c0 + kk) << (8 * cnt);
                  ++cnt;
                }
              }
            }
          }
          if (ref) nc = (cnt > 4 || cnt == 0) ? 255 : cnt;
        }
        tc_fence_before();
        mbar_arrive(acc_empty + b);
        if (valid) {
          lab[p] = (i1 >= 0 && i1 < C) ? i1 : 0;
          jsum += (double)b1;
          if (ref) {
            const int c0 = cpk & 0xFF, c1 = (cpk >> 8) & 0xFF, c2 = (cpk >> 16) & 0xFF, c3 = cpk >> 24;
            const int slot = atomicAdd(&s_nflag, 1);
            flags[slot] = make_int4(p, __float_as_int(b1), nc | (c0 << 8) | (c1 << 18), c2 | (c3 << 16));
          }
        }
      }
      jsum = warp_sum(jsum);
      if (lane == 0) s_red[warp] = jsum;
    }
  };

  // ------------------------------------------------------------- fp64 re-decision of flagged points
  auto x_at = [&](int p, int a) -> const __nv_bfloat16* {  // element a of resident point p (swizzled)
    const int t = p >> 7, row = p & 127, kb = a >> 6, w = a & 63;
    return (const __nv_bfloat16*)(sX + ((size_t)t * KB + kb) * kKlTile * 128 + row * 128 +
                                  ((((w >> 3) ^ (row & 7)) << 4) | ((w & 7) << 1)));
  };
  auto redecide = [&](double& jcorr) {
    const int nflag = s_nflag;
    double* xs = xs_all + warp * 128;
    const double* W64 = (kKeys ? L.kW64 : L.qU64) + (size_t)bh * C * D;
    const double* B64 = (kKeys ? L.kbias64 : L.qbias64) + (size_t)bh * C;
    for (int li = warp; li < nflag; li += kKlWarps) {
      const int4 en = flags[li];
      const int p = en.x;
      for (int a = lane; a < D; a += 32) xs[a] = (double)__bfloat162float(*x_at(p, a));
      __syncwarp();
      int best;
      double bv;
      const int nc = en.z & 0xFF;
      if (nc <= 4) {
        int cand[4] = {(en.z >> 8) & 0x3FF, (en.z >> 18) & 0x3FF, en.w & 0xFFFF, (en.w >> 16) & 0xFFFF};
        double scale = 1.0;
        if (!kKeys && !L.semantic) {
          double xl[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) xl[k] = lane + 32 * k < D ? xs[lane + 32 * k] : 0.0;
          scale = query_scale_fp64(L.Gc + (size_t)bh * D * D, xs, xl, D);
        }
        redecide_candidates<true>(xs, D, W64, B64, scale, cand, nc, best, bv);
      } else {
        redecide_fp64<kKeys, true>(L, bh, xs, D, C, W64, B64, best, bv);
      }
      if (lane == 0) {
        lab[p] = (best >= 0 && best < C) ? best : 0;
        jcorr += bv - (double)__int_as_float(en.y);
      }
      __syncwarp();
    }
  };

  // ------------------------------------------------------------- partial group sums of the CTA
  auto group_sums = [&]() {
    for (int j = tid; j <= C; j += kKlThreads) cursor[j] = 0;
    __syncthreads();
    // histogram: lanes holding the same label add once (labels are spatially coherent)
    for (int p0 = 0; p0 < npts; p0 += kKlThreads) {
      const int p = p0 + tid;
      const bool v = p < npts;
      const int g = v ? lab[p] : -1;
      const unsigned act = __ballot_sync(0xffffffffu, v);
      if (v) {
        const unsigned same = __match_any_sync(act, g);
        if (lane == __ffs(same) - 1) atomicAdd(&cursor[g], __popc(same));
      }
    }
    __syncthreads();
    if (warp == 0) {  // exclusive prefix over the groups
      int run = 0;
      for (int c0 = 0; c0 < C; c0 += 32) {
        const int j = c0 + lane;
        const int v = j < C ? cursor[j] : 0;
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        if (j < C) {
          offs[j] = run + x - v;
          cursor[j] = run + x - v;
        }
        run += __shfl_sync(0xffffffffu, x, 31);
      }
      if (lane == 0) offs[C] = run;
    }
    __syncthreads();
    for (int p0 = 0; p0 < npts; p0 += kKlThreads) {  // scatter: one atomic per label per warp
      const int p = p0 + tid;
      const bool v = p < npts;
      const int g = v ? lab[p] : -1;
      const unsigned act = __ballot_sync(0xffffffffu, v);
      if (v) {
        const unsigned same = __match_any_sync(act, g);
        const int leader = __ffs(same) - 1;
        int base = 0;
        if (lane == leader) base = atomicAdd(&cursor[g], __popc(same));
        base = __shfl_sync(same, base, leader);
        order[base + __popc(same & ((1u << lane) - 1))] = p;
      }
    }
    __syncthreads();
    // Balanced sums.  Warp w takes the sorted positions [s0, s1) = [w n / 12, (w + 1) n / 12);
    // lanes run over the dimensions (d = 64: two per lane, d = 128: four), four rows in flight.
    // A run (one group's points) that lies inside the slice is written to the CTA's partial sums
    // at once.  A run that crosses a slice boundary leaves its piece in shared memory: slot 0 for
    // the run the slice starts in when it began before s0, slot 1 for the run the slice ends in
    // when it goes on past s1.  After a barrier the pieces of each crossing run are added in warp
    // order, and absent groups get zeros.
    const int per = D / 32, a0 = lane * per;
    double* pieces = xs_all;  // [kKlWarps][2][D]: the re-decision staging, free here
    auto slice_lo = [&](int w) { return (int)((long long)npts * w / kKlWarps); };
    auto add_row = [&](double (&ac)[4], int p) {
      const double sc = kKeys ? 1.0 : sig[p];
      const __nv_bfloat16* xp = x_at(p, a0);  // `per` consecutive dimensions of one 16-byte piece
      if (per == 2) {
        const uint32_t v = *(const uint32_t*)xp;
        ac[0] = fma(bf16_bits_to_f64(v & 0xFFFFu), sc, ac[0]);
        ac[1] = fma(bf16_bits_to_f64(v >> 16), sc, ac[1]);
      } else {
        const uint2 v = *(const uint2*)xp;
        ac[0] = fma(bf16_bits_to_f64(v.x & 0xFFFFu), sc, ac[0]);
        ac[1] = fma(bf16_bits_to_f64(v.x >> 16), sc, ac[1]);
        ac[2] = fma(bf16_bits_to_f64(v.y & 0xFFFFu), sc, ac[2]);
        ac[3] = fma(bf16_bits_to_f64(v.y >> 16), sc, ac[3]);
      }
    };
    const int s0 = slice_lo(warp), s1 = slice_lo(warp + 1);
    if (s0 < s1) {
      int g = lab[order[s0]];
      while (true) {
        const int q0 = offs[g], q1 = offs[g + 1];
        const int b0 = max(q0, s0), b1 = min(q1, s1);
        double acc[4][4];
#pragma unroll
        for (int u2 = 0; u2 < 4; ++u2)
#pragma unroll
          for (int k = 0; k < 4; ++k) acc[u2][k] = 0.0;
        int qq = b0;
        for (; qq + 4 <= b1; qq += 4) {
          const int pa = order[qq], pb2 = order[qq + 1], pc = order[qq + 2], pd = order[qq + 3];
          add_row(acc[0], pa);
          add_row(acc[1], pb2);
          add_row(acc[2], pc);
          add_row(acc[3], pd);
        }
        if (qq < b1) add_row(acc[0], order[qq]);  // the last 0..3 rows
        if (qq + 1 < b1) add_row(acc[1], order[qq + 1]);
        if (qq + 2 < b1) add_row(acc[2], order[qq + 2]);
        const bool inside = q0 >= s0 && q1 <= s1;
        double* dst = inside ? L.klp_sum + ((hc + r) * C + g) * D + a0 : pieces + ((size_t)warp * 2 + (q0 < s0 ? 0 : 1)) * D + a0;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (k < per) {
            const double v = (acc[0][k] + acc[1][k]) + (acc[2][k] + acc[3][k]);
            if (inside) __stcg(dst + k, v);
            else dst[k] = v;
          }
        if (inside && lane == 0) __stcg(L.klp_cnt + (hc + r) * C + g, q1 - q0);
        if (b1 >= s1) break;
        g = lab[order[b1]];  // the next group present (the sort is by group)
      }
    }
    __syncthreads();
    for (int g = warp; g < C; g += kKlWarps) {
      const int q0 = offs[g], q1 = offs[g + 1];
      int wf = 0, wl = 0;  // slices holding the run's first and last positions
      for (int w2 = 1; w2 < kKlWarps; ++w2) {
        if (slice_lo(w2) <= q0) wf = w2;
        if (slice_lo(w2) <= q1 - 1) wl = w2;
      }
      if (q1 > q0 && wf == wl) continue;  // inside one slice: written by its warp
      double v[4] = {0.0, 0.0, 0.0, 0.0};
      if (q1 > q0)
        for (int w2 = wf; w2 <= wl; ++w2) {
          if (slice_lo(w2) == slice_lo(w2 + 1)) continue;  // an empty slice (fewer points than warps)
          const double* pc = pieces + ((size_t)w2 * 2 + (q0 < slice_lo(w2) ? 0 : 1)) * D + a0;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (k < per) v[k] += pc[k];
        }
      double* dst = L.klp_sum + ((hc + r) * C + g) * D + a0;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (k < per) __stcg(dst + k, v[k]);
      if (lane == 0) __stcg(L.klp_cnt + (hc + r) * C + g, q1 - q0);
    }
  };

  // ------------------------------------------------------------- partial sums by label changes
  // From the second iteration of the launch on, the CTA's partial sums and counts (its own
  // slice of klp_sum / klp_cnt, kept from the iteration before) move only by the points whose
  // label changed: the point leaves its old group's sum and joins its new group's (fp64 atomics,
  // one warp per point, lanes over the dimensions).  Key sums of bf16 inputs are exact in fp64,
  // so this equals summing every point again; query sums (scaled by 1/rms) agree to rounding.
  // `prev` (the sort's order array, free after the first iteration) holds the labels of the
  // iteration before; the changed points are listed in the re-decision entries' space.
  auto delta_sums = [&]() {
    int* prev = order;
    int* changed = (int*)flags;
    if (tid == 0) s_nchg = 0;
    __syncthreads();
    for (int p0 = 0; p0 < npts; p0 += kKlThreads) {
      const int p = p0 + tid;
      const bool ch = p < npts && lab[p] != prev[p];
      const unsigned m = __ballot_sync(0xffffffffu, ch);
      int base = 0;
      if (lane == 0 && m) base = atomicAdd(&s_nchg, __popc(m));
      base = __shfl_sync(0xffffffffu, base, 0);
      if (ch) changed[base + __popc(m & ((1u << lane) - 1))] = p;
    }
    __syncthreads();
    const int nchg = s_nchg;
    const int per = D / 32, a0 = lane * per;
    double* part = L.klp_sum + (hc + r) * C * D;
    int* pcnt = L.klp_cnt + (hc + r) * C;
    for (int i = warp; i < nchg; i += kKlWarps) {
      const int p = changed[i];
      const int g0 = prev[p], g1 = lab[p];
      const double sc = kKeys ? 1.0 : sig[p];
      const __nv_bfloat16* xp = x_at(p, a0);
      double v[4];
      if (per == 2) {
        const uint32_t u = *(const uint32_t*)xp;
        v[0] = bf16_bits_to_f64(u & 0xFFFFu) * sc;
        v[1] = bf16_bits_to_f64(u >> 16) * sc;
        v[2] = v[3] = 0.0;
      } else {
        const uint2 u = *(const uint2*)xp;
        v[0] = bf16_bits_to_f64(u.x & 0xFFFFu) * sc;
        v[1] = bf16_bits_to_f64(u.x >> 16) * sc;
        v[2] = bf16_bits_to_f64(u.y & 0xFFFFu) * sc;
        v[3] = bf16_bits_to_f64(u.y >> 16) * sc;
      }
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (k < per) {
          atomicAdd(part + (size_t)g0 * D + a0 + k, -v[k]);
          atomicAdd(part + (size_t)g1 * D + a0 + k, v[k]);
        }
      if (lane == 0) {
        atomicAdd(pcnt + g0, -1);
        atomicAdd(pcnt + g1, 1);
      }
    }
    __syncthreads();  // every warp has read its points' previous labels
    for (int i = tid; i < nchg; i += kKlThreads) prev[changed[i]] = lab[changed[i]];
  };

  // ------------------------------------------------------------- head-wide W into shared memory
  auto load_weights = [&]() {
    const __nv_bfloat16* Wb = kKeys ? L.kWb : L.qWb;
    const size_t plane = (size_t)L.BH * Npg * D;
    const int nchunk = KB * 2 * Np * 8;  // 16-byte pieces of both terms
    const float* B32 = (kKeys ? L.kbias32 : L.qbias32) + (size_t)bh * C;
    const float* WN = (kKeys ? L.kwnorm : L.qwnorm) + (size_t)bh * C;
    // the bias of group tid and (warp 0) the inputs of the bound's maxima, loaded with W
    const float bj = tid < C ? __ldcg(B32 + tid) : INFINITY;
    float bmx[4], wmx[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int j = lane + 32 * k;
      const bool on = warp == 0 && j < C;
      bmx[k] = on ? fabsf(__ldcg(B32 + j)) : 0.f;
      wmx[k] = on ? __ldcg(WN + j) : 0.f;
    }
#pragma unroll 4
    for (int e = tid; e < nchunk; e += kKlThreads) {
      const int c = e & 7, n = (e >> 3) % Np, rest = (e >> 3) / Np, term = rest & 1, kb = rest >> 1;
      const uint4 v = n < Npg ? __ldcg((const uint4*)(Wb + term * plane + ((size_t)bh * Npg + n) * D + kb * 64 + c * 8))
                              : make_uint4(0u, 0u, 0u, 0u);  // rows past the global padding
      *(uint4*)(sW + ((size_t)(kb * 2 + term) * Np + n) * 128 + ((c ^ (n & 7)) << 4)) = v;
    }
    if (tid < Np) sbias[tid] = bj;  // padded groups: +inf (Np <= 128 < the block's threads)
    if (warp == 0) {  // maxima of the rounding bound over all groups (C <= 128)
      float wm = fmaxf(fmaxf(wmx[0], wmx[1]), fmaxf(wmx[2], wmx[3]));
      float bm = fmaxf(fmaxf(bmx[0], bmx[1]), fmaxf(bmx[2], bmx[3]));
      wm = warp_max(wm);
      bm = warp_max(bm);
      if (lane == 0) {
        s_wmax = wm;
        s_bmax = bm;
      }
    }
    fence_proxy_async_smem();  // generic writes of W before the tensor core reads them
    if (tid == 0) s_nflag = 0;
    __syncthreads();
  };

  // ================================================================ the loop
  bool ok = true;
  centroid_step(false, true);  // weights of the first assignment from the initial centroids
  ok = head_barrier(hbar, G * ++nbar, gabort, &s_abort, blim);
  if (ok && !mbar_wait(x_full, 0, &s_abort)) ok = false;  // the resident tiles have landed
  ok = !__syncthreads_or(!ok);
  int it = 0;
  for (; ok; ++it) {
    load_weights();
    assign(it);
    __syncthreads();
    if (s_abort) break;
    double jcorr = 0.0;
    redecide(jcorr);
    if (lane == 0) s_redc[warp] = jcorr;
    __syncthreads();  // labels final; the objective's pieces are in s_red (epilogue) and s_redc
    if (tid == 0) {   // summed in a fixed order
      double js = 0.0;
      for (int w = 4; w < kKlWarps; ++w) js += s_red[w];
      for (int w = 0; w < kKlWarps; ++w) js += s_redc[w];
      s_J = js;
    }
    if (it == 0) {
      group_sums();
      __syncthreads();
      for (int p = tid; p < npts; p += kKlThreads) order[p] = lab[p];  // the labels the next deltas start from
    } else {
      delta_sums();
    }
    __syncthreads();
    if (tid == 0) {
      __stcg(L.klp_J + hc + r, s_J);
      if (s_nflag) atomicAdd((kKeys ? L.krefined : L.qrefined) + bh, s_nflag);
    }
    if (!head_barrier(hbar, G * ++nbar, gabort, &s_abort, blim)) break;
    // the objective of this assignment: warp 0 loads the head's G shares at once (lane q takes
    // CTAs q, q + 32, ...) and adds them in a fixed order, so every CTA of the head gets the same
    // value
    if (warp == 0) {
      double js = 0.0;
      for (int q = lane; q < G; q += 32) js += __ldcg(L.klp_J + hc + q);
      js = warp_sum(js);
      if (lane == 0) s_J = T0 + js;
    }
    __syncthreads();
    const double Jc = s_J;
    if (r == 0 && tid == 0) Jarr[it] = Jc;
    const int nx = it + 1;  // the stop test before assignment nx
    const bool stop = nx >= P.iters || (nx >= 2 && L.km_tol >= 0.f && Jprev - Jc <= (double)L.km_tol * Jprev);
    Jprev = Jc;
    centroid_step(true, !stop);
    if (stop) {
      if (r == 0 && tid == 0) L.stop_at[bh * 2 + (kKeys ? 0 : 1)] = nx;
      break;
    }
    if (!head_barrier(hbar, G * ++nbar, gabort, &s_abort, blim)) break;
  }
  __syncthreads();
  {  // an aborted loop leaves label 0 (a valid group) on every point: later kernels index by it
    int* labels = kKeys ? L.klabel : L.qlabel;
    const bool good = !s_abort;
    for (int p = tid; p < npts; p += kKlThreads) labels[row0 + p] = good ? lab[p] : 0;
  }
  if (tid == 0) {
    if (s_abort) {
      atomicCAS(L.status, kDevOk, kDevTimeout);
      mbar_wait_drain(x_full, 0);  // never leave with the tile copies in flight
    }
  }
  if (warp == 1 && lane == 0) {  // every MMA issued has completed before TMEM is released
    mma_commit(mma_done);
    mbar_wait_drain(mma_done, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}

// ----------------------------------------------------------------------------------- host
// CTAs per head and resident tiles per CTA of the loop on a device with `ctas` co-resident CTAs
// (one per SM); 0 when the call does not qualify: bf16 inputs, at most 128 groups (padded to a
// multiple of 32 in shared memory, so that both W terms form one MMA operand of at most 256
// rows), the query step with at most kKlMaxKGroups key groups, and every CTA's tiles in shared
// memory.
int km_loop_ctas_per_head(int BH, int N, int d, int dtype, int C, int Ck, bool keys, int ctas, int* cap_out) {
  if (dtype != SPARSEPR_BF16 || (d != 64 && d != 128) || BH < 1) return 0;
  const int Np = ((C + 15) / 16 * 16 + 31) & ~31;
  if (Np > 128) return 0;
  if (!keys && Ck > kKlMaxKGroups) return 0;
  const int tph = (N + kKlTile - 1) / kKlTile;
  int G = std::min(tph, ctas / BH);
  if (G < 1) return 0;
  const int cap = (tph + G - 1) / G;
  G = (tph + cap - 1) / cap;  // the fewest CTAs with that many tiles each: fewer partials per group
  if (km_loop_smem(d, Np, C, cap) + kKlStaticSmem > (size_t)227 * 1024) return 0;
  if (cap_out) *cap_out = cap;
  return G;
}

static int device_sms() {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 1;
  }
  return sms;
}

// The launch shape of one side's whole loop on the current device: CTAs per head, resident tiles
// per CTA and shared memory, or false when the side does not qualify (shape, workspace, test
// hook) or its CTAs could not all be co-resident (cooperative launch support, occupancy).
static bool km_loop_config(const Layout& L, bool keys, int& G, int& cap, size_t& smem) {
  if (!L.klp_sum || L.km_steps) return false;
  const int C = keys ? L.Ck : L.Cq;
  cap = 0;
  G = km_loop_ctas_per_head(L.BH, L.N, L.d, L.dtype, C, L.Ck, keys, std::min(device_sms(), kKmLoopMaxCtas), &cap);
  if (G < 1 || G > L.klp_G) return false;
  int dev = 0, coop = 0;
  cudaGetDevice(&dev);
  if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess || !coop) {
    (void)cudaGetLastError();  // a failed query must not read as a failed launch later
    return false;
  }
  const int Np = ((keys ? L.Ckp : L.Cqp) + 31) & ~31;
  smem = km_loop_smem(L.d, Np, C, cap);
  auto kern = keys ? kmeans_loop_kernel<true> : kmeans_loop_kernel<false>;
  // A failure here falls back to the per-iteration launches, so its error must not linger for
  // their launch checks to report.
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kKlThreads, smem) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  return occ >= 1 && (long long)occ * device_sms() >= (long long)L.BH * G;
}

bool km_loop_supported(const Layout& L, bool keys) {
  int G, cap;
  size_t smem;
  return km_loop_config(L, keys, G, cap, smem);
}

sparsepr_status launch_kmeans_loop(const Layout& L, bool keys, const void* X, int iters, cudaStream_t st) {
  int G, cap;
  size_t smem;
  if (!km_loop_config(L, keys, G, cap, smem)) return SPARSEPR_ERR_UNSUPPORTED;
  auto kern = keys ? kmeans_loop_kernel<true> : kmeans_loop_kernel<false>;
  CUtensorMap mX;
  if (!make_tmap_bf16(&mX, X, (long long)L.BH * L.N, L.d, kKlTile)) return SPARSEPR_ERR_CUDA;
  // head barrier counters and the abort flag start at zero
  cudaMemsetAsync(L.klp_bar, 0, (size_t)(L.BH + 1) * sizeof(unsigned), st);
  KmLoopArgs P{G, cap, iters};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // all CTAs co-resident: they wait on one another
  attr[0].val.cooperative = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L.BH * G);
  cfg.blockDim = dim3(kKlThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kern, mX, L, P);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  SPR_LAUNCH_CHECK();
  return SPARSEPR_OK;
}

}  // namespace sparsepr
