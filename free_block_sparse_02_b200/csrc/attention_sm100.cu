// Block-sparse attention and dense probe-row attention on the 5th-generation tensor cores
// (tcgen05, TMEM accumulators, TMA tile loads), bf16 inputs, fp32 accumulation and softmax.
//
// "Partition the Support, Reconstruct the Residual" (arXiv 2608.18484), abstract: attention is
// evaluated for the selected group pairs only (every query of a query group attends to the keys
// of the key groups its group keeps, softmax over the retained keys only), and exactly, over
// all keys, for the few probe rows.
//
// Work item = 256 query rows of one query group (block-sparse pass) or of one head's probe rows
// (dense pass), as two 128-row MMA tiles Q0, Q1 that share every KV tile.  The keys are the
// concatenation of the kept key groups' rows in the group-permuted K/V, streamed in 128-key
// tiles assembled from 64-row TMA boxes, so a kept key group costs at most 63 padded (masked)
// rows wherever it starts.
//
// CTA of 384 threads: warp 0 = TMA producer, warp 1 = MMA issuer (and TMEM owner), warps 4..7
// = softmax of Q0, warps 8..11 = softmax of Q1 (thread t of a group owns query row t of its tile:
// TMEM lane t).  TMEM (512 columns): S0 [0,128), S1 [128,256), O0 at 256, O1 at 256 + d.
// P_t (bf16, packed) overwrites the first 64 columns of S_t and feeds O_t += P_t V from TMEM.
// The MMA warp issues  PV0(j), S0(j+1), PV1(j), S1(j+1)  so each softmax warpgroup works while
// the tensor core runs the other tile's two MMAs (ping-pong).  tcgen05.mma operations of one
// thread execute in issue order, which orders S_t(j+1) after the PV_t(j) that reads P_t(j).
// Online softmax in base 2 with lazy rescaling: the running max only moves (and O is rescaled
// in TMEM) when a tile's max exceeds it by more than 8 (a factor 256).
// Every mbarrier wait is bounded; a wait that gives up sets the device status to
// SPARSEPR_ERR_TIMEOUT and the CTA drains its copies, frees TMEM and exits.
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace sparsepr {

using namespace sm100;

constexpr int kTcTileM = 128;   // query rows per MMA tile
constexpr int kTcTileN = 128;   // keys per KV tile (MMA N of S, K of PV)
constexpr int kSubRows = 64;    // rows per TMA box of K/V (64: 1.5% faster than 32 at the 13B-DiT
                                // shape, which was 3% faster than 16)
constexpr int kSubPerTile = kTcTileN / kSubRows;
constexpr int kTmemCols = 512;
constexpr int kRegsCtl = 152;      // registers per thread of warps 0-3 (TMA, MMA, two idle warps)
constexpr int kRegsSoftmax = 176;  // ... of the two softmax warpgroups
static_assert(128 * kRegsCtl + 256 * kRegsSoftmax <= 384 * 168, "register split above the launch's registers");
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kExpPolyEvery = 0;           // in tiles whose keys are all real, 1 in n exponential
                                           // pairs runs on the FMA pipe (0: none)

// 2^x for a pair of x <= kRescaleThreshold on the FMA pipe (f32x2), for x >= -125 (smaller x
// give 2^-125 instead of 0: far below the bf16 rounding of P and of any row sum, which is
// >= 1).  Cody-Waite style reduction x = n + f with n = round(x) (adding 1.5 * 2^23 leaves n in
// the low mantissa bits) and f in [-1/2, 1/2], then a cubic in f fitted to 2^f by least squares
// on relative error at Chebyshev nodes with Lawson reweighting (max relative error 7.5e-5 in fp32
// Horner evaluation, 26 times below the bf16 rounding of P), and n added to the exponent field.
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x) {
  float x0, x1;
  f2_unpack(x, x0, x1);
  const uint64_t xc = f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t t = f2_add(xc, f2_pack(12582912.f, 12582912.f));
  const uint64_t n = f2_add(t, f2_pack(-12582912.f, -12582912.f));
  const uint64_t f = f2_fma(n, f2_pack(-1.f, -1.f), xc);
  uint64_t p = f2_fma(f2_pack(0.05517166853f, 0.05517166853f), f, f2_pack(0.24261114001f, 0.24261114001f));
  p = f2_fma(p, f, f2_pack(0.69326096773f, 0.69326096773f));
  p = f2_fma(p, f, f2_pack(0.99992805719f, 0.99992805719f));
  float p0, p1, t0, t1;
  f2_unpack(p, p0, p1);
  f2_unpack(t, t0, t1);
  return f2_pack(__int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23)),
                 __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23)));
}

// Exponentials of 64 scores of a row of S (fp32 bits) into 32 packed bf16 pairs, adding them to
// the row sum.  kFull: every key of the tile is real (no -inf scores), so the polynomial pairs
// may run; otherwise every exponential is on the special-function unit, where 2^-inf = 0
// exactly.
template <bool kFull>
__device__ __forceinline__ void exp_half(const uint32_t (&sv)[64], float scale2, float neg_m, uint32_t (&pk)[32],
                                         uint64_t (&acc)[2]) {
  const uint64_t sc = f2_pack(scale2, scale2), nm = f2_pack(neg_m, neg_m);
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const uint64_t x = f2_fma(f2_pack(__uint_as_float(sv[2 * k]), __uint_as_float(sv[2 * k + 1])), sc, nm);
    uint64_t e;
    if (kFull && kExpPolyEvery > 0 && (k % (kExpPolyEvery > 0 ? kExpPolyEvery : 1)) == kExpPolyEvery - 1) {
      e = exp2_poly2(x);
    } else {
      float x0, x1;
      f2_unpack(x, x0, x1);
      e = f2_pack(ex2(x0), ex2(x1));
    }
    acc[k & 1] = f2_add(acc[k & 1], e);
    float p0, p1;
    f2_unpack(e, p0, p1);
    pk[k] = pack_bf16x2(p0, p1);
  }
}

static_assert(kAttnTileMTc == 2 * kTcTileM, "a work item is two MMA tiles");

template <int D>
struct TcCfg {
  static constexpr int kKB = D / 64;                    // 64-column (128-byte) blocks of a row
  static constexpr int kKS = D == 64 ? 4 : 3;           // K stages
  static constexpr int kVS = D == 64 ? 4 : 2;           // V stages (K runs one tile ahead of V)
  static constexpr int kQTileBytes = kTcTileM * D * 2;
  static constexpr int kQBytes = 2 * kQTileBytes;
  static constexpr int kKVTileBytes = kTcTileN * D * 2;  // one K or V tile
  static constexpr int kSmemTiles = kQBytes + (kKS + kVS) * kKVTileBytes;
  static constexpr int kSmemBytes = kSmemTiles + 1024 /* align */ + 512 /* barriers, tile validity */;
};

// The keys of a work item: probe items attend to all N keys of the head (one segment);
// sparse items to the kept key groups' segments of the group-permuted K/V (offset, length),
// read from the route list and the group offsets in global memory.
struct Segs {
  const int* list;  // kept key groups (sparse items)
  const int* koff;  // key-group offsets of the head
  int n;            // segments
  int probe_len;    // > 0: probe item, one segment [0, probe_len)
  __device__ __forceinline__ int2 at(int i) const {
    if (probe_len > 0) return make_int2(0, probe_len);
    const int j = list[i];
    const int o = koff[j];
    return make_int2(o, koff[j + 1] - o);
  }
};

struct SegState {
  int seg;   // index of the current segment
  int off;   // rows already consumed in it
  int2 cur;  // the current segment (offset, length)
};

// Next KV tile: row of each kSubRows-row box (global row of the 2D [BH*N, d] view) and its valid
// row count (0 = box not used; it is then loaded from past the end of the tensor, all zeros).
__device__ __forceinline__ void next_tile(SegState& s, const Segs& sg, int row_base, int oob_row,
                                          int (&rows)[kSubPerTile], int (&valid)[kSubPerTile]) {
#pragma unroll
  for (int b = 0; b < kSubPerTile; ++b) {
    while (s.seg < sg.n && s.off >= s.cur.y) {
      ++s.seg;
      s.off = 0;
      if (s.seg < sg.n) s.cur = sg.at(s.seg);
    }
    if (s.seg < sg.n) {
      rows[b] = row_base + s.cur.x + s.off;
      valid[b] = min(kSubRows, s.cur.y - s.off);
      s.off += kSubRows;
    } else {
      rows[b] = oob_row;
      valid[b] = 0;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(384, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQprobe,
                   const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, Layout L,
                   int probe_items_per_head, int sparse_items_per_head) {
  pdl_entry();
  using C = TcCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = smem;                            // tile t at t * kQTileBytes
  uint8_t* sK = smem + C::kQBytes;               // K stage s at s * kKVTileBytes
  uint8_t* sV = sK + C::kKS * C::kKVTileBytes;   // V stage s at s * kKVTileBytes
  uint64_t* bars = (uint64_t*)(smem + C::kSmemTiles);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + C::kKS;
  uint64_t* v_full = k_empty + C::kKS;
  uint64_t* v_empty = v_full + C::kVS;
  uint64_t* s_full = v_empty + C::kVS;       // [2] per query tile
  uint64_t* p_full = s_full + 2;             // [2]
  uint64_t* o_bar = p_full + 2;              // [2]
  uint64_t* mma_done = o_bar + 2;
  uint32_t* tmem_slot = (uint32_t*)(mma_done + 1);
  // valid rows of each box of the tile held in V stage s, written by the producer before
  // the V copy (the softmax reads it after waiting on that copy)
  int* tvalid = (int*)(tmem_slot + 2);       // [kVS][kSubPerTile]
  __shared__ int s_nseg, s_ntiles, s_qrow0, s_rows0, s_rows1, s_mode, s_bh;
  __shared__ volatile int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Every wait below gives up after the default limit, or after L.attn_wait_limit cycles when
  // the test hook of the timeout path sets one; a wait that gives up sets s_abort.
  const long long wlim = L.attn_wait_limit;
  auto wt = [wlim](uint64_t* bar, uint32_t parity) -> bool {
    return wlim > 0 ? mbar_wait_limit(bar, parity, &s_abort, wlim) : mbar_wait(bar, parity, &s_abort);
  };

  // ---- work item
  if (tid == 0) {
    const int nprobe_items = L.BH * probe_items_per_head;
    int item = blockIdx.x;
    int mode, bh, qrow0 = 0, end = 0;
    if (item < nprobe_items) {
      mode = 1;
      bh = item / probe_items_per_head;
      qrow0 = (item % probe_items_per_head) * kAttnTileMTc;
      end = L.P;
    } else {
      item -= nprobe_items;
      mode = 0;
      bh = item / sparse_items_per_head;
      const int x = item % sparse_items_per_head;
      const int* toff = L.tile_off + (size_t)bh * (L.Cq + 1);
      if (x < toff[L.Cq]) {
        int lo = 0, hi = L.Cq - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (toff[mid] <= x) lo = mid;
          else hi = mid - 1;
        }
        const int* qoff = L.qoff + (size_t)bh * (L.Cq + 1);
        qrow0 = qoff[lo] + (x - toff[lo]) * kAttnTileMTc;
        end = qoff[lo + 1];
        s_nseg = lo;  // group id, replaced by the segment count below
      }
    }
    s_mode = mode;
    s_bh = bh;
    s_qrow0 = qrow0;
    s_rows0 = min(kTcTileM, end - qrow0);
    s_rows1 = min(kTcTileM, end - qrow0 - kTcTileM);
    s_abort = 0;
  }
  __syncthreads();
  if (s_rows0 <= 0) return;  // uniform: no barrier, TMEM or copy has been touched yet
  const int mode = s_mode, bh = s_bh;
  const int ntq = s_rows1 > 0 ? 2 : 1;
  const int g_item = s_nseg;  // sparse items: the query group
  __syncthreads();
  Segs sg;
  sg.probe_len = mode == 1 ? L.N : 0;
  sg.list = L.route_list + ((size_t)bh * L.Cq + (mode == 1 ? 0 : g_item)) * L.Ck;
  sg.koff = L.koff + (size_t)bh * (L.Ck + 1);
  sg.n = mode == 1 ? 1 : L.route_cnt[(size_t)bh * L.Cq + g_item];
  if (tid == 0) {
    int nsub = 0;
    for (int i = 0; i < sg.n; ++i) nsub += (sg.at(i).y + kSubRows - 1) / kSubRows;
    s_ntiles = (nsub + kSubPerTile - 1) / kSubPerTile;
    mbar_init(q_full, 1);
    for (int s = 0; s < C::kKS; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
    }
    for (int s = 0; s < C::kVS; ++s) {
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(s_full + t, 1);
      mbar_init(p_full + t, 128);
      mbar_init(o_bar + t, 1);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int ntiles = s_ntiles, qrow0 = s_qrow0;
  const int row_base = bh * L.N;   // first row of this head in the 2D K/V view
  const int oob_row = L.BH * L.N;  // a box starting here is entirely zero-filled
  // registers: the TMA / MMA warpgroup gives a share to the two softmax warpgroups, which hold a
  // whole row of S in registers (128 x kRegsCtl + 256 x kRegsSoftmax = 384 x 168, the launch's)
  if (warp < 4)
    regs_release<kRegsCtl>();
  else
    regs_take<kRegsSoftmax>();

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0 && ntiles > 0) {
      const CUtensorMap* qm = mode == 1 ? &tmQprobe : &tmQ;
      prefetch_tmap(qm);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(q_full, ntq * C::kQTileBytes);
      const int qy = (mode == 1 ? bh * L.P : bh * L.N) + qrow0;
      for (int t = 0; t < ntq; ++t)
#pragma unroll
        for (int kb = 0; kb < C::kKB; ++kb)
          tma_load_2d(sQ + t * C::kQTileBytes + kb * kTcTileM * 128, qm, q_full, kb * 64, qy + t * kTcTileM);
      // K(0), K(1), V(0), K(2), V(1), ...: K runs one tile ahead of V
      SegState st{0, 0, sg.n > 0 ? sg.at(0) : make_int2(0, 0)};
      int rows[kSubPerTile], valid[kSubPerTile], prows[kSubPerTile], pvalid[kSubPerTile];
      int nk = 0, nv = 0;  // K and V tiles issued
      auto load_k = [&](int i) -> bool {
        const int s = i % C::kKS;
        if (!wt(k_empty + s, ((i / C::kKS) & 1) ^ 1)) return false;
        uint8_t* dst = sK + s * C::kKVTileBytes;
        mbar_arrive_expect_tx(k_full + s, C::kKVTileBytes);
#pragma unroll
        for (int b = 0; b < kSubPerTile; ++b)
#pragma unroll
          for (int kb = 0; kb < C::kKB; ++kb)
            tma_load_2d(dst + kb * kTcTileN * 128 + b * kSubRows * 128, &tmK, k_full + s, kb * 64, rows[b]);
        ++nk;
        return true;
      };
      auto load_v = [&](int i) -> bool {
        const int s = i % C::kVS;
        if (!wt(v_empty + s, ((i / C::kVS) & 1) ^ 1)) return false;
#pragma unroll
        for (int b = 0; b < kSubPerTile; ++b) tvalid[s * kSubPerTile + b] = pvalid[b];
        uint8_t* dst = sV + s * C::kKVTileBytes;
        mbar_arrive_expect_tx(v_full + s, C::kKVTileBytes);  // (release: tvalid is visible to its waiters)
#pragma unroll
        for (int b = 0; b < kSubPerTile; ++b)
#pragma unroll
          for (int kb = 0; kb < C::kKB; ++kb)
            tma_load_2d(dst + kb * kTcTileN * 128 + b * kSubRows * 128, &tmV, v_full + s, kb * 64, prows[b]);
        ++nv;
        return true;
      };
      bool okp = true;
      for (int i = 0; okp && i < ntiles; ++i) {
        next_tile(st, sg, row_base, oob_row, rows, valid);
        okp = load_k(i);
        if (okp && i > 0) okp = load_v(i - 1);
#pragma unroll
        for (int b = 0; b < kSubPerTile; ++b) {
          prows[b] = rows[b];
          pvalid[b] = valid[b];
        }
      }
      if (okp && ntiles > 0) load_v(ntiles - 1);
      // drain: never leave with copies in flight into this CTA's shared memory
      mbar_wait_drain(q_full, 0);
      for (int i = max(0, nk - C::kKS); i < nk; ++i) mbar_wait_drain(k_full + (i % C::kKS), (i / C::kKS) & 1);
      for (int i = max(0, nv - C::kVS); i < nv; ++i) mbar_wait_drain(v_full + (i % C::kVS), (i / C::kVS) & 1);
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0 && ntiles > 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kTcTileM, kTcTileN, 0, 0);
      const uint32_t idesc_o = idesc_bf16_f32(kTcTileM, D, 0, 1);
      const uint32_t q_addr = smem_u32(sQ);
      auto issue_s = [&](int t, int j) {  // S_t(j) = Q_t K_j^T
        const uint32_t k_addr = smem_u32(sK + (j % C::kKS) * C::kKVTileBytes);
        const uint32_t qa = q_addr + t * C::kQTileBytes;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t koff = (ks >> 2) * (kTcTileN * 128) + (ks & 3) * 32;
          const uint32_t qoff = (ks >> 2) * (kTcTileM * 128) + (ks & 3) * 32;
          mma_ss(tmem + t * 128, sdesc_sw128(qa + qoff, 16, 1024), sdesc_sw128(k_addr + koff, 16, 1024), idesc_s,
                 ks > 0 ? 1u : 0u);
        }
        mma_commit(s_full + t);
      };
      auto issue_pv = [&](int t, int j) -> bool {  // O_t += P_t(j) V_j
        if (!wt(p_full + t, j & 1)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sV + (j % C::kVS) * C::kKVTileBytes);
#pragma unroll
        for (int ks = 0; ks < kTcTileN / 16; ++ks) {
          // B = V (keys x d, d contiguous): 16 keys per step = 2048 bytes; LBO = next 64 d-columns
          const uint64_t bdesc = sdesc_sw128(v_addr + ks * 2048, kTcTileN * 128, 1024);
          mma_ts(tmem + 256 + t * D, tmem + t * 128 + ks * 8, bdesc, idesc_o, (j > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(o_bar + t);
        return true;
      };
      bool ok = wt(q_full, 0) && wt(k_full, 0);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        if (ntq == 2) issue_s(1, 0);
        mma_commit(k_empty);  // K_0 is free once S(0) completes
      }
      for (int j = 0; ok && j < ntiles; ++j) {
        const bool more = j + 1 < ntiles;
        if (!wt(v_full + j % C::kVS, (j / C::kVS) & 1)) break;
        if (!issue_pv(0, j)) break;
        if (more) {
          if (!wt(k_full + (j + 1) % C::kKS, ((j + 1) / C::kKS) & 1)) break;
          tc_fence_after();
          issue_s(0, j + 1);
        }
        if (ntq == 2 && !issue_pv(1, j)) break;
        mma_commit(v_empty + j % C::kVS);  // V_j is no longer read once these complete
        if (more) {
          if (ntq == 2) issue_s(1, j + 1);
          mma_commit(k_empty + (j + 1) % C::kKS);  // nor K_{j+1}
        }
      }
      // every MMA issued by this thread has completed before TMEM is released
      mma_commit(mma_done);
      mbar_wait_drain(mma_done, 0);
    }
  } else if (warp >= 4) {
    // ================================================================ softmax + epilogue
    const int t = (warp - 4) >> 2;  // query tile of this warpgroup
    const int row = tid - 128 - t * 128;
    const int rows_t = t == 0 ? s_rows0 : s_rows1;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + t * 128;
    const uint32_t tO = tmem + lane_base + 256 + t * D;
    const float scale2 = 1.4426950408889634f / sqrtf((float)D);
    float m_used = -INFINITY, l = 0.f;
    bool ok = ntiles > 0 && t < ntq;
    for (int j = 0; ok && j < ntiles; ++j) {
      // warp-uniform: the tcgen05.ld below needs every lane of the warp.  The V copy of tile j
      // is waited on too: it orders the producer's tile-validity words before their read.
      const bool okw = wt(s_full + t, j & 1) &&
                       wt(v_full + j % C::kVS, (j / C::kVS) & 1);
      if (!__all_sync(0xffffffffu, okw)) {
        ok = false;
        break;
      }
      int valid[kSubPerTile];
      bool full = true;  // every key of the tile is real (the same for every thread of the CTA)
#pragma unroll
      for (int b = 0; b < kSubPerTile; ++b) {
        valid[b] = tvalid[(j % C::kVS) * kSubPerTile + b];
        full = full && valid[b] == kSubRows;
      }
      tc_fence_after();
      // the row's kTcTileN scores in registers: four loads, one wait
      uint32_t sv[kTcTileN];
#pragma unroll
      for (int c = 0; c < kTcTileN / 32; ++c)
        tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(sv + c * 32));
      tmem_wait_ld();
      if (!full) {  // padded keys of partial boxes take no part: -inf, probability exactly 0
#pragma unroll
        for (int k = 0; k < kTcTileN; ++k)
          if ((k & (kSubRows - 1)) >= valid[k / kSubRows]) sv[k] = __float_as_uint(-INFINITY);
      }
      // row max: eight chains over columns c + 8i, three inputs per maximum
      float tmax;
      {
        float mx[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float m = fmax3(__uint_as_float(sv[c]), __uint_as_float(sv[c + 8]), __uint_as_float(sv[c + 16]));
#pragma unroll
          for (int i = 3; i + 1 < kTcTileN / 8; i += 2)
            m = fmax3(m, __uint_as_float(sv[c + 8 * i]), __uint_as_float(sv[c + 8 * i + 8]));
          if ((kTcTileN / 8 - 3) % 2) m = fmaxf(m, __uint_as_float(sv[c + kTcTileN - 8]));
          mx[c] = m;
        }
        tmax = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(fmax3(mx[3], mx[4], mx[5]), mx[6], mx[7]));
      }
      tmax *= scale2;
      // lazy rescale: move the running max only when this tile exceeds it by > 2^8
      const bool need = (m_used == -INFINITY) ? (tmax > -INFINITY) : (tmax > m_used + kRescaleThreshold);
      float factor = 1.f;
      float m_new = m_used;
      if (need) {
        m_new = tmax;
        factor = (m_used == -INFINITY) ? 0.f : ex2(m_used - m_new);
      }
      l *= factor;
      m_used = m_new;
      // P = 2^(s*scale - m) as packed bf16 over the first kTcTileN/2 columns of S_t (every score
      // is already in registers, so the packed columns may overwrite them)
      uint64_t acc[2] = {0ull, 0ull};
#pragma unroll
      for (int h = 0; h < kTcTileN / 64; ++h) {  // 64 scores -> 32 packed columns at a time
        uint32_t pk[32];
        if (full)
          exp_half<true>(*reinterpret_cast<const uint32_t(*)[64]>(sv + h * 64), scale2, -m_used, pk, acc);
        else
          exp_half<false>(*reinterpret_cast<const uint32_t(*)[64]>(sv + h * 64), scale2, -m_used, pk, acc);
        tmem_st32(tS + h * 32, pk);
      }
      // a moved maximum rescales O_t before PV_t(j) adds to it (the arrival below releases that
      // MMA); here, after P, the row's scores no longer occupy registers
      if (__any_sync(0xffffffffu, need && j > 0)) {
        // O_t holds P_t(0..j-1) V (complete: S_t(j) was issued after the last of them)
        const bool okw2 = wt(o_bar + t, (j - 1) & 1);
        if (!__all_sync(0xffffffffu, okw2)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + c * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * factor);
          tmem_st32(tO + c * 32, r);
        }
      }
      float a0, a1, a2, a3;
      f2_unpack(acc[0], a0, a1);
      f2_unpack(acc[1], a2, a3);
      l += (a0 + a1) + (a2 + a3);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full + t);
    }
    // epilogue: O_t / l for the rows of this tile (a tile without keys outputs zeros)
    if (t < ntq) {
      float* out = (mode == 1 ? L.Odense + ((size_t)bh * L.P + qrow0 + t * kTcTileM) * D
                              : L.Osp + ((size_t)bh * L.N + qrow0 + t * kTcTileM) * D);
      if (ntiles == 0 && row < rows_t)
        for (int c = 0; c < D; c += 4) *(float4*)(out + (size_t)row * D + c) = make_float4(0.f, 0.f, 0.f, 0.f);
      // warp-uniform: the tcgen05.ld below needs every lane of the warp
      const bool oke = ok && wt(o_bar + t, (ntiles - 1) & 1);
      if (__all_sync(0xffffffffu, oke)) {
        tc_fence_after();
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + c * 32, r);
          tmem_wait_ld();
          if (row < rows_t) {
            float4* o4 = (float4*)(out + (size_t)row * D + c * 32);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              o4[k] = make_float4(__uint_as_float(r[4 * k]) * inv, __uint_as_float(r[4 * k + 1]) * inv,
                                  __uint_as_float(r[4 * k + 2]) * inv, __uint_as_float(r[4 * k + 3]) * inv);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  // after the barrier every wait of the CTA has ended, so a late give-up is not missed
  if (s_abort && tid == 0) atomicCAS(L.status, kDevOk, kDevTimeout);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ----------------------------------------------------------------------------------- host
template <int D>
static sparsepr_status launch_tc(const Layout& L, cudaStream_t st, cudaEvent_t ev0, cudaEvent_t ev1) {
  using C = TcCfg<D>;
  CUtensorMap mQ, mQp, mK, mV;
  const long long rows = (long long)L.BH * L.N;
  if (!make_tmap_bf16(&mQ, L.Qp, rows, D, kTcTileM) || !make_tmap_bf16(&mK, L.Kp, rows, D, kSubRows) ||
      !make_tmap_bf16(&mV, L.Vp, rows, D, kSubRows))
    return SPARSEPR_ERR_CUDA;
  const int probe_items = (L.P + kAttnTileMTc - 1) / kAttnTileMTc;
  if (probe_items > 0) {
    if (!make_tmap_bf16(&mQp, L.Qprobe, (long long)L.BH * L.P, D, kTcTileM)) return SPARSEPR_ERR_CUDA;
  } else {
    mQp = mQ;
  }
  const int sparse_items = max_query_tiles(L, kAttnTileMTc);
  const int items = L.BH * (probe_items + sparse_items);
  cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (ev0) cudaEventRecord(ev0, st);
  launch(attn_tc_kernel<D>, dim3(items), dim3(384), (size_t)C::kSmemBytes, st, mQ, mQp, mK, mV, L, probe_items,
         sparse_items);
  if (ev1) cudaEventRecord(ev1, st);
  SPR_LAUNCH_CHECK();
  return SPARSEPR_OK;
}

sparsepr_status launch_attention_tc(const Layout& L, cudaStream_t st, cudaEvent_t ev0, cudaEvent_t ev1) {
  return L.d == 64 ? launch_tc<64>(L, st, ev0, ev1) : launch_tc<128>(L, st, ev0, ev1);
}

}  // namespace sparsepr
