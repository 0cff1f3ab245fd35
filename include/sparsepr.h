/*
 * sparsepr.h -- C ABI of the B200 (sm_100a) SparsePR per-call sparse attention operator.
 *
 * The operator is the one described in "Partition the Support, Reconstruct the Residual:
 * Training-Free Sparse Attention for Video Generation and World Models" (Taghavi, Langari,
 * Pandey, arXiv 2608.18484): abstract, and the method pipeline of the project page
 * "SparsePR: Training-Free Sparse Attention for Video Generation" (steps 01 sample responses,
 * 02 partition support, 03 execute sparse routes, 04 reconstruct residual).
 *
 * One call on Q, K, V of shape [B, H, N, d] runs, independently for every (b, h) head:
 *   sparsepr_plan       Response-Coupled Partitioning and routing (abstract: K/V tokens are
 *                       grouped in pairs by the responses of their keys to sampled queries;
 *                       queries are grouped by their responses to those key groups' centroids,
 *                       and each query group shares one sparse route), plus the choice of probe
 *                       rows (Table 4).
 *   sparsepr_attention  block-sparse attention over the kept (query group, key group) cells
 *                       and exact dense attention of the probe rows (abstract: a few query
 *                       rows are evaluated exactly).
 *   sparsepr_fit_apply  Probe-Fitted Residual Reconstruction: weighted ridge fit of an affine
 *                       map [O_sp, 1] -> O_dense - O_sp on the probe rows, restricted to the
 *                       span of the probe residuals, added to every unprobed row; probe rows
 *                       take their exact output.
 *
 * Conventions
 *   - All tensor arguments are DEVICE pointers to contiguous row-major [B, H, N, d] arrays of
 *     the configured dtype (SPARSEPR_F32 or SPARSEPR_BF16); d is 64 or 128.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  Every
 *     call only enqueues work on that stream and returns without waiting, except
 *     sparsepr_plan_query and sparsepr_sync, which wait for the stream.
 *   - The caller owns Q, K, V, O and the workspace; the plan owns a small host structure and
 *     pointers into the caller's workspace.  Inputs are never written.
 *   - Errors: arguments are checked before anything is enqueued (SPARSEPR_ERR_INVALID_ARG /
 *     _UNSUPPORTED / _WORKSPACE, nothing launched).  Launch failures return SPARSEPR_ERR_CUDA.
 *     Faults found by the kernels themselves (a ridge system that stays indefinite after the
 *     jitter retries, a bounded wait that expired) are written to a device status word in the
 *     workspace and returned by the next sparsepr_sync or sparsepr_plan_query.  No exception
 *     crosses the ABI; no call allocates device memory.
 */
#ifndef SPARSEPR_H_
#define SPARSEPR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sparsepr_status {
  SPARSEPR_OK = 0,
  SPARSEPR_ERR_INVALID_ARG = 1,  /* null pointer, size out of range, inconsistent config     */
  SPARSEPR_ERR_UNSUPPORTED = 2,  /* valid but not built: d not in {64,128}, or B*H*N above 2^31 rows */
  SPARSEPR_ERR_CUDA = 3,         /* a CUDA runtime call or kernel launch failed               */
  SPARSEPR_ERR_WORKSPACE = 4,    /* workspace null, too small or not 256-byte aligned         */
  SPARSEPR_ERR_NUMERIC = 5,      /* ridge system not positive definite after jitter retries  */
  SPARSEPR_ERR_TIMEOUT = 6,      /* a bounded device-side wait gave up                       */
  SPARSEPR_ERR_STATE = 7         /* call out of order (attention before plan, ...)           */
} sparsepr_status;

enum { SPARSEPR_F32 = 0, SPARSEPR_BF16 = 1 };
/* Probe rows (Table 4, probe selection): uniform rows floor((2i+1)N/(2P)); query-group stratified
   (the paper's reference setting); or P distinct rows drawn at random (partial Fisher-Yates on
   SplitMix64 stream seed + 2^63 + 2*(b*H+h)), weight 1 each. */
enum { SPARSEPR_PROBE_UNIFORM = 0, SPARSEPR_PROBE_STRATIFIED = 1, SPARSEPR_PROBE_RANDOM = 2 };

/* Parameters of one call, as the paper states the problem (abstract; Table C.1; Table 4). */
typedef struct sparsepr_config {
  int32_t B, H, N, d;       /* Q/K/V shape [B,H,N,d]; N >= 1, d in {64, 128}                   */
  int32_t dtype;            /* SPARSEPR_F32 or SPARSEPR_BF16 for Q, K, V                        */
  int32_t s;                /* sampled queries per head, 1 <= s <= N; rows floor((2i+1)N/(2s)) */
  int32_t n_kgroups;        /* C_k paired K/V groups, 1 <= C_k <= min(N, 1024)                */
  int32_t n_qgroups;        /* C_q query groups,      1 <= C_q <= min(N, 1024)                */
  float density;            /* target executed-pair density in (0, 1], counting the s*N routing,
                               C_k*N centroid and P*N probe pairs; per-row key budget
                               kappa = density*N - (s + C_k + P)                                */
  int32_t fixed_k;          /* > 0: every query group keeps exactly min(fixed_k, non-empty)
                               key groups and `density` is ignored                              */
  int32_t P;                /* probe rows per head, 0 <= P <= min(N, 4096)                     */
  int32_t probe_mode;       /* SPARSEPR_PROBE_UNIFORM, _STRATIFIED or _RANDOM                   */
  double lambda;            /* ridge lambda >= 0; < 0 selects 1e-3 * tr(X^T W X) / (d+1)       */
  int32_t km_iters;         /* Lloyd iteration limit of a cold plan (>= 1)                     */
  int32_t km_iters_warm;    /* limit of a re-plan warm-started from the previous centroids;
                               0 = every plan starts cold                                      */
  float km_tol;             /* stop when J_prev - J <= km_tol * J_prev; < 0 = never early      */
  uint64_t seed;            /* k-means initial points: SplitMix64 stream seed + 2*(b*H+h) + stage */
  int32_t partition;        /* SPARSEPR_PARTITION_RESPONSE (the paper's response-coupled
                               partition) or SPARSEPR_PARTITION_SEMANTIC (k-means on the raw keys
                               and the raw queries: the semantic baseline of Table 2)           */
  int32_t repair;           /* 1: fit and add the probe-residual correction (the paper's method);
                               0: unprobed rows keep their block-sparse output                  */
  int32_t correction;       /* SPARSEPR_CORRECTION_AFFINE (the affine map of [O_sp, 1], the
                               paper's method) or SPARSEPR_CORRECTION_MEAN (Table 4 "Mean-only":
                               the weighted mean probe residual, (sum w + lambda)^-1 sum w R,
                               lambda < 0 selecting 1e-3 * sum w)                               */
  int32_t trunc_rank;       /* 0: the map's outputs restricted to the whole probe-residual span
                               (the identity on the ridge solution); 1 <= r <= d: to the r leading
                               eigenvectors of R^T W R (Table D.2's output truncation)           */
  int32_t key_rank;         /* Table C.1's key response rank r_K.  0 (or d): the key k-means sees
                               the full key responses; 0 < r < d: the N x s key responses are taken
                               in the basis of their r leading right singular vectors (the best
                               rank-r approximation, not centred) before the key k-means.  0..d;
                               the semantic partition ignores it                                */
} sparsepr_config;

enum { SPARSEPR_CORRECTION_AFFINE = 0, SPARSEPR_CORRECTION_MEAN = 1 };

enum { SPARSEPR_PARTITION_RESPONSE = 0, SPARSEPR_PARTITION_SEMANTIC = 1 };

/* Per-head statistics, read with sparsepr_plan_query(SPARSEPR_Q_STATS). */
typedef struct sparsepr_head_stats {
  int32_t k_iters;          /* Lloyd iterations run for the key groups                          */
  int32_t q_iters;          /* ... for the query groups                                         */
  int32_t k_refined;        /* key labels decided by the float64 tie-break at the last pass     */
  int32_t q_refined;        /* query labels decided by the float64 tie-break at the last pass   */
  int32_t fit_retries;      /* ridge jitter retries, 0..3; 0 normally.  A failed attempt retries
                               with lambda x10 (lambda = 0: 1e-12 tr(G)/(d+1) first); when the
                               third retry fails too the head's A is zero and the status word
                               is SPARSEPR_ERR_NUMERIC                                           */
  int32_t span_rank;        /* rank of the probe-residual span                                  */
  int64_t sparse_pairs;     /* executed (query, key) pairs of the block-sparse pass             */
  double density;           /* realised density: (s*N + C_k*N + P*N + sparse_pairs) / N^2      */
  double k_objective;       /* J at the last key assignment                                     */
  double q_objective;       /* J at the last query assignment                                   */
  double lambda;            /* ridge lambda used                                                */
} sparsepr_head_stats;

/* What sparsepr_plan_query copies to host memory (all heads, head-major). */
enum {
  SPARSEPR_Q_KLABELS = 1,   /* int32  [B*H, N]       key-group label of every key token        */
  SPARSEPR_Q_QLABELS = 2,   /* int32  [B*H, N]       query-group label of every query token    */
  SPARSEPR_Q_ROUTE = 3,     /* uint8  [B*H, C_q, C_k] 1 = key group kept by the query group     */
  SPARSEPR_Q_PROBES = 4,    /* int32  [B*H, P]       probe token ids, ascending                 */
  SPARSEPR_Q_PROBE_W = 5,   /* double [B*H, P]       probe weights (sum P per head)             */
  SPARSEPR_Q_FIT = 6,       /* double [B*H, d+1, d]  fitted affine map A (last row: intercept) */
  SPARSEPR_Q_KCENT = 7,     /* double [B*H, C_k, d]  key-group centroids (key space)            */
  SPARSEPR_Q_QCENT = 8,     /* double [B*H, C_q, C_k] query-group centroids (response space)    */
  SPARSEPR_Q_OSP = 9,       /* float  [B*H, N, d]    block-sparse output, original token order */
  SPARSEPR_Q_ODENSE = 10,   /* float  [B*H, P, d]    exact output of the probe rows            */
  SPARSEPR_Q_STATS = 11,    /* sparsepr_head_stats [B*H]                                        */
  SPARSEPR_Q_KOBJ = 12,     /* double [B*H, km_iters] key objective per iteration (0 = not run) */
  SPARSEPR_Q_QOBJ = 13,     /* double [B*H, km_iters] query objective per iteration             */
  SPARSEPR_Q_KM_PATH = 14   /* int32  [2]            k-means path of the keys, then the queries:
                             * 0 one launch per step of every iteration, 1 one launch for the
                             * whole loop (see SPARSEPR_KERNEL_KMEANS_LOOP)                      */
};

typedef struct sparsepr_plan_s sparsepr_plan_t;

/* Bytes of device workspace the configuration needs.  Returns INVALID_ARG / UNSUPPORTED for a
 * configuration that the other calls would reject. */
sparsepr_status sparsepr_workspace_size(const sparsepr_config* cfg, size_t* bytes);

/* Creates a plan bound to `workspace` (device memory of at least sparsepr_workspace_size
 * bytes, 256-byte aligned, owned by the caller and kept alive until sparsepr_plan_destroy).
 * Allocates the small host plan structure and clears the device status word and statistics
 * with a blocking cudaMemset; enqueues nothing on any stream. */
sparsepr_status sparsepr_plan_create(const sparsepr_config* cfg, void* workspace,
                                     size_t ws_bytes, sparsepr_plan_t** plan);

/* Response-Coupled Partitioning, routing and probe choice for Q, K (device pointers).
 * The first plan of a plan object starts k-means from SplitMix64-drawn points and runs up
 * to km_iters; later plans start from the previous call's centroids and run up to
 * km_iters_warm when km_iters_warm > 0 (Table C.1: 25 initial / 2 subsequent iterations). */
sparsepr_status sparsepr_plan(sparsepr_plan_t* plan, const void* Q, const void* K, void* stream);

/* Debug/injection entry: installs a partition given in HOST memory instead of computing one
 * (klabels, qlabels int32 [B*H, N] with values in [0, C_k) / [0, C_q); route uint8
 * [B*H, C_q, C_k]; probes int32 [B*H, P] distinct token ids; probe_w double [B*H, P]).
 * Copies synchronously; afterwards attention / fit_apply run as after sparsepr_plan. */
sparsepr_status sparsepr_set_partition(sparsepr_plan_t* plan, const int32_t* klabels,
                                       const int32_t* qlabels, const uint8_t* route,
                                       const int32_t* probes, const double* probe_w,
                                       void* stream);

/* Block-sparse attention of every query over the keys of its group's kept key groups, and
 * exact dense attention of the probe rows.  Q, K, V: the same tensors as the plan's. */
sparsepr_status sparsepr_attention(sparsepr_plan_t* plan, const void* Q, const void* K,
                                   const void* V, void* stream);

/* Weighted ridge fit on the probe rows, projection onto the probe-residual span, and the
 * corrected output O [B,H,N,d] in original token order (out_dtype SPARSEPR_F32 or _BF16). */
sparsepr_status sparsepr_fit_apply(sparsepr_plan_t* plan, void* O, int32_t out_dtype,
                                   void* stream);

/* Waits for the plan's last stream and copies one result (SPARSEPR_Q_*) to host memory;
 * `bytes` must equal the item's size.  Returns a pending device fault if there is one. */
sparsepr_status sparsepr_plan_query(const sparsepr_plan_t* plan, int32_t what, void* host_dst,
                                    size_t bytes);

/* Waits for the plan's last stream and returns (and clears) the device status word. */
sparsepr_status sparsepr_sync(sparsepr_plan_t* plan);

/* Frees the host plan structure (not the caller's workspace).  NULL is ignored. */
void sparsepr_plan_destroy(sparsepr_plan_t* plan);

/* Static string naming a status code. */
const char* sparsepr_status_string(sparsepr_status status);

/* Library version, e.g. 100 for 0.1.0. */
int32_t sparsepr_version(void);

/* Kernels whose launches sparsepr_set_kernel_events can bracket:
 *   BLOCK_SPARSE   the block-sparse (and probe-row) attention launch of sparsepr_attention;
 *   KMEANS_ASSIGN  the first key-group k-means assignment launch of sparsepr_plan (bf16
 *                  inputs, tensor-core path: one pass over all keys);
 *   KMEANS_UPDATE  the first key-group k-means update launch of sparsepr_plan (group sums
 *                  and counts: one pass over all keys);
 *   KMEANS_LOOP    the key-group k-means launch of sparsepr_plan when the whole loop runs in
 *                  one launch (bf16 calls whose keys fit in the shared memory of the SMs,
 *                  at most 128 groups; SPARSEPR_Q_KM_PATH tells which path ran): every
 *                  iteration, the stop test included.  The two hooks above are then not
 *                  recorded. */
enum {
  SPARSEPR_KERNEL_BLOCK_SPARSE = 0,
  SPARSEPR_KERNEL_KMEANS_ASSIGN = 1,
  SPARSEPR_KERNEL_KMEANS_UPDATE = 2,
  SPARSEPR_KERNEL_KMEANS_LOOP = 3
};

/* Optional timing hook for measurement.  When set, the library records `start_event` on its
 * stream immediately before launching the named kernel and `stop_event` immediately after it,
 * so cudaEventElapsedTime gives that kernel's duration.  Events are cudaEvent_t handles passed
 * as void*, created and owned by the caller; passing NULL for both removes the hook.  Returns
 * INVALID_ARG for an unknown kernel id. */
sparsepr_status sparsepr_set_kernel_events(sparsepr_plan_t* plan, int32_t kernel, void* start_event,
                                           void* stop_event);

/* Number of CUDA kernels this library has launched since it was loaded (all plans). */
int64_t sparsepr_launch_count(void);

/* Test hook of the timeout path (no counterpart in the paper).  Every device-side wait of the
 * library is bounded: by default it gives up after about 2e9 SM cycles (about 1 s), sets the
 * device status word to SPARSEPR_ERR_TIMEOUT, lets the copies and tensor-core operations it
 * started finish, frees its tensor memory and returns, so the context stays usable.  This call
 * sets, for the plan's later launches of `kernel`, a limit of `cycles` SM cycles on each such
 * wait (0 restores the default).  SPARSEPR_KERNEL_BLOCK_SPARSE (the attention launch's waits)
 * and SPARSEPR_KERNEL_KMEANS_LOOP (the barriers between the CTAs of one head in the whole-loop
 * k-means launch) are accepted; other ids give SPARSEPR_ERR_UNSUPPORTED, cycles < 0
 * SPARSEPR_ERR_INVALID_ARG.  With a limit of a few hundred cycles the attention launch gives
 * up and its output rows are left unwritten; the whole-loop k-means gives up at its first head
 * barrier and leaves every point of the side in group 0.  The next sparsepr_sync then returns
 * SPARSEPR_ERR_TIMEOUT (and clears it); the plan, its workspace and the context stay usable for
 * the next call.  Enqueues nothing. */
sparsepr_status sparsepr_set_wait_limit(sparsepr_plan_t* plan, int32_t kernel, int64_t cycles);

/* Test hook of the k-means paths (no counterpart in the paper).  A bf16 call with at most 128
 * groups on a side, whose points fit in the shared memory of the SMs (mid-size calls), runs that
 * side's whole Lloyd loop in one cooperative launch; other calls launch the steps of every
 * iteration separately.  Both compute the same labels and centroids.  mode 1 makes the plan's
 * later sparsepr_plan calls use the per-iteration launches everywhere (so that both paths can be
 * checked on the same inputs); mode 0 restores the automatic choice.  Other modes:
 * SPARSEPR_ERR_INVALID_ARG.  Enqueues nothing. */
sparsepr_status sparsepr_set_kmeans_path(sparsepr_plan_t* plan, int32_t mode);

/* Allocation-free weighted ridge fit (no counterpart in the paper: an interface for callers
 * that cannot allocate device memory).  Some callers cannot call cudaMalloc or hand this
 * library scratch memory at the point where they fit the correction -- e.g. code running under
 * a fixed memory pool that must not grow during a step, or a host runtime that only passes the
 * tensors it already owns.  This entry point fits, for each of n_heads heads, the affine map A
 * that sparsepr_fit_apply fits with the default settings (correction SPARSEPR_CORRECTION_AFFINE,
 * trunc_rank 0): the weighted ridge of O_dense - O_sp on [O_sp, 1], lambda as in
 * sparsepr_config, restricted to the whole span of the probe residuals.  It has no mean-only
 * family and no output truncation; for plans that use either, its A differs from theirs.  The
 * probe rows come from the caller and nothing is allocated.
 *   osp_probe    float  [n_heads, P, d]   device: block-sparse output of the probe rows
 *   odense_probe float  [n_heads, P, d]   device: exact output of the probe rows
 *   probe_w      double [n_heads, P]      device: probe weights
 *   A            double [n_heads, d+1, d] device, written (last row: intercept)
 *   status_out   int32  [1] device or NULL: receives 0, or SPARSEPR_ERR_NUMERIC if a head's
 *                system stayed indefinite after the jitter retries (that head's A is zero)
 * Scratch: one fixed __device__ array inside the library (about 7.4 MB) that every GPU which
 * loads the library reserves until the process exits.  Limits: 1 <= n_heads <= 16,
 * 0 <= P <= 4096 (larger sizes return SPARSEPR_ERR_WORKSPACE and launch nothing); d must be 64
 * or 128 (else SPARSEPR_ERR_UNSUPPORTED).  The first call on a device looks up the array's
 * device address (cudaGetSymbolAddress) with that device current and keeps it for that device's
 * context, so make that first call before any stream capture.  All calls share the one array
 * and it keeps the last call's contents: calls that overlap on the GPU (e.g. on two streams at
 * once) race and give wrong results; serialise them.  Enqueued on `stream` (cudaStream_t as
 * void*); returns without waiting. */
sparsepr_status sparsepr_ridge_fit_static(const float* osp_probe, const float* odense_probe,
                                          const double* probe_w, int32_t n_heads, int32_t P,
                                          int32_t d, double lambda, double* A, int32_t* status_out,
                                          void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SPARSEPR_H_ */
