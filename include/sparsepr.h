/*
 * sparsepr.h -- C ABI of the B200 SparsePR per-call sparse attention library.
 *
 * SparsePR ("Partition the Support, Reconstruct the Residual: Training-Free Sparse
 * Attention for Video Generation and World Models") replaces one dense attention call
 * O = softmax(Q K^T / sqrt(d)) V, per head, by four stages:
 *
 *   sparsepr_plan       Response-Coupled Partitioning and routing (paper S4.1, App. B):
 *                       key response metric from M_s evenly spaced query rows, its
 *                       eigen-weighted rank-r_K factor, k-means of the key coordinates
 *                       into C_k paired K/V groups, the query metric of the centred
 *                       non-empty K/V centroids, RMS-normalised rank-r_Q query
 *                       coordinates, k-means into C_q query groups; routing scores per
 *                       (query group, K/V group) cell and the shortest score-ranked
 *                       prefix reaching the per-query key budget (App. B.3, S4.3);
 *                       group-major permutation of Q, K, V; Algorithm A.1 probe rows.
 *   sparsepr_attend     renormalised hard-drop block-sparse attention over the
 *                       selected cells (paper S2).
 *   sparsepr_probe_fit  exact attention of the M probe rows against all keys, the
 *                       coverage-weighted statistics and ridge fit of the residual on
 *                       the sparse output, and the leading-r residual subspace
 *                       (paper S4.2, App. A.2-A.3, App. D.2).
 *   sparsepr_correct    corrected output for unprobed rows, dense output for probe
 *                       rows, restored to the original token order.
 *
 * Conventions (every entry point):
 *   - Q is [H, N_q, d], K and V are [H/G, N_k, d] (G = sparsepr_params.G, 1 unless
 *     grouped-query attention), contiguous row-major DEVICE memory in the dtype of
 *     sparsepr_params.dtype (fp32 or bf16).  Out is [H, N_q, d] in the same dtype.  d must
 *     be a multiple of 8 and at most 128.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     Every call except sparsepr_get_stats, sparsepr_export and sparsepr_check only
 *     enqueues work on it and never synchronises the host.
 *   - Q, K, V and Out must be 16-byte aligned (SPARSEPR_ERR_ARG otherwise).
 *   - The caller owns Q, K, V, Out and the workspace (device memory of at least
 *     sparsepr_workspace_size bytes, 256-byte aligned).  A plan handle is host memory
 *     owned by the library until sparsepr_destroy; it refers to, but does not own, the
 *     workspace and the input tensors, which must stay valid until the last call on the
 *     plan has completed on the GPU.
 *   - Errors: arguments are validated on the host before any launch (SPARSEPR_ERR_ARG,
 *     SPARSEPR_ERR_SHAPE, SPARSEPR_ERR_DTYPE, SPARSEPR_ERR_WORKSPACE); a CUDA launch
 *     error returns SPARSEPR_ERR_CUDA; calls out of order return SPARSEPR_ERR_STATE.
 *     Inconsistencies found on the device (a metric with no positive eigenvalue,
 *     non-finite values, injected labels out of range, a warm state saved for other
 *     dimensions, a pipeline wait that timed out) set a device error word that
 *     sparsepr_check and sparsepr_get_stats report as SPARSEPR_ERR_DEVICE_CHECK.  No call
 *     traps or aborts the CUDA context.
 */
#ifndef SPARSEPR_H
#define SPARSEPR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SPARSEPR_OK = 0,
  SPARSEPR_ERR_ARG = 1,          /* a parameter is out of its valid range */
  SPARSEPR_ERR_SHAPE = 2,        /* H, N, d or a group count is unsupported */
  SPARSEPR_ERR_DTYPE = 3,        /* dtype is neither SPARSEPR_F32 nor SPARSEPR_BF16 */
  SPARSEPR_ERR_WORKSPACE = 4,    /* workspace missing, misaligned or too small */
  SPARSEPR_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed */
  SPARSEPR_ERR_DEVICE_CHECK = 6, /* the device error word is set (see sparsepr_check) */
  SPARSEPR_ERR_STATE = 7         /* call out of order for this plan */
} sparsepr_status;

typedef enum { SPARSEPR_F32 = 0, SPARSEPR_BF16 = 1 } sparsepr_dtype;

/* Attention engine used by sparsepr_attend and sparsepr_dense_attention. */
typedef enum {
  SPARSEPR_ENGINE_AUTO = 0,   /* tensor-core engine for bf16, CUDA-core engine for fp32 */
  SPARSEPR_ENGINE_SIMT = 1    /* fp32 CUDA-core engine for every dtype (reference path) */
} sparsepr_engine;

/* Residual estimator of sparsepr_probe_fit (paper S4.2; App. D.3, Table 4). */
typedef enum {
  SPARSEPR_EST_RIDGE = 0,     /* full weighted ridge B, projected on Psi_r (the method) */
  SPARSEPR_EST_MEAN = 1,      /* weighted mean residual only (B = 0) */
  SPARSEPR_EST_SCALAR = 2,    /* B = a I, penalty lambda d a^2, no projection */
  SPARSEPR_EST_DIAGONAL = 3   /* B = diag(b), penalty lambda |b|^2, no projection */
} sparsepr_estimator;

/* Partition of sparsepr_plan ("Partition the Support, Reconstruct the Residual", S3 and
 * the ablation tables): the method's response-coupled partition, or the semantic
 * reference partition, which runs the same k-means on the raw key rows and the raw query
 * rows (no metric, no eigen factor, no RMS step; requires d <= 64). */
typedef enum {
  SPARSEPR_PARTITION_RESPONSE = 0,
  SPARSEPR_PARTITION_SEMANTIC = 1
} sparsepr_partition;

/* Routing budget of sparsepr_plan ("Partition the Support, Reconstruct the Residual",
 * S4.3 and App. B.3: every query group keeps the shortest score-ranked prefix of K/V
 * groups whose key count reaches a common budget beta).
 *   PREFIX      beta = (target_density - M/N_q) N_k: the realised rho_exec is at or above
 *               the target.
 *   CALIBRATED  App. D.2 calibrates the budget toward the target: per head, the integer
 *               beta in [1, N_k] whose selection brings rho_exec nearest the target (of two
 *               selections equally near, the denser; of the betas giving one selection,
 *               the smallest), found by bisection on beta (rho_exec never decreases in
 *               beta).  The realised density may then fall on either side of the target. */
typedef enum {
  SPARSEPR_BUDGET_PREFIX = 0,
  SPARSEPR_BUDGET_CALIBRATED = 1
} sparsepr_budget;

/*
 * Problem and hyper-parameters of one call (paper S2, S4; values of the review page's
 * hyper-parameter table: r_K=48, r_Q=64, M=64, r=16, lambda=0.1).
 *   H                 query heads (each head is an independent problem, but for the K/V
 *                     partition it shares with the other heads of its group when G > 1)
 *   N_q, N_k          query and key/value tokens per head
 *   d                 head dimension (multiple of 8, <= 128)
 *   dtype             sparsepr_dtype of Q, K, V and Out
 *   M_s               sampled query rows for the key metric (rows floor(s*N_q/M_s))
 *   r_K, r_Q          ranks of the key and query response coordinates (1..min(d,64))
 *   C_q, C_k          requested query / K-V group counts (1..1024, <= N_q / N_k)
 *   M                 probe rows (1..128, <= N_q)
 *   r                 residual-subspace rank (0 = no projection; else 1..M)
 *   lambda            ridge strength (>= 0)
 *   target_density    executed-pair target rho* including probes (M/N_q < rho* <= 1)
 *   kmeans_max_iter   Lloyd assignment steps at most (1..1000; the paper uses 25)
 *   engine            sparsepr_engine
 *   seed              seed of the SplitMix64 stream that draws the k-means initial rows
 *   estimator         sparsepr_estimator (0, the method's weighted ridge, unless comparing)
 *   G                 query heads per K/V head (grouped-query attention; 0 or 1 = none).
 *                     H must be a multiple of G; K and V are then [H/G, N_k, d], query head
 *                     h reads K/V head h/G.  Paper App. C: the shared key response metric
 *                     of a K/V head is built from its G query heads' rows, concatenated in
 *                     head order, of which G*M_s evenly spaced rows are taken; the K/V
 *                     groups, their centroids, the query metric and F_Q are shared by the
 *                     G heads, and everything from the query coordinates on is per query
 *                     head.  Exports of the K/V side (LABELS_K, PERM_K, GROUPS_K, SIZES_K,
 *                     FACTOR_K, EIG_K, METRIC_K, PHI_K, KBAR, METRIC_Q, FACTOR_Q, EIG_Q)
 *                     then have H/G rows; KMEANS_ITERS and OBJECTIVE keep H rows, the key
 *                     column of row h being that of K/V head h/G.  Warm starts take G <= 1.
 *   partition         sparsepr_partition (0 unless comparing).  With the semantic partition
 *                     r_K and r_Q are ignored (the coordinates are the d raw channels),
 *                     FACTOR_K / FACTOR_Q export the identity and METRIC_* / EIG_* are not
 *                     computed; warm starts take the response partition.
 *   budget            sparsepr_budget (0, the plain prefix rule, unless calibrating)
 */
typedef struct {
  int32_t H, N_q, N_k, d;
  int32_t dtype;
  int32_t M_s, r_K, r_Q, C_q, C_k, M, r;
  double lambda;
  double target_density;
  int32_t kmeans_max_iter;
  int32_t engine;
  uint64_t seed;
  int32_t estimator;
  int32_t G;
  int32_t partition;
  int32_t budget;
} sparsepr_params;

typedef struct sparsepr_plan_s* sparsepr_plan_t;

/* Whole-call statistics (summed over heads).  Realised densities follow paper S2/S4.3:
 * rho_route = routed pairs / (H N_q N_k), rho_exec = (routed pairs + H M N_k)/(H N_q N_k). */
typedef struct {
  int64_t pairs_route;
  int64_t pairs_exec;
  double rho_route;
  double rho_exec;
  int32_t kmeans_iters_k_max;
  int32_t kmeans_iters_q_max;
  int32_t groups_k_min;      /* smallest per-head count of non-empty K/V groups */
  int32_t groups_q_min;      /* smallest per-head count of non-empty query groups */
  int32_t device_error;      /* device error word (0 = none) */
} sparsepr_stats;

/* Bytes of device workspace a plan with these parameters needs.  Host only. */
sparsepr_status sparsepr_workspace_size(const sparsepr_params* params, size_t* bytes);

/*
 * Response-Coupled Partitioning, routing, permutation and probe selection for all heads.
 * Q, K, V: device [H,N,d].  workspace: device, >= sparsepr_workspace_size bytes.
 * On success *out receives a new plan handle (host memory).  Asynchronous on `stream`.
 */
sparsepr_status sparsepr_plan(const sparsepr_params* params, const void* Q, const void* K,
                              const void* V, void* workspace, size_t workspace_bytes,
                              void* stream, sparsepr_plan_t* out);

/*
 * As sparsepr_plan, but the k-means labels are given: labQ [H,N_q] and labK [H/G,N_k] are
 * device int32 arrays with values in [0,C_q) and [0,C_k).  Every later step (groups,
 * centroids, query coordinates, routing, permutation, probes) is computed from them
 * exactly as sparsepr_plan computes it from its own k-means labels.  For testing the
 * stages after clustering against a reference given identical labels.
 */
sparsepr_status sparsepr_plan_from_labels(const sparsepr_params* params, const void* Q,
                                          const void* K, const void* V,
                                          const int32_t* labQ, const int32_t* labK,
                                          void* workspace, size_t workspace_bytes,
                                          void* stream, sparsepr_plan_t* out);

/*
 * Cross-call warm start ("Partition the Support, Reconstruct the Residual", App. C:
 * later calls of a denoising sequence start the k-means from the previous centroids in
 * the original space, mapped into the current response coordinates, and refresh the
 * metric factors by two subspace iterations with a Cholesky factorisation instead of a
 * full eigendecomposition).
 *
 * The state is caller-owned DEVICE memory of sparsepr_state_size bytes, 256-byte
 * aligned.  It holds a header (the dimensions it was saved for), the fp64 factors F_K
 * [H,d,r_K] and F_Q [H,d,r_Q], and for every k-means label its original-space centroid
 * (fp64 [H,C_k,d] and [H,C_q,d]) with a non-empty flag; the layout is internal.
 *
 * sparsepr_save_state writes a planned call's state (asynchronous, any time after
 * sparsepr_plan*; the plan keeps its own copies).  sparsepr_plan_warm is sparsepr_plan
 * started from a saved state: per head, the factor update is
 * F <- Z L^-T with Z = M F, L L^T = F^T Z, twice, then scaled to unit mean eigenvalue;
 * label c of each k-means starts at phi(cbar_c) when it was non-empty, else at the fresh
 * draw c.  A head whose F^T M F is not positive definite takes the full
 * eigendecomposition.  A state saved for other dimensions (or never saved) makes every
 * head start cold and sets the device error word (SPARSEPR_ERR_DEVICE_CHECK from
 * sparsepr_check).  The state is read by work enqueued on `stream`; saving the new
 * plan's state into the same buffer later on the same stream is allowed.  After a warm
 * plan, the EIG_K / EIG_Q exports are zero for the heads updated this way.
 * Errors: SPARSEPR_ERR_ARG for a null or misaligned state, or for parameters with G > 1 or
 * the semantic partition (both calls); otherwise as sparsepr_plan.
 */
sparsepr_status sparsepr_state_size(const sparsepr_params* params, size_t* bytes);
sparsepr_status sparsepr_save_state(sparsepr_plan_t plan, void* state, void* stream);
sparsepr_status sparsepr_plan_warm(const sparsepr_params* params, const void* Q, const void* K,
                                   const void* V, const void* state, void* workspace,
                                   size_t workspace_bytes, void* stream, sparsepr_plan_t* out);

/* Renormalised hard-drop attention over the selected cells; the sparse output stays in
 * the workspace (group-major, fp32).  Requires a plan.  Asynchronous. */
sparsepr_status sparsepr_attend(sparsepr_plan_t plan, void* stream);

/* Exact probe attention, residual statistics, ridge fit, residual subspace and the folded
 * correction.  Requires sparsepr_attend.  Asynchronous. */
sparsepr_status sparsepr_probe_fit(sparsepr_plan_t plan, void* stream);

/* Writes the corrected output Out (device [H,N_q,d], params dtype) in the original token
 * order: O_sp + mu_R + ((O_sp - mu_x)/s) B P for unprobed rows, the exact dense output
 * for probe rows.  Requires sparsepr_probe_fit.  Asynchronous. */
sparsepr_status sparsepr_correct(sparsepr_plan_t plan, void* Out, void* stream);

/* The four calls above in order, on one stream, followed by sparsepr_destroy of the
 * internal plan (host memory only).  Asynchronous. */
sparsepr_status sparsepr_forward(const sparsepr_params* params, const void* Q, const void* K,
                                 const void* V, void* Out, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* Dense attention softmax(Q K^T / sqrt(d)) V for all rows through the same attention
 * engine (every key selected).  Only H, N_q, N_k, d, dtype, engine and G of params are
 * read (K and V are [H/G, N_k, d] when G > 1).  Needs no workspace.  Asynchronous.  A
 * pipeline wait of the tensor-core engine that timed out (its work abandoned, part of Out
 * unwritten) sets a sticky per-device error word that sparsepr_dense_check reports. */
sparsepr_status sparsepr_dense_attention(const sparsepr_params* params, const void* Q,
                                         const void* K, const void* V, void* Out,
                                         void* stream);

/*
 * Exact attention of selected query rows without any device allocation.  The paper has
 * no counterpart: this is a library convenience for callers that cannot allocate device
 * memory around the call -- code whose device memory is owned by another allocator (a
 * framework's caching pool that has reserved the GPU) and latency-critical loops that
 * must not pay the implicit device synchronisation of cudaMalloc/cudaFree.
 *   Q [H,N_q,d], K, V [H/G,N_k,d]: device, params dtype; only H, N_q, N_k, d, dtype,
 *   engine and G of params are read (G = query heads per K/V head, 0 or 1 = none; H must
 *   be a multiple of G and at most 65535).  rows: device int32 [nrows], 1 <= nrows <= 128,
 *   indices into [0,N_q) (an index below 0 reads row 0 and one at or above N_q reads row
 *   N_q-1, never outside Q).  Out: device [H,nrows,d], params dtype:
 *   softmax(q K^T / sqrt(d)) V for each requested row.
 * Work space is a fixed 16 MiB device array inside the library, held on every GPU that
 * loads it until the process exits; a call needing more (about
 * H * nrows * ceil(N_k/4096) * (d+2) * 4 bytes) returns SPARSEPR_ERR_WORKSPACE before
 * launching anything.  The first call on a device looks up that array's address (with
 * that device current), so make it before any stream capture.  All calls share the
 * array: calls whose work overlaps on the GPU race and must be serialised by the caller.
 * A call whose attention kernel timed out on a pipeline wait writes NaN rows, and a
 * non-finite result row is reported too: both set bits of a sticky per-device word that
 * sparsepr_dense_check reads.  Asynchronous on `stream`; calls no allocator.
 */
sparsepr_status sparsepr_dense_rows_noalloc(const sparsepr_params* params, const void* Q,
                                            const void* K, const void* V,
                                            const int32_t* rows, int32_t nrows, void* Out,
                                            void* stream);

/* The paper has no counterpart: error reporting of the two plan-free entry points.
 * Synchronises `stream`, then reads and clears, on the current device, the error words of
 * sparsepr_dense_attention and sparsepr_dense_rows_noalloc (bits as for a plan: 4 a
 * non-finite output row, 32 a pipeline wait that timed out).  Returns SPARSEPR_OK when
 * both were zero, else SPARSEPR_ERR_DEVICE_CHECK with their OR in *device_error (when
 * non-NULL).  The words collect every call since the last check; work still running on
 * other streams may set them after the read.  Allocates nothing. */
sparsepr_status sparsepr_dense_check(void* stream, int32_t* device_error);

/* The paper has no counterpart: a self-test of the failure path every tensor-core kernel
 * takes when a pipeline wait gives up.  Launches, on `stream` and the current device, one
 * warp that waits through the engines' bounded mbarrier wait on a barrier nothing ever
 * completes, with no copy or product in flight; after about one second (2e9 SM clocks)
 * the wait returns and sets bit 32 of the error word that sparsepr_dense_check reads.
 * No fault, no hang: the warp then exits.  Asynchronous; allocates nothing. */
sparsepr_status sparsepr_wait_selftest(void* stream);

/*
 * Diagnostics of "Partition the Support, Reconstruct the Residual" S3 (observations O1,
 * O3), in fp64.  They measure a partition; they are not part of the attention call.
 *
 * O1 support densities.  For query row i of head h, D_i(alpha) is the smallest set of
 * keys whose dense attention weights softmax(q_i K^T / sqrt(d)) reach the fraction alpha
 * of the row's mass: keys by decreasing weight, the lowest index first among equal
 * weights, the mass compared with alpha (1 - 1e-15) times the row's total.  rows [H][nrows]
 * (device int32, indices into [0, N_q), clamped) picks each head's rows, pool [H][nrows]
 * (device int32 in [0, npools); a row outside marks nothing) assigns them to pools.
 * Outputs (device int32): sizes [H][nrows] = |D_i(alpha)| (tau_i = sizes / N_k) and
 * pooled [H][npools] = |union of the D_i of the pool's rows| (gamma = pooled / N_k).
 * Only H, N_q, N_k, d, dtype and G of params are read (K is [H/G, N_k, d]).  workspace:
 * device, 256-byte aligned, sparsepr_support_workspace_size bytes (about
 * 8 H nrows N_k).  SPARSEPR_ERR_ARG for 0 < alpha <= 1 violated, nrows < 1 or
 * npools outside [1, nrows].  Asynchronous.
 */
sparsepr_status sparsepr_support_workspace_size(const sparsepr_params* params, int32_t nrows,
                                                int32_t npools, size_t* bytes);
sparsepr_status sparsepr_support_densities(const sparsepr_params* params, const void* Q,
                                           const void* K, const int32_t* rows,
                                           const int32_t* pool, int32_t nrows, int32_t npools,
                                           double alpha, void* workspace, size_t workspace_bytes,
                                           int32_t* sizes, int32_t* pooled, void* stream);

/*
 * O3 oracle affine fit (S3 O3, App. D.5), per head over all N_q rows: the least-squares
 * fit R ~ 1 b + O_sp B of the hard-drop residual R = dense - O_sp, with the centred sparse
 * output's non-zero columns scaled to unit norm and directions whose singular value is
 * at most 1e-10 times the largest left out.  The directions come from the
 * eigendecomposition of the scaled Gram matrix, so only singular values above about
 * 1e-8 of the largest are resolved (an ill-conditioned O_sp fits its leading directions
 * only).  plan: after sparsepr_attend (its sparse output is used).  dense: device
 * [H,N_q,d] in params dtype, the exact attention output in original order (for example
 * from sparsepr_dense_attention).  Outputs (device fp64 [H]): explained = 1 - err / |R|^2
 * and err = the remaining squared error.  workspace: device, 256-byte aligned,
 * sparsepr_affine_workspace_size bytes.  Asynchronous.
 */
sparsepr_status sparsepr_affine_workspace_size(sparsepr_plan_t plan, size_t* bytes);
sparsepr_status sparsepr_affine_fit(sparsepr_plan_t plan, const void* dense, void* workspace,
                                    size_t workspace_bytes, double* explained, double* err,
                                    void* stream);

/* Synchronises `stream` and reports the device error word: SPARSEPR_OK or
 * SPARSEPR_ERR_DEVICE_CHECK (with the word in *device_error when non-NULL). */
sparsepr_status sparsepr_check(sparsepr_plan_t plan, void* stream, int32_t* device_error);

/* Synchronises `stream` and fills *stats.  Valid after sparsepr_plan. */
sparsepr_status sparsepr_get_stats(sparsepr_plan_t plan, void* stream, sparsepr_stats* stats);

/* Internal arrays a plan exposes for inspection (all per head, leading dimension H). */
typedef enum {
  SPARSEPR_X_LABELS_K = 0,    /* int32 [H,N_k]   final k-means labels of the keys */
  SPARSEPR_X_LABELS_Q = 1,    /* int32 [H,N_q]   final k-means labels of the queries */
  SPARSEPR_X_PERM_K = 2,      /* int32 [H,N_k]   group-major order: row at each position */
  SPARSEPR_X_PERM_Q = 3,      /* int32 [H,N_q] */
  SPARSEPR_X_GROUPS_K = 4,    /* int32 [H]       non-empty K/V groups C_k' */
  SPARSEPR_X_GROUPS_Q = 5,    /* int32 [H]       non-empty query groups C_q' */
  SPARSEPR_X_SIZES_K = 6,     /* int32 [H,C_k]   sizes of compact K/V groups (first C_k') */
  SPARSEPR_X_SIZES_Q = 7,     /* int32 [H,C_q] */
  SPARSEPR_X_CELL_COUNT = 8,  /* int32 [H,C_q]   selected K/V groups per compact query group */
  SPARSEPR_X_CELL_IDS = 9,    /* int32 [H,C_q,C_k] selected compact K/V ids, ascending */
  SPARSEPR_X_PROBES = 10,     /* int32 [H,M]     probe rows in selection order */
  SPARSEPR_X_PROBE_COUNT = 11,/* int32 [H,C_q]   probes per compact query group m_a */
  SPARSEPR_X_KMEANS_ITERS = 12,/* int32 [H,2]    assignment steps (keys, queries) */
  SPARSEPR_X_OBJECTIVE = 13,  /* double [H,2]    final k-means objectives (keys, queries) */
  SPARSEPR_X_PAIRS = 14,      /* int64 [H]       routed pairs per head */
  SPARSEPR_X_FACTOR_K = 15,   /* double [H,d,r_K] F_K */
  SPARSEPR_X_FACTOR_Q = 16,   /* double [H,d,r_Q] F_Q */
  SPARSEPR_X_EIG_K = 17,      /* double [H,r_K]  kept eigenvalues of M_K (descending) */
  SPARSEPR_X_EIG_Q = 18,      /* double [H,r_Q]  kept eigenvalues of M_Q */
  SPARSEPR_X_METRIC_K = 19,   /* double [H,d,d]  M_K */
  SPARSEPR_X_METRIC_Q = 20,   /* double [H,d,d]  M_Q */
  SPARSEPR_X_PHI_K = 21,      /* double [H,N_k,r_K] key coordinates */
  SPARSEPR_X_PHI_Q = 22,      /* double [H,N_q,r_Q] query coordinates */
  SPARSEPR_X_CENTRES_Q = 23,  /* double [H,C_q,r_Q] query-group centres in phi_Q space (raw labels) */
  SPARSEPR_X_SCORES = 24,     /* double [H,C_q,C_k] routing scores (compact ids) */
  SPARSEPR_X_OSP = 25,        /* float [H,N_q,d] sparse output, group-major order */
  SPARSEPR_X_ODENSE_PROBE = 26,/* float [H,M,d]  exact output of the probe rows */
  SPARSEPR_X_FIT_MU_X = 27,   /* double [H,d] */
  SPARSEPR_X_FIT_MU_R = 28,   /* double [H,d] */
  SPARSEPR_X_FIT_S = 29,      /* double [H,d] */
  SPARSEPR_X_FIT_B = 30,      /* double [H,d,d] ridge coefficients B_lambda */
  SPARSEPR_X_FIT_P = 31,      /* double [H,d,d] projector Psi_r Psi_r^T */
  SPARSEPR_X_FIT_REFF = 32,   /* int32 [H]      rank kept in the projector */
  SPARSEPR_X_PROBE_DIST = 33, /* double [H,N_q] squared phi_Q distance to the group centre */
  SPARSEPR_X_KBAR = 34,       /* double [H,C_k,d] K/V group key centroids (compact ids) */
  SPARSEPR_X_QBAR = 35,       /* double [H,C_q,d] query group centroids (compact ids) */
  SPARSEPR_X_KM_REASSIGNED = 36,/* int64 [2,H]: row 0 keys (by K/V head), row 1 queries:
                                   points the tensor-core k-means listed for re-assignment,
                                   summed over its steps, when it keeps distance bounds
                                   (warm plans; zero otherwise); the others kept their
                                   label by the bounds */
  SPARSEPR_X_BETA = 37,       /* double [H]    per-query key budget beta the routing used */
  SPARSEPR_X_COUNT = 38
} sparsepr_export_what;

/* Size in bytes of an exported array for this plan. Host only. */
sparsepr_status sparsepr_export_size(sparsepr_plan_t plan, int32_t what, size_t* bytes);

/* Synchronises `stream`, then copies the array `what` into HOST memory `dst` of exactly
 * sparsepr_export_size bytes (SPARSEPR_ERR_ARG otherwise). */
sparsepr_status sparsepr_export(sparsepr_plan_t plan, int32_t what, void* dst, size_t bytes,
                                void* stream);

/* Frees the plan handle (host memory only; the workspace stays the caller's). */
void sparsepr_destroy(sparsepr_plan_t plan);

/* Static text for a status code. */
const char* sparsepr_status_string(sparsepr_status status);

/* Number of CUDA kernels this library has enqueued since it was loaded, over all threads
 * and devices (a relaxed atomic counter; the difference of two readings around a region
 * counts that region's launches when no other thread calls the library meanwhile).
 * The paper has no counterpart: it serves measurement.  Never fails. */
unsigned long long sparsepr_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* SPARSEPR_H */
