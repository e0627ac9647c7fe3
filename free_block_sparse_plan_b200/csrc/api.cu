// C ABI of the SparsePR library: argument validation, workspace layout, stage order.
#include <atomic>
#include <cmath>
#include <cstring>
#include <new>

#include "common.cuh"

using namespace spr;

namespace spr {
// Kernels launched by this library since it was loaded (all threads, all devices).
std::atomic<unsigned long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
}  // namespace spr

struct sparsepr_plan_s {
  Plan p;
};

namespace {

// Bump allocator over the caller's workspace; with base == nullptr it only measures.
// The kernels read Q, K, V and write Out with 16-byte vector accesses.
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

struct Carver {
  char* base;
  size_t off = 0;
  template <class T>
  T* take(size_t count) {
    off = (off + 255) & ~size_t(255);
    T* ptr = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += count * sizeof(T);
    return ptr;
  }
};

sparsepr_status validate(const sparsepr_params* q) {
  if (!q) return SPARSEPR_ERR_ARG;
  if (q->dtype != SPARSEPR_F32 && q->dtype != SPARSEPR_BF16) return SPARSEPR_ERR_DTYPE;
  if (q->H < 1 || q->N_q < 1 || q->N_k < 1) return SPARSEPR_ERR_SHAPE;
  if (q->d < 8 || q->d > kMaxD || q->d % 8) return SPARSEPR_ERR_SHAPE;
  if ((long long)q->H * q->N_q * q->d > (1LL << 40)) return SPARSEPR_ERR_SHAPE;
  if (q->N_q > (1 << 28) || q->N_k > (1 << 28)) return SPARSEPR_ERR_SHAPE;
  const int rmax = q->d < kMaxR ? q->d : kMaxR;
  if (q->M_s < 1) return SPARSEPR_ERR_ARG;
  if (q->r_K < 1 || q->r_K > rmax || q->r_Q < 1 || q->r_Q > rmax) return SPARSEPR_ERR_ARG;
  if (q->C_q < 1 || q->C_q > kMaxC || q->C_q > q->N_q) return SPARSEPR_ERR_ARG;
  if (q->C_k < 1 || q->C_k > kMaxC || q->C_k > q->N_k) return SPARSEPR_ERR_ARG;
  if (q->M < 1 || q->M > kMaxM || q->M > q->N_q) return SPARSEPR_ERR_ARG;
  if (q->r < 0 || q->r > q->M) return SPARSEPR_ERR_ARG;
  if (!(q->lambda >= 0.0) || !std::isfinite(q->lambda)) return SPARSEPR_ERR_ARG;
  if (!(q->target_density <= 1.0) || !(q->target_density > (double)q->M / (double)q->N_q))
    return SPARSEPR_ERR_ARG;
  if (q->kmeans_max_iter < 1 || q->kmeans_max_iter > 1000) return SPARSEPR_ERR_ARG;
  if (q->engine != SPARSEPR_ENGINE_AUTO && q->engine != SPARSEPR_ENGINE_SIMT) return SPARSEPR_ERR_ARG;
  if (q->estimator < SPARSEPR_EST_RIDGE || q->estimator > SPARSEPR_EST_DIAGONAL) return SPARSEPR_ERR_ARG;
  if (q->G < 0 || (q->G > 1 && q->H % q->G != 0)) return SPARSEPR_ERR_SHAPE;
  if (q->partition != SPARSEPR_PARTITION_RESPONSE && q->partition != SPARSEPR_PARTITION_SEMANTIC)
    return SPARSEPR_ERR_ARG;
  if (q->partition == SPARSEPR_PARTITION_SEMANTIC && q->d > kMaxR) return SPARSEPR_ERR_ARG;
  if (q->budget != SPARSEPR_BUDGET_PREFIX && q->budget != SPARSEPR_BUDGET_CALIBRATED) return SPARSEPR_ERR_ARG;
  return SPARSEPR_OK;
}

Dims make_dims(const sparsepr_params* q) {
  Dims d{};
  d.H = q->H; d.Nq = q->N_q; d.Nk = q->N_k; d.d = q->d; d.dtype = q->dtype;
  d.Ms = q->M_s; d.rK = q->r_K; d.rQ = q->r_Q; d.Cq = q->C_q; d.Ck = q->C_k;
  d.M = q->M; d.r = q->r; d.lambda = q->lambda; d.rho = q->target_density;
  d.max_iter = q->kmeans_max_iter; d.engine = q->engine; d.seed = q->seed;
  d.estimator = q->estimator;
  d.G = q->G > 1 ? q->G : 1;
  d.Hk = d.H / d.G;
  d.semantic = q->partition == SPARSEPR_PARTITION_SEMANTIC;
  if (d.semantic) d.rK = d.rQ = d.d;        // coordinates are the raw channels
  d.nchK = cdiv(q->N_k, kSortChunk);
  d.nchQ = cdiv(q->N_q, kSortChunk);
  d.nsplit = cdiv(q->N_k, kProbeSplit);
  // paper S4.3: the router reserves the probe cost; common per-query key budget
  d.beta = (q->target_density - (double)q->M / (double)q->N_q) * (double)q->N_k;
  d.budget = q->budget;
  return d;
}

size_t carve(const Dims& m, char* base, Buffers* b) {
  Carver c{base};
  const size_t H = m.H, d = m.d, Nq = m.Nq, Nk = m.Nk, Cq = m.Cq, Ck = m.Ck, M = m.M;
  const size_t es = m.dtype == SPARSEPR_BF16 ? 2 : 4;
  b->MK = c.take<double>(H * d * d);
  b->MQ = c.take<double>(H * d * d);
  b->lamK = c.take<double>(H * m.rK);
  b->lamQ = c.take<double>(H * m.rQ);
  b->FK64 = c.take<double>(H * d * m.rK);
  b->FQ64 = c.take<double>(H * d * m.rQ);
  b->FK = c.take<float>(H * d * m.rK);
  b->FQ = c.take<float>(H * d * m.rQ);
  b->phiK = c.take<double>(H * Nk * m.rK);
  b->phiQ = c.take<double>(H * Nq * m.rQ);
  b->centK = c.take<double>(H * Ck * m.rK);
  b->centQ = c.take<double>(H * Cq * m.rQ);
  b->labK = c.take<int>(H * Nk);
  b->labQ = c.take<int>(H * Nq);
  b->histK = c.take<int>(H * Ck * m.nchK);
  b->histQ = c.take<int>(H * Cq * m.nchQ);
  b->permK = c.take<int>(H * Nk);
  b->permQ = c.take<int>(H * Nq);
  b->invQ = c.take<int>(H * Nq);
  b->offK = c.take<int>(H * (Ck + 1));
  b->offQ = c.take<int>(H * (Cq + 1));
  b->poffK = c.take<int>(H * (Ck + 1));
  b->kmK = c.take<int>(H * 4);
  b->kmQ = c.take<int>(H * 4);
  b->objK = c.take<double>(H * Ck);
  b->objQ = c.take<double>(H * Cq);
  b->objH = c.take<double>(H * 2);
  b->compK = c.take<int>(H * Ck);
  b->compQ = c.take<int>(H * Cq);
  b->usedK = c.take<int>(H * Ck);
  b->usedQ = c.take<int>(H * Cq);
  b->nK = c.take<int>(H);
  b->nQ = c.take<int>(H);
  b->sizeK = c.take<int>(H * Ck);
  b->sizeQ = c.take<int>(H * Cq);
  b->kbar = c.take<double>(H * Ck * d);
  b->vbar = c.take<double>(H * Ck * d);
  b->qbar = c.take<double>(H * Cq * d);
  b->scores = c.take<double>(H * Cq * Ck);
  b->cellCnt = c.take<int>(H * Cq);
  b->cellIds = c.take<int>(H * Cq * Ck);
  b->rankPref = m.budget == SPARSEPR_BUDGET_CALIBRATED ? c.take<int>(H * Cq * Ck) : nullptr;
  b->betaH = c.take<double>(H);
  b->pairs = c.take<long long>(H);
  b->Qp = c.take<char>(H * Nq * d * es);
  {
    const size_t plain = H * Nk * d * es;
    const size_t tiled = tc_engine_applies(m.dtype, m.d, m.engine) ? (size_t)m.Hk * kv_tiled_rows(m.Nk, m.Ck) * d * 2 : 0;
    b->Kp = c.take<char>(plain > tiled ? plain : tiled);
    b->Vp = c.take<char>(plain > tiled ? plain : tiled);
  }
  b->dist = c.take<double>(H * Nq);
  b->probeTop = c.take<int>(H * Cq * M);
  b->probes = c.take<int>(H * M);
  b->probeA = c.take<int>(H * M);
  b->mA = c.take<int>(H * Cq);
  b->wP = c.take<double>(H * M);
  b->Osp = c.take<float>(H * Nq * d);
  b->Opart = c.take<float>(H * M * m.nsplit * d);
  b->MLpart = c.take<float>(H * M * m.nsplit * 2);
  b->Odense = c.take<float>(H * M * d);
  b->fitA = c.take<double>(H * M * d);
  b->fitY = c.take<double>(H * M * d);
  b->fitZ = c.take<double>(H * (M > d ? M : d) * d);
  b->muX = c.take<double>(H * d);
  b->muR = c.take<double>(H * d);
  b->sX = c.take<double>(H * d);
  b->Bm = c.take<double>(H * d * d);
  b->Pm = c.take<double>(H * d * d);
  b->sig = c.take<double>(H * kMaxM);
  b->reff = c.take<int>(H);
  b->Bp = c.take<float>(H * d * d);
  b->BpT = c.take<float>(H * d * d);
  b->cvec = c.take<float>(H * d);
  b->work = c.take<int>(H * (size_t)tc_max_items(m));
  b->nwork = c.take<int>(H);
  {
    const size_t Nm = Nk > Nq ? Nk : Nq, Cm = Ck > Cq ? Ck : Cq;
    const size_t Np = (size_t)km_tc_npad((int)Nm), Cp = (size_t)km_tc_cpad((int)Cm);
    b->kmXhi = c.take<__nv_bfloat16>(H * Np * 64);
    b->kmXlo = c.take<__nv_bfloat16>(H * Np * 64);
    b->kmXn = c.take<float>(H * Nm);
    b->kmChi = c.take<__nv_bfloat16>(H * Cp * 64);
    b->kmClo = c.take<__nv_bfloat16>(H * Cp * 64);
    b->kmCn = c.take<float>(H * Cp);
    b->kmCmaxb = c.take<int>(2 * H);
    b->kmQueue = c.take<int4>((size_t)km_tc_queue_cap((int)H, (int)Nm));
    b->kmQcnt = c.take<int>(2);
    b->kmU = c.take<double>(H * Nm);
    b->kmL = c.take<float>(H * Nm * (size_t)cdiv((int)Cm, 32));
    b->kmDelta = c.take<double>(H * Cm);
    b->kmDmax = c.take<unsigned long long>(2 * H * (size_t)cdiv((int)Cm, 32));
    b->kmAidx = c.take<int>(H * Np);
    b->kmAcnt = c.take<int>(2 * H);
    b->kmReassigned = c.take<long long>(2 * H);
    b->kmShi = c.take<__nv_bfloat16>(H * Np * 64);
    b->kmSlo = c.take<__nv_bfloat16>(H * Np * 64);
  }
  b->warmCold = c.take<int>(2 * H);
  {
    const size_t Nm = Nk > Nq ? Nk : Nq, Cm = Ck > Cq ? Ck : Cq;
    b->kmFx = c.take<unsigned long long>(H * Cm * 64 * 3);
    b->kmFxCnt = c.take<int>(H * Cm);
    b->kmChg = c.take<unsigned long long>(H * Nm);
  }
  b->err = c.take<int>(64);
  return (c.off + 255) & ~size_t(255);
}

sparsepr_status make_plan(const sparsepr_params* q, const void* Q, const void* K,
                          const void* V, void* ws, size_t ws_bytes, sparsepr_plan_t* out,
                          Plan* plan) {
  sparsepr_status s = validate(q);
  if (s != SPARSEPR_OK) return s;
  if (!Q || !K || !V || !out) return SPARSEPR_ERR_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V)) return SPARSEPR_ERR_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return SPARSEPR_ERR_WORKSPACE;
  plan->dm = make_dims(q);
  const size_t need = carve(plan->dm, nullptr, &plan->b);
  if (ws_bytes < need) return SPARSEPR_ERR_WORKSPACE;
  carve(plan->dm, reinterpret_cast<char*>(ws), &plan->b);
  plan->Q = Q; plan->K = K; plan->V = V;
  plan->warm = nullptr;
  plan->stage = 0;
  return SPARSEPR_OK;
}

#define SPR_TRY(expr)                                  \
  do {                                                 \
    sparsepr_status s_ = (expr);                       \
    if (s_ != SPARSEPR_OK) return s_;                  \
  } while (0)

sparsepr_status run_plan(Plan& p, const int32_t* labQ, const int32_t* labK, cudaStream_t st) {
  const Dims& m = p.dm;
  SPR_CUDA_OK(cudaMemsetAsync(p.b.err, 0, 64 * sizeof(int), st));
  SPR_CUDA_OK(cudaMemsetAsync(p.b.kmK, 0, m.H * 4 * sizeof(int), st));
  SPR_CUDA_OK(cudaMemsetAsync(p.b.kmQ, 0, m.H * 4 * sizeof(int), st));
  SPR_CUDA_OK(cudaMemsetAsync(p.b.pairs, 0, m.H * sizeof(long long), st));
  SPR_CUDA_OK(cudaMemsetAsync(p.b.kmReassigned, 0, 2 * m.H * sizeof(long long), st));
  // key side (paper S4.1, App. B.1)
  if (m.semantic) {
    SPR_TRY(launch_identity_factors(p, st));       // F_K = F_Q = I: raw rows as coordinates
  } else {
    SPR_TRY(launch_key_metric(p, st));
    SPR_TRY(p.warm ? launch_warm_factor(p, false, st) : launch_eigen_factor(p, false, st));
  }
  SPR_TRY(launch_project_keys(p, st));
  if (labK) {
    SPR_CUDA_OK(cudaMemcpyAsync(p.b.labK, labK, sizeof(int) * m.Hk * m.Nk,
                                cudaMemcpyDeviceToDevice, st));
    SPR_TRY(launch_check_labels(p, false, st));
  } else {
    SPR_TRY(launch_kmeans(p, false, st));
  }
  SPR_TRY(launch_finalize_groups(p, false, st));
  SPR_TRY(launch_centroids(p, false, st));
  // query side (paper S4.1, App. B.2)
  if (!m.semantic) {
    SPR_TRY(launch_query_metric(p, st));
    SPR_TRY(p.warm ? launch_warm_factor(p, true, st) : launch_eigen_factor(p, true, st));
  }
  SPR_TRY(launch_project_queries(p, st));
  if (labQ) {
    SPR_CUDA_OK(cudaMemcpyAsync(p.b.labQ, labQ, sizeof(int) * m.H * m.Nq,
                                cudaMemcpyDeviceToDevice, st));
    SPR_TRY(launch_check_labels(p, true, st));
  } else {
    SPR_TRY(launch_kmeans(p, true, st));
  }
  SPR_TRY(launch_finalize_groups(p, true, st));
  SPR_TRY(launch_centroids(p, true, st));
  // routing (App. B.3, S4.3), group-major layout, probes (App. A.2)
  SPR_TRY(launch_route(p, st));
  SPR_TRY(launch_permute(p, st));
  SPR_TRY(launch_select_probes(p, st));
  p.stage = 1;
  return SPARSEPR_OK;
}

struct ExportDesc {
  const void* ptr;
  size_t bytes;
};

ExportDesc export_desc(const Plan& p, int what) {
  const Dims& m = p.dm;
  const Buffers& b = p.b;
  const size_t H = m.H, Hk = m.Hk, d = m.d, I = sizeof(int), D = sizeof(double), F = sizeof(float);
  switch (what) {
    case SPARSEPR_X_LABELS_K: return {b.labK, Hk * m.Nk * I};
    case SPARSEPR_X_LABELS_Q: return {b.labQ, H * m.Nq * I};
    case SPARSEPR_X_PERM_K: return {b.permK, Hk * m.Nk * I};
    case SPARSEPR_X_PERM_Q: return {b.permQ, H * m.Nq * I};
    case SPARSEPR_X_GROUPS_K: return {b.nK, Hk * I};
    case SPARSEPR_X_GROUPS_Q: return {b.nQ, H * I};
    case SPARSEPR_X_SIZES_K: return {b.sizeK, Hk * m.Ck * I};
    case SPARSEPR_X_SIZES_Q: return {b.sizeQ, H * m.Cq * I};
    case SPARSEPR_X_CELL_COUNT: return {b.cellCnt, H * m.Cq * I};
    case SPARSEPR_X_CELL_IDS: return {b.cellIds, H * m.Cq * m.Ck * I};
    case SPARSEPR_X_PROBES: return {b.probes, H * m.M * I};
    case SPARSEPR_X_PROBE_COUNT: return {b.mA, H * m.Cq * I};
    case SPARSEPR_X_KMEANS_ITERS: return {nullptr, H * 2 * I};   // gathered specially
    case SPARSEPR_X_OBJECTIVE: return {nullptr, H * 2 * D};      // gathered specially
    case SPARSEPR_X_PAIRS: return {b.pairs, H * sizeof(long long)};
    case SPARSEPR_X_FACTOR_K: return {b.FK64, Hk * d * m.rK * D};
    case SPARSEPR_X_FACTOR_Q: return {b.FQ64, Hk * d * m.rQ * D};
    case SPARSEPR_X_EIG_K: return {b.lamK, Hk * m.rK * D};
    case SPARSEPR_X_EIG_Q: return {b.lamQ, Hk * m.rQ * D};
    case SPARSEPR_X_METRIC_K: return {b.MK, Hk * d * d * D};
    case SPARSEPR_X_METRIC_Q: return {b.MQ, Hk * d * d * D};
    case SPARSEPR_X_PHI_K: return {b.phiK, Hk * m.Nk * m.rK * D};
    case SPARSEPR_X_PHI_Q: return {b.phiQ, H * m.Nq * m.rQ * D};
    case SPARSEPR_X_CENTRES_Q: return {b.centQ, H * m.Cq * m.rQ * D};
    case SPARSEPR_X_SCORES: return {b.scores, H * m.Cq * m.Ck * D};
    case SPARSEPR_X_OSP: return {b.Osp, H * m.Nq * d * F};
    case SPARSEPR_X_ODENSE_PROBE: return {b.Odense, H * m.M * d * F};
    case SPARSEPR_X_FIT_MU_X: return {b.muX, H * d * D};
    case SPARSEPR_X_FIT_MU_R: return {b.muR, H * d * D};
    case SPARSEPR_X_FIT_S: return {b.sX, H * d * D};
    case SPARSEPR_X_FIT_B: return {b.Bm, H * d * d * D};
    case SPARSEPR_X_FIT_P: return {b.Pm, H * d * d * D};
    case SPARSEPR_X_FIT_REFF: return {b.reff, H * I};
    case SPARSEPR_X_PROBE_DIST: return {b.dist, H * m.Nq * D};
    case SPARSEPR_X_KBAR: return {b.kbar, Hk * m.Ck * d * D};
    case SPARSEPR_X_QBAR: return {b.qbar, H * m.Cq * d * D};
    case SPARSEPR_X_KM_REASSIGNED: return {b.kmReassigned, H * 2 * sizeof(long long)};
    case SPARSEPR_X_BETA: return {b.betaH, H * D};
    default: return {nullptr, 0};
  }
}

}  // namespace

extern "C" {

sparsepr_status sparsepr_workspace_size(const sparsepr_params* params, size_t* bytes) {
  sparsepr_status s = validate(params);
  if (s != SPARSEPR_OK) return s;
  if (!bytes) return SPARSEPR_ERR_ARG;
  Buffers b;
  *bytes = carve(make_dims(params), nullptr, &b);
  return SPARSEPR_OK;
}

static sparsepr_status plan_common(const sparsepr_params* params, const void* Q, const void* K,
                                   const void* V, const int32_t* labQ, const int32_t* labK,
                                   const void* warm, void* ws, size_t ws_bytes, void* stream,
                                   sparsepr_plan_t* out) {
  if (out) *out = nullptr;
  sparsepr_plan_s* h = new (std::nothrow) sparsepr_plan_s();
  if (!h) return SPARSEPR_ERR_ARG;
  sparsepr_status s = make_plan(params, Q, K, V, ws, ws_bytes, out, &h->p);
  h->p.warm = warm;
  if (s == SPARSEPR_OK) s = run_plan(h->p, labQ, labK, reinterpret_cast<cudaStream_t>(stream));
  if (s != SPARSEPR_OK) {
    delete h;
    return s;
  }
  *out = h;
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_plan(const sparsepr_params* params, const void* Q, const void* K,
                              const void* V, void* workspace, size_t workspace_bytes,
                              void* stream, sparsepr_plan_t* out) {
  return plan_common(params, Q, K, V, nullptr, nullptr, nullptr, workspace, workspace_bytes, stream, out);
}

sparsepr_status sparsepr_state_size(const sparsepr_params* params, size_t* bytes) {
  sparsepr_status s = validate(params);
  if (s != SPARSEPR_OK) return s;
  if (!bytes) return SPARSEPR_ERR_ARG;
  *bytes = state_layout(make_dims(params)).total;
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_plan_warm(const sparsepr_params* params, const void* Q, const void* K,
                                   const void* V, const void* state, void* workspace,
                                   size_t workspace_bytes, void* stream, sparsepr_plan_t* out) {
  if (!state || (reinterpret_cast<uintptr_t>(state) & 255)) return SPARSEPR_ERR_ARG;
  if (params && (params->G > 1 || params->partition != SPARSEPR_PARTITION_RESPONSE)) return SPARSEPR_ERR_ARG;
  return plan_common(params, Q, K, V, nullptr, nullptr, state, workspace, workspace_bytes, stream, out);
}

sparsepr_status sparsepr_save_state(sparsepr_plan_t plan, void* state, void* stream) {
  if (!plan || !state || (reinterpret_cast<uintptr_t>(state) & 255)) return SPARSEPR_ERR_ARG;
  if (plan->p.dm.G > 1 || plan->p.dm.semantic) return SPARSEPR_ERR_ARG;   // as sparsepr_plan_warm
  if (plan->p.stage < 1) return SPARSEPR_ERR_STATE;
  return launch_save_state(plan->p, state, reinterpret_cast<cudaStream_t>(stream));
}

sparsepr_status sparsepr_plan_from_labels(const sparsepr_params* params, const void* Q,
                                          const void* K, const void* V,
                                          const int32_t* labQ, const int32_t* labK,
                                          void* workspace, size_t workspace_bytes,
                                          void* stream, sparsepr_plan_t* out) {
  if (!labQ || !labK) return SPARSEPR_ERR_ARG;
  return plan_common(params, Q, K, V, labQ, labK, nullptr, workspace, workspace_bytes, stream, out);
}

sparsepr_status sparsepr_attend(sparsepr_plan_t plan, void* stream) {
  if (!plan) return SPARSEPR_ERR_ARG;
  if (plan->p.stage < 1) return SPARSEPR_ERR_STATE;
  SPR_TRY(launch_sparse_attention(plan->p, reinterpret_cast<cudaStream_t>(stream)));
  plan->p.stage = 2;
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_probe_fit(sparsepr_plan_t plan, void* stream) {
  if (!plan) return SPARSEPR_ERR_ARG;
  if (plan->p.stage < 2) return SPARSEPR_ERR_STATE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  SPR_TRY(launch_probe_attention(plan->p, st));
  SPR_TRY(launch_fit(plan->p, st));
  plan->p.stage = 3;
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_correct(sparsepr_plan_t plan, void* Out, void* stream) {
  if (!plan || !Out || !aligned16(Out)) return SPARSEPR_ERR_ARG;
  if (plan->p.stage < 3) return SPARSEPR_ERR_STATE;
  return launch_correct(plan->p, Out, reinterpret_cast<cudaStream_t>(stream));
}

sparsepr_status sparsepr_forward(const sparsepr_params* params, const void* Q, const void* K,
                                 const void* V, void* Out, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  if (!Out) return SPARSEPR_ERR_ARG;
  sparsepr_plan_t plan = nullptr;
  SPR_TRY(sparsepr_plan(params, Q, K, V, workspace, workspace_bytes, stream, &plan));
  sparsepr_status s = sparsepr_attend(plan, stream);
  if (s == SPARSEPR_OK) s = sparsepr_probe_fit(plan, stream);
  if (s == SPARSEPR_OK) s = sparsepr_correct(plan, Out, stream);
  sparsepr_destroy(plan);
  return s;
}

sparsepr_status sparsepr_dense_attention(const sparsepr_params* params, const void* Q,
                                         const void* K, const void* V, void* Out,
                                         void* stream) {
  if (!params || !Q || !K || !V || !Out) return SPARSEPR_ERR_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(Out)) return SPARSEPR_ERR_ARG;
  if (params->dtype != SPARSEPR_F32 && params->dtype != SPARSEPR_BF16) return SPARSEPR_ERR_DTYPE;
  if (params->H < 1 || params->N_q < 1 || params->N_k < 1) return SPARSEPR_ERR_SHAPE;
  if (params->d < 8 || params->d > kMaxD || params->d % 8) return SPARSEPR_ERR_SHAPE;
  if (params->engine != SPARSEPR_ENGINE_AUTO && params->engine != SPARSEPR_ENGINE_SIMT)
    return SPARSEPR_ERR_ARG;
  if (params->G < 0 || (params->G > 1 && params->H % params->G != 0)) return SPARSEPR_ERR_SHAPE;
  Dims m{};
  m.H = params->H; m.Nq = params->N_q; m.Nk = params->N_k; m.d = params->d;
  m.dtype = params->dtype; m.engine = params->engine;
  m.G = params->G > 1 ? params->G : 1;
  m.Hk = m.H / m.G;
  return launch_dense_attention(m, Q, K, V, Out, reinterpret_cast<cudaStream_t>(stream));
}

sparsepr_status sparsepr_affine_workspace_size(sparsepr_plan_t plan, size_t* bytes) {
  if (!plan || !bytes) return SPARSEPR_ERR_ARG;
  *bytes = affine_ws_doubles(plan->p.dm) * sizeof(double);
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_affine_fit(sparsepr_plan_t plan, const void* dense, void* workspace,
                                    size_t workspace_bytes, double* explained, double* err,
                                    void* stream) {
  if (!plan || !dense || !explained || !err) return SPARSEPR_ERR_ARG;
  if (plan->p.stage < 2) return SPARSEPR_ERR_STATE;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) ||
      workspace_bytes < affine_ws_doubles(plan->p.dm) * sizeof(double))
    return SPARSEPR_ERR_WORKSPACE;
  return launch_affine_fit(plan->p, dense, reinterpret_cast<double*>(workspace), explained, err,
                           reinterpret_cast<cudaStream_t>(stream));
}

sparsepr_status sparsepr_dense_check(void* stream, int32_t* device_error) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int* words[2] = {nullptr, nullptr};
  SPR_TRY(dense_error_address(&words[0]));
  SPR_TRY(noalloc_error_address(&words[1]));
  int v[2] = {0, 0};
  SPR_CUDA_OK(cudaStreamSynchronize(st));
  for (int k = 0; k < 2; ++k) {
    SPR_CUDA_OK(cudaMemcpyAsync(&v[k], words[k], sizeof(int), cudaMemcpyDeviceToHost, st));
    SPR_CUDA_OK(cudaMemsetAsync(words[k], 0, sizeof(int), st));
  }
  SPR_CUDA_OK(cudaStreamSynchronize(st));
  const int e = v[0] | v[1];
  if (device_error) *device_error = e;
  return e ? SPARSEPR_ERR_DEVICE_CHECK : SPARSEPR_OK;
}

sparsepr_status sparsepr_wait_selftest(void* stream) {
  return launch_wait_selftest(reinterpret_cast<cudaStream_t>(stream));
}

sparsepr_status sparsepr_check(sparsepr_plan_t plan, void* stream, int32_t* device_error) {
  if (!plan) return SPARSEPR_ERR_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int e = 0;
  SPR_CUDA_OK(cudaMemcpyAsync(&e, plan->p.b.err, sizeof(int), cudaMemcpyDeviceToHost, st));
  SPR_CUDA_OK(cudaStreamSynchronize(st));
  if (device_error) *device_error = e;
  return e ? SPARSEPR_ERR_DEVICE_CHECK : SPARSEPR_OK;
}

sparsepr_status sparsepr_get_stats(sparsepr_plan_t plan, void* stream, sparsepr_stats* stats) {
  if (!plan || !stats) return SPARSEPR_ERR_ARG;
  if (plan->p.stage < 1) return SPARSEPR_ERR_STATE;
  const Plan& p = plan->p;
  const int H = p.dm.H;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  long long* pairs = new long long[H];
  int* km = new int[H * 8 + 2 * H + 1];
  int *kmK = km, *kmQ = km + 4 * H, *nK = km + 8 * H, *nQ = km + 9 * H, *err = km + 10 * H;
  cudaError_t e = cudaMemcpyAsync(pairs, p.b.pairs, H * sizeof(long long), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(kmK, p.b.kmK, 4 * H * sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(kmQ, p.b.kmQ, 4 * H * sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(nK, p.b.nK, H * sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(nQ, p.b.nQ, H * sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(err, p.b.err, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) {
    delete[] pairs;
    delete[] km;
    return SPARSEPR_ERR_CUDA;
  }
  sparsepr_stats s{};
  s.groups_k_min = 1 << 30;
  s.groups_q_min = 1 << 30;
  for (int h = 0; h < H; ++h) {
    s.pairs_route += pairs[h];
    s.kmeans_iters_q_max = kmQ[4 * h + 3] > s.kmeans_iters_q_max ? kmQ[4 * h + 3] : s.kmeans_iters_q_max;
    s.groups_q_min = nQ[h] < s.groups_q_min ? nQ[h] : s.groups_q_min;
  }
  for (int hk = 0; hk < p.dm.Hk; ++hk) {          // K/V heads
    s.kmeans_iters_k_max = kmK[4 * hk + 3] > s.kmeans_iters_k_max ? kmK[4 * hk + 3] : s.kmeans_iters_k_max;
    s.groups_k_min = nK[hk] < s.groups_k_min ? nK[hk] : s.groups_k_min;
  }
  const double total = (double)H * p.dm.Nq * p.dm.Nk;
  s.pairs_exec = s.pairs_route + (long long)H * p.dm.M * p.dm.Nk;
  s.rho_route = (double)s.pairs_route / total;
  s.rho_exec = (double)s.pairs_exec / total;
  s.device_error = *err;
  *stats = s;
  delete[] pairs;
  delete[] km;
  return *err ? SPARSEPR_ERR_DEVICE_CHECK : SPARSEPR_OK;
}

sparsepr_status sparsepr_export_size(sparsepr_plan_t plan, int32_t what, size_t* bytes) {
  if (!plan || !bytes || what < 0 || what >= SPARSEPR_X_COUNT) return SPARSEPR_ERR_ARG;
  *bytes = export_desc(plan->p, what).bytes;
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_export(sparsepr_plan_t plan, int32_t what, void* dst, size_t bytes,
                                void* stream) {
  if (!plan || !dst || what < 0 || what >= SPARSEPR_X_COUNT) return SPARSEPR_ERR_ARG;
  const Plan& p = plan->p;
  ExportDesc x = export_desc(p, what);
  if (bytes != x.bytes) return SPARSEPR_ERR_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // row h: key side of its K/V head h / G, query side of h
  if (what == SPARSEPR_X_KMEANS_ITERS) {
    const int H = p.dm.H, G = p.dm.G;
    int* km = new int[8 * H];
    cudaError_t e = cudaMemcpyAsync(km, p.b.kmK, 4 * H * sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(km + 4 * H, p.b.kmQ, 4 * H * sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess) {
      int* o = reinterpret_cast<int*>(dst);
      for (int h = 0; h < H; ++h) {
        o[2 * h] = km[4 * (h / G) + 3];
        o[2 * h + 1] = km[4 * H + 4 * h + 3];
      }
    }
    delete[] km;
    return e == cudaSuccess ? SPARSEPR_OK : SPARSEPR_ERR_CUDA;
  }
  if (what == SPARSEPR_X_OBJECTIVE) {
    const int H = p.dm.H, G = p.dm.G;
    double* ob = new double[2 * H];
    cudaError_t e = cudaMemcpyAsync(ob, p.b.objH, 2 * H * sizeof(double), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess) {
      double* o = reinterpret_cast<double*>(dst);
      for (int h = 0; h < H; ++h) {
        o[2 * h] = ob[2 * (h / G)];
        o[2 * h + 1] = ob[2 * h + 1];
      }
    }
    delete[] ob;
    return e == cudaSuccess ? SPARSEPR_OK : SPARSEPR_ERR_CUDA;
  }
  SPR_CUDA_OK(cudaMemcpyAsync(dst, x.ptr, x.bytes, cudaMemcpyDeviceToHost, st));
  SPR_CUDA_OK(cudaStreamSynchronize(st));
  return SPARSEPR_OK;
}

void sparsepr_destroy(sparsepr_plan_t plan) { delete plan; }

const char* sparsepr_status_string(sparsepr_status status) {
  switch (status) {
    case SPARSEPR_OK: return "ok";
    case SPARSEPR_ERR_ARG: return "invalid argument";
    case SPARSEPR_ERR_SHAPE: return "unsupported shape";
    case SPARSEPR_ERR_DTYPE: return "unsupported dtype";
    case SPARSEPR_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case SPARSEPR_ERR_CUDA: return "CUDA error";
    case SPARSEPR_ERR_DEVICE_CHECK: return "device-side check failed";
    case SPARSEPR_ERR_STATE: return "call out of order for this plan";
  }
  return "unknown status";
}

}  // extern "C"

extern "C" unsigned long long sparsepr_launch_count(void) { return spr::g_launches.load(); }
