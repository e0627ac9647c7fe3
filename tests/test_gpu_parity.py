"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on a B200.

Two modes, as the acceptance rules of the method's reproduction fix them:
  * free running: the GPU runs its own k-means (same SplitMix64 initial rows as the
    oracle); labels must agree on >= 99.9% of rows and objectives within 1e-4 relative;
  * labels injected: the GPU plan is built from the ORACLE's final labels; then every
    indexing result (permutations, group sizes, selected cells, routed pairs, probe rows)
    must be bit-exact and the corrected output within 1e-5 (fp32) / 1e-2 (bf16) relative
    Frobenius error.
Full-size workloads (the shapes the benchmark times) are checked on sampled heads and
2048 evenly spaced rows per head, the oracle computing only those rows.
"""
import math

import numpy as np
import pytest
import torch

from free_block_sparse_plan_b200 import native as N
from free_block_sparse_plan_b200 import workloads as W
from oracle import sparsepr_oracle as O

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 1e-2}
_oracle_cache = {}


RAN = []                  # set once the module's GPU tests start (for the summary)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    RAN.append(True)


def oracle_head(w: W.Workload, h: int, rows=None):
    """Oracle call for head h of workload w (cached partition per head)."""
    key = (w, h)
    p = O.Params.from_dict(w.params())
    if key not in _oracle_cache:
        q, k, v = W.make_head(w, h)
        _oracle_cache[key] = (q, k, v, O.partition(q, k, v, p, h))
    q, k, v, part = _oracle_cache[key]
    return q, k, v, O.sparsepr_call(q, k, v, p, head=h, rows=rows, part=part)


def gpu_call(w, inputs=None, labels=None, engine=N.SPARSEPR_ENGINE_AUTO, params=None):
    Q, K, V = inputs if inputs is not None else W.make_inputs_torch(w, device="cuda")
    params = params or N.params_from_dict(w.params(), engine)
    plan = N.Plan(params, Q, K, V, labels=labels)
    plan.attend()
    plan.probe_fit()
    out = plan.correct()
    torch.cuda.synchronize()
    return plan, out, (Q, K, V)


def rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


PROBE_TIE_TOL = 1e-6      # both sides compute the probe distances in fp64
SWAPS_EXCUSED = []        # (test id, head, positions) of every tie-ambiguous swap excused


def tie_ambiguous_probes(res: O.CallResult, gpu_probes: np.ndarray, tol=PROBE_TIE_TOL,
                         where="") -> bool:
    """True if the probe lists are equal, or if every position where they differ swaps
    two rows of one query group whose oracle distances agree to `tol` relative (the
    radial order of Algorithm A.1 is then decided by rounding).  Each excused swap is
    recorded in SWAPS_EXCUSED and printed."""
    if np.array_equal(gpu_probes, res.probes):
        return True
    comp = res.part.gq.compact
    swaps = []
    for pos, (g, o) in enumerate(zip(gpu_probes, res.probes)):
        if g == o:
            continue
        if comp[g] != comp[o]:
            return False
        dg, do = res.probe_dist[g], res.probe_dist[o]
        if abs(dg - do) > tol * max(abs(dg), abs(do), 1e-30):
            return False
        swaps.append(pos)
    SWAPS_EXCUSED.append((where, swaps))
    print(f"tie-ambiguous probe swaps excused {where}: positions {swaps}")
    return True


def check_injected_head(plan, out_h, res: O.CallResult, h, w, exact_probes=True):
    """Bit-exact indexing and output tolerance for head h of a label-injected plan."""
    gq, gk = res.part.gq, res.part.gk
    ex = {k: plan.export(k) for k in ("PERM_Q", "PERM_K", "GROUPS_Q", "GROUPS_K", "SIZES_Q",
                                      "SIZES_K", "CELL_COUNT", "CELL_IDS", "PAIRS", "PROBES",
                                      "PROBE_COUNT")}
    assert np.array_equal(ex["PERM_Q"][h], res.permQ)
    assert np.array_equal(ex["PERM_K"][h], res.permK)
    assert ex["GROUPS_Q"][h] == gq.sizes.size and ex["GROUPS_K"][h] == gk.sizes.size
    assert np.array_equal(ex["SIZES_Q"][h][:gq.sizes.size], gq.sizes)
    assert np.array_equal(ex["SIZES_K"][h][:gk.sizes.size], gk.sizes)
    for a, sel in enumerate(res.sel):
        assert ex["CELL_COUNT"][h][a] == sel.size, a
        assert np.array_equal(ex["CELL_IDS"][h][a][:sel.size], sel), a
    assert int(ex["PAIRS"][h]) == res.pairs_route
    if exact_probes:
        assert tie_ambiguous_probes(res, ex["PROBES"][h], where=f"{w.name} head {h}"), \
            (ex["PROBES"][h], res.probes)
        if np.array_equal(ex["PROBES"][h], res.probes):
            assert np.array_equal(ex["PROBE_COUNT"][h][:gq.sizes.size], res.m_a)
    err = rel(out_h[res.rows], res.out)
    assert err < TOL[w.dtype], err
    return err


# ---------------------------------------------------------------------------------- tiny
def test_tiny_free_running_matches_oracle():
    w = W.TINY
    plan, out, _ = gpu_call(w)
    _, _, _, res = oracle_head(w, 0)
    labK, labQ = plan.export("LABELS_K")[0], plan.export("LABELS_Q")[0]
    assert np.mean(labK == res.part.km_K.labels) >= 0.999
    assert np.mean(labQ == res.part.km_Q.labels) >= 0.999
    obj = plan.export("OBJECTIVE")[0]
    assert abs(obj[0] - res.part.km_K.objective) <= 1e-4 * res.part.km_K.objective
    assert abs(obj[1] - res.part.km_Q.objective) <= 1e-4 * res.part.km_Q.objective
    iters = plan.export("KMEANS_ITERS")[0]
    assert tuple(iters) == (res.part.km_K.iterations, res.part.km_Q.iterations)
    assert plan.check() == 0
    if np.array_equal(labK, res.part.km_K.labels) and np.array_equal(labQ, res.part.km_Q.labels):
        assert rel(out[0].double().cpu().numpy(), res.out) < 1e-5


def _align_signs(F_gpu, F_ref):
    s = np.sign((F_gpu * F_ref).sum(axis=0))
    s[s == 0] = 1
    return s


def test_tiny_injected_stagewise():
    w = W.TINY
    _, _, _, res = oracle_head(w, 0)
    part = res.part
    labQ = torch.tensor(part.km_Q.labels[None], dtype=torch.int32, device="cuda")
    labK = torch.tensor(part.km_K.labels[None], dtype=torch.int32, device="cuda")
    plan, out, _ = gpu_call(w, labels=(labQ, labK))
    assert plan.check() == 0
    # key metric and factor (fp64 on both sides)
    assert rel(plan.export("METRIC_K")[0], part.M_K) < 1e-12
    assert rel(plan.export("EIG_K")[0], part.lam_K) < 1e-10
    FK = plan.export("FACTOR_K")[0]
    s = _align_signs(FK, part.F_K)
    assert rel(FK * s, part.F_K) < 1e-8
    assert rel(plan.export("PHI_K")[0] * s, part.phiK) < 1e-7
    # centroids, query metric, factor, coordinates
    nk, nq = part.gk.sizes.size, part.gq.sizes.size
    assert rel(plan.export("KBAR")[0][:nk], part.kbar) < 1e-13
    assert rel(plan.export("QBAR")[0][:nq], part.qbar) < 1e-13
    assert rel(plan.export("METRIC_Q")[0], part.M_Q) < 1e-12
    FQ = plan.export("FACTOR_Q")[0]
    sq = _align_signs(FQ, part.F_Q)
    assert rel(FQ * sq, part.F_Q) < 1e-8
    assert rel(plan.export("PHI_Q")[0] * sq, part.phiQ) < 1e-7
    # routing scores (fp64), then indexing bit-exact and output
    assert rel(plan.export("SCORES")[0][:nq, :nk], res.scores) < 1e-12
    assert rel(plan.export("PROBE_DIST")[0], res.probe_dist) < 1e-7
    perm = plan.export("PERM_Q")[0]
    osp = plan.export("OSP")[0]
    osp_rows = np.empty_like(osp)
    osp_rows[perm] = osp
    assert rel(osp_rows, res.osp) < 1e-5
    assert rel(plan.export("ODENSE_PROBE")[0], res.dense_probe) < 1e-5
    assert rel(plan.export("FIT_MU_X")[0], res.fit.mu_x) < 1e-5
    assert rel(plan.export("FIT_S")[0], res.fit.s) < 1e-5
    assert int(plan.export("FIT_REFF")[0]) == res.fit.r_eff
    # the ridge B and the projector P element by element: the oracle's fit ([P] S4.2,
    # App. D.2) run on the GPU's own probe outputs, so only the fit stage is compared
    assert np.array_equal(plan.export("PROBES")[0], res.probes)
    x_gpu = osp_rows[res.probes]
    R_gpu = plan.export("ODENSE_PROBE")[0].astype(np.float64) - x_gpu
    fit = O.fit_residual(x_gpu.astype(np.float64), R_gpu, res.weights, w.lam, w.r)
    assert rel(plan.export("FIT_MU_X")[0], fit.mu_x) < 1e-12
    assert rel(plan.export("FIT_MU_R")[0], fit.mu_R) < 1e-12
    assert rel(plan.export("FIT_S")[0], fit.s) < 1e-12
    assert rel(plan.export("FIT_B")[0], fit.B) < 1e-8
    sig = fit.sigma
    assert sig[w.r - 1] > (1 + 1e-6) * sig[w.r]          # no singular-value tie at r
    assert np.abs(plan.export("FIT_P")[0] - fit.P).max() < 1e-8
    check_injected_head(plan, out[0].double().cpu().numpy(), res, 0, w)


@pytest.mark.parametrize("est", [N.SPARSEPR_EST_MEAN, N.SPARSEPR_EST_SCALAR, N.SPARSEPR_EST_DIAGONAL])
def test_restricted_estimators_match_oracle(est):
    # App. D.3's mean-only, scalar and diagonal corrections, oracle labels injected
    for w in (W.TINY.with_(estimator=est), W.MID.with_(H=2, estimator=est)):
        inputs = W.make_inputs_torch(w, device="cuda")
        ref = [oracle_head(w, h)[3] for h in range(w.H)]
        labQ = torch.tensor(np.stack([r.part.km_Q.labels for r in ref]), dtype=torch.int32, device="cuda")
        labK = torch.tensor(np.stack([r.part.km_K.labels for r in ref]), dtype=torch.int32, device="cuda")
        plan, out, _ = gpu_call(w, inputs=inputs, labels=(labQ, labK))
        assert plan.check() == 0
        B = plan.export("FIT_B")
        for h, res in enumerate(ref):
            if est == N.SPARSEPR_EST_MEAN:
                assert np.all(B[h] == 0.0)
            elif np.array_equal(plan.export("PROBES")[h], res.probes):
                # B is a least-squares coefficient of the residuals R = dense - sparse on the
                # standardised features; where the two barely correlate B is near zero and
                # its relative error means nothing.  Its error is measured on what it
                # predicts, x_bar (B - B_ref), against what it fits, R_bar (both weighted by
                # omega).  To first order a weighted least-squares fit moves by at most the
                # perturbation of its targets plus twice that of its features, so the bound
                # is taken from the GPU's own residuals and features against the oracle's.
                om = np.sqrt(w.M * res.weights / res.weights.sum())[:, None]
                osp = plan.export("OSP")[h]
                rows = np.empty_like(osp)
                rows[plan.export("PERM_Q")[h]] = osp
                x_gpu = rows[res.probes]
                R_gpu = plan.export("ODENSE_PROBE")[h] - x_gpu
                x, R = res.x_probe, res.dense_probe - res.x_probe
                xb = (x - res.fit.mu_x) / res.fit.s
                Rb_n = np.linalg.norm(om * (R - res.fit.mu_R))
                err = np.linalg.norm(om * (xb @ (B[h] - res.fit.B))) / Rb_n
                eps_R = np.linalg.norm(om * (R_gpu - R)) / Rb_n
                eps_x = np.linalg.norm(x_gpu - x) / np.linalg.norm(x - res.fit.mu_x)
                # on the bf16 path the residual (0.35% of the output at the mid shape) is
                # as small as the rounding of the bf16 probabilities, so eps_R is large
                # there and only the bound below (and the output check) apply
                if w.dtype == "f32":
                    assert eps_R < 1e-3, (h, eps_R)
                assert err < 3.0 * (eps_R + eps_x) + 1e-4, (h, err, eps_R, eps_x)
            assert np.array_equal(plan.export("FIT_P")[h], np.eye(w.d))
            check_injected_head(plan, out[h].double().cpu().numpy(), res, h, w)


def _ff(F):
    return F @ F.T


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_warm_start_sequence_matches_oracle(name):
    # App. C warm start: call 0 cold, call 1 on drifted inputs from call 0's saved state
    # (factors by two Cholesky subspace iterations, k-means from the previous centroids)
    w0 = W.TINY if name == "tiny" else W.MID.with_(H=2)
    w1 = w0.with_(step=1)
    params = N.params_from_dict(w0.params())
    P = O.Params.from_dict(w0.params())
    plan0 = N.Plan(params, *W.make_inputs_torch(w0, device="cuda"))
    state = plan0.save_state()
    plan1 = N.Plan(params, *W.make_inputs_torch(w1, device="cuda"), warm=state)
    plan1.attend()
    plan1.probe_fit()
    out = plan1.correct()
    torch.cuda.synchronize()
    assert plan1.check() == 0
    FK, FQ = plan1.export("FACTOR_K"), plan1.export("FACTOR_Q")
    labK, labQ = plan1.export("LABELS_K"), plan1.export("LABELS_Q")
    iters, obj = plan1.export("KMEANS_ITERS"), plan1.export("OBJECTIVE")
    rows = None if w0.N <= 4096 else (np.arange(2048) * w0.N) // 2048
    for h in range(w0.H):
        q0, k0, v0 = W.make_head(w0, h)
        st = O.warm_state(O.partition(q0, k0, v0, P, h), P)
        res = O.sparsepr_call(*W.make_head(w1, h), P, head=h, rows=rows, warm=st)
        part = res.part
        assert rel(_ff(FK[h]), _ff(part.F_K)) < 1e-10
        assert rel(_ff(FQ[h]), _ff(part.F_Q)) < 1e-10
        assert np.mean(labK[h] == part.km_K.labels) >= 0.999
        assert np.mean(labQ[h] == part.km_Q.labels) >= 0.999
        assert abs(obj[h][0] - part.km_K.objective) <= 1e-4 * part.km_K.objective
        assert abs(obj[h][1] - part.km_Q.objective) <= 1e-4 * part.km_Q.objective
        if np.array_equal(labK[h], part.km_K.labels) and np.array_equal(labQ[h], part.km_Q.labels):
            assert tuple(iters[h]) == (part.km_K.iterations, part.km_Q.iterations)
            assert rel(out[h].double().cpu().numpy()[res.rows], res.out) < TOL[w0.dtype]


def test_warm_state_that_was_never_saved_starts_cold_and_is_flagged():
    w = W.TINY
    inputs = W.make_inputs_torch(w, device="cuda")
    params = N.params_from_dict(w.params())
    cold, out_c, _ = gpu_call(w, inputs=inputs)
    state = torch.zeros(N.sparsepr_state_size(params), dtype=torch.uint8, device="cuda")
    plan = N.Plan(params, *inputs, warm=state)
    plan.attend()
    plan.probe_fit()
    out = plan.correct()
    torch.cuda.synchronize()
    assert plan.check() == 64                                  # the warm-state bit alone
    assert np.array_equal(plan.export("LABELS_K"), cold.export("LABELS_K"))
    assert np.array_equal(plan.export("LABELS_Q"), cold.export("LABELS_Q"))
    assert torch.equal(out, out_c)


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_gqa_shared_key_partition_matches_oracle(name):
    # App. C GQA: G query heads share each K/V head; the key metric comes from their
    # concatenated rows, the K/V groups and F_Q are shared, the rest is per query head
    w = (W.TINY.with_(H=2, G=2) if name == "tiny" else W.MID.with_(H=4, G=2))
    P = O.Params.from_dict(w.params())
    Q, K, V = W.make_inputs_torch(w, device="cuda")
    assert K.shape[0] == w.H_kv
    rows = None if w.N <= 4096 else (np.arange(2048) * w.N) // 2048
    groups = [W.make_kv_group(w, hk) for hk in range(w.H_kv)]
    parts = [O.partition(groups[h // w.G][0][h % w.G], groups[h // w.G][1], groups[h // w.G][2], P, h,
                         Qgroup=groups[h // w.G][0], kv_head=h // w.G) for h in range(w.H)]
    # free running: labels, objectives, iterations
    plan, out, _ = gpu_call(w, inputs=(Q, K, V))
    assert plan.check() == 0
    labK, labQ = plan.export("LABELS_K"), plan.export("LABELS_Q")
    MK = plan.export("METRIC_K")
    obj, iters = plan.export("OBJECTIVE"), plan.export("KMEANS_ITERS")
    for h, part in enumerate(parts):
        hk = h // w.G
        assert rel(MK[hk], part.M_K) < 1e-12
        assert np.mean(labK[hk] == part.km_K.labels) >= 0.999
        assert np.mean(labQ[h] == part.km_Q.labels) >= 0.999
        assert abs(obj[h][0] - part.km_K.objective) <= 1e-4 * part.km_K.objective
        assert abs(obj[h][1] - part.km_Q.objective) <= 1e-4 * part.km_Q.objective
        if np.array_equal(labK[hk], part.km_K.labels) and np.array_equal(labQ[h], part.km_Q.labels):
            assert tuple(iters[h]) == (part.km_K.iterations, part.km_Q.iterations)
    # oracle labels injected: bit-exact indexing and the output
    labQi = torch.tensor(np.stack([p_.km_Q.labels for p_ in parts]), dtype=torch.int32, device="cuda")
    labKi = torch.tensor(np.stack([parts[hk * w.G].km_K.labels for hk in range(w.H_kv)]),
                         dtype=torch.int32, device="cuda")
    plan, out, _ = gpu_call(w, inputs=(Q, K, V), labels=(labQi, labKi))
    assert plan.check() == 0
    for h, part in enumerate(parts):
        g = groups[h // w.G]
        res = O.sparsepr_call(g[0][h % w.G], g[1], g[2], P, head=h, rows=rows, part=part)
        check_injected_head_gqa(plan, out[h].double().cpu().numpy(), res, h, w)


def check_injected_head_gqa(plan, out_h, res, h, w):
    """check_injected_head with the K/V-side exports read at the K/V head h / G."""
    hk = h // w.G
    gq, gk = res.part.gq, res.part.gk
    assert np.array_equal(plan.export("PERM_Q")[h], res.permQ)
    assert np.array_equal(plan.export("PERM_K")[hk], res.permK)
    assert plan.export("GROUPS_Q")[h] == gq.sizes.size and plan.export("GROUPS_K")[hk] == gk.sizes.size
    cc, ci = plan.export("CELL_COUNT")[h], plan.export("CELL_IDS")[h]
    for a, sel in enumerate(res.sel):
        assert cc[a] == sel.size and np.array_equal(ci[a][:sel.size], sel), a
    assert int(plan.export("PAIRS")[h]) == res.pairs_route
    assert tie_ambiguous_probes(res, plan.export("PROBES")[h], where=f"{w.name} head {h} (GQA)")
    assert rel(out_h[res.rows], res.out) < TOL[w.dtype]


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_semantic_partition_matches_oracle(name):
    # the reference partition of the paper's S3 and ablations: k-means on raw rows
    w = (W.TINY if name == "tiny" else W.MID.with_(H=2)).with_(partition=1)
    P = O.Params.from_dict(w.params())
    assert P.partition == "semantic"
    Q, K, V = W.make_inputs_torch(w, device="cuda")
    rows = None if w.N <= 4096 else (np.arange(2048) * w.N) // 2048
    heads = [W.make_head(w, h) for h in range(w.H)]
    parts = [O.partition_semantic(*heads[h], P, h) for h in range(w.H)]
    plan, out, _ = gpu_call(w, inputs=(Q, K, V))
    assert plan.check() == 0
    labK, labQ = plan.export("LABELS_K"), plan.export("LABELS_Q")
    obj = plan.export("OBJECTIVE")
    for h, part in enumerate(parts):
        assert np.mean(labK[h] == part.km_K.labels) >= 0.999
        assert np.mean(labQ[h] == part.km_Q.labels) >= 0.999
        assert abs(obj[h][0] - part.km_K.objective) <= 1e-4 * part.km_K.objective
        assert abs(obj[h][1] - part.km_Q.objective) <= 1e-4 * part.km_Q.objective
    assert np.array_equal(plan.export("PHI_Q")[0], heads[0][0])      # raw rows, no RMS step
    labQi = torch.tensor(np.stack([p_.km_Q.labels for p_ in parts]), dtype=torch.int32, device="cuda")
    labKi = torch.tensor(np.stack([p_.km_K.labels for p_ in parts]), dtype=torch.int32, device="cuda")
    plan, out, _ = gpu_call(w, inputs=(Q, K, V), labels=(labQi, labKi))
    assert plan.check() == 0
    for h, part in enumerate(parts):
        res = O.sparsepr_call(*heads[h], P, head=h, rows=rows, part=part)
        check_injected_head(plan, out[h].double().cpu().numpy(), res, h, w)


def test_tiny_simt_engine_equals_auto():
    w = W.TINY
    _, out_a, inputs = gpu_call(w)
    _, out_s, _ = gpu_call(w, inputs=inputs, engine=N.SPARSEPR_ENGINE_SIMT)
    assert rel(out_a.cpu().numpy(), out_s.cpu().numpy()) < 1e-6


def test_deterministic_reruns():
    w = W.MID.with_(H=3)
    _, o1, inputs = gpu_call(w)
    _, o2, _ = gpu_call(w, inputs=inputs)
    assert torch.equal(o1, o2)


# ---------------------------------------------------------------------------------- mid
@pytest.fixture(scope="module")
def mid_runs():
    w = W.MID
    inputs = W.make_inputs_torch(w, device="cuda")
    free_plan, free_out, _ = gpu_call(w, inputs=inputs)
    ref = [oracle_head(w, h)[3] for h in range(w.H)]
    labQ = torch.tensor(np.stack([r.part.km_Q.labels for r in ref]), dtype=torch.int32, device="cuda")
    labK = torch.tensor(np.stack([r.part.km_K.labels for r in ref]), dtype=torch.int32, device="cuda")
    inj_plan, inj_out, _ = gpu_call(w, inputs=inputs, labels=(labQ, labK))
    return w, ref, free_plan, free_out, inj_plan, inj_out


def test_mid_free_running_labels_and_objective(mid_runs):
    w, ref, plan, _, _, _ = mid_runs
    labK, labQ, obj = plan.export("LABELS_K"), plan.export("LABELS_Q"), plan.export("OBJECTIVE")
    for h, r in enumerate(ref):
        assert np.mean(labK[h] == r.part.km_K.labels) >= 0.999, h
        assert np.mean(labQ[h] == r.part.km_Q.labels) >= 0.999, h
        assert abs(obj[h, 0] - r.part.km_K.objective) <= 1e-4 * r.part.km_K.objective
        assert abs(obj[h, 1] - r.part.km_Q.objective) <= 1e-4 * r.part.km_Q.objective


def test_mid_injected_bit_exact_and_output(mid_runs):
    w, ref, _, _, plan, out = mid_runs
    assert plan.check() == 0
    out_np = out.float().cpu().numpy()
    errs = [check_injected_head(plan, out_np[h], r, h, w) for h, r in enumerate(ref)]
    pairs = sum(r.pairs_route for r in ref)
    st = plan.stats()
    assert st["pairs_route"] == pairs
    assert st["pairs_exec"] == pairs + w.H * w.M * w.N
    assert max(errs) < TOL["bf16"]


# ---------------------------------------------------------------------------------- full size
def _full_size_check(w, heads, nrows=2048):
    inputs = W.make_inputs_torch(w, device="cuda")
    free_plan, _, _ = gpu_call(w, inputs=inputs)
    labK = free_plan.export("LABELS_K")
    labQ = free_plan.export("LABELS_Q")
    obj = free_plan.export("OBJECTIVE")
    rows = np.unique(np.linspace(0, w.N - 1, nrows).astype(np.int64))
    refs = {}
    for h in heads:
        _, _, _, res = oracle_head(w, h, rows=rows)
        refs[h] = res
        assert np.mean(labK[h] == res.part.km_K.labels) >= 0.999, h
        assert np.mean(labQ[h] == res.part.km_Q.labels) >= 0.999, h
        assert abs(obj[h, 0] - res.part.km_K.objective) <= 1e-4 * res.part.km_K.objective
        assert abs(obj[h, 1] - res.part.km_Q.objective) <= 1e-4 * res.part.km_Q.objective
        labK[h] = res.part.km_K.labels
        labQ[h] = res.part.km_Q.labels
    del free_plan
    plan, out, _ = gpu_call(w, inputs=inputs, labels=(torch.tensor(labQ, device="cuda"),
                                                      torch.tensor(labK, device="cuda")))
    assert plan.check() == 0
    for h in heads:
        check_injected_head(plan, out[h].float().cpu().numpy(), refs[h], h, w)


def test_wan_full_size_sampled_heads():
    _full_size_check(W.WAN, heads=(0, 20, 39))


def test_hunyuan_full_size_sampled_heads():
    _full_size_check(W.HUNYUAN, heads=(0, 23))


def test_operating_point_sweep_head0():
    # every (rho*, M) point of the operating-point sweep on the Wan-like head 0, oracle
    # labels injected (the partition does not depend on rho* or M)
    base = W.WAN
    q, k, v, _ = oracle_head(base, 0, rows=np.arange(4))
    part = _oracle_cache[(base, 0)][3]
    dt = torch.bfloat16
    Q, K, V = (torch.from_numpy(x.astype(np.float32))[None].to(dt).cuda() for x in (q, k, v))
    labQ = torch.tensor(part.km_Q.labels[None], dtype=torch.int32, device="cuda")
    labK = torch.tensor(part.km_K.labels[None], dtype=torch.int32, device="cuda")
    rows = np.unique(np.linspace(0, base.N - 1, 1024).astype(np.int64))
    points = [(rho, M) for rho in W.SWEEP_RHO for M in W.SWEEP_M]
    assert len(points) == 15
    for rho, M in points:
        w = base.with_(H=1, rho=rho, M=M)
        p = O.Params.from_dict(w.params())
        res = O.sparsepr_call(q, k, v, p, head=0, rows=rows, part=part)
        plan, out, _ = gpu_call(w, inputs=(Q, K, V), labels=(labQ, labK))
        check_injected_head(plan, out[0].float().cpu().numpy(), res, 0, w)
        st = plan.stats()
        assert abs(st["rho_exec"] - res.rho_exec) < 1e-15


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_calibrated_budget_matches_oracle(name):
    # App. D.2's budget calibrated toward the target (reading S13): the per-head budget,
    # the selected cells and the routed pairs bit-exact with oracle labels injected, the
    # output within tolerance, and the realised density no farther from the target than
    # the plain prefix rule's.
    base = W.TINY if name == "tiny" else W.MID.with_(H=3)
    w = base.with_(budget=1)
    inputs = W.make_inputs_torch(w, device="cuda")
    ref = [oracle_head(w, h)[3] for h in range(w.H)]
    labQ = torch.tensor(np.stack([r.part.km_Q.labels for r in ref]), dtype=torch.int32, device="cuda")
    labK = torch.tensor(np.stack([r.part.km_K.labels for r in ref]), dtype=torch.int32, device="cuda")
    plan, out, _ = gpu_call(w, inputs=inputs, labels=(labQ, labK))
    assert plan.check() == 0
    beta = plan.export("BETA")
    out_np = out.double().cpu().numpy()
    for h, r in enumerate(ref):
        assert beta[h] == r.beta, (h, beta[h], r.beta)
        check_injected_head(plan, out_np[h], r, h, w)
    plain, _, _ = gpu_call(base, inputs=inputs, labels=(labQ, labK))
    assert np.all(plain.export("BETA") == (base.rho - base.M / base.N) * base.N)
    pairs_cal, pairs_plain = plan.export("PAIRS"), plain.export("PAIRS")
    for h in range(w.H):
        T = w.rho * w.N * w.N - w.M * w.N
        assert abs(pairs_cal[h] - T) <= abs(pairs_plain[h] - T)


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_support_densities_match_oracle(name):
    # O1 ([P] S3): |D_i(0.9)| of sampled rows and the pooled union per query group,
    # against the oracle on fp64 weights of the same stored values.  Sizes are exact
    # unless the oracle's sorted running sum sits within 1e-12 of the mass target at the
    # boundary (a rounding tie); pooled sizes are compared where every size matched.
    w = W.TINY if name == "tiny" else W.MID.with_(H=2)
    Q, K, V = W.make_inputs_torch(w, device="cuda")
    nrows = 256 if name == "tiny" else 64
    idx = np.unique(np.linspace(0, w.N - 1, nrows).astype(np.int64))
    rows_h, pool_h, refs = [], [], []
    for h in range(w.H):
        _, _, _, res = oracle_head(w, h, rows=np.arange(4))
        comp = res.part.gq.compact[idx]
        uniq, pool = np.unique(comp, return_inverse=True)
        rows_h.append(idx)
        pool_h.append(pool)
        refs.append((uniq.size, pool))
    npools = max(u for u, _ in refs)
    rows = torch.tensor(np.stack(rows_h), dtype=torch.int32, device="cuda")
    pool = torch.tensor(np.stack(pool_h), dtype=torch.int32, device="cuda")
    sizes, pooled = N.support_densities(Q, K, rows, pool, npools, 0.9)
    sizes, pooled = sizes.cpu().numpy(), pooled.cpu().numpy()
    for h in range(w.H):
        q, k, _ = W.make_head(w, h)
        a = O.attention_probs(q[idx], k)
        ref = O.support_size(a, 0.9)
        exact = np.array_equal(sizes[h], ref)
        if not exact:
            srt = -np.sort(-a, axis=1)
            cum = np.cumsum(srt, axis=1)
            for i in np.flatnonzero(sizes[h] != ref):
                assert abs(int(sizes[h][i]) - int(ref[i])) == 1, (h, i)
                k0 = min(sizes[h][i], ref[i]) - 1
                gap = abs(cum[i, k0] - 0.9 * cum[i, -1] * (1 - 1e-15)) / cum[i, -1]
                assert gap < 1e-12, (h, i, gap)
        else:
            npool_h, pid = refs[h]
            for c in range(npool_h):
                sel = pid == c
                _, gamma = O.support_densities(a[sel], 0.9)
                assert pooled[h][c] == round(gamma * w.N), (h, c)


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_affine_fit_matches_oracle(name):
    # O3 ([P] S3, App. D.5): the affine fit of R = dense - O_sp on O_sp over all rows, on
    # the GPU's own sparse and dense outputs, against the oracle's SVD-based fit.
    w = W.TINY if name == "tiny" else W.MID.with_(H=2)
    Q, K, V = W.make_inputs_torch(w, device="cuda")
    plan = N.Plan(N.params_from_dict(w.params()), Q, K, V)
    plan.attend()
    dense = N.dense_attention(Q, K, V)
    expl, err = plan.affine_fit(dense)
    expl, err = expl.cpu().numpy(), err.cpu().numpy()
    assert plan.check() == 0
    osp = plan.export("OSP")
    perm = plan.export("PERM_Q")
    dn = dense.double().cpu().numpy()
    for h in range(w.H):
        orig = np.empty_like(osp[h], dtype=np.float64)
        orig[perm[h]] = osp[h]
        e_ref, err_ref = O.oracle_affine_fit(orig, dn[h])
        assert abs(expl[h] - e_ref) < 1e-9, (h, expl[h], e_ref)
        assert abs(err[h] - err_ref) <= 1e-6 * err_ref + 1e-300, (h, err[h], err_ref)


# ---------------------------------------------------------------------------------- edges
def test_negative_logits_padding_columns_masked():
    # Every query-key logit below zero: the zero K rows that pad each K/V group to a
    # multiple of 8 in the tensor-core layout score 0 and would decide the row max, so the
    # kernel masks them in TMEM and takes the max again (the path other data rarely take).
    # bf16, d = 64, oracle labels injected; output and sparse output against the oracle.
    w = W.TINY.with_(dtype="bf16", N=2048)
    rng = np.random.default_rng(21)
    mu = rng.standard_normal(w.d)
    mu *= 8.0 / np.linalg.norm(mu)                          # |mu|^2 = 64
    k = W.round_to_bf16(mu + 0.5 * rng.standard_normal((w.N, w.d)))
    q = W.round_to_bf16(-0.5 * mu + 0.5 * rng.standard_normal((w.N, w.d)))
    v = W.round_to_bf16(rng.standard_normal((w.N, w.d)))
    assert (q @ k.T).max() < 0.0
    p = O.Params.from_dict(w.params())
    res = O.sparsepr_call(q, k, v, p, head=0, part=O.partition(q, k, v, p, 0))
    assert np.any(res.part.gk.sizes % 8 != 0)               # some groups are padded
    td = W.torch_dtype(w.dtype)
    inputs = tuple(torch.from_numpy(a[None].astype(np.float32)).to(td).cuda() for a in (q, k, v))
    labQ = torch.tensor(res.part.km_Q.labels[None], dtype=torch.int32, device="cuda")
    labK = torch.tensor(res.part.km_K.labels[None], dtype=torch.int32, device="cuda")
    plan, out, _ = gpu_call(w, inputs=inputs, labels=(labQ, labK))
    assert plan.check() == 0
    osp = plan.export("OSP")[0]
    rows = np.empty_like(osp)
    rows[plan.export("PERM_Q")[0]] = osp
    assert rel(rows[res.rows], res.osp) < 1e-2
    check_injected_head(plan, out[0].float().cpu().numpy(), res, 0, w)


def test_full_density_returns_dense():
    # rho* = 1 with every group larger than M: every cell is selected, residuals vanish
    # and the whole call returns dense attention (paper S2: all cells recover dense).
    w = W.MID.with_(H=2, rho=1.0, M=16, C_q=32, C_k=32)
    plan, out, (Q, K, V) = gpu_call(w)
    sizes = plan.export("SIZES_K")
    ng = plan.export("GROUPS_K")
    assert all(sizes[h][:ng[h]].min() > w.M for h in range(w.H))
    st = plan.stats()
    assert st["rho_route"] == 1.0
    dense = N.dense_attention(Q, K, V)
    assert rel(out.float().cpu().numpy(), dense.float().cpu().numpy()) < 1e-2
    q, k, v = W.make_head(w, 1)
    rows = np.arange(0, w.N, 97)
    ref = O.dense_attention(q, k, v, rows)
    assert rel(out[1].float().cpu().numpy()[rows], ref) < 1e-2


@pytest.mark.parametrize("dtype,d", [("f32", 64), ("bf16", 64), ("bf16", 128)])
def test_dense_attention_engine_ragged(dtype, d):
    rng = np.random.default_rng(5)
    H, Nq, Nk = 2, 333, 517
    arrs = [rng.standard_normal((H, n, d)) * s for n, s in ((Nq, 0.7), (Nk, 0.7), (Nk, 1.0))]
    if dtype == "bf16":
        arrs = [W.round_to_bf16(a) for a in arrs]
    td = W.torch_dtype(dtype)
    Q, K, V = (torch.from_numpy(a.astype(np.float32)).to(td).cuda() for a in arrs)
    out = N.dense_attention(Q, K, V).float().cpu().numpy()
    for h in range(H):
        ref = O.dense_attention(arrs[0][h], arrs[1][h], arrs[2][h])
        assert rel(out[h], ref) < (1e-5 if dtype == "f32" else 1e-2)


@pytest.mark.parametrize("d", [64, 128])
def test_tensor_core_engine_matches_cuda_core_engine(d):
    # Same plan (oracle labels injected), attention by both engines: the sparse outputs
    # agree to bf16 rounding of the probabilities, the corrected outputs to the tolerance.
    w = (W.MID if d == 64 else W.WAN.with_(N=16800, grid=(21, 20, 40), C_q=128, C_k=128)).with_(H=2)
    inputs = W.make_inputs_torch(w, device="cuda")
    ref = [oracle_head(w, h)[3] for h in range(w.H)]
    labQ = torch.tensor(np.stack([r.part.km_Q.labels for r in ref]), dtype=torch.int32, device="cuda")
    labK = torch.tensor(np.stack([r.part.km_K.labels for r in ref]), dtype=torch.int32, device="cuda")
    p_tc, o_tc, _ = gpu_call(w, inputs=inputs, labels=(labQ, labK))
    p_ct, o_ct, _ = gpu_call(w, inputs=inputs, labels=(labQ, labK), engine=N.SPARSEPR_ENGINE_SIMT)
    assert p_tc.check() == 0 and p_ct.check() == 0
    assert rel(p_tc.export("OSP"), p_ct.export("OSP")) < 5e-3
    assert rel(p_tc.export("ODENSE_PROBE"), p_ct.export("ODENSE_PROBE")) < 5e-3
    for h, r in enumerate(ref):
        check_injected_head(p_tc, o_tc[h].float().cpu().numpy(), r, h, w)


def test_ragged_cross_attention_and_empty_groups():
    # N_q != N_k, neither a multiple of any tile, more requested groups than the data
    # supports (empty clusters), d = 32, fp32: labels injected from the oracle.
    rng = np.random.default_rng(9)
    Nq, Nk, d = 301, 457, 32
    mu = rng.standard_normal((12, d)) * 2
    q = mu[rng.integers(0, 12, Nq)] + 0.3 * rng.standard_normal((Nq, d))
    k = mu[rng.integers(0, 12, Nk)] + 0.3 * rng.standard_normal((Nk, d))
    v = rng.standard_normal((Nk, d))
    q, k, v = (x.astype(np.float32).astype(np.float64) for x in (q, k, v))
    pdict = dict(H=1, N_q=Nq, N_k=Nk, d=d, dtype="f32", M_s=50, r_K=6, r_Q=5, C_q=40, C_k=60,
                 M=24, r=5, lam=0.1, target_density=0.3, kmeans_max_iter=25, seed=3)
    p = O.Params.from_dict(pdict)
    res = O.sparsepr_call(q, k, v, p, head=0)
    assert res.part.gk.sizes.size < 60 or res.part.gq.sizes.size < 40   # empty groups occurred
    Q, K, V = (torch.from_numpy(x.astype(np.float32))[None].cuda() for x in (q, k, v))
    labQ = torch.tensor(res.part.km_Q.labels[None], dtype=torch.int32, device="cuda")
    labK = torch.tensor(res.part.km_K.labels[None], dtype=torch.int32, device="cuda")
    params = N.params_from_dict(pdict)
    plan = N.Plan(params, Q, K, V, labels=(labQ, labK))
    plan.attend()
    plan.probe_fit()
    out = plan.correct()
    torch.cuda.synchronize()
    w = W.TINY.with_(N=Nq)
    check_injected_head(plan, out[0].double().cpu().numpy(), res, 0, w)
    # free running on the same problem: labels agree with the oracle's own k-means
    plan2 = N.Plan(params, Q, K, V)
    assert np.mean(plan2.export("LABELS_K")[0] == res.part.km_K.labels) >= 0.999
    assert np.mean(plan2.export("LABELS_Q")[0] == res.part.km_Q.labels) >= 0.999


def test_probe_rows_are_exact_dense_rows():
    # Probe rows carry the exact dense output (review page step 5), here with most rows
    # probed (M = 120 of 128).
    w = W.TINY.with_(N=128, grid=(2, 8, 8), M=120, r=4, rho=1.0, C_q=8, C_k=8)
    plan, out, _ = gpu_call(w)
    q, k, v = W.make_head(w, 0)
    probes = plan.export("PROBES")[0]
    assert len(set(probes.tolist())) == 120
    assert rel(out[0].double().cpu().numpy()[probes], O.dense_attention(q, k, v, probes)) < 1e-5


def test_zero_queries_set_device_error_without_fault():
    # A zero query sample makes the key metric zero: no positive eigenvalue.  The call
    # completes, the device error word is set and the context stays usable.
    w = W.TINY
    Q, K, V = W.make_inputs_torch(w, device="cuda")
    Q.zero_()
    params = N.params_from_dict(w.params())
    plan = N.Plan(params, Q, K, V)
    assert plan.check() & 1
    assert torch.cuda.is_available() and float(torch.ones(1, device="cuda").sum()) == 1.0


def test_out_of_range_injected_labels_are_flagged():
    w = W.TINY
    Q, K, V = W.make_inputs_torch(w, device="cuda")
    labQ = torch.zeros((1, w.N), dtype=torch.int32, device="cuda")
    labK = torch.zeros((1, w.N), dtype=torch.int32, device="cuda")
    labK[0, 5] = w.C_k + 3
    plan = N.Plan(N.params_from_dict(w.params()), Q, K, V, labels=(labQ, labK))
    assert plan.check() & 16


@pytest.mark.parametrize("case", ["mid", "wan2", "ragged"])
def test_tensor_core_kmeans_equals_full_scan(case):
    # The tensor-core assignment (bf16 split scores + exact rescoring of near ties) must
    # give the same labels, objectives and iteration counts as the fp32 full scan.
    w = {"mid": W.MID.with_(H=3), "wan2": W.WAN.with_(H=2),
         "ragged": W.TINY.with_(N=1000, grid=(10, 10, 10), C_q=100, C_k=70, M=16)}[case]
    inputs = W.make_inputs_torch(w, device="cuda")
    p_tc = N.Plan(N.params_from_dict(w.params()), *inputs)
    p_ct = N.Plan(N.params_from_dict(w.params(), N.SPARSEPR_ENGINE_SIMT), *inputs)
    assert p_tc.check() == 0 and p_ct.check() == 0
    for name in ("LABELS_K", "LABELS_Q", "KMEANS_ITERS", "OBJECTIVE", "PERM_Q", "CELL_COUNT"):
        assert np.array_equal(p_tc.export(name), p_ct.export(name)), name
