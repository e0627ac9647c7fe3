"""Pins of the fp64 oracle against what the SparsePR pages and the mathematics fix.

Every check here uses something other than the oracle's own formula: hand-worked
values (tests/golden/), closed forms, library routines on special cases, identities the
paper states, and brute force on tiny inputs.  CPU only.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from conftest import GOLDEN
from oracle import sparsepr_oracle as O


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- sampling / RNG
def test_sample_rows_evenly_spaced():
    assert O.sample_rows(10, 4).tolist() == [0, 2, 5, 7]          # floor(s*10/4)
    assert O.sample_rows(1024, 64).tolist() == list(range(0, 1024, 16))
    assert O.sample_rows(5, 8).tolist() == [0, 1, 2, 3, 4]        # all rows if fewer


def test_splitmix64_published_vector():
    g = _golden("splitmix64_seed1234567.json")
    x = g["seed"]
    outs = []
    for _ in range(5):
        x = (x + O._GAMMA) & O._M64
        outs.append(O._mix64(x))
    assert outs == [int(v) for v in g["outputs"]]


def test_kmeans_init_indices_range_and_uniformity():
    idx = O.kmeans_init_indices(0, 3, 1, 20000, 1000)
    assert idx.min() >= 0 and idx.max() < 1000
    counts = np.bincount(idx, minlength=1000)
    chi2 = ((counts - 20.0) ** 2 / 20.0).sum()
    assert 850 < chi2 < 1150          # 999 dof: mean 999, sd ~45
    # streams of different heads / stages differ
    assert not np.array_equal(O.kmeans_init_indices(0, 0, 0, 64, 1000),
                              O.kmeans_init_indices(0, 0, 1, 64, 1000))


# ---------------------------------------------------------------- key metric / factor
def test_key_metric_is_average_squared_response_difference():
    rng = _rng(1)
    Q = rng.standard_normal((50, 6))
    rows = O.sample_rows(50, 7)
    MK = O.key_metric(Q, rows)
    for _ in range(5):
        dk = rng.standard_normal(6)
        brute = sum(float(np.dot(Q[i], dk)) ** 2 for i in rows) / len(rows)
        assert abs(dk @ MK @ dk - brute) <= 1e-12 * brute


def test_eigen_factor_diagonal_closed_form():
    M = np.diag([4.0, 1.0, 9.0])
    F, lam, _ = O.eigen_factor(M, 2)
    assert np.allclose(lam, [9.0, 4.0])
    expect = np.zeros((3, 2))
    expect[2, 0] = math.sqrt(9.0 / 6.5)
    expect[0, 1] = math.sqrt(4.0 / 6.5)
    assert np.allclose(np.abs(F), expect, atol=1e-14)


def test_eigen_factor_full_rank_reproduces_metric_up_to_scale():
    rng = _rng(2)
    A = rng.standard_normal((40, 8))
    M = A.T @ A / 40
    F, lam, U = O.eigen_factor(M, 8)
    scale = lam.mean()
    for _ in range(5):
        x, y = rng.standard_normal(8), rng.standard_normal(8)
        lhs = np.sum(((x - y) @ F) ** 2)
        rhs = (x - y) @ M @ (x - y) / scale
        assert abs(lhs - rhs) <= 1e-12 * rhs
    # F F^T = U_r diag(lam_hat) U_r^T and eigen-residuals vanish
    assert np.allclose(F @ F.T, U @ np.diag(lam / scale) @ U.T, atol=1e-13)
    assert np.abs(M @ U - U * lam[None, :]).max() < 1e-12


def test_eigen_factor_rejects_zero_metric():
    with pytest.raises(ValueError):
        O.eigen_factor(np.zeros((4, 4)), 2)


# ---------------------------------------------------------------- k-means
def test_kmeans_hand_worked():
    g = _golden("kmeans_1d.json")
    X = np.array(g["points"])
    res = O.kmeans(X, np.array(g["init_idx"]), g["max_iter"])
    assert res.labels.tolist() == g["labels"]
    assert np.allclose(res.centres, g["centres"], atol=0)
    assert res.iterations == g["iterations"]
    assert res.objective == g["objective"]
    one = O.kmeans(X, np.array(g["init_idx"]), 1)
    assert one.labels.tolist() == g["labels_max_iter_1"]
    assert np.allclose(one.centres, g["centres_max_iter_1"], rtol=1e-15)


def test_kmeans_assignment_is_the_exact_argmin_of_direct_distances():
    # S5: label = argmin_c sum_j (x_j - c_j)^2 taken in the direct form.  With a large
    # common offset the differences x_j - c_j are exact (Sterbenz) and the sums of their
    # squares resolve the nearest centre, which exact rational arithmetic confirms; the
    # expanded form |x|^2 - 2 x.c + |c|^2 loses it to cancellation (checked below, so the
    # case has teeth).  Equal distances go to the lowest centre index.
    from fractions import Fraction
    rng = _rng(40)
    off = float(2 ** 30)
    X = off + rng.random((300, 5))
    Cn = off + rng.random((7, 5))
    lab = O._assign(X, Cn)
    Xf = [[Fraction(v) for v in row] for row in X]
    Cf = [[Fraction(v) for v in row] for row in Cn]
    exact = []
    for x in Xf:
        d = [sum((a - b) ** 2 for a, b in zip(x, c)) for c in Cf]
        exact.append(min(range(len(d)), key=lambda c: (d[c], c)))
    assert lab.tolist() == exact
    expanded = ((X * X).sum(1)[:, None] - 2.0 * X @ Cn.T + (Cn * Cn).sum(1)[None, :]).argmin(1)
    assert (expanded != np.array(exact)).sum() > 10
    # ties: two centres at the same distance from every point -> the lower index
    Xt = np.array([[0.0, 0.0], [1.0, 1.0]])
    Ct = np.array([[5.0, 5.0], [1.0, 0.0], [0.0, 1.0]])
    assert O._assign(Xt, Ct).tolist() == [1, 1]


def test_kmeans_matches_sklearn_lloyd():
    from sklearn.cluster import KMeans
    rng = _rng(3)
    centres = rng.standard_normal((6, 4)) * 6
    X = np.concatenate([c + rng.standard_normal((40, 4)) for c in centres])
    init = np.array([0, 41, 85, 130, 170, 201])
    res = O.kmeans(X, init, 50)
    km = KMeans(n_clusters=6, init=X[init], n_init=1, algorithm="lloyd", max_iter=50, tol=0.0)
    km.fit(X)
    assert res.iterations < 50
    assert np.array_equal(res.labels, km.labels_)
    assert np.allclose(res.centres, km.cluster_centers_, atol=1e-12)


def test_kmeans_brute_force_fixed_point_tiny():
    rng = _rng(4)
    for trial in range(30):
        N, C = rng.integers(3, 9), rng.integers(1, 4)
        X = rng.standard_normal((N, 2))
        init = rng.integers(0, N, C)
        res = O.kmeans(X, init, 100)
        # objective never increases
        assert all(b <= a + 1e-12 for a, b in zip(res.history, res.history[1:]))
        if res.iterations < 100:
            # Lloyd fixed point: each point's label is its nearest centre (lowest on ties)
            for i in range(N):
                dists = [sum((X[i][k] - res.centres[c][k]) ** 2 for k in range(2)) for c in range(C)]
                best = min(dists)
                assert res.labels[i] == dists.index(best)
            # each non-empty centre is its members' mean
            for c in range(C):
                mem = [i for i in range(N) if res.labels[i] == c]
                if mem:
                    assert np.allclose(res.centres[c], X[mem].mean(axis=0), atol=1e-14)


def test_kmeans_empty_cluster_keeps_centre():
    # Duplicate init: centre 1 loses every tie (lowest index wins), stays empty after step
    # 1 and keeps its value 0.0 (S6); step 2 it is nearer to point 0 than centre 0 (now
    # 0.05), regains it, and step 3 changes nothing.
    X = np.array([[0.0], [0.1], [5.0]])
    one = O.kmeans(X, np.array([0, 0, 2]), 1)
    assert one.labels.tolist() == [0, 0, 2]
    assert one.centres[:, 0].tolist() == [0.05, 0.0, 5.0]
    res = O.kmeans(X, np.array([0, 0, 2]), 10)
    assert res.labels.tolist() == [1, 0, 2]
    assert res.centres[:, 0].tolist() == [0.1, 0.0, 5.0]
    assert res.iterations == 3


# ---------------------------------------------------------------- query side
def test_groups_and_centring():
    g = O.compact_groups(np.array([3, 3, 0, 5]), 6)
    assert g.compact.tolist() == [1, 1, 0, 2]
    assert g.sizes.tolist() == [1, 2, 1]
    assert g.labels_used.tolist() == [0, 3, 5]
    rng = _rng(5)
    kbar = rng.standard_normal((7, 5))
    Kt = O.centred_key_centroids(kbar)
    assert np.abs(Kt.sum(axis=0)).max() < 1e-14
    q = rng.standard_normal(5)
    sm = lambda z: np.exp(z - z.max()) / np.exp(z - z.max()).sum()
    assert np.allclose(sm(kbar @ q), sm(Kt @ q), atol=1e-15)   # [P] App. B.2


def test_query_metric_is_average_squared_centred_logit_difference():
    rng = _rng(6)
    Kt = O.centred_key_centroids(rng.standard_normal((9, 4)))
    MQ = O.query_metric(Kt)
    for _ in range(5):
        dq = rng.standard_normal(4)
        brute = sum(float(np.dot(Kt[b], dq)) ** 2 for b in range(9)) / 9
        assert abs(dq @ MQ @ dq - brute) <= 1e-12 * brute


def test_query_coords_rms_normalisation():
    rng = _rng(7)
    Q = rng.standard_normal((20, 6))
    F = rng.standard_normal((6, 4))
    phi = O.query_coords(Q, F)
    assert np.allclose((phi ** 2).mean(axis=1), 1.0, atol=1e-14)
    assert np.allclose(O.query_coords(3.5 * Q, F), phi, atol=1e-14)   # scale invariant
    Q[0] = 0.0
    assert np.all(O.query_coords(Q, F)[0] == 0.0)                   # floor, no NaN
    tiny = O.query_coords(np.full((1, 6), 1e-9), np.eye(6)[:, :4])
    assert np.allclose(tiny, 1e-9 / 1e-6)                           # max(rms, eps)


# ---------------------------------------------------------------- routing
def test_route_score_hand_worked():
    g = _golden("route_score_example.json")
    for c in g["cases"]:
        S = O.route_scores(np.array(c["qbar"]), np.array(c["kbar"]), np.array(c["vbar"]),
                           np.array(c["sizes"]), 1)
        assert np.allclose(S, c["scores"], atol=1e-15)


def test_route_score_singletons_match_hard_drop_of_one_key():
    # With one key per group and the query at its centroid, pi is the exact attention and
    # the score equals || O_dense - O_sp(without b) || (App. A.1 identity, U = {b}).
    rng = _rng(8)
    d = 4
    q = rng.standard_normal((1, d)) * 3
    K = rng.standard_normal((6, d))
    V = rng.standard_normal((6, d))
    S = O.route_scores(q, K, V, np.ones(6, dtype=np.int64), d)[0]
    dense = O.attention_rows(q, K, V)[0]
    for b in range(6):
        keep = [j for j in range(6) if j != b]
        osp = O.attention_rows(q, K[keep], V[keep])[0]
        assert abs(S[b] - np.linalg.norm(dense - osp)) < 1e-12


def test_route_score_matches_definition_by_brute_force():
    # ohat^(-b) formed literally from the other groups for every b, including a group
    # holding nearly all the mass (where the closed form would cancel).
    rng = _rng(81)
    C, d = 7, 5
    kbar = rng.standard_normal((C, d))
    kbar[3] *= 12.0
    qbar = np.vstack([kbar[3] * 2.0, rng.standard_normal(d)])
    vbar = rng.standard_normal((C, d))
    sizes = rng.integers(1, 50, C)
    S = O.route_scores(qbar, kbar, vbar, sizes, d)
    for a in range(2):
        l = [float(qbar[a] @ kbar[b]) / math.sqrt(d) + math.log(sizes[b]) for b in range(C)]
        mx = max(l)
        z = [math.exp(x - mx) for x in l]
        for b in range(C):
            pb = z[b] / sum(z)
            zo = [(c, math.exp(l[c] - max(l[cc] for cc in range(C) if cc != b))) for c in range(C) if c != b]
            tot = sum(x for _, x in zo)
            orest = sum(x * vbar[c] for c, x in zo) / tot
            want = pb * float(np.linalg.norm(vbar[b] - orest))
            assert abs(S[a, b] - want) <= 1e-12 * max(want, 1e-300) + 1e-300, (a, b, S[a, b], want)
    assert S[0, 3] > 0.1 and np.argmax(S[0]) == 3    # the dominant group ranks first


def test_select_cells_hand_worked():
    g = _golden("cell_selection_example.json")
    for c in g["cases"]:
        sel = O.select_cells(np.array(g["scores"]), np.array(g["sizes"]), c["beta"])
        assert sel[0].tolist() == c["selected"]


def test_select_cells_prefix_minimal_and_full_budget():
    rng = _rng(9)
    S = rng.random((12, 15))
    sizes = rng.integers(1, 30, 15)
    beta = 0.3 * sizes.sum()
    for a, sel in enumerate(O.select_cells(S, sizes, beta)):
        assert sizes[sel].sum() >= beta
        worst = sel[np.argmin(S[a, sel])]
        assert sizes[sel].sum() - sizes[worst] < beta         # shortest prefix
        others = np.setdiff1d(np.arange(15), sel)
        if others.size:
            assert S[a, sel].min() >= S[a, others].max()
    for sel in O.select_cells(S, sizes, float(sizes.sum())):
        assert sel.tolist() == list(range(15))


# ---------------------------------------------------------------- permutation
def test_calibrated_budget_hand_worked():
    g = _golden("calibrated_budget_example.json")
    S = np.array(g["scores"], dtype=np.float64)
    sa, sb = np.array(g["sizes_q"]), np.array(g["sizes_k"])
    for c in g["cases"]:
        beta, sel = O.calibrated_selection(S, sa, sb, c["rho"], g["M"], g["N_q"], g["N_k"])
        assert beta == c["beta"], c
        assert [s.tolist() for s in sel] == c["sel"], c
        assert O.executed_pairs(sa, sb, sel) == c["pairs"]


def test_calibrated_budget_is_the_nearest_achievable_density():
    # S13: among the selections of the prefix rule over every integer budget (found here
    # by running select_cells at each beta), the calibrated one is nearest rho*; rho_exec
    # never decreases in beta; the calibrated distance is at most the plain rule's.
    rng = _rng(41)
    for trial in range(6):
        Cq, Ck = rng.integers(3, 9), rng.integers(3, 9)
        sa = rng.integers(1, 7, Cq)
        sb = rng.integers(1, 7, Ck)
        S = rng.random((Cq, Ck))
        S[0, 1] = S[0, 0]                                      # a score tie
        N_q, N_k, M = int(sa.sum()), int(sb.sum()), 1
        for rho in (0.2, 0.35, 0.5, 0.8):
            if rho <= M / N_q:
                continue
            T = rho * N_q * N_k - M * N_k
            pairs = [O.executed_pairs(sa, sb, O.select_cells(S, sb, float(b))) for b in range(1, N_k + 1)]
            assert all(x <= y for x, y in zip(pairs, pairs[1:]))
            beta, sel = O.calibrated_selection(S, sa, sb, rho, M, N_q, N_k)
            got = O.executed_pairs(sa, sb, sel)
            assert got == pairs[beta - 1]
            assert abs(got - T) == min(abs(x - T) for x in pairs)
            plain = O.executed_pairs(sa, sb, O.select_cells(S, sb, O.route_budget(rho, M, N_q, N_k)))
            assert abs(got - T) <= abs(plain - T)


def test_calibrated_budget_full_call_lands_near_the_target():
    Q, K, V = _clustered(42, N=400)
    p = _small_workload_params(rho=0.3, M=8)
    plain = O.sparsepr_call(Q, K, V, p)
    cal = O.sparsepr_call(Q, K, V, O.Params(**{**p.__dict__, "budget": "calibrated"}), part=plain.part)
    assert abs(cal.rho_exec - p.rho) <= abs(plain.rho_exec - p.rho)
    assert cal.pairs_exec == cal.pairs_route + p.M * Q.shape[0]


def test_group_major_permutation():
    perm, off = O.group_major_permutation(np.array([2, 0, 1, 0, 2, 1]), 3)
    assert perm.tolist() == [1, 3, 2, 5, 0, 4]
    assert off.tolist() == [0, 2, 4, 6]
    inv = np.empty_like(perm)
    inv[perm] = np.arange(6)
    assert np.array_equal(perm[inv], np.arange(6))


# ---------------------------------------------------------------- attention
def test_dense_attention_matches_torch_sdpa():
    rng = _rng(10)
    Q, K, V = (rng.standard_normal((33, 16)) for _ in range(3))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None])[0].numpy()
    assert np.abs(O.dense_attention(Q, K, V) - ref).max() < 1e-13


def test_attention_small_closed_forms():
    rng = _rng(11)
    q = rng.standard_normal((1, 4))
    k = rng.standard_normal((1, 4))
    v = rng.standard_normal((1, 4))
    assert np.allclose(O.attention_rows(q, k, v), v, atol=1e-15)          # one key
    K2, V2 = rng.standard_normal((2, 4)), rng.standard_normal((2, 4))
    delta = float(q[0] @ (K2[0] - K2[1])) / 2.0                           # tau = 1/2
    p0 = 1.0 / (1.0 + math.exp(-delta))
    assert np.allclose(O.attention_rows(q, K2, V2)[0], p0 * V2[0] + (1 - p0) * V2[1], atol=1e-14)
    K5 = rng.standard_normal((5, 4))
    probs = O.attention_rows(q, K5, np.eye(5))[0]                         # one-hot V
    z = np.exp(K5 @ q[0] / 2.0)
    assert np.allclose(probs, z / z.sum(), atol=1e-15)


def _tiny_problem(seed=12, N=96, d=8, C=6):
    rng = _rng(seed)
    Q, K, V = (rng.standard_normal((N, d)) * 1.5 for _ in range(3))
    gq = O.compact_groups(rng.integers(0, C, N), C)
    gk = O.compact_groups(rng.integers(0, C, N), C)
    return Q, K, V, gq, gk


def test_hard_drop_residual_identity():
    # [P] App. A.1: O_dense - O_sp = p_U (O_U - O_sp), p_U the omitted dense mass.
    Q, K, V, gq, gk = _tiny_problem()
    rng = _rng(13)
    n = gk.sizes.size
    sel = [np.sort(rng.choice(n, size=rng.integers(1, n), replace=False)) for _ in range(gq.sizes.size)]
    osp = O.sparse_attention(Q, K, V, gq, gk, sel)
    dense = O.dense_attention(Q, K, V)
    comp = [np.setdiff1d(np.arange(n), s) for s in sel]
    d = Q.shape[1]
    for i in range(Q.shape[0]):
        a = gq.compact[i]
        if comp[a].size == 0:
            assert np.allclose(osp[i], dense[i], atol=1e-14)
            continue
        U = np.flatnonzero(np.isin(gk.compact, comp[a]))
        z = np.exp(Q[i] @ K.T / math.sqrt(d))
        pU = z[U].sum() / z.sum()
        oU = (z[U] @ V[U]) / z[U].sum()
        lhs = dense[i] - osp[i]
        rhs = pU * (oU - osp[i])
        assert np.abs(lhs - rhs).max() <= 1e-12 * max(1.0, np.abs(lhs).max())


def test_all_cells_selected_is_dense():
    Q, K, V, gq, gk = _tiny_problem(seed=14)
    sel = [np.arange(gk.sizes.size) for _ in range(gq.sizes.size)]
    assert np.abs(O.sparse_attention(Q, K, V, gq, gk, sel) - O.dense_attention(Q, K, V)).max() < 1e-13


# ---------------------------------------------------------------- probes
def test_probe_selection_hand_worked():
    g = _golden("probe_selection_example.json")
    gq = O.compact_groups(np.array(g["labels"]), 3)
    for c in g["cases"]:
        probes, m_a = O.select_probes(np.array(g["dist"]), gq, c["M"])
        assert probes.tolist() == c["probes"]
        assert m_a.tolist() == c["m_a"]


def test_probe_distances_selection_and_weights_hand_worked():
    # [P] App. A.2 (distance of a row's query coordinates to its group's centre, then
    # Algorithm A.1) and [R] step 4 (w_p = |G_a^Q| / m_a), on values worked out by hand.
    g = _golden("probe_distance_example.json")
    gq = O.compact_groups(np.array(g["labels"]), 2)
    dist = O.probe_distances(np.array(g["phi"], dtype=np.float64),
                             np.array(g["centres"], dtype=np.float64), gq)
    assert dist.tolist() == g["dist"]
    probes, m_a = O.select_probes(dist, gq, g["M"])
    assert probes.tolist() == g["probes"]
    assert m_a.tolist() == g["m_a"]
    w = O.coverage_weights(gq, probes, m_a)
    assert np.allclose(w, g["weights"], rtol=1e-15, atol=0)


def test_probe_weights_of_a_group_add_up_to_its_size_in_a_full_call():
    # Each probe stands for an equal share of its group ([R] step 4): within a group the
    # weights are equal and they add up to the group's size, so with a probe in every
    # group they add up to N_q.  The group-major centres the call measures distances to
    # are the member means of the final query labels in phi_Q space.
    Q, K, V = _clustered(31, N=300)
    res = O.sparsepr_call(Q, K, V, _small_workload_params(M=12), head=0)
    gq = res.part.gq
    a_of = gq.compact[res.probes]
    for a in np.unique(a_of):
        wa = res.weights[a_of == a]
        assert np.all(wa == wa[0])
        assert abs(wa.sum() - gq.sizes[a]) <= 1e-12 * gq.sizes[a]
    for a in range(gq.sizes.size):
        mem = gq.compact == a
        c = res.part.phiQ[mem].mean(axis=0)
        d = ((res.part.phiQ[mem] - c) ** 2).sum(axis=1)
        assert np.allclose(res.probe_dist[mem], d, rtol=1e-12, atol=1e-14)


def test_probe_selection_many_groups_takes_nearest_of_largest():
    # [P] App. A.2: with at least M non-empty groups, the row nearest the centroid of
    # each of the M largest groups.
    rng = _rng(15)
    lab = rng.integers(0, 40, 2000)
    gq = O.compact_groups(lab, 40)
    dist = rng.random(2000)
    probes, m_a = O.select_probes(dist, gq, 16)
    largest = sorted(range(gq.sizes.size), key=lambda a: (-gq.sizes[a], a))[:16]
    expect = []
    for a in largest:
        mem = [i for i in range(2000) if gq.compact[i] == a]
        expect.append(min(mem, key=lambda i: (dist[i], i)))
    assert probes.tolist() == expect
    assert m_a.sum() == 16 and len(set(probes.tolist())) == 16


# ---------------------------------------------------------------- fit / correction
def _fit_inputs(seed=16, M=40, d=6):
    rng = _rng(seed)
    x = rng.standard_normal((M, d)) * rng.random(d) * 3
    R = rng.standard_normal((M, d))
    w = rng.integers(1, 9, M).astype(np.float64)
    return x, R, w


def test_ridge_matches_augmented_least_squares_and_dual():
    x, R, w = _fit_inputs()
    lam = 0.1
    f = O.fit_residual(x, R, w, lam, 0)
    M, d = x.shape
    # brute force from the definition: minimise sum omega ||Rb - xb B||^2 + lam ||B||^2
    wt = w / w.sum()
    mu_x = sum(wt[p] * x[p] for p in range(M))
    mu_R = sum(wt[p] * R[p] for p in range(M))
    var = sum(wt[p] * (x[p] - mu_x) ** 2 for p in range(M))
    s = np.sqrt(var + 1e-6)
    xb = (x - mu_x) / s
    Rb = R - mu_R
    om = w * M / w.sum()
    assert abs(om.mean() - 1.0) < 1e-15 and abs(wt.sum() - 1.0) < 1e-15
    A = np.vstack([np.sqrt(om)[:, None] * xb, math.sqrt(lam) * np.eye(d)])
    Y = np.vstack([np.sqrt(om)[:, None] * Rb, np.zeros((d, d))])
    B_ls = np.linalg.lstsq(A, Y, rcond=None)[0]
    assert np.abs(f.B - B_ls).max() < 1e-10
    Xo = np.sqrt(om)[:, None] * xb
    B_dual = Xo.T @ np.linalg.inv(Xo @ Xo.T + lam * np.eye(M)) @ (np.sqrt(om)[:, None] * Rb)
    assert np.abs(f.B - B_dual).max() < 1e-10
    assert np.allclose(f.mu_x, mu_x) and np.allclose(f.mu_R, mu_R) and np.allclose(f.s, s)


def test_ridge_large_lambda_is_mean_only():
    x, R, w = _fit_inputs(seed=17)
    f = O.fit_residual(x, R, w, 1e12, 0)
    assert np.abs(f.B).max() < 1e-9
    xs = np.random.default_rng(1).standard_normal((5, x.shape[1]))
    assert np.allclose(O.correct_rows(xs, f), xs + f.mu_R, atol=1e-9)


def test_planted_affine_residual_is_recovered():
    # If the residual is exactly affine in the sparse output, a near-unregularised fit
    # with r = d recovers it, so corrected outputs are exact on unseen rows.
    rng = _rng(18)
    M, d = 60, 5
    Bt = rng.standard_normal((d, d))          # non-symmetric: a transposed B fails
    bt = rng.standard_normal(d)
    x = rng.standard_normal((M, d)) * 2 + 1
    R = bt + x @ Bt
    w = rng.integers(1, 5, M).astype(np.float64)
    f = O.fit_residual(x, R, w, 1e-12, d)
    xs = rng.standard_normal((7, d))
    truth = xs + bt + xs @ Bt
    assert np.abs(O.correct_rows(xs, f) - truth).max() < 1e-8


def test_subspace_projector_properties():
    x, R, w = _fit_inputs(seed=19, M=30, d=10)
    f = O.fit_residual(x, R, w, 0.1, 4)
    P = f.P
    assert f.r_eff == 4
    assert np.abs(P @ P - P).max() < 1e-13 and np.abs(P - P.T).max() < 1e-14
    assert abs(np.trace(P) - 4) < 1e-12
    # with r >= rank(Y), Y P = Y
    full = O.fit_residual(x, R, w, 0.1, 10)
    om = w * len(w) / w.sum()
    Y = np.sqrt(om)[:, None] * (R - full.mu_R)
    assert np.abs(Y @ full.P - Y).max() < 1e-12
    # centring makes rank(Y) <= M - 1: a rank-deficient case keeps only real directions
    x2, R2, w2 = _fit_inputs(seed=20, M=4, d=10)
    f2 = O.fit_residual(x2, R2, w2, 0.1, 16)
    assert f2.r_eff == 3


# ---------------------------------------------------------------- whole call
def _small_workload_params(**kw):
    base = dict(d=8, M_s=32, r_K=4, r_Q=4, C_q=8, C_k=8, M=8, r=3, lam=0.1, rho=0.3,
                kmeans_max_iter=25, seed=0)
    base.update(kw)
    return O.Params(**base)


def _clustered(seed, N=240, d=8, C=8):
    rng = _rng(seed)
    mu = rng.standard_normal((C, d)) * 2
    cid = rng.integers(0, C, N)
    Q = mu[cid] + 0.4 * rng.standard_normal((N, d))
    K = mu[cid] + 0.4 * rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    return Q, K, V


def test_full_call_at_full_density_is_dense():
    Q, K, V = _clustered(21)
    res = O.sparsepr_call(Q, K, V, _small_workload_params(rho=1.0))
    dense = O.dense_attention(Q, K, V)
    assert res.rho_route == 1.0
    assert np.abs(res.out - dense).max() < 1e-12
    assert np.abs(res.fit.mu_R).max() < 1e-13


def test_full_call_probe_rows_exact_and_density_identity():
    Q, K, V = _clustered(22)
    p = _small_workload_params()
    res = O.sparsepr_call(Q, K, V, p)
    dense = O.dense_attention(Q, K, V, res.probes)
    assert np.array_equal(res.out[res.probes], res.dense_probe)
    assert np.abs(res.dense_probe - dense).max() < 1e-14
    N = Q.shape[0]
    assert res.pairs_exec == res.pairs_route + p.M * N                  # integer identity
    assert abs(res.rho_exec - (res.rho_route + p.M / N)) < 1e-15
    assert res.rho_exec >= p.rho                                       # prefix reaches budget
    assert sorted(res.probes.tolist()) == sorted(set(res.probes.tolist()))
    assert res.m_a.sum() == p.M


def test_full_call_correction_reduces_error():
    # PFRR's purpose ([P] S4.2, Table 2): the fitted correction moves unprobed rows toward
    # the dense output.  A flipped residual sign or a dropped mean term fails this.
    for seed in (23, 24, 25):
        Q, K, V = _clustered(seed, N=600)
        p = _small_workload_params(rho=0.3, M=64, r=8, lam=0.1)
        res = O.sparsepr_call(Q, K, V, p)
        dense = O.dense_attention(Q, K, V)
        unprobed = np.setdiff1d(np.arange(Q.shape[0]), res.probes)
        err = lambda A: np.linalg.norm(A[unprobed] - dense[unprobed]) / np.linalg.norm(dense[unprobed])
        assert err(res.out) < 0.9 * err(res.osp)


# ----------------------------------------------------------------------------------
# Restricted estimators ([P] App. D.3, Table 4): each is the minimiser of the weighted
# objective over its family, pinned against an augmented least-squares solve.

def _fit_inputs(seed=3, M=12, d=5):
    rng = np.random.default_rng(seed)
    x = rng.normal(size=(M, d))
    R = 0.3 * x @ rng.normal(size=(d, d)) + 0.05 * rng.normal(size=(M, d)) + 0.2
    w = rng.uniform(0.5, 2.0, size=M)
    return x, R, w


def _standardised(x, R, w):
    wt = w / w.sum()
    mu_x, mu_R = wt @ x, wt @ R
    s = np.sqrt(wt @ ((x - mu_x) ** 2) + O.STD_EPS)
    return (x - mu_x) / s, R - mu_R, x.shape[0] * w / w.sum()


def test_mean_only_estimator_predicts_the_weighted_mean_residual():
    x, R, w = _fit_inputs()
    f = O.fit_residual(x, R, w, 0.1, 4, "mean")
    assert np.all(f.B == 0) and np.array_equal(f.P, np.eye(x.shape[1]))
    xs = np.random.default_rng(9).normal(size=(7, x.shape[1]))
    np.testing.assert_allclose(O.correct_rows(xs, f), xs + (w / w.sum()) @ R, rtol=1e-13)


def test_scalar_estimator_matches_augmented_least_squares():
    x, R, w = _fit_inputs()
    lam, d = 0.7, x.shape[1]
    xb, Rb, om = _standardised(x, R, w)
    A = np.concatenate([(np.sqrt(om)[:, None] * xb).ravel(), [np.sqrt(lam * d)]])[:, None]
    y = np.concatenate([(np.sqrt(om)[:, None] * Rb).ravel(), [0.0]])
    a = np.linalg.lstsq(A, y, rcond=None)[0][0]
    f = O.fit_residual(x, R, w, lam, 4, "scalar")
    np.testing.assert_allclose(f.B, a * np.eye(d), rtol=1e-12, atol=1e-14)
    assert np.array_equal(f.P, np.eye(d))


def test_diagonal_estimator_matches_augmented_least_squares():
    x, R, w = _fit_inputs(seed=5)
    lam, d = 0.4, x.shape[1]
    xb, Rb, om = _standardised(x, R, w)
    b = np.empty(d)
    for j in range(d):
        A = np.concatenate([np.sqrt(om) * xb[:, j], [np.sqrt(lam)]])[:, None]
        y = np.concatenate([np.sqrt(om) * Rb[:, j], [0.0]])
        b[j] = np.linalg.lstsq(A, y, rcond=None)[0][0]
    f = O.fit_residual(x, R, w, lam, 4, "diagonal")
    np.testing.assert_allclose(f.B, np.diag(b), rtol=1e-12, atol=1e-14)


def test_restricted_estimators_never_beat_ridge_on_the_weighted_objective():
    # ridge minimises over all B, so its penalised objective is the smallest (r = d, P = I)
    x, R, w = _fit_inputs(seed=11, M=20, d=4)
    lam = 0.3
    xb, Rb, om = _standardised(x, R, w)

    def obj(B):
        return float(np.sum(om[:, None] * (Rb - xb @ B) ** 2) + lam * np.sum(B * B))

    ridge = O.fit_residual(x, R, w, lam, 4, "ridge")
    for est in ("mean", "scalar", "diagonal"):
        assert obj(ridge.B) <= obj(O.fit_residual(x, R, w, lam, 4, est).B) + 1e-12


# ---------------------------------------------------------------- warm start ([P] App. C)
def _spd_with_spectrum(seed, lam):
    rng = _rng(seed)
    U, _ = np.linalg.qr(rng.standard_normal((lam.size, lam.size)))
    return U @ np.diag(lam) @ U.T, U


def test_subspace_factor_from_the_leading_eigenspace_is_the_eigen_factor():
    # started anywhere inside the leading r-dimensional eigenspace (any basis), the
    # update returns U_r diag(lam_r / mean lam_r) U_r^T, built here from the spectrum
    lam = np.array([9.0, 7.0, 5.5, 4.0, 1.0, 0.5, 0.25, 0.1, 0.05, 0.01])
    M, U = _spd_with_spectrum(21, lam)
    r = 4
    T = _rng(22).standard_normal((r, r)) + 3.0 * np.eye(r)
    F = O.subspace_factor(M, U[:, :r] @ T)
    want = U[:, :r] @ np.diag(lam[:r] / lam[:r].mean()) @ U[:, :r].T
    assert np.abs(F @ F.T - want).max() < 1e-12 * np.abs(want).max()
    assert abs(np.trace(F.T @ F) - r) < 1e-12


def test_subspace_factor_at_full_rank_reproduces_the_metric():
    # r = d: M F (F^T M F)^-1 F^T M = M for any invertible F, scaled to unit mean
    lam = np.array([3.0, 2.0, 1.5, 0.7, 0.2, 0.1])
    M, _ = _spd_with_spectrum(23, lam)
    F = O.subspace_factor(M, _rng(24).standard_normal((6, 6)))
    assert np.abs(F @ F.T - M / lam.mean()).max() < 1e-11


def test_subspace_factor_iterated_converges_to_the_leading_eigenspace():
    lam = np.array([10.0, 8.0, 6.0, 1.0, 0.8, 0.5, 0.3, 0.1])
    M, U = _spd_with_spectrum(25, lam)
    r = 3
    F = O.subspace_factor(M, _rng(26).standard_normal((8, r)), steps=60)
    want = U[:, :r] @ np.diag(lam[:r] / lam[:r].mean()) @ U[:, :r].T
    assert np.abs(F @ F.T - want).max() < 1e-10


def test_subspace_factor_depends_only_on_the_span_of_its_start():
    lam = np.linspace(5.0, 0.1, 9)
    M, _ = _spd_with_spectrum(27, lam)
    F0 = _rng(28).standard_normal((9, 4))
    T = _rng(29).standard_normal((4, 4)) + 2.0 * np.eye(4)
    A = O.subspace_factor(M, F0)
    B = O.subspace_factor(M, F0 @ T)
    assert np.abs(A @ A.T - B @ B.T).max() < 1e-11


def test_subspace_factor_reports_a_singular_projected_metric():
    M = np.diag([1.0, 0.0, 2.0])
    assert O.subspace_factor(M, np.array([[0.0], [1.0], [0.0]])) is None


def test_warm_key_kmeans_restarts_at_its_fixed_point():
    # the same inputs again: the previous key centroids in the original space, mapped by
    # the (same) factor, are the converged centres, so the first assignment reproduces
    # the converged labels and the second one confirms them
    from free_block_sparse_plan_b200 import workloads as W
    w = W.TINY
    p = O.Params.from_dict(w.params())
    Q, K, V = W.make_head(w, 0)
    cold = O.partition(Q, K, V, p, 0)
    assert cold.km_K.iterations < p.kmeans_max_iter        # converged
    warm = O.partition(Q, K, V, p, 0, O.warm_state(cold, p))
    assert np.array_equal(warm.km_K.labels, cold.km_K.labels)
    assert warm.km_K.iterations == 2
    assert np.abs(warm.F_K @ warm.F_K.T - cold.F_K @ cold.F_K.T).max() < 1e-10


def test_warm_kmeans_objective_is_monotone_and_empty_labels_redraw():
    from free_block_sparse_plan_b200 import workloads as W
    w = W.TINY
    p = O.Params.from_dict(w.params())
    Q, K, V = W.make_head(w, 0)
    st = O.warm_state(O.partition(Q, K, V, p, 0), p)
    st.k_used[3] = False                                   # label 3 had no members
    Q1, K1, V1 = W.make_head(w.with_(step=1), 0)
    part = O.partition(Q1, K1, V1, p, 0, st)
    h = part.km_K.history
    assert all(b <= a * (1 + 1e-12) for a, b in zip(h, h[1:]))
    idx = O.kmeans_init_indices(p.seed, 0, 0, p.C_k, w.N)
    c0 = O.warm_centres(part.phiK, idx, st.k_used, st.kbar @ part.F_K)
    assert np.array_equal(c0[3], part.phiK[idx[3]])
    c = int(np.flatnonzero(st.k_used)[0])
    assert np.allclose(c0[c], st.kbar[c] @ part.F_K, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- GQA ([P] App. C)
def test_gqa_key_metric_is_the_mean_of_the_heads_metrics():
    # G * M_s evenly spaced rows of the head-major concatenation take, when M_s divides
    # N_q, exactly each head's own M_s sample rows, so the shared metric is the mean of
    # the G per-head metrics
    from free_block_sparse_plan_b200 import workloads as W
    w = W.TINY.with_(H=3, G=3)
    p = O.Params.from_dict(w.params())
    qs, K, V = W.make_kv_group(w, 0)
    part = O.partition(qs[1], K, V, p, 1, Qgroup=qs, kv_head=0)
    want = sum(O.key_metric(q, O.sample_rows(w.N, p.M_s)) for q in qs) / 3.0
    assert np.abs(part.M_K - want).max() < 1e-13 * np.abs(want).max()


def test_gqa_with_identical_query_heads_reproduces_the_single_head_partition():
    from free_block_sparse_plan_b200 import workloads as W
    w = W.TINY
    p = O.Params.from_dict(w.params())
    Q, K, V = W.make_head(w, 0)
    single = O.partition(Q, K, V, p, 0)
    shared = O.partition(Q, K, V, p, 0, Qgroup=[Q, Q], kv_head=0)
    assert np.abs(shared.M_K - single.M_K).max() < 1e-13 * np.abs(single.M_K).max()
    assert np.array_equal(shared.km_K.labels, single.km_K.labels)
    assert np.array_equal(shared.km_Q.labels, single.km_Q.labels)


def test_gqa_query_heads_share_the_key_partition_and_keep_their_own_query_groups():
    from free_block_sparse_plan_b200 import workloads as W
    w = W.TINY.with_(H=2, G=2)
    p = O.Params.from_dict(w.params())
    qs, K, V = W.make_kv_group(w, 0)
    a = O.partition(qs[0], K, V, p, 0, Qgroup=qs, kv_head=0)
    b = O.partition(qs[1], K, V, p, 1, Qgroup=qs, kv_head=0)
    assert np.array_equal(a.km_K.labels, b.km_K.labels)
    assert np.array_equal(a.F_Q, b.F_Q)                    # M_Q comes from the K/V groups
    assert not np.array_equal(a.km_Q.labels, b.km_Q.labels)
    assert not np.array_equal(qs[0], qs[1])


# ---------------------------------------------------------------- semantic partition, O1, O3
def test_semantic_partition_clusters_raw_rows_and_full_density_is_dense():
    Q, K, V = _clustered(31)
    p = _small_workload_params(rho=1.0)
    p.partition = "semantic"
    res = O.sparsepr_call(Q, K, V, p)
    assert np.abs(res.out - O.dense_attention(Q, K, V)).max() < 1e-12
    # the key groups are the k-means of the raw key rows, and every value follows its key
    km = O.kmeans(K, O.kmeans_init_indices(p.seed, 0, 0, p.C_k, K.shape[0]), p.kmeans_max_iter)
    assert np.array_equal(res.part.km_K.labels, km.labels)
    assert np.allclose(res.part.vbar, O.group_means(V, res.part.gk), rtol=0, atol=0)


def test_attention_probs_rows_sum_to_one_and_weigh_the_values():
    # a one-hot V turns attention output into the weights themselves ([P] S2)
    rng = _rng(43)
    q, K = rng.standard_normal((5, 4)), rng.standard_normal((9, 4))
    a = O.attention_probs(q, K)
    assert np.allclose(a.sum(axis=1), 1.0, atol=1e-15)
    assert np.allclose(a, O.attention_rows(q, K, np.eye(9)), atol=1e-15)
    z = np.exp(q @ K.T / 2.0)
    assert np.allclose(a, z / z.sum(axis=1, keepdims=True), atol=1e-15)


def test_support_size_hand_worked():
    a = np.array([[0.5, 0.3, 0.1, 0.1],          # 0.5 + 0.3 + 0.1 >= 0.9
                  [0.25, 0.25, 0.25, 0.25],      # ceil(0.9 * 4) = 4 keys
                  [0.0, 1.0, 0.0, 0.0],          # one key
                  [0.1, 0.2, 0.3, 0.4]])         # 0.4 + 0.3 + 0.2 >= 0.9
    assert O.support_size(a, 0.9).tolist() == [3, 4, 1, 3]
    assert O.support_size(a, 0.95).tolist() == [4, 4, 1, 4]
    assert O.support_size(a[:1], 0.5).tolist() == [1]


def test_pooled_support_density_is_the_union_of_the_supports():
    n = 8
    one_hot = np.eye(n)[[1, 5, 5]]
    tau, gamma = O.support_densities(one_hot, 0.9)
    assert tau.tolist() == [1 / n] * 3 and gamma == 2 / n      # keys {1, 5}
    a = np.array([[0.6, 0.3, 0.1, 0, 0, 0, 0, 0],
                  [0, 0, 0.1, 0.3, 0.6, 0, 0, 0]])
    tau, gamma = O.support_densities(a, 0.85)                   # {0, 1} and {4, 3}
    assert tau.tolist() == [2 / n, 2 / n] and gamma == 4 / n


def test_oracle_affine_fit_recovers_a_planted_affine_residual_and_matches_lstsq():
    rng = _rng(41)
    n, d = 200, 6
    osp = rng.standard_normal((n, d))
    B = rng.standard_normal((d, d))
    b = rng.standard_normal(d)
    frac, err = O.oracle_affine_fit(osp, osp + b + osp @ B)
    assert abs(frac - 1.0) < 1e-12 and err < 1e-20 * n
    # a generic residual: the explained part is the least-squares projection on [1, O_sp]
    R = rng.standard_normal((n, d))
    frac, err = O.oracle_affine_fit(osp, osp + R)
    A = np.hstack([np.ones((n, 1)), osp])
    coef, *_ = np.linalg.lstsq(A, R, rcond=None)
    rem = float(((R - A @ coef) ** 2).sum())
    assert abs(err - rem) < 1e-10 * rem
    assert abs(frac - (1.0 - rem / float((R * R).sum()))) < 1e-12
    # a duplicated (rank-deficient) feature column changes nothing
    frac2, err2 = O.oracle_affine_fit(np.hstack([osp, osp[:, :1]]), np.hstack([osp, osp[:, :1]]) + np.hstack([R, R[:, :1]]))
    A2 = np.hstack([np.ones((n, 1)), osp])
    coef2, *_ = np.linalg.lstsq(A2, np.hstack([R, R[:, :1]]), rcond=None)
    rem2 = float(((np.hstack([R, R[:, :1]]) - A2 @ coef2) ** 2).sum())
    assert abs(err2 - rem2) < 1e-10 * rem2


def test_warm_query_centres_pass_the_rms_step():
    # W2: a non-empty query label restarts at phi_Q(qbar) = (qbar F_Q) / rms, a point of the
    # RMS sphere (raw qbar F_Q is not), and the partition's query k-means starts there
    from free_block_sparse_plan_b200 import workloads as W
    w = W.TINY
    p = O.Params.from_dict(w.params())
    Q, K, V = W.make_head(w, 0)
    st = O.warm_state(O.partition(Q, K, V, p, 0), p)
    Q1, K1, V1 = W.make_head(w.with_(step=1), 0)
    part = O.partition(Q1, K1, V1, p, 0, st)
    mapped = O.query_coords(st.qbar, part.F_Q)
    used = np.flatnonzero(st.q_used)
    assert np.allclose(np.sqrt((mapped[used] ** 2).mean(axis=1)), 1.0, rtol=1e-12)
    raw = st.qbar[used] @ part.F_Q
    assert not np.allclose(np.sqrt((raw ** 2).mean(axis=1)), 1.0, rtol=1e-3)
    idx = O.kmeans_init_indices(p.seed, 0, 1, p.C_q, w.N)
    again = O.kmeans(part.phiQ, idx, p.kmeans_max_iter, O.warm_centres(part.phiQ, idx, st.q_used, mapped))
    assert np.array_equal(again.labels, part.km_Q.labels) and again.iterations == part.km_Q.iterations
