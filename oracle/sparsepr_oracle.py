"""SparsePR per-call sparse attention: a plain fp64 CPU oracle.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import or call this
module: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg use it.  It shares no code with the CUDA library (no kernels, headers, tables or
helpers) and imports nothing from the product package.

Sources.  [P] = "Partition the Support, Reconstruct the Residual: Training-Free Sparse
Attention for Video Generation and World Models" (the paper text; its display
equations were lost in extraction, so several formulas are re-derived from the
sentences around them).  [R] = the paper.rainbus.top review of the same paper, which
restates the pipeline with concrete values (w_p = |G_a^Q|/m_a, lambda = 0.1, r = 16,
the subspace Psi_r, dense output on probe rows).  Section labels of [P] are inferred
from its content: S2 problem setup, S4.1 Response-Coupled Partitioning (RCP), S4.2
Probe-Fitted Residual Reconstruction (PFRR), S4.3 routing budget, App. A.1 hard-drop
derivation, App. A.2 probe selection (Algorithm A.1), App. A.3 estimator statistics,
App. B.1 key metric, App. B.2 query metric and RMS normalisation, App. B.3 routing,
App. C implementation, App. D ablations.

Readings where the pages are silent:
  S1  evenly spaced sample rows are floor(s*N_q/M_s), s = 0..M_s-1 (all rows if M_s >= N_q)
  S2  M_K = (1/M_s) Q_s^T Q_s, the unique symmetric matrix with
      dk M_K dk^T = mean_s (q_s . dk)^2
  S3  eigenvalues normalised to unit mean over the retained r; negatives clamped to 0
  S5  k-means assignment: label = argmin_c sum_j (x_j - c_j)^2 in the direct form (the
      sum over ascending j, one fused multiply-add per term), ties to the lowest
      centre index; computed by the plain C routine in kmeans_direct.c
  S6  an empty cluster keeps its previous centre
  S7  k-means stops after max_iter assignment steps or when an assignment changes no label
  S8  k-means init: C rows drawn with replacement by SplitMix64 (counter-based)
  S9  phi_Q = z / max(rms(z), 1e-6)
  S11 routing score (the SVG-EAR value error score is not on the pages): the centroid
      estimate of the hard-drop residual of omitting K/V group b alone,
      l_ab = tau qbar_a.kbar_b + ln|G_b|, pi_ab = softmax_b l_ab,
      ohat_a^(-b) = sum_{c != b} pi_ac vbar_c / (1 - pi_ab),
      score_ab = pi_ab * ||vbar_b - ohat_a^(-b)||_2
  S12 score ties ranked by ascending KV group id
  S13 the calibrated budget (optional): the common integer budget beta in [1, N_k] whose
      prefix selection brings rho_exec nearest rho* (ties to the denser selection)
  S14 group-major order keeps ascending original index inside a group
  S16 probe distance d_i is the squared distance to the group centre in phi_Q space
  S20 r = 0 means no subspace projection (P = I)
  S21 singular values <= 1e-10 * sigma_max are dropped before taking the leading r
  W1  a warm factor update is F <- Z L^-T with Z = M F and L L^T = F^T Z (a Cholesky
      factor), twice, then scaled to unit mean eigenvalue: F F^T = M F (F^T M F)^-1 F^T M,
      which depends only on span(F); if F^T M F is not positive definite the call takes
      the full eigendecomposition instead
  G1  GQA: the key metric of a K/V head is built from the concatenation (head-major) of
      the query rows of its G query heads, sampled by S1 with G*M_s rows out of G*N_q;
      the K/V partition, its centroids, the query metric and F_Q are shared by the G
      heads; query coordinates, query k-means (init stream of the query head), routing,
      probes and fit stay per query head
  S25 the semantic (reference) partition runs the same k-means on the raw key and query
      rows; probe distances are then taken on raw query rows
  S26 O1 support densities are fractions of the keys: tau_i = |D_i(alpha)| / N_k and the
      pooled gamma = |union of the D_i| / N_k
  W2  warm k-means starts label c at the previous call's original-space centroid of
      label c mapped into the current coordinates (phi_K linear, phi_Q with its RMS
      step); a label that was empty in the previous call has no centroid and takes the
      fresh draw c of the counter-based init stream

Parity status: every function here is pinned by tests in ``tests/test_oracle_*.py``
except ``route_scores``, whose formula is a reading (S11) of a score the pages only
name: its parity against the SVG-EAR definition is UNPINNED (its stated properties and
a hand-worked value are pinned).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np

RMS_EPS = 1e-6            # [P] App. B.2: floor of the RMS denominator
STD_EPS = 1e-6            # [P] App. D.3: sqrt(weighted variance + 1e-6)
SV_REL_TOL = 1e-10        # [P] App. D.5: relative singular-value tolerance

# ----------------------------------------------------------------------------------
# S8: SplitMix64 (Steele, Lea & Flood, "Fast Splittable Pseudorandom Number
# Generators", OOPSLA 2014), used in counter form: output n of a generator whose
# state starts at `key` is mix(key + n * GAMMA), n = 1, 2, ...
_M64 = (1 << 64) - 1
_GAMMA = 0x9E3779B97F4A7C15


def _mix64(z: int) -> int:
    z &= _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def kmeans_init_indices(seed: int, head: int, stage: int, C: int, N: int) -> np.ndarray:
    """Initial centre rows: C draws with replacement from [0, N) ([P] App. C: "initial
    k means centers are sampled uniformly with replacement from feature rows").

    stage 0 = key clustering, 1 = query clustering.  The stream key is output number
    (2*head + stage + 1) of SplitMix64 seeded with `seed`; draw c uses output c+1 of
    the generator keyed by it, mapped to an index by the high 32 bits:
    idx = (hi32 * N) >> 32.
    """
    key = _mix64(seed + (2 * head + stage + 1) * _GAMMA)
    out = np.empty(C, dtype=np.int64)
    for c in range(C):
        z = _mix64(key + (c + 1) * _GAMMA)
        out[c] = ((z >> 32) * N) >> 32
    return out


# ----------------------------------------------------------------------------------
# RCP: key side ([P] S4.1 "Key-response coordinates", App. B.1)

def sample_rows(N_q: int, M_s: int) -> np.ndarray:
    """S1: M_s query rows at deterministic evenly spaced token positions."""
    if M_s >= N_q:
        return np.arange(N_q, dtype=np.int64)
    return (np.arange(M_s, dtype=np.int64) * N_q) // M_s


def key_metric(Q: np.ndarray, rows: np.ndarray) -> np.ndarray:
    """S2: key response metric M_K = (1/M_s) Q_s^T Q_s ([P] S4.1, App. B.1)."""
    Qs = Q[rows]
    return (Qs.T @ Qs) / Qs.shape[0]


def eigen_factor(Msym: np.ndarray, r: int):
    """Eigenvalue-weighted factor F (d x r) of a symmetric PSD metric.

    [P] S4.1 / App. B.1: keep the leading r eigenvectors, normalise their eigenvalues
    to unit mean (S3: mean over the r kept), and scale each eigenvector by the square
    root of its normalised eigenvalue.  Returns (F, kept eigenvalues, eigenvectors).
    """
    w, U = np.linalg.eigh(Msym)
    order = np.argsort(-w, kind="stable")[:r]
    lam = np.maximum(w[order], 0.0)
    mean = lam.mean()
    if not mean > 0.0:
        raise ValueError("metric has no positive eigenvalue among the leading r")
    Ur = U[:, order]
    return Ur * np.sqrt(lam / mean)[None, :], lam, Ur


def subspace_factor(Msym: np.ndarray, F_prev: np.ndarray, steps: int = 2):
    """Warm update of an eigenvalue-weighted factor ([P] App. C: later calls refresh the
    metric factors with two subspace iterations started from the previous factors, using
    a Cholesky factorisation).

    Reading W1: each iteration multiplies by the metric, Z = M F, factors the projected
    metric F^T M F = F^T Z = L L^T and takes F <- Z L^-T, so that
    F F^T = M F (F^T M F)^-1 F^T M.  That product depends only on the subspace spanned
    by F, and equals U_r Lambda_r U_r^T when the subspace is the leading eigenspace, i.e.
    the eigen-weighted factor of `eigen_factor` up to a rotation of its columns (which
    leaves every distance in the coordinates unchanged).  The result is scaled so its
    eigenvalues, those of F^T F, have unit mean (S3).  Returns None when F^T M F is not
    positive definite (the caller falls back to the full eigendecomposition).
    """
    F = np.array(F_prev, dtype=np.float64)
    for _ in range(steps):
        Z = Msym @ F
        try:
            L = np.linalg.cholesky(F.T @ Z)
        except np.linalg.LinAlgError:
            return None
        F = np.linalg.solve(L, Z.T).T
    r = F.shape[1]
    mean = float(np.trace(F.T @ F)) / r
    if not mean > 0.0:
        return None
    return F / math.sqrt(mean)


# ----------------------------------------------------------------------------------
# k-means ([P] S4.1, App. C: Lloyd iterations, fresh centres, at most 25 iterations)

@dataclass
class KMeansResult:
    labels: np.ndarray          # int64 [N], in [0, C)
    centres: np.ndarray         # fp64 [C, r], means of the final labels (S6 for empties)
    iterations: int             # assignment steps taken
    objective: float            # sum_i ||x_i - c_label(i)||^2 at the final centres
    history: List[float] = field(default_factory=list)  # objective after each update


_C_SRC = os.path.join(os.path.dirname(os.path.abspath(__file__)), "kmeans_direct.c")
_C_LIB = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_build", "libkmeans_direct.so")
_clib_handle = None


def _clib():
    """The direct-form assignment of ``kmeans_direct.c`` (plain C, OpenMP over rows),
    compiled with gcc on first use when the shared object is missing or older than its
    source."""
    global _clib_handle
    if _clib_handle is None:
        if not os.path.exists(_C_LIB) or os.path.getmtime(_C_LIB) < os.path.getmtime(_C_SRC):
            os.makedirs(os.path.dirname(_C_LIB), exist_ok=True)
            tmp = f"{_C_LIB}.{os.getpid()}.tmp"
            subprocess.run(["gcc", "-O3", "-fopenmp", "-ffp-contract=off", "-shared", "-fPIC",
                            _C_SRC, "-o", tmp, "-lm"], check=True)
            os.replace(tmp, _C_LIB)
        lib = ctypes.CDLL(_C_LIB)
        lib.oracle_assign_direct.restype = None
        lib.oracle_assign_direct.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                             ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p]
        _clib_handle = lib
    return _clib_handle


def _assign(X: np.ndarray, centres: np.ndarray) -> np.ndarray:
    """S5: label = argmin_c sum_j (x_j - c_j)^2, the sum over ascending j with one fused
    multiply-add per term, ties to the lowest centre index (computed in plain C)."""
    X = np.ascontiguousarray(X, dtype=np.float64)
    CT = np.ascontiguousarray(np.asarray(centres, dtype=np.float64).T)
    n, r = X.shape
    k = CT.shape[1]
    labels = np.empty(n, dtype=np.int64)
    if n:
        _clib().oracle_assign_direct(X.ctypes.data, CT.ctypes.data, n, k, r, labels.ctypes.data)
    return labels


def _update(X: np.ndarray, labels: np.ndarray, centres: np.ndarray) -> np.ndarray:
    C = centres.shape[0]
    counts = np.bincount(labels, minlength=C)
    sums = np.zeros_like(centres)
    np.add.at(sums, labels, X)
    new = centres.copy()
    nz = counts > 0
    new[nz] = sums[nz] / counts[nz][:, None]          # S6: empty clusters keep theirs
    return new


def objective(X: np.ndarray, labels: np.ndarray, centres: np.ndarray) -> float:
    diff = X - centres[labels]
    return float((diff * diff).sum())


def kmeans(X: np.ndarray, init_idx: np.ndarray, max_iter: int,
           centres0: Optional[np.ndarray] = None) -> KMeansResult:
    """Lloyd's algorithm: assign to the nearest centre, move centres to member means.

    Starts from the feature rows `init_idx`, or from `centres0` when given (warm start).
    S7: stop after `max_iter` assignment steps or as soon as an assignment step leaves
    every label unchanged.  The returned centres are the means of the returned labels.
    """
    centres = X[init_idx].copy() if centres0 is None else np.array(centres0, dtype=np.float64)
    labels = None
    it = 0
    history = []
    for _ in range(max_iter):
        new = _assign(X, centres)
        it += 1
        if labels is not None and np.array_equal(new, labels):
            break
        labels = new
        centres = _update(X, labels, centres)
        history.append(objective(X, labels, centres))
    return KMeansResult(labels, centres, it, objective(X, labels, centres), history)


# ----------------------------------------------------------------------------------
# RCP: query side ([P] S4.1 "Query-response coordinates", App. B.2)

@dataclass
class Groups:
    """Non-empty groups of a labelling, renumbered 0..C'-1 in ascending label order."""
    compact: np.ndarray      # int64 [N] compact group id of each row
    sizes: np.ndarray        # int64 [C'] member counts
    labels_used: np.ndarray  # int64 [C'] original label of each compact id


def compact_groups(labels: np.ndarray, C: int) -> Groups:
    counts = np.bincount(labels, minlength=C)
    used = np.flatnonzero(counts > 0)
    remap = -np.ones(C, dtype=np.int64)
    remap[used] = np.arange(used.size)
    return Groups(remap[labels], counts[used], used)


def group_means(X: np.ndarray, g: Groups) -> np.ndarray:
    sums = np.zeros((g.sizes.size, X.shape[1]))
    np.add.at(sums, g.compact, X)
    return sums / g.sizes[:, None]


def centred_key_centroids(kbar: np.ndarray) -> np.ndarray:
    """[P] S4.1 / App. B.2: subtract the uniform mean of the non-empty group centroids."""
    return kbar - kbar.mean(axis=0, keepdims=True)


def query_metric(Ktil: np.ndarray) -> np.ndarray:
    """M_Q = (1/C_k') K~^T K~: each non-empty KV group weighs equally ([P] App. B.2)."""
    return (Ktil.T @ Ktil) / Ktil.shape[0]


def query_coords(Q: np.ndarray, F_Q: np.ndarray) -> np.ndarray:
    """phi_Q(q) = z / max(rms(z), eps), z = q F_Q; no gain, no bias ([P] S4.1, App. B.2)."""
    z = Q @ F_Q
    rms = np.sqrt((z * z).mean(axis=1))
    return z / np.maximum(rms, RMS_EPS)[:, None]


# ----------------------------------------------------------------------------------
# Routing ([P] App. B.3, S4.3)

def route_scores(qbar: np.ndarray, kbar: np.ndarray, vbar: np.ndarray,
                 size_b: np.ndarray, d: int) -> np.ndarray:
    """S11 (reading; the SVG-EAR formula is not on the pages; parity unpinned against it).

    Centroid estimate of the residual left by omitting K/V group b alone from query group
    a: by the hard-drop identity of [P] App. A.1 with U = {b}, ||R|| = p_b ||O_b - O_sp||,
    estimated with pi_ab = softmax_b(tau qbar_a.kbar_b + ln|G_b|) for p_b, vbar_b for O_b
    and ohat_a^(-b) = sum_{c != b} pi_ac vbar_c / (1 - pi_ab) for O_sp:
        score_ab = pi_ab * ||vbar_b - ohat_a^(-b)||.
    For every b but the largest-mass one, vbar_b - ohat^(-b) = (vbar_b - ohat)/(1 - pi_b)
    exactly, with ohat the estimate over all groups and 1 - pi_b >= 1/2; for the largest-
    mass group ohat^(-b) is formed directly from the other groups.  One group: score 0.
    """
    tau = 1.0 / math.sqrt(d)
    L = tau * (qbar @ kbar.T) + np.log(size_b.astype(np.float64))[None, :]
    n = L.shape[1]
    S = np.zeros_like(L)
    if n == 1:
        return S
    for a in range(L.shape[0]):
        l = L[a]
        top = int(np.argmax(l))                      # first index of the maximum
        z = np.exp(l - l[top])
        Z = z.sum()
        ohat = (z @ vbar) / Z
        rest = Z - z
        rest[top] = 1.0                              # replaced below
        S[a] = z * np.sqrt(((vbar - ohat[None, :]) ** 2).sum(axis=1)) / rest
        others = np.arange(n) != top
        zo = np.exp(l[others] - l[others].max())
        ohat_rest = (zo @ vbar[others]) / zo.sum()
        S[a, top] = (z[top] / Z) * np.linalg.norm(vbar[top] - ohat_rest)
    return S


def route_budget(rho_target: float, M: int, N_q: int, N_k: int) -> float:
    """[P] S4.3: the router reserves the probe cost, rho*_route = rho* - M/N_q; the common
    per-query key-token budget is rho*_route * N_k."""
    return (rho_target - float(M) / float(N_q)) * float(N_k)


def select_cells(S: np.ndarray, size_b: np.ndarray, beta: float) -> List[np.ndarray]:
    """[P] App. B.3: rank non-empty KV groups by decreasing score (S12: ties by id) and keep
    the shortest prefix whose key-token count reaches beta (all groups if none does).
    Each query group's selected ids are returned in ascending order."""
    C_k = S.shape[1]
    ids = np.arange(C_k)
    sel = []
    for a in range(S.shape[0]):
        order = np.lexsort((ids, -S[a]))
        csum = np.cumsum(size_b[order]).astype(np.float64)
        hit = np.flatnonzero(csum >= beta)
        k = (hit[0] + 1) if hit.size else C_k
        sel.append(np.sort(order[:k]))
    return sel


def calibrated_selection(S: np.ndarray, size_a: np.ndarray, size_b: np.ndarray, rho_target: float,
                         M: int, N_q: int, N_k: int):
    """S13, the calibrated budget ([P] App. D.2 speaks of a budget calibrated toward the
    target density; [Site] Table 1's realised densities fall on both sides of it).

    The prefix rule of `select_cells` with a common per-query budget beta selects, for
    every integer beta in [1, N_k], some set of cells; the realised density
    rho_exec(beta) = (routed pairs + M N_k) / (N_q N_k) never decreases as beta grows.
    The calibrated budget is the beta whose selection brings rho_exec nearest rho*, i.e.
    minimises |routed pairs - T| with T = rho* N_q N_k - M N_k (in that fp64 order);
    between a selection below T and one above at equal distance the denser is taken, and
    among the betas giving one selection the smallest.  Returns (beta, selection).
    """
    T = rho_target * N_q * N_k - M * N_k
    C_k = S.shape[1]
    ids = np.arange(C_k)
    betas = np.arange(1, N_k + 1, dtype=np.int64)
    pairs = np.zeros(betas.size, dtype=np.int64)
    for a in range(S.shape[0]):
        order = np.lexsort((ids, -S[a]))
        pref = np.cumsum(size_b[order]).astype(np.int64)          # pref[-1] = N_k
        k = np.searchsorted(pref, betas, side="left")             # first prefix >= beta
        pairs += int(size_a[a]) * pref[k]
    dist = np.abs(pairs.astype(np.float64) - T)
    best = dist.min()
    cand = np.flatnonzero(dist == best)
    pick = cand[np.argmax(pairs[cand])]                            # the denser on a tie
    pick = np.flatnonzero(pairs == pairs[pick])[0]                 # its smallest beta
    beta = int(betas[pick])
    return beta, select_cells(S, size_b, float(beta))


def executed_pairs(size_a: np.ndarray, size_b: np.ndarray, sel: List[np.ndarray]) -> int:
    """Routed query-key interactions: each selected cell costs |G_a^Q| |G_b^KV| ([P] S2)."""
    return int(sum(int(size_a[a]) * int(size_b[s].sum()) for a, s in enumerate(sel)))


# ----------------------------------------------------------------------------------
# Group-major permutation ([R] step 3: Q, K, V rearranged group-major, output restored)

def group_major_permutation(compact: np.ndarray, n_groups: int):
    """S14: stable order by group id; returns (perm, offsets) with perm[pos] = row."""
    perm = np.argsort(compact, kind="stable")
    sizes = np.bincount(compact, minlength=n_groups)
    offsets = np.concatenate([[0], np.cumsum(sizes)])
    return perm, offsets


# ----------------------------------------------------------------------------------
# Attention ([P] S2: dense attention and renormalised hard drop)

def attention_probs(q: np.ndarray, K: np.ndarray) -> np.ndarray:
    """Dense attention weights softmax(tau q K^T) of rows q over every key ([P] S2),
    tau = 1/sqrt(d): the matrix whose rows the O1 support densities of [P] S3 measure."""
    tau = 1.0 / math.sqrt(q.shape[1])
    logits = tau * (q @ K.T)
    logits -= logits.max(axis=1, keepdims=True)
    p = np.exp(logits)
    return p / p.sum(axis=1, keepdims=True)


def attention_rows(q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """softmax(tau q K^T) V for rows q, with tau = 1/sqrt(d) ([P] S4.1: the common 1/sqrt(d)
    scale).  Renormalised hard drop is this same formula over the retained keys only."""
    tau = 1.0 / math.sqrt(q.shape[1])
    logits = tau * (q @ K.T)
    logits -= logits.max(axis=1, keepdims=True)
    p = np.exp(logits)
    return (p @ V) / p.sum(axis=1, keepdims=True)


def sparse_attention(Q, K, V, gq: Groups, gk: Groups, sel: List[np.ndarray],
                     rows: Optional[np.ndarray] = None) -> np.ndarray:
    """O^sp for `rows` (default all): row i in query group a attends, with softmax
    renormalised over them, to the keys of the KV groups selected for a ([P] S2)."""
    rows = np.arange(Q.shape[0]) if rows is None else np.asarray(rows)
    out = np.empty((rows.size, V.shape[1]))
    members_k = [np.flatnonzero(gk.compact == b) for b in range(gk.sizes.size)]
    ga = gq.compact[rows]
    for a in np.unique(ga):
        pos = np.flatnonzero(ga == a)
        keys = np.concatenate([members_k[b] for b in sel[a]])
        out[pos] = attention_rows(Q[rows[pos]], K[keys], V[keys])
    return out


def dense_attention(Q, K, V, rows: Optional[np.ndarray] = None) -> np.ndarray:
    rows = np.arange(Q.shape[0]) if rows is None else np.asarray(rows)
    out = np.empty((rows.size, V.shape[1]))
    for s in range(0, rows.size, 512):
        out[s:s + 512] = attention_rows(Q[rows[s:s + 512]], K, V)
    return out


# ----------------------------------------------------------------------------------
# PFRR ([P] S4.2, App. A.2-A.3, App. D; [R] step 4)

def probe_distances(phiQ: np.ndarray, cQ_compact: np.ndarray, gq: Groups) -> np.ndarray:
    """S16: d_i = ||phi_Q(q_i) - c_a||^2 for i in G_a, c_a the group's phi_Q centre."""
    diff = phiQ - cQ_compact[gq.compact]
    return (diff * diff).sum(axis=1)


def select_probes(dist: np.ndarray, gq: Groups, M: int):
    """Algorithm A.1 ([P] App. A.2): stratified radial round robin.

    Rows inside a group by increasing d_i (ties by row index); non-empty groups by
    decreasing size (ties by group index); each pass takes the next row of every group
    that still has one; stop after M distinct probes.  Returns (probes in selection
    order, m_a = number of probes per compact group).
    """
    n_groups = gq.sizes.size
    if M > gq.compact.size:
        raise ValueError("more probes than query rows")
    ranked = []
    for a in range(n_groups):
        mem = np.flatnonzero(gq.compact == a)
        ranked.append(mem[np.lexsort((mem, dist[mem]))])
    order = np.lexsort((np.arange(n_groups), -gq.sizes))
    probes = []
    t = 0
    while len(probes) < M:
        for a in order:
            if t < ranked[a].size:
                probes.append(int(ranked[a][t]))
                if len(probes) == M:
                    break
        t += 1
    probes = np.array(probes, dtype=np.int64)
    m_a = np.bincount(gq.compact[probes], minlength=n_groups)
    return probes, m_a


def coverage_weights(gq: Groups, probes: np.ndarray, m_a: np.ndarray) -> np.ndarray:
    """[R] step 4 ([P] App. A.3, whose formula was lost): probe p of query group a stands
    for its group's rows, w_p = |G_a^Q| / m_a, so the weights of a group's probes sum to
    the group's size."""
    a_of = gq.compact[probes]
    return gq.sizes[a_of].astype(np.float64) / m_a[a_of]


@dataclass
class Fit:
    mu_x: np.ndarray
    mu_R: np.ndarray
    s: np.ndarray
    B: np.ndarray          # d x d weighted ridge coefficients on standardised features
    P: np.ndarray          # d x d projector Psi_r Psi_r^T (identity when r == 0)
    r_eff: int
    sigma: np.ndarray      # singular values of Omega^{1/2} R_bar


ESTIMATORS = ("ridge", "mean", "scalar", "diagonal")   # codes 0..3 of the C ABI
PARTITIONS = ("response", "semantic")                  # codes 0..1 of the C ABI
BUDGETS = ("prefix", "calibrated")                     # codes 0..1 of the C ABI


def fit_residual(x: np.ndarray, R: np.ndarray, w: np.ndarray, lam: float, r: int,
                 estimator: str = "ridge") -> Fit:
    """Coverage-weighted ridge fit of the residual on the sparse output.

    [P] App. A.3: weights normalised to unit sum give mu_x, mu_R and the elementwise
    scale s = sqrt(weighted variance + 1e-6) ([P] App. D.3); x_bar = (x - mu_x) / s,
    R_bar = R - mu_R.  Weights normalised to unit mean (omega) weigh the ridge objective
    sum_p omega_p ||R_bar_p - x_bar_p B||^2 + lambda ||B||_F^2 ([P] S4.2), whose
    minimiser is (X^T Omega X + lambda I)^-1 X^T Omega R.  [P] App. D.2 / [R] step 4: the
    centred prediction is projected on the leading r right singular vectors of
    Omega^{1/2} R_bar.

    `estimator` selects the restricted corrections of [P] App. D.3 (Table 4), which
    minimise the same weighted objective over a smaller family, with the same lambda, no
    penalty on the mean and no projection (P = I): "mean" (B = 0, predict mu_R),
    "scalar" (B = a I, penalty lambda d a^2), "diagonal" (B = diag(b), penalty
    lambda sum_j b_j^2).
    """
    M, d = x.shape
    wt = w / w.sum()
    mu_x = wt @ x
    mu_R = wt @ R
    s = np.sqrt(wt @ ((x - mu_x) ** 2) + STD_EPS)
    xb = (x - mu_x) / s
    Rb = R - mu_R
    omega = M * w / w.sum()
    if estimator != "ridge":
        if estimator == "mean":
            B = np.zeros((d, d))
        elif estimator == "scalar":
            # d/da [sum_p omega_p ||Rb_p - a xb_p||^2 + lam d a^2] = 0
            a = float(np.sum(omega[:, None] * xb * Rb)) / (float(np.sum(omega[:, None] * xb * xb)) + lam * d)
            B = a * np.eye(d)
        elif estimator == "diagonal":
            # one column at a time: sum_p omega_p (Rb_pj - b_j xb_pj)^2 + lam b_j^2
            b = (omega @ (xb * Rb)) / (omega @ (xb * xb) + lam)
            B = np.diag(b)
        else:
            raise ValueError(estimator)
        return Fit(mu_x, mu_R, s, B, np.eye(d), d, np.zeros(0))
    lhs = xb.T @ (omega[:, None] * xb) + lam * np.eye(d)
    rhs = xb.T @ (omega[:, None] * Rb)
    B = np.linalg.solve(lhs, rhs)
    Y = np.sqrt(omega)[:, None] * Rb
    _, sig, Vt = np.linalg.svd(Y, full_matrices=False)
    if r == 0:
        return Fit(mu_x, mu_R, s, B, np.eye(d), d, sig)
    keep = int((sig > SV_REL_TOL * sig[0]).sum()) if sig[0] > 0 else 0
    r_eff = min(r, keep)
    Psi = Vt[:r_eff].T
    return Fit(mu_x, mu_R, s, B, Psi @ Psi.T, r_eff, sig)


def correct_rows(xs: np.ndarray, fit: Fit) -> np.ndarray:
    """Unprobed rows: O_hat = O^sp + mu_R + ((O^sp - mu_x) / s) B P ([R] step 5; [P] App. D.2)."""
    return xs + fit.mu_R[None, :] + (((xs - fit.mu_x) / fit.s) @ fit.B) @ fit.P


# ----------------------------------------------------------------------------------
# The whole call for one head

@dataclass
class Params:
    d: int
    M_s: int
    r_K: int
    r_Q: int
    C_q: int
    C_k: int
    M: int
    r: int
    lam: float
    rho: float
    kmeans_max_iter: int = 25
    seed: int = 0
    estimator: str = "ridge"
    partition: str = "response"     # "response" (RCP) or "semantic" (the reference partition)
    budget: str = "prefix"          # "prefix" (beta = rho*_route N_k) or "calibrated" (S13)

    @classmethod
    def from_dict(cls, p: Dict) -> "Params":
        return cls(d=p["d"], M_s=p["M_s"], r_K=p["r_K"], r_Q=p["r_Q"], C_q=p["C_q"],
                   C_k=p["C_k"], M=p["M"], r=p["r"], lam=p["lam"],
                   rho=p["target_density"], kmeans_max_iter=p["kmeans_max_iter"],
                   seed=p["seed"], estimator=ESTIMATORS[int(p.get("estimator", 0))],
                   partition=PARTITIONS[int(p.get("partition", 0))],
                   budget=BUDGETS[int(p.get("budget", 0))])


@dataclass
class Partition:
    """Response-Coupled Partitioning of one head ([P] S4.1)."""
    sample: np.ndarray
    M_K: np.ndarray
    F_K: np.ndarray
    lam_K: np.ndarray
    phiK: np.ndarray
    km_K: KMeansResult
    gk: Groups
    kbar: np.ndarray
    vbar: np.ndarray
    Ktil: np.ndarray
    M_Q: np.ndarray
    F_Q: np.ndarray
    lam_Q: np.ndarray
    phiQ: np.ndarray
    km_Q: KMeansResult
    gq: Groups
    qbar: np.ndarray


@dataclass
class WarmState:
    """What one call of a sequence hands to the next ([P] App. C warm start), per head."""
    F_K: np.ndarray          # d x r_K key factor
    F_Q: np.ndarray          # d x r_Q query factor
    kbar: np.ndarray         # C_k x d original-space key centroid of each label
    k_used: np.ndarray       # bool C_k: label non-empty (rows of empty labels are unused)
    qbar: np.ndarray         # C_q x d original-space query centroid of each label
    q_used: np.ndarray       # bool C_q


def warm_state(part: Partition, p: Params) -> WarmState:
    """The state a finished partition leaves for the next call of the sequence."""
    d = part.F_K.shape[0]
    kb = np.zeros((p.C_k, d))
    qb = np.zeros((p.C_q, d))
    ku = np.zeros(p.C_k, dtype=bool)
    qu = np.zeros(p.C_q, dtype=bool)
    kb[part.gk.labels_used] = part.kbar
    qb[part.gq.labels_used] = part.qbar
    ku[part.gk.labels_used] = True
    qu[part.gq.labels_used] = True
    return WarmState(part.F_K.copy(), part.F_Q.copy(), kb, ku, qb, qu)


def warm_centres(X: np.ndarray, fresh_idx: np.ndarray, used: np.ndarray,
                 mapped: np.ndarray) -> np.ndarray:
    """W2: label c starts at `mapped[c]` (the previous original-space centroid in the
    current coordinates) when it was non-empty, else at the fresh draw X[fresh_idx[c]]."""
    return np.where(used[:, None], mapped, X[fresh_idx])


def partition(Q, K, V, p: Params, head: int, warm: Optional[WarmState] = None,
              Qgroup: Optional[List[np.ndarray]] = None, kv_head: Optional[int] = None) -> Partition:
    """Response-Coupled Partitioning of query head `head`.

    GQA ([P] App. C, reading G1): `Qgroup` holds the query rows of the G heads sharing
    this K/V head (in head order) and `kv_head` its index; the key metric is built from
    G*M_s evenly spaced rows of their concatenation and the key k-means draws its initial
    rows from the K/V head's stream.  Without them (G = 1) both are this head's own.
    """
    N_q, N_k = Q.shape[0], K.shape[0]
    if Qgroup is None:
        Qcat, M_s, kv_head = Q, p.M_s, head if kv_head is None else kv_head
    else:
        Qcat, M_s = np.concatenate(Qgroup, axis=0), p.M_s * len(Qgroup)
    rows = sample_rows(Qcat.shape[0], M_s)
    M_K = key_metric(Qcat, rows)
    F_K = subspace_factor(M_K, warm.F_K) if warm is not None else None
    if F_K is None:
        F_K, lam_K, _ = eigen_factor(M_K, p.r_K)
    else:
        lam_K = np.sort(np.linalg.eigvalsh(F_K.T @ F_K))[::-1]
    phiK = K @ F_K
    idxK = kmeans_init_indices(p.seed, kv_head, 0, p.C_k, N_k)
    c0K = None if warm is None else warm_centres(phiK, idxK, warm.k_used, warm.kbar @ F_K)
    km_K = kmeans(phiK, idxK, p.kmeans_max_iter, c0K)
    gk = compact_groups(km_K.labels, p.C_k)
    kbar = group_means(K, gk)
    vbar = group_means(V, gk)
    Ktil = centred_key_centroids(kbar)
    M_Q = query_metric(Ktil)
    F_Q = subspace_factor(M_Q, warm.F_Q) if warm is not None else None
    if F_Q is None:
        F_Q, lam_Q, _ = eigen_factor(M_Q, p.r_Q)
    else:
        lam_Q = np.sort(np.linalg.eigvalsh(F_Q.T @ F_Q))[::-1]
    phiQ = query_coords(Q, F_Q)
    idxQ = kmeans_init_indices(p.seed, head, 1, p.C_q, N_q)
    c0Q = None if warm is None else warm_centres(phiQ, idxQ, warm.q_used, query_coords(warm.qbar, F_Q))
    km_Q = kmeans(phiQ, idxQ, p.kmeans_max_iter, c0Q)
    gq = compact_groups(km_Q.labels, p.C_q)
    qbar = group_means(Q, gq)
    return Partition(rows, M_K, F_K, lam_K, phiK, km_K, gk, kbar, vbar, Ktil, M_Q, F_Q,
                     lam_Q, phiQ, km_Q, gq, qbar)


def partition_semantic(Q, K, V, p: Params, head: int, kv_head: Optional[int] = None) -> Partition:
    """The reference (semantic) partition of [P] S3 and of its ablations: k-means applied
    separately to the raw key rows and to the raw query rows, each value following its
    key.  Reading S25: the same Lloyd steps, init streams and stop rule as the response
    coordinates' k-means, on the stored rows themselves (no metric, no RMS step); the
    coordinate maps are the identity, so probe distances (S16) are taken on raw query rows.
    """
    N_q, N_k, d = Q.shape[0], K.shape[0], Q.shape[1]
    kv = head if kv_head is None else kv_head            # GQA: the K/V head's init stream
    km_K = kmeans(K, kmeans_init_indices(p.seed, kv, 0, p.C_k, N_k), p.kmeans_max_iter)
    gk = compact_groups(km_K.labels, p.C_k)
    kbar = group_means(K, gk)
    vbar = group_means(V, gk)
    km_Q = kmeans(Q, kmeans_init_indices(p.seed, head, 1, p.C_q, N_q), p.kmeans_max_iter)
    gq = compact_groups(km_Q.labels, p.C_q)
    qbar = group_means(Q, gq)
    eye = np.eye(d)
    none = np.zeros((0,))
    return Partition(none, none, eye, np.ones(d), K, km_K, gk, kbar, vbar,
                     centred_key_centroids(kbar), none, eye, np.ones(d), Q, km_Q, gq, qbar)


def support_size(a: np.ndarray, alpha: float) -> np.ndarray:
    """|D_i(alpha)|: the fewest highest-weight keys whose dense attention mass reaches
    alpha, per row of the attention matrix `a` ([P] S3, O1).  Ties in weight do not change
    the count."""
    srt = -np.sort(-a, axis=1)
    cum = np.cumsum(srt, axis=1)
    return np.argmax(cum >= alpha * cum[:, -1:] * (1.0 - 1e-15), axis=1) + 1


def support_densities(a: np.ndarray, alpha: float):
    """O1 ([P] S3): individual support densities tau_i(alpha) = |D_i(alpha)| / N_k of
    the rows of `a`, and the pooled density gamma(alpha) = |union_i D_i(alpha)| / N_k of
    those rows taken together (reading S26: the equations were lost; the text defines
    both as fractions of the keys).  D_i keeps the keys of largest weight, lowest index
    first among equal weights."""
    n = a.shape[1]
    sizes = support_size(a, alpha)
    order = np.lexsort((np.broadcast_to(np.arange(n), a.shape), -a), axis=1)
    union = np.zeros(n, dtype=bool)
    for i in range(a.shape[0]):
        union[order[i, :sizes[i]]] = True
    return sizes / n, float(union.sum()) / n


def oracle_affine_fit(osp: np.ndarray, dense: np.ndarray, tol: float = SV_REL_TOL):
    """O3 ([P] S3, App. D.5): least-squares affine fit R ~ 1 b + O_sp B of the residual
    R = dense - O_sp over all given rows, in fp64: the columns of the centred sparse
    output are scaled to unit norm (zero columns left out), singular values below `tol`
    times the largest are dropped, the fit is the projection of the centred residual on
    the remaining left singular vectors, and the residual mean is the intercept.  Returns
    (explained fraction of the residual's squared norm, remaining squared error)."""
    R = dense - osp
    Xc = osp - osp.mean(axis=0, keepdims=True)
    nrm = np.linalg.norm(Xc, axis=0)
    Xs = Xc[:, nrm > 0] / nrm[nrm > 0]
    Rc = R - R.mean(axis=0, keepdims=True)
    if Xs.shape[1]:
        U, sig, _ = np.linalg.svd(Xs, full_matrices=False)
        U = U[:, sig > tol * sig[0]] if sig[0] > 0 else U[:, :0]
        fit = U @ (U.T @ Rc)
    else:
        fit = np.zeros_like(Rc)
    err = float(((Rc - fit) ** 2).sum())
    tot = float((R * R).sum())
    return (1.0 - err / tot if tot > 0 else 0.0), err


@dataclass
class CallResult:
    part: Partition
    scores: np.ndarray
    beta: float
    sel: List[np.ndarray]
    pairs_route: int
    pairs_exec: int
    rho_route: float
    rho_exec: float
    permQ: np.ndarray
    offQ: np.ndarray
    permK: np.ndarray
    offK: np.ndarray
    probes: np.ndarray
    m_a: np.ndarray
    probe_dist: np.ndarray
    weights: np.ndarray
    x_probe: np.ndarray
    dense_probe: np.ndarray
    fit: Fit
    rows: np.ndarray         # rows of `out`, `osp`
    osp: np.ndarray          # sparse output on `rows`
    out: np.ndarray          # corrected output on `rows`


def sparsepr_call(Q, K, V, p: Params, head: int = 0, rows: Optional[np.ndarray] = None,
                  part: Optional[Partition] = None,
                  warm: Optional[WarmState] = None) -> CallResult:
    """One SparsePR attention call for one head, in the pages' order.

    `rows` limits the rows whose sparse and corrected outputs are formed (the fit only
    needs the probe rows); `part` reuses a partition computed earlier for this head;
    `warm` is the previous call's state in a sequence ([P] App. C warm start).
    """
    N_q, N_k = Q.shape[0], K.shape[0]
    if part is None:
        part = (partition_semantic(Q, K, V, p, head) if p.partition == "semantic"
                else partition(Q, K, V, p, head, warm))
    gq, gk = part.gq, part.gk
    S = route_scores(part.qbar, part.kbar, part.vbar, gk.sizes, p.d)
    if p.budget == "calibrated":
        beta, sel = calibrated_selection(S, gq.sizes, gk.sizes, p.rho, p.M, N_q, N_k)
    else:
        beta = route_budget(p.rho, p.M, N_q, N_k)
        sel = select_cells(S, gk.sizes, beta)
    pairs = executed_pairs(gq.sizes, gk.sizes, sel)
    pairs_exec = pairs + p.M * N_k                       # [P] S4.3: probes add M/N_q
    permQ, offQ = group_major_permutation(gq.compact, gq.sizes.size)
    permK, offK = group_major_permutation(gk.compact, gk.sizes.size)
    cQ = part.km_Q.centres[gq.labels_used]
    dist = probe_distances(part.phiQ, cQ, gq)
    probes, m_a = select_probes(dist, gq, p.M)
    w = coverage_weights(gq, probes, m_a)
    x_probe = sparse_attention(Q, K, V, gq, gk, sel, probes)
    dense_probe = dense_attention(Q, K, V, probes)
    fit = fit_residual(x_probe, dense_probe - x_probe, w, p.lam, p.r, p.estimator)
    rows = np.arange(N_q) if rows is None else np.asarray(rows)
    osp = sparse_attention(Q, K, V, gq, gk, sel, rows)
    out = correct_rows(osp, fit)
    is_probe = np.zeros(N_q, dtype=bool)
    is_probe[probes] = True
    where = np.flatnonzero(is_probe[rows])
    if where.size:                                       # [R] step 5: probes keep dense output
        lookup = {int(pr): k for k, pr in enumerate(probes)}
        out[where] = dense_probe[[lookup[int(i)] for i in rows[where]]]
    return CallResult(part, S, beta, sel, pairs, pairs_exec, pairs / (N_q * N_k),
                      pairs_exec / (N_q * N_k), permQ, offQ, permK, offK, probes, m_a,
                      dist, w, x_probe, dense_probe, fit, rows, osp, out)


def cell_csr(sel: List[np.ndarray]):
    """Selected cells as (row pointer, KV group ids) with ids ascending per query group."""
    ptr = np.concatenate([[0], np.cumsum([s.size for s in sel])]).astype(np.int64)
    ids = np.concatenate(sel).astype(np.int64) if sel else np.zeros(0, np.int64)
    return ptr, ids
