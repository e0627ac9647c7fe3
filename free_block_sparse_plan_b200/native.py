"""ctypes binding of libsparsepr.so: the C ABI in include/sparsepr.h, same names.

Argument marshalling only.  Every step of the SparsePR call runs in the library's CUDA
kernels; torch supplies device memory and the stream handle.  If the library is not
built, loading raises: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_double, c_int32, c_int64, c_size_t, c_uint64, c_void_p
from typing import Optional

import numpy as np

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsparsepr.so")

SPARSEPR_OK = 0
SPARSEPR_ERR_ARG = 1
SPARSEPR_ERR_SHAPE = 2
SPARSEPR_ERR_DTYPE = 3
SPARSEPR_ERR_WORKSPACE = 4
SPARSEPR_ERR_CUDA = 5
SPARSEPR_ERR_DEVICE_CHECK = 6
SPARSEPR_ERR_STATE = 7

SPARSEPR_F32 = 0
SPARSEPR_BF16 = 1
SPARSEPR_ENGINE_AUTO = 0
SPARSEPR_EST_RIDGE, SPARSEPR_EST_MEAN, SPARSEPR_EST_SCALAR, SPARSEPR_EST_DIAGONAL = 0, 1, 2, 3
SPARSEPR_PARTITION_RESPONSE, SPARSEPR_PARTITION_SEMANTIC = 0, 1
SPARSEPR_BUDGET_PREFIX, SPARSEPR_BUDGET_CALIBRATED = 0, 1
SPARSEPR_ENGINE_SIMT = 1

EXPORTS = [
    "LABELS_K", "LABELS_Q", "PERM_K", "PERM_Q", "GROUPS_K", "GROUPS_Q", "SIZES_K", "SIZES_Q",
    "CELL_COUNT", "CELL_IDS", "PROBES", "PROBE_COUNT", "KMEANS_ITERS", "OBJECTIVE", "PAIRS",
    "FACTOR_K", "FACTOR_Q", "EIG_K", "EIG_Q", "METRIC_K", "METRIC_Q", "PHI_K", "PHI_Q",
    "CENTRES_Q", "SCORES", "OSP", "ODENSE_PROBE", "FIT_MU_X", "FIT_MU_R", "FIT_S", "FIT_B",
    "FIT_P", "FIT_REFF", "PROBE_DIST", "KBAR", "QBAR", "KM_REASSIGNED", "BETA",
]
EXPORT_ID = {name: i for i, name in enumerate(EXPORTS)}

# The public entry points, exactly as include/sparsepr.h declares them.
SYMBOLS = [
    "sparsepr_workspace_size", "sparsepr_plan", "sparsepr_plan_from_labels", "sparsepr_attend",
    "sparsepr_probe_fit", "sparsepr_correct", "sparsepr_forward", "sparsepr_dense_attention",
    "sparsepr_check", "sparsepr_get_stats", "sparsepr_export_size", "sparsepr_export",
    "sparsepr_destroy", "sparsepr_status_string", "sparsepr_dense_rows_noalloc",
    "sparsepr_launch_count", "sparsepr_state_size", "sparsepr_save_state", "sparsepr_plan_warm",
    "sparsepr_dense_check", "sparsepr_wait_selftest", "sparsepr_support_workspace_size", "sparsepr_support_densities",
    "sparsepr_affine_workspace_size", "sparsepr_affine_fit",
]


class sparsepr_params(ctypes.Structure):
    _fields_ = [("H", c_int32), ("N_q", c_int32), ("N_k", c_int32), ("d", c_int32),
                ("dtype", c_int32), ("M_s", c_int32), ("r_K", c_int32), ("r_Q", c_int32),
                ("C_q", c_int32), ("C_k", c_int32), ("M", c_int32), ("r", c_int32),
                ("lam", c_double), ("target_density", c_double),
                ("kmeans_max_iter", c_int32), ("engine", c_int32), ("seed", c_uint64),
                ("estimator", c_int32), ("G", c_int32), ("partition", c_int32),
                ("budget", c_int32)]


class sparsepr_stats(ctypes.Structure):
    _fields_ = [("pairs_route", c_int64), ("pairs_exec", c_int64), ("rho_route", c_double),
                ("rho_exec", c_double), ("kmeans_iters_k_max", c_int32),
                ("kmeans_iters_q_max", c_int32), ("groups_k_min", c_int32),
                ("groups_q_min", c_int32), ("device_error", c_int32)]


class SparsePRError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib = None


def lib():
    """The loaded library (loads on first use; raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is not built; run "
                               "`python -c 'import __graft_entry__ as g; g.build()'`")
        L = ctypes.CDLL(_LIB_PATH)
        P = POINTER(sparsepr_params)
        sig = {
            "sparsepr_workspace_size": (c_int32, [P, POINTER(c_size_t)]),
            "sparsepr_plan": (c_int32, [P, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                        c_void_p, POINTER(c_void_p)]),
            "sparsepr_plan_from_labels": (c_int32, [P, c_void_p, c_void_p, c_void_p, c_void_p,
                                                    c_void_p, c_void_p, c_size_t, c_void_p,
                                                    POINTER(c_void_p)]),
            "sparsepr_attend": (c_int32, [c_void_p, c_void_p]),
            "sparsepr_probe_fit": (c_int32, [c_void_p, c_void_p]),
            "sparsepr_correct": (c_int32, [c_void_p, c_void_p, c_void_p]),
            "sparsepr_forward": (c_int32, [P, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                           c_size_t, c_void_p]),
            "sparsepr_dense_attention": (c_int32, [P, c_void_p, c_void_p, c_void_p, c_void_p,
                                                   c_void_p]),
            "sparsepr_check": (c_int32, [c_void_p, c_void_p, POINTER(c_int32)]),
            "sparsepr_dense_check": (c_int32, [c_void_p, POINTER(c_int32)]),
            "sparsepr_wait_selftest": (c_int32, [c_void_p]),
            "sparsepr_support_workspace_size": (c_int32, [P, c_int32, c_int32, POINTER(c_size_t)]),
            "sparsepr_support_densities": (c_int32, [P, c_void_p, c_void_p, c_void_p, c_void_p,
                                                     c_int32, c_int32, c_double, c_void_p, c_size_t,
                                                     c_void_p, c_void_p, c_void_p]),
            "sparsepr_affine_workspace_size": (c_int32, [c_void_p, POINTER(c_size_t)]),
            "sparsepr_affine_fit": (c_int32, [c_void_p, c_void_p, c_void_p, c_size_t, c_void_p,
                                              c_void_p, c_void_p]),
            "sparsepr_get_stats": (c_int32, [c_void_p, c_void_p, POINTER(sparsepr_stats)]),
            "sparsepr_export_size": (c_int32, [c_void_p, c_int32, POINTER(c_size_t)]),
            "sparsepr_export": (c_int32, [c_void_p, c_int32, c_void_p, c_size_t, c_void_p]),
            "sparsepr_destroy": (None, [c_void_p]),
            "sparsepr_dense_rows_noalloc": (c_int32, [P, c_void_p, c_void_p, c_void_p, c_void_p,
                                                      c_int32, c_void_p, c_void_p]),
            "sparsepr_status_string": (c_char_p, [c_int32]),
            "sparsepr_launch_count": (ctypes.c_ulonglong, []),
            "sparsepr_state_size": (c_int32, [P, POINTER(c_size_t)]),
            "sparsepr_save_state": (c_int32, [c_void_p, c_void_p, c_void_p]),
            "sparsepr_plan_warm": (c_int32, [P, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                             c_size_t, c_void_p, POINTER(c_void_p)]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def launch_count() -> int:
    """Kernels the library has enqueued since it was loaded."""
    return int(lib().sparsepr_launch_count())


def status_string(status: int) -> str:
    return lib().sparsepr_status_string(status).decode()


def _check(status: int, where: str):
    if status != SPARSEPR_OK:
        raise SparsePRError(status, where)


def make_params(H, N_q, N_k, d, dtype, M_s, r_K, r_Q, C_q, C_k, M, r, lam, target_density,
                kmeans_max_iter=25, seed=0, engine=SPARSEPR_ENGINE_AUTO, estimator=0,
                G=1, partition=0, budget=0) -> sparsepr_params:
    if isinstance(dtype, str):
        dtype = {"f32": SPARSEPR_F32, "bf16": SPARSEPR_BF16}[dtype]
    return sparsepr_params(H=H, N_q=N_q, N_k=N_k, d=d, dtype=dtype, M_s=M_s, r_K=r_K, r_Q=r_Q,
                           C_q=C_q, C_k=C_k, M=M, r=r, lam=lam, target_density=target_density,
                           kmeans_max_iter=kmeans_max_iter, engine=engine, seed=seed,
                           estimator=estimator, G=G, partition=partition, budget=budget)


def params_from_dict(p: dict, engine=SPARSEPR_ENGINE_AUTO) -> sparsepr_params:
    return make_params(p["H"], p["N_q"], p["N_k"], p["d"], p["dtype"], p["M_s"], p["r_K"],
                       p["r_Q"], p["C_q"], p["C_k"], p["M"], p["r"], p["lam"],
                       p["target_density"], p["kmeans_max_iter"], p["seed"], engine,
                       p.get("estimator", 0), p.get("G", 1), p.get("partition", 0),
                       p.get("budget", 0))


# ----------------------------------------------------------------------------------
# Functions with the C names (pointers as ints / ctypes, streams as ints)

def sparsepr_workspace_size(params: sparsepr_params) -> int:
    n = c_size_t()
    _check(lib().sparsepr_workspace_size(ctypes.byref(params), ctypes.byref(n)),
           "sparsepr_workspace_size")
    return n.value


def sparsepr_plan(params, Q, K, V, workspace, workspace_bytes, stream) -> c_void_p:
    h = c_void_p()
    _check(lib().sparsepr_plan(ctypes.byref(params), Q, K, V, workspace, workspace_bytes, stream,
                               ctypes.byref(h)), "sparsepr_plan")
    return h


def sparsepr_plan_from_labels(params, Q, K, V, labQ, labK, workspace, workspace_bytes, stream):
    h = c_void_p()
    _check(lib().sparsepr_plan_from_labels(ctypes.byref(params), Q, K, V, labQ, labK, workspace,
                                           workspace_bytes, stream, ctypes.byref(h)),
           "sparsepr_plan_from_labels")
    return h


def sparsepr_state_size(params: sparsepr_params) -> int:
    n = c_size_t()
    _check(lib().sparsepr_state_size(ctypes.byref(params), ctypes.byref(n)), "sparsepr_state_size")
    return n.value


def sparsepr_save_state(plan, state, stream):
    _check(lib().sparsepr_save_state(plan, state, stream), "sparsepr_save_state")


def sparsepr_plan_warm(params, Q, K, V, state, workspace, workspace_bytes, stream):
    h = c_void_p()
    _check(lib().sparsepr_plan_warm(ctypes.byref(params), Q, K, V, state, workspace,
                                    workspace_bytes, stream, ctypes.byref(h)), "sparsepr_plan_warm")
    return h


def sparsepr_attend(plan, stream):
    _check(lib().sparsepr_attend(plan, stream), "sparsepr_attend")


def sparsepr_probe_fit(plan, stream):
    _check(lib().sparsepr_probe_fit(plan, stream), "sparsepr_probe_fit")


def sparsepr_correct(plan, Out, stream):
    _check(lib().sparsepr_correct(plan, Out, stream), "sparsepr_correct")


def sparsepr_forward(params, Q, K, V, Out, workspace, workspace_bytes, stream):
    _check(lib().sparsepr_forward(ctypes.byref(params), Q, K, V, Out, workspace, workspace_bytes,
                                  stream), "sparsepr_forward")


def sparsepr_dense_attention(params, Q, K, V, Out, stream):
    _check(lib().sparsepr_dense_attention(ctypes.byref(params), Q, K, V, Out, stream),
           "sparsepr_dense_attention")


def sparsepr_check(plan, stream) -> int:
    e = c_int32()
    st = lib().sparsepr_check(plan, stream, ctypes.byref(e))
    if st not in (SPARSEPR_OK, SPARSEPR_ERR_DEVICE_CHECK):
        _check(st, "sparsepr_check")
    return e.value


def sparsepr_get_stats(plan, stream) -> dict:
    s = sparsepr_stats()
    st = lib().sparsepr_get_stats(plan, stream, ctypes.byref(s))
    if st not in (SPARSEPR_OK, SPARSEPR_ERR_DEVICE_CHECK):
        _check(st, "sparsepr_get_stats")
    return {name: getattr(s, name) for name, _ in sparsepr_stats._fields_}


def sparsepr_export_size(plan, what: int) -> int:
    n = c_size_t()
    _check(lib().sparsepr_export_size(plan, what, ctypes.byref(n)), "sparsepr_export_size")
    return n.value


def sparsepr_export(plan, what: int, dst, nbytes: int, stream):
    _check(lib().sparsepr_export(plan, what, dst, nbytes, stream), "sparsepr_export")


def sparsepr_destroy(plan):
    lib().sparsepr_destroy(plan)


def sparsepr_status_string(status: int) -> str:
    return status_string(status)


def sparsepr_dense_rows_noalloc(params, Q, K, V, rows, nrows, Out, stream):
    _check(lib().sparsepr_dense_rows_noalloc(ctypes.byref(params), Q, K, V, rows, nrows, Out,
                                             stream), "sparsepr_dense_rows_noalloc")


def sparsepr_dense_check(stream=None) -> int:
    """Reads and clears the error words of the plan-free entry points (dense attention and
    the workspace-free rows); returns the word (0 = none)."""
    e = c_int32(0)
    st = lib().sparsepr_dense_check(stream, ctypes.byref(e))
    if st not in (SPARSEPR_OK, SPARSEPR_ERR_DEVICE_CHECK):
        raise SparsePRError(st, "sparsepr_dense_check")
    return int(e.value)


def wait_selftest(stream=None):
    """Launches the bounded-wait self-test (a wait nothing completes gives up after about
    one second and sets bit 32 of the word sparsepr_dense_check reads)."""
    _check(lib().sparsepr_wait_selftest(stream), "sparsepr_wait_selftest")


def support_densities(Q, K, rows, pool, npools, alpha=0.9, stream=None):
    """O1 support sizes |D_i(alpha)| of rows [H, nrows] (device int32) and the pooled
    union sizes of each pool [H, npools] (pool: device int32 [H, nrows]); see
    sparsepr_support_densities."""
    import torch
    H, Nq, d = Q.shape
    dt = SPARSEPR_BF16 if Q.dtype == torch.bfloat16 else SPARSEPR_F32
    p = make_params(H, Nq, K.shape[1], d, dt, 1, 1, 1, 1, 1, 1, 0, 0.0, 1.0, G=H // K.shape[0])
    nrows = rows.shape[1]
    nb = c_size_t(0)
    _check(lib().sparsepr_support_workspace_size(ctypes.byref(p), nrows, npools, ctypes.byref(nb)),
           "sparsepr_support_workspace_size")
    ws = torch.empty(nb.value, dtype=torch.uint8, device=Q.device)
    sizes = torch.empty((H, nrows), dtype=torch.int32, device=Q.device)
    pooled = torch.empty((H, npools), dtype=torch.int32, device=Q.device)
    _check(lib().sparsepr_support_densities(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(rows), _ptr(pool),
                                            nrows, npools, alpha, _ptr(ws), nb.value, _ptr(sizes),
                                            _ptr(pooled), _stream(stream)), "sparsepr_support_densities")
    return sizes, pooled


# ----------------------------------------------------------------------------------
# Torch convenience layer (still marshalling only)

def _ptr(t) -> int:
    return t.data_ptr()


def _stream(stream=None) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _export_layout(p: sparsepr_params, name: str):
    H, d = p.H, p.d
    Hk = H // max(p.G, 1)                # K/V heads
    rK, rQ = (d, d) if p.partition == SPARSEPR_PARTITION_SEMANTIC else (p.r_K, p.r_Q)
    i32, f64, f32, i64 = np.int32, np.float64, np.float32, np.int64
    return {
        "LABELS_K": (i32, (Hk, p.N_k)), "LABELS_Q": (i32, (H, p.N_q)),
        "PERM_K": (i32, (Hk, p.N_k)), "PERM_Q": (i32, (H, p.N_q)),
        "GROUPS_K": (i32, (Hk,)), "GROUPS_Q": (i32, (H,)),
        "SIZES_K": (i32, (Hk, p.C_k)), "SIZES_Q": (i32, (H, p.C_q)),
        "CELL_COUNT": (i32, (H, p.C_q)), "CELL_IDS": (i32, (H, p.C_q, p.C_k)),
        "PROBES": (i32, (H, p.M)), "PROBE_COUNT": (i32, (H, p.C_q)),
        "KMEANS_ITERS": (i32, (H, 2)), "OBJECTIVE": (f64, (H, 2)), "PAIRS": (i64, (H,)),
        "FACTOR_K": (f64, (Hk, d, rK)), "FACTOR_Q": (f64, (Hk, d, rQ)),
        "EIG_K": (f64, (Hk, rK)), "EIG_Q": (f64, (Hk, rQ)),
        "METRIC_K": (f64, (Hk, d, d)), "METRIC_Q": (f64, (Hk, d, d)),
        "PHI_K": (f64, (Hk, p.N_k, rK)), "PHI_Q": (f64, (H, p.N_q, rQ)),
        "CENTRES_Q": (f64, (H, p.C_q, rQ)), "SCORES": (f64, (H, p.C_q, p.C_k)),
        "OSP": (f32, (H, p.N_q, d)), "ODENSE_PROBE": (f32, (H, p.M, d)),
        "FIT_MU_X": (f64, (H, d)), "FIT_MU_R": (f64, (H, d)), "FIT_S": (f64, (H, d)),
        "FIT_B": (f64, (H, d, d)), "FIT_P": (f64, (H, d, d)), "FIT_REFF": (i32, (H,)),
        "PROBE_DIST": (f64, (H, p.N_q)), "KBAR": (f64, (Hk, p.C_k, d)),
        "QBAR": (f64, (H, p.C_q, d)),
        "KM_REASSIGNED": (i64, (2, H)), "BETA": (f64, (H,)),
    }[name]


class Plan:
    """A planned SparsePR call over device tensors Q, K, V [H, N, d] (fp32 or bf16)."""

    def __init__(self, params: sparsepr_params, Q, K, V, workspace=None, labels=None, stream=None,
                 warm=None):
        """`warm`: a state tensor written by `save_state` of the previous call of a sequence
        (cross-call warm start); `labels`: injected k-means labels (testing)."""
        import torch
        self.params = params
        self.inputs = (Q, K, V)          # keep alive until the plan is destroyed
        nbytes = sparsepr_workspace_size(params)
        if workspace is None:
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=Q.device)
        self.workspace = workspace
        st = _stream(stream)
        if warm is not None:
            self._warm = warm
            self.handle = sparsepr_plan_warm(params, _ptr(Q), _ptr(K), _ptr(V), _ptr(warm),
                                             _ptr(workspace), workspace.numel(), st)
        elif labels is None:
            self.handle = sparsepr_plan(params, _ptr(Q), _ptr(K), _ptr(V), _ptr(workspace),
                                        workspace.numel(), st)
        else:
            labQ, labK = labels
            self._labels = (labQ, labK)
            self.handle = sparsepr_plan_from_labels(params, _ptr(Q), _ptr(K), _ptr(V), _ptr(labQ),
                                                    _ptr(labK), _ptr(workspace),
                                                    workspace.numel(), st)

    def attend(self, stream=None):
        sparsepr_attend(self.handle, _stream(stream))

    def save_state(self, state=None, stream=None):
        """Writes this call's warm state into `state` (a device uint8 tensor of
        `state_size(params)` bytes, allocated when None) and returns it."""
        if state is None:
            state = new_state(self.params, self.inputs[0].device)
        sparsepr_save_state(self.handle, _ptr(state), _stream(stream))
        return state

    def probe_fit(self, stream=None):
        sparsepr_probe_fit(self.handle, _stream(stream))

    def correct(self, out=None, stream=None):
        import torch
        if out is None:
            Q = self.inputs[0]
            out = torch.empty_like(Q)
        sparsepr_correct(self.handle, _ptr(out), _stream(stream))
        return out

    def stats(self, stream=None) -> dict:
        return sparsepr_get_stats(self.handle, _stream(stream))

    def check(self, stream=None) -> int:
        return sparsepr_check(self.handle, _stream(stream))

    def affine_fit(self, dense, stream=None):
        """O3 affine fit of the residual dense - O_sp (dense: [H, N_q, d] device tensor in
        original order); returns (explained fraction [H], remaining squared error [H])."""
        import torch
        nb = c_size_t(0)
        _check(lib().sparsepr_affine_workspace_size(self.handle, ctypes.byref(nb)),
               "sparsepr_affine_workspace_size")
        ws = torch.empty(nb.value, dtype=torch.uint8, device=dense.device)
        H = self.params.H
        expl = torch.empty(H, dtype=torch.float64, device=dense.device)
        err = torch.empty(H, dtype=torch.float64, device=dense.device)
        _check(lib().sparsepr_affine_fit(self.handle, _ptr(dense), _ptr(ws), nb.value, _ptr(expl),
                                         _ptr(err), _stream(stream)), "sparsepr_affine_fit")
        return expl, err

    def export(self, name: str, stream=None) -> np.ndarray:
        dtype, shape = _export_layout(self.params, name)
        arr = np.empty(shape, dtype=dtype)
        nbytes = sparsepr_export_size(self.handle, EXPORT_ID[name])
        assert nbytes == arr.nbytes, (name, nbytes, arr.nbytes)
        sparsepr_export(self.handle, EXPORT_ID[name], arr.ctypes.data, arr.nbytes, _stream(stream))
        return arr

    def close(self):
        if getattr(self, "handle", None):
            sparsepr_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def new_state(params: sparsepr_params, device):
    """An uninitialised warm-state buffer (torch allocations are 256-byte aligned)."""
    import torch
    return torch.empty(sparsepr_state_size(params), dtype=torch.uint8, device=device)


def forward(params: sparsepr_params, Q, K, V, out=None, workspace=None, stream=None):
    """One SparsePR attention call: plan, attend, probe fit and correct on one stream."""
    import torch
    if workspace is None:
        workspace = torch.empty(sparsepr_workspace_size(params), dtype=torch.uint8, device=Q.device)
    if out is None:
        out = torch.empty_like(Q)
    sparsepr_forward(params, _ptr(Q), _ptr(K), _ptr(V), _ptr(out), _ptr(workspace),
                     workspace.numel(), _stream(stream))
    return out


def dense_attention(Q, K, V, out=None, engine=SPARSEPR_ENGINE_AUTO, stream=None):
    """softmax(Q K^T / sqrt(d)) V through the library's attention engine."""
    import torch
    H, Nq, d = Q.shape
    dt = SPARSEPR_BF16 if Q.dtype == torch.bfloat16 else SPARSEPR_F32
    G = H // K.shape[0]                  # query heads per K/V head
    p = make_params(H, Nq, K.shape[1], d, dt, 1, 1, 1, 1, 1, 1, 0, 0.0, 1.0, engine=engine, G=G)
    if out is None:
        out = torch.empty_like(Q)
    sparsepr_dense_attention(p, _ptr(Q), _ptr(K), _ptr(V), _ptr(out), _stream(stream))
    return out
