"""The workspace-free entry point sparsepr_dense_rows_noalloc, through the C ABI.

It serves callers that cannot allocate device memory around the call (memory owned by
another allocator, or loops that must not pay cudaMalloc's implicit synchronisation).
Its rows must match exact fp64 attention (the oracle's dense rows) within the tests'
tolerances on two calls in a row (the calls share the library's fixed scratch array),
and agree with the library's dense engine.  This file is collected last so a failure
here never hides an earlier test.
"""
import ctypes

import numpy as np
import pytest
import torch

from free_block_sparse_plan_b200 import native as N
from free_block_sparse_plan_b200 import workloads as W
from oracle import sparsepr_oracle as O

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 1e-2}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import __graft_entry__
    __graft_entry__.build()


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def _inputs(dtype, H, Hk, Nq, Nk, d, seed):
    """Stored values (fp64 arrays of exactly the device values) and the device tensors."""
    rng = np.random.default_rng(seed)
    arrs = [rng.standard_normal((h, n, d)) * s for h, n, s in ((H, Nq, 0.8), (Hk, Nk, 0.8), (Hk, Nk, 1.0))]
    if dtype == "bf16":
        arrs = [W.round_to_bf16(a) for a in arrs]
    else:
        arrs = [a.astype(np.float32).astype(np.float64) for a in arrs]
    td = W.torch_dtype(dtype)
    return arrs, [torch.from_numpy(a.astype(np.float32)).to(td).cuda() for a in arrs]


def _call(params, Q, K, V, rows, out):
    st = torch.cuda.current_stream().cuda_stream
    N.sparsepr_dense_rows_noalloc(params, Q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                  rows.data_ptr(), rows.numel(), out.data_ptr(), st)
    torch.cuda.synchronize()


@pytest.mark.parametrize("dtype,d,H,G,Nq,Nk,nrows", [
    ("bf16", 128, 4, 1, 3000, 20000, 96),
    ("bf16", 64, 3, 1, 1000, 5003, 17),
    ("bf16", 64, 4, 2, 900, 4500, 33),
    ("f32", 64, 2, 1, 777, 3001, 128),
])
def test_noalloc_rows_match_exact_attention_twice(dtype, d, H, G, Nq, Nk, nrows):
    (q, k, v), (Q, K, V) = _inputs(dtype, H, H // G, Nq, Nk, d, seed=nrows)
    idx = np.linspace(0, Nq - 1, nrows).astype(np.int32)
    rows = torch.tensor(idx, device="cuda")
    params = N.make_params(H, Nq, Nk, d, dtype, 1, 1, 1, 1, 1, 1, 0, 0.0, 1.0, G=G)
    # exact fp64 attention of the requested rows (query head h reads K/V head h / G)
    ref = np.stack([O.dense_attention(q[h], k[h // G], v[h // G], idx) for h in range(H)])
    outs = []
    for _ in range(2):
        out = torch.empty((H, nrows, d), dtype=Q.dtype, device="cuda")
        _call(params, Q, K, V, rows, out)
        outs.append(out)
        assert _rel(out.double().cpu().numpy(), ref) < TOL[dtype]
    assert torch.equal(outs[0], outs[1])
    assert N.sparsepr_dense_check() == 0
    if G == 1:
        dense = N.dense_attention(Q, K, V)[:, rows.long()]
        assert _rel(outs[0].double().cpu().numpy(), dense.double().cpu().numpy()) < TOL[dtype]
        assert N.sparsepr_dense_check() == 0


def test_noalloc_clamps_rows_outside_the_queries():
    # An index below 0 reads row 0, one at or above N_q reads row N_q - 1.
    (q, k, v), (Q, K, V) = _inputs("bf16", 2, 2, 300, 1000, 64, seed=3)
    idx = np.array([-1, 0, 299, 300, 12345, -7], dtype=np.int32)
    rows = torch.tensor(idx, device="cuda")
    params = N.make_params(2, 300, 1000, 64, "bf16", 1, 1, 1, 1, 1, 1, 0, 0.0, 1.0)
    out = torch.empty((2, idx.size, 64), dtype=Q.dtype, device="cuda")
    _call(params, Q, K, V, rows, out)
    clamped = np.clip(idx, 0, 299)
    ref = np.stack([O.dense_attention(q[h], k[h], v[h], clamped) for h in range(2)])
    assert _rel(out.double().cpu().numpy(), ref) < TOL["bf16"]
    o = out.cpu()
    assert torch.equal(o[:, 0], o[:, 1]) and torch.equal(o[:, 0], o[:, 5])
    assert torch.equal(o[:, 2], o[:, 3]) and torch.equal(o[:, 2], o[:, 4])


def test_noalloc_reports_a_non_finite_row_and_the_check_clears_it():
    # A NaN key makes every requested row non-finite: the call completes, the rows are
    # NaN, the error word read by sparsepr_dense_check carries the non-finite bit, and the
    # check clears it (the next check and a clean call report nothing).
    _, (Q, K, V) = _inputs("bf16", 1, 1, 64, 512, 64, seed=4)
    rows = torch.arange(8, dtype=torch.int32, device="cuda")
    params = N.make_params(1, 64, 512, 64, "bf16", 1, 1, 1, 1, 1, 1, 0, 0.0, 1.0)
    out = torch.empty((1, 8, 64), dtype=Q.dtype, device="cuda")
    assert N.sparsepr_dense_check() == 0
    Kbad = K.clone()
    Kbad[0, 7, 3] = float("nan")
    _call(params, Q, Kbad, V, rows, out)
    assert torch.isnan(out.float()).all()
    assert N.sparsepr_dense_check() & 4
    assert N.sparsepr_dense_check() == 0
    _call(params, Q, K, V, rows, out)
    assert torch.isfinite(out.float()).all()
    assert N.sparsepr_dense_check() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    _, (Q, K, V) = _inputs("bf16", 1, 1, 16, 16, 64, seed=1)
    rows = torch.zeros(8, dtype=torch.int32, device="cuda")
    out = torch.empty((1, 8, 64), dtype=Q.dtype, device="cuda")
    big = N.make_params(64, 16, 4_000_000, 128, "bf16", 1, 1, 1, 1, 1, 1, 0, 0.0, 1.0)
    st = N.lib().sparsepr_dense_rows_noalloc(ctypes.byref(big), Q.data_ptr(), K.data_ptr(),
                                             V.data_ptr(), rows.data_ptr(), 128, out.data_ptr(), None)
    assert st == N.SPARSEPR_ERR_WORKSPACE
    p = N.make_params(1, 16, 16, 64, "bf16", 1, 1, 1, 1, 1, 1, 0, 0.0, 1.0)
    st = N.lib().sparsepr_dense_rows_noalloc(ctypes.byref(p), Q.data_ptr(), K.data_ptr(),
                                             V.data_ptr(), rows.data_ptr(), 129, out.data_ptr(), None)
    assert st == N.SPARSEPR_ERR_ARG
    many = N.make_params(70000, 16, 16, 8, "bf16", 1, 1, 1, 1, 1, 1, 0, 0.0, 1.0)
    st = N.lib().sparsepr_dense_rows_noalloc(ctypes.byref(many), Q.data_ptr(), K.data_ptr(),
                                             V.data_ptr(), rows.data_ptr(), 1, out.data_ptr(), None)
    assert st == N.SPARSEPR_ERR_SHAPE


def test_bounded_wait_gives_up_and_reports_without_fault():
    # A pipeline wait that nothing completes (no copy or product in flight): the self-test
    # warp waits through the engines' bounded mbarrier wait, gives up after about one
    # second and sets the timeout bit (32) of the word sparsepr_dense_check reads and
    # clears; the CUDA context stays usable afterwards.
    assert N.sparsepr_dense_check() == 0
    N.wait_selftest()
    assert N.sparsepr_dense_check() & 32
    assert N.sparsepr_dense_check() == 0
    x = torch.arange(8, dtype=torch.float32, device="cuda")
    assert float(x.sum()) == 28.0
