"""The workspace-free entry point sparsepr_dense_rows_noalloc, through the C ABI.

It serves callers that cannot allocate device memory around the call (memory owned by
another allocator, or loops that must not pay cudaMalloc's implicit synchronisation).
Its output must match the library's dense attention on the same rows, within the tests'
tolerances, on two calls in a row (the calls share the library's fixed scratch array).
This file is collected last so a failure here never hides an earlier test.
"""
import ctypes

import numpy as np
import pytest
import torch

from free_block_sparse_plan_b200 import native as N
from free_block_sparse_plan_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 1e-2}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import __graft_entry__
    __graft_entry__.build()


def _rel(a, b):
    a, b = a.double().cpu().numpy(), b.double().cpu().numpy()
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def _inputs(dtype, H, Nq, Nk, d, seed):
    rng = np.random.default_rng(seed)
    arrs = [rng.standard_normal((H, n, d)) * s for n, s in ((Nq, 0.8), (Nk, 0.8), (Nk, 1.0))]
    if dtype == "bf16":
        arrs = [W.round_to_bf16(a) for a in arrs]
    td = W.torch_dtype(dtype)
    return [torch.from_numpy(a.astype(np.float32)).to(td).cuda() for a in arrs]


@pytest.mark.parametrize("dtype,d,H,Nq,Nk,nrows", [
    ("bf16", 128, 4, 3000, 20000, 96),
    ("bf16", 64, 3, 1000, 5003, 17),
    ("f32", 64, 2, 777, 3001, 128),
])
def test_noalloc_rows_match_dense_attention_twice(dtype, d, H, Nq, Nk, nrows):
    Q, K, V = _inputs(dtype, H, Nq, Nk, d, seed=nrows)
    rows = torch.tensor(np.linspace(0, Nq - 1, nrows).astype(np.int32), device="cuda")
    params = N.make_params(H, Nq, Nk, d, dtype, 1, 1, 1, 1, 1, 1, 0, 0.0, 1.0)
    ref = N.dense_attention(Q, K, V)[:, rows.long()]
    st = torch.cuda.current_stream().cuda_stream
    outs = []
    for _ in range(2):
        out = torch.empty((H, nrows, d), dtype=Q.dtype, device="cuda")
        N.sparsepr_dense_rows_noalloc(params, Q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                      rows.data_ptr(), nrows, out.data_ptr(), st)
        torch.cuda.synchronize()
        outs.append(out)
        assert _rel(out, ref) < TOL[dtype]
    assert torch.equal(outs[0], outs[1])


def test_noalloc_rejects_sizes_beyond_its_scratch():
    Q, K, V = _inputs("bf16", 1, 16, 16, 64, seed=1)
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
