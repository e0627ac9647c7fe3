"""The C-ABI library on a machine without a GPU: it loads, exports every entry point
include/sparsepr.h declares, and validates arguments on the host before any launch."""
import ctypes
import os
import re

import numpy as np
import pytest

from conftest import ROOT
from free_block_sparse_plan_b200 import native as N
from free_block_sparse_plan_b200 import workloads as W


@pytest.fixture(scope="module", autouse=True)
def built():
    import __graft_entry__
    __graft_entry__.build()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "sparsepr.h")).read()
    return sorted(set(re.findall(r"^\s*(?:sparsepr_status|void|const char\*|unsigned long long)\s+"
                                 r"(sparsepr_\w+)\s*\(", text, re.M)))


def test_every_declared_symbol_is_exported():
    declared = _declared_functions()
    assert len(declared) >= 14
    lib = ctypes.CDLL(N._LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(N.SYMBOLS) == sorted(declared)


def test_struct_layout_matches_header():
    assert ctypes.sizeof(N.sparsepr_params) == 96
    assert N.sparsepr_params.estimator.offset == 80
    assert N.sparsepr_params.G.offset == 84
    assert N.sparsepr_params.partition.offset == 88
    assert N.sparsepr_params.lam.offset == 48
    assert N.sparsepr_params.seed.offset == 72


def test_status_strings():
    assert N.status_string(0) == "ok"
    assert "argument" in N.status_string(1)
    assert N.status_string(99) == "unknown status"


def _params(**kw):
    base = W.TINY.params()
    base.update(kw)
    return N.params_from_dict(base)


def test_workspace_size_positive_and_monotone():
    small = N.sparsepr_workspace_size(_params())
    big = N.sparsepr_workspace_size(N.params_from_dict(W.HUNYUAN.params()))
    assert 0 < small < big
    assert big % 256 == 0


@pytest.mark.parametrize("field,value,status", [
    ("d", 60, N.SPARSEPR_ERR_SHAPE), ("d", 256, N.SPARSEPR_ERR_SHAPE),
    ("dtype", 7, N.SPARSEPR_ERR_DTYPE), ("H", 0, N.SPARSEPR_ERR_SHAPE),
    ("r_K", 0, N.SPARSEPR_ERR_ARG), ("r_Q", 65, N.SPARSEPR_ERR_ARG),
    ("C_q", 2000, N.SPARSEPR_ERR_ARG), ("C_k", 0, N.SPARSEPR_ERR_ARG),
    ("M", 0, N.SPARSEPR_ERR_ARG), ("M", 129, N.SPARSEPR_ERR_ARG),
    ("r", 17, N.SPARSEPR_ERR_ARG), ("r", -1, N.SPARSEPR_ERR_ARG),
    ("lam", -0.5, N.SPARSEPR_ERR_ARG), ("lam", float("nan"), N.SPARSEPR_ERR_ARG),
    ("target_density", 1.5, N.SPARSEPR_ERR_ARG), ("target_density", 0.01, N.SPARSEPR_ERR_ARG),
    ("kmeans_max_iter", 0, N.SPARSEPR_ERR_ARG), ("engine", 3, N.SPARSEPR_ERR_ARG),
    ("G", -1, N.SPARSEPR_ERR_SHAPE), ("G", 5, N.SPARSEPR_ERR_SHAPE),
    ("partition", 2, N.SPARSEPR_ERR_ARG), ("budget", 2, N.SPARSEPR_ERR_ARG),
])
def test_invalid_parameters_rejected_on_host(field, value, status):
    p = _params()
    setattr(p, field, value)
    with pytest.raises(N.SparsePRError) as ei:
        N.sparsepr_workspace_size(p)
    assert ei.value.status == status
    # the plan entry point rejects them before touching the (fake) device pointers
    h = ctypes.c_void_p()
    st = N.lib().sparsepr_plan(ctypes.byref(p), 256, 256, 256, 256, 1 << 40, None, ctypes.byref(h))
    assert st == status and not h.value


def test_plan_rejects_missing_or_small_workspace():
    p = _params()
    h = ctypes.c_void_p()
    need = N.sparsepr_workspace_size(p)
    L = N.lib()
    assert L.sparsepr_plan(ctypes.byref(p), 256, 256, 256, None, need, None, ctypes.byref(h)) == N.SPARSEPR_ERR_WORKSPACE
    assert L.sparsepr_plan(ctypes.byref(p), 256, 256, 256, 512 + 8, need, None, ctypes.byref(h)) == N.SPARSEPR_ERR_WORKSPACE
    assert L.sparsepr_plan(ctypes.byref(p), 256, 256, 256, 512, need - 1, None, ctypes.byref(h)) == N.SPARSEPR_ERR_WORKSPACE
    assert L.sparsepr_plan(ctypes.byref(p), None, 256, 256, 512, need, None, ctypes.byref(h)) == N.SPARSEPR_ERR_ARG


def test_calls_out_of_order_or_null_are_rejected():
    L = N.lib()
    assert L.sparsepr_attend(None, None) == N.SPARSEPR_ERR_ARG
    assert L.sparsepr_probe_fit(None, None) == N.SPARSEPR_ERR_ARG
    assert L.sparsepr_correct(None, 256, None) == N.SPARSEPR_ERR_ARG
    L.sparsepr_destroy(None)


def test_gqa_group_sizes_and_warm_start_restriction():
    # H = 4 query heads: groups of 1, 2 and 4 are valid; a warm start takes G <= 1
    for g in (0, 1, 2, 4):
        p = _params()
        p.H, p.G = 4, g
        assert N.sparsepr_workspace_size(p) > 0
    p = _params()
    p.H, p.G = 4, 2
    h = ctypes.c_void_p()
    st = N.lib().sparsepr_plan_warm(ctypes.byref(p), 256, 256, 256, 256, 256, 1 << 40, None, ctypes.byref(h))
    assert st == N.SPARSEPR_ERR_ARG and not h.value


def test_semantic_partition_limits():
    # the raw channels are the coordinates: d <= 64; warm starts take the response partition
    p = _params(partition=1)
    assert N.sparsepr_workspace_size(p) > 0
    q = N.params_from_dict(dict(W.WAN.params(), partition=1))
    with pytest.raises(N.SparsePRError) as ei:
        N.sparsepr_workspace_size(q)
    assert ei.value.status == N.SPARSEPR_ERR_ARG
    h = ctypes.c_void_p()
    st = N.lib().sparsepr_plan_warm(ctypes.byref(p), 256, 256, 256, 256, 256, 1 << 40, None, ctypes.byref(h))
    assert st == N.SPARSEPR_ERR_ARG and not h.value


def test_bench_traffic_record_matches_kernel_source_by_hash(tmp_path, monkeypatch):
    # the recorded DRAM traffic is used only while the kernel source is the one captured,
    # scaled by heads, and only for the captured workload family and shape
    import hashlib
    import json
    import bench
    src = b"// kernel source\n"
    (tmp_path / "free_block_sparse_plan_b200" / "csrc").mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (tmp_path / "free_block_sparse_plan_b200" / "csrc" / "k.cu").write_bytes(src)
    rec = {"k.cu": [{"family": "mid", "N": 16384, "d": 64, "H": 12, "bytes_per_launch": 1200,
                     "sha256": hashlib.sha256(src).hexdigest()}]}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("k.cu", W.MID) == 1200.0
    assert bench.measured_traffic("k.cu", W.MID.with_(H=6)) == 600.0
    assert bench.measured_traffic("k.cu", W.WAN) is None
    (tmp_path / "free_block_sparse_plan_b200" / "csrc" / "k.cu").write_bytes(src + b"//")
    assert bench.measured_traffic("k.cu", W.MID) is None


def test_bench_tile_pair_accounting():
    import bench
    sizes_q = np.array([[148, 20, 0]])             # two query groups
    n_q = np.array([2])
    cell_cnt = np.array([[2, 1, 0]])
    cell_ids = np.array([[[0, 2, 0], [1, 0, 0], [0, 0, 0]]])
    sizes_k = np.array([[100, 300, 60]])
    proc, routed = bench.tile_pairs(sizes_q, n_q, cell_cnt, cell_ids, sizes_k)
    # group 0: 148 rows -> 256, keys 100 + 60 = 160 -> 256; group 1: 20 -> 128, 300 -> 384
    assert proc == 256 * 256 + 128 * 384
    assert routed == 148 * 160 + 20 * 300
    # GQA: query head h reads the key sizes of K/V head h // G
    proc2, _ = bench.tile_pairs(np.vstack([sizes_q, sizes_q]), np.array([2, 2]),
                                np.vstack([cell_cnt, cell_cnt]), np.vstack([cell_ids, cell_ids]),
                                sizes_k, G=2)
    assert proc2 == 2 * proc


def test_bench_tile_accounting_from_plan_exports():
    import bench

    class FakePlan:
        def export(self, name):
            return {"SIZES_Q": np.array([[148, 20, 0]]), "GROUPS_Q": np.array([2]),
                    "CELL_COUNT": np.array([[2, 1, 0]]),
                    "CELL_IDS": np.array([[[0, 2, 0], [1, 0, 0], [0, 0, 0]]]),
                    "SIZES_K": np.array([[100, 300, 60]]), "GROUPS_K": np.array([3])}[name]

    acc = bench.attention_tile_accounting(FakePlan(), W.MID, 1)
    assert acc["groups_q"] == [2] and acc["groups_kv"] == [3]
    assert acc["processed_pairs"] == 256 * 256 + 128 * 384
    assert acc["routed_pairs"] == 148 * 160 + 20 * 300
    assert abs(acc["fraction"] - (1 - acc["routed_pairs"] / acc["processed_pairs"])) < 1e-15
    assert "unavailable" in bench.attention_tile_accounting(FakePlan(), W.TINY, 1)   # fp32: CUDA cores

    class Broken:
        def export(self, name):
            raise RuntimeError("no such export")

    assert "unavailable" in bench.attention_tile_accounting(Broken(), W.MID, 1)


def test_exp2_poly_meets_its_stated_error_bound():
    # The attention softmax evaluates part of its exponentials as 2^x = 2^n * p(f) with a
    # cubic p on [-1/2, 1/2] (tc_ptx.cuh, exp2_poly / exp2_poly2).  Its comment states a
    # relative error of 2.4e-4, under bf16's 2^-9.  The coefficients are read from the
    # source and the fp32 steps emulated (fused multiply-adds exactly rounded once).
    import re
    src = open(os.path.join(ROOT, "free_block_sparse_plan_b200", "csrc", "tc_ptx.cuh")).read()
    body = src[src.index("float exp2_poly(float x)"):]
    body = body[:body.index("}")]
    coef = [float(c) for c in re.findall(r"([0-9.]+e[-+][0-9]+)f", body)]
    assert len(coef) == 4
    c3, c2, c1, c0 = (np.float32(c) for c in coef)
    x = np.concatenate([np.linspace(-126.0, 8.0, 2_000_001), np.linspace(-1.0, 1.0, 200_001)])
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    C = np.float32(12582912.0)
    t = (x + C).astype(np.float32)
    f = (x - (t - C)).astype(np.float32)

    def fma(a, b, c):
        return (a.astype(np.float64) * b.astype(np.float64) + np.float64(c)).astype(np.float32)

    p = fma(np.full_like(f, c3), f, c2)
    p = fma(p, f, c1)
    p = fma(p, f, c0)
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    y = bits.astype(np.uint32).view(np.float32).astype(np.float64)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(y - exact) / exact
    normal = exact >= 2.0 ** -125          # results in the denormal range are not claimed
    assert rel[normal].max() < 2.5e-4, rel[normal].max()
    assert rel[normal].max() < 2.0 ** -9
