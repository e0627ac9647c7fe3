"""The seeded synthetic generator: determinism, storage rounding, calibration."""
import math

import numpy as np
import torch

from free_block_sparse_plan_b200 import workloads as W


def test_bf16_rounding_matches_torch_on_fp32_inputs():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(100000) * 10).astype(np.float32).astype(np.float64)
    ours = W.round_to_bf16(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)


def test_bf16_rounding_ties_to_even():
    # 1 + 2^-8 is halfway between bf16 neighbours 1 and 1 + 2^-7: ties go to the even one
    assert W.round_to_bf16(np.array([1 + 2.0 ** -8]))[0] == 1.0
    assert W.round_to_bf16(np.array([1 + 3 * 2.0 ** -8]))[0] == 1 + 2.0 ** -6
    assert W.round_to_bf16(np.array([1 + 2.0 ** -8 + 2.0 ** -30]))[0] == 1 + 2.0 ** -7


def test_tiny_workload_deterministic_and_calibrated():
    w = W.TINY
    q1, k1, v1 = W.make_head(w, 0)
    q2, k2, v2 = W.make_head(w, 0)
    assert np.array_equal(q1, q2) and np.array_equal(k1, k2) and np.array_equal(v1, v2)
    assert q1.shape == (1024, 64)
    assert np.array_equal(q1, q1.astype(np.float32).astype(np.float64))
    std = np.std(q1 @ k1.T / math.sqrt(64))
    assert abs(std - 4.0) < 0.01


def test_mid_workload_head_stream_and_storage():
    w = W.MID.with_(H=2, N=2048, grid=(2, 32, 32))
    q, k, v = W.make_head(w, 1)
    assert np.array_equal(q, W.round_to_bf16(q))
    q0, _, _ = W.make_head(w, 0)
    assert not np.array_equal(q, q0)
    tq, tk, tv = W.make_inputs_torch(w)
    assert tq.dtype == torch.bfloat16 and tq.shape == (2, 2048, 64)
    assert np.array_equal(tq[1].to(torch.float64).numpy(), q)


def test_centre_layout_counts():
    for w in (W.TINY, W.MID, W.WAN, W.HUNYUAN):
        cid = W._centre_ids(w)
        assert cid.size == w.N and cid.min() == 0 and cid.max() == w.centres - 1
        assert np.unique(cid).size == w.centres
