"""Seeded synthetic workloads shaped like the video-DiT attention calls SparsePR targets.

This module only draws inputs. It holds none of SparsePR's arithmetic, so both the
fp64 oracle (under ``oracle/``) and the CUDA path can consume it without sharing
method code.

The SparsePR paper ("Partition the Support, Reconstruct the Residual: Training-Free
Sparse Attention for Video Generation and World Models") measures on captured
activations of Wan2.2, HunyuanVideo and Cosmos models, which are not available here.
These generators stand in for them with the same shapes (a 21x45x80 latent grid is
75600 tokens, 33x45x80 is 118800), head dimension, and target densities (the
review page's hyper-parameter table: r_K=48, r_Q=64, M=64, r=16, lambda=0.1,
22%/26% targets).

Recipe (one head; every head draws from its own child seed):
  * tokens in raster order n = (t*GH + y)*GW + x over a (T, GH, GW) grid;
  * centre id c(n) = (floor(t*a_t/T)*a_y + floor(y*a_y/GH))*a_x + floor(x*a_x/GW);
  * centres mu_c ~ N(0, I_d); K_n = mu_c(n) + sigma_K*eps, Q_n = mu_c(n) + sigma_Q*eps';
  * optional local spatial bias: e_n @ G added to Q_n and K_n with
    e_n = [sin(pi t/T), cos(pi t/T), sin(2 pi y/GH), cos(2 pi y/GH), sin(2 pi x/GW),
    cos(2 pi x/GW)] and G ~ N(0,1) of shape [6, d];
  * V ~ N(0, 1);
  * call `step` s > 0 of a sequence (denoising steps) adds s * drift * (dmu_c(n) +
    sigma * e_n) to K and Q and s * drift * e_n to V, with dmu ~ N(0, I_d) per centre and
    e_n ~ N(0, I_d) drawn from the head's second seed stream (step 0 is unchanged);
  * logit-std calibration: sigma_hat = std(q_i . k_j / sqrt(d)) over 65536 random
    (i, j) pairs (all pairs when N*N <= 65536 * 16), then Q and K are each multiplied
    by sqrt(target / sigma_hat);
  * drawn in fp64 with numpy PCG64, then rounded once (round-to-nearest-even) to the
    storage dtype (fp32 or bf16).  Every consumer reads exactly the stored values.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Tuple

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    H: int
    N: int
    d: int
    dtype: str                  # "f32" or "bf16"
    grid: Tuple[int, int, int]  # (T, GH, GW)
    blocks: Tuple[int, int, int]  # (a_t, a_y, a_x): centres = a_t*a_y*a_x
    sigma_k: float
    sigma_q: float
    logit_std: float
    spatial_bias: bool
    # SparsePR hyper-parameters
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
    estimator: int = 0          # 0 ridge, 1 mean-only, 2 scalar affine, 3 diagonal affine
    # position in a sequence of calls (denoising steps) and the drift per step
    step: int = 0
    drift: float = 0.05
    # grouped-query attention: G query heads share each K/V head (H/G K/V heads)
    G: int = 1
    # 0 response-coupled partition (the method), 1 semantic reference partition
    partition: int = 0
    # 0 plain prefix budget, 1 budget calibrated toward the target density
    budget: int = 0

    @property
    def H_kv(self) -> int:
        return self.H // self.G

    @property
    def centres(self) -> int:
        a_t, a_y, a_x = self.blocks
        return a_t * a_y * a_x

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def params(self) -> Dict[str, object]:
        """SparsePR parameter set, in the C-ABI's field names."""
        return dict(H=self.H, N_q=self.N, N_k=self.N, d=self.d, dtype=self.dtype,
                    M_s=self.M_s, r_K=self.r_K, r_Q=self.r_Q, C_q=self.C_q,
                    C_k=self.C_k, M=self.M, r=self.r, lam=self.lam,
                    target_density=self.rho, kmeans_max_iter=self.kmeans_max_iter,
                    seed=self.seed, estimator=self.estimator, G=self.G, partition=self.partition,
                    budget=self.budget)


TINY = Workload("tiny-f32-1x1024x64", H=1, N=1024, d=64, dtype="f32",
                grid=(8, 8, 16), blocks=(2, 2, 4), sigma_k=0.3, sigma_q=0.5,
                logit_std=4.0, spatial_bias=False,
                M_s=64, r_K=8, r_Q=8, C_q=16, C_k=16, M=16, r=4, lam=0.1, rho=0.25)

MID = Workload("mid-bf16-12x16384x64", H=12, N=16384, d=64, dtype="bf16",
               grid=(16, 32, 32), blocks=(4, 4, 8), sigma_k=0.3, sigma_q=0.3,
               logit_std=4.0, spatial_bias=False,
               M_s=256, r_K=48, r_Q=64, C_q=128, C_k=128, M=64, r=16, lam=0.1, rho=0.22)

WAN = Workload("wan-bf16-40x75600x128", H=40, N=75600, d=128, dtype="bf16",
               grid=(21, 45, 80), blocks=(8, 8, 8), sigma_k=0.3, sigma_q=0.3,
               logit_std=5.0, spatial_bias=True,
               M_s=256, r_K=48, r_Q=64, C_q=512, C_k=512, M=64, r=16, lam=0.1, rho=0.22)

HUNYUAN = Workload("hunyuan-bf16-24x118800x128", H=24, N=118800, d=128, dtype="bf16",
                   grid=(33, 45, 80), blocks=(8, 8, 12), sigma_k=0.3, sigma_q=0.3,
                   logit_std=5.0, spatial_bias=False,
                   M_s=256, r_K=48, r_Q=64, C_q=768, C_k=768, M=64, r=16, lam=0.1, rho=0.26)

WORKLOADS: Dict[str, Workload] = {w.name: w for w in (TINY, MID, WAN, HUNYUAN)}
ALIASES = {"tiny": TINY.name, "mid": MID.name, "wan": WAN.name, "hunyuan": HUNYUAN.name}

# Operating-point sweep on the Wan-like shapes and data.
SWEEP_RHO = (0.12, 0.17, 0.22, 0.26, 0.35)
SWEEP_M = (32, 64, 128)


def get(name: str) -> Workload:
    return WORKLOADS[ALIASES.get(name, name)]


def sweep_points(base: Workload = WAN):
    return [base.with_(name=f"{base.name}-rho{int(round(rho * 100))}-M{m}", rho=rho, M=m)
            for rho in SWEEP_RHO for m in SWEEP_M]


# ----------------------------------------------------------------------------------
def _centre_ids(w: Workload) -> np.ndarray:
    T, GH, GW = w.grid
    a_t, a_y, a_x = w.blocks
    t = np.arange(T)[:, None, None]
    y = np.arange(GH)[None, :, None]
    x = np.arange(GW)[None, None, :]
    c = ((t * a_t) // T * a_y + (y * a_y) // GH) * a_x + (x * a_x) // GW
    return np.broadcast_to(c, (T, GH, GW)).reshape(-1).astype(np.int64)


def _position_features(w: Workload) -> np.ndarray:
    T, GH, GW = w.grid
    t = np.repeat(np.arange(T), GH * GW).astype(np.float64)
    y = np.tile(np.repeat(np.arange(GH), GW), T).astype(np.float64)
    x = np.tile(np.arange(GW), T * GH).astype(np.float64)
    return np.stack([np.sin(np.pi * t / T), np.cos(np.pi * t / T),
                     np.sin(2 * np.pi * y / GH), np.cos(2 * np.pi * y / GH),
                     np.sin(2 * np.pi * x / GW), np.cos(2 * np.pi * x / GW)], axis=1)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values once, to nearest-even, onto the bf16 grid (returned as fp64).

    Works on the fp64 bit pattern directly so there is no intermediate fp32 rounding.
    Values are assumed finite and inside bf16's normal range (true for these draws).
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    bits = x.view(np.uint64)
    shift = np.uint64(52 - 7)
    half = np.uint64(1) << (shift - np.uint64(1))
    lsb = (bits >> shift) & np.uint64(1)
    rounded = (bits + (half - np.uint64(1)) + lsb) & ~((np.uint64(1) << shift) - np.uint64(1))
    return rounded.view(np.float64)


def _round_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    if dtype == "bf16":
        return round_to_bf16(x)
    raise ValueError(dtype)


def make_head(w: Workload, h: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Q of query head ``h`` and K, V of its K/V head (``h // G``) as fp64 arrays holding
    exactly the stored (rounded) values."""
    if w.G > 1:
        qs, k, v = make_kv_group(w, h // w.G)
        return qs[h % w.G], k, v
    return _make_kv_head(w, h, 0)


def make_kv_group(w: Workload, hk: int):
    """GQA: the G query heads of K/V head ``hk`` (a list) and its K, V.  Query head 0 of
    the group is drawn exactly as a head of the G = 1 recipe; query head j > 0 draws its
    own noise (and nothing else) from the stream (hk, 2, j) and shares the group's
    mixture centres, positional bias and logit scale."""
    assert w.step == 0, "drifting sequences are drawn for G = 1 only"
    q0, k, v, extra = _make_kv_head(w, hk, w.G - 1)
    return [q0] + extra, k, v


def _make_kv_head(w: Workload, h: int, n_extra: int):
    N, d = w.N, w.d
    assert N == w.grid[0] * w.grid[1] * w.grid[2]
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(w.seed, spawn_key=(h,))))
    mu = rng.standard_normal((w.centres, d))
    cid = _centre_ids(w)
    base = mu[cid]
    K = base + w.sigma_k * rng.standard_normal((N, d))
    Q = base + w.sigma_q * rng.standard_normal((N, d))
    if w.spatial_bias:
        G = rng.standard_normal((6, d))
        bias = _position_features(w) @ G
        Q += bias
        K += bias
    V = rng.standard_normal((N, d))
    if w.step > 0:
        # drift along a sequence of calls: the mixture centres and the token noise move
        # by drift * step along fixed directions drawn from the head's second stream
        drng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(w.seed, spawn_key=(h, 1))))
        a = w.drift * w.step
        K += a * (drng.standard_normal((w.centres, d))[cid] + w.sigma_k * drng.standard_normal((N, d)))
        Q += a * (drng.standard_normal((w.centres, d))[cid] + w.sigma_q * drng.standard_normal((N, d)))
        V += a * drng.standard_normal((N, d))
    if N * N <= 65536 * 16:
        logits = (Q @ K.T) / math.sqrt(d)
        sigma_hat = float(np.std(logits))
    else:
        i = rng.integers(0, N, 65536)
        j = rng.integers(0, N, 65536)
        sigma_hat = float(np.std(np.einsum("nd,nd->n", Q[i], K[j]) / math.sqrt(d)))
    scale = math.sqrt(w.logit_std / sigma_hat)
    Q *= scale
    K *= scale
    out = (_round_storage(Q, w.dtype), _round_storage(K, w.dtype), _round_storage(V, w.dtype))
    if n_extra == 0:
        return out
    extra = []
    for j in range(1, n_extra + 1):
        erng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(w.seed, spawn_key=(h, 2, j))))
        Qj = base + w.sigma_q * erng.standard_normal((N, d))
        if w.spatial_bias:
            Qj += bias
        extra.append(_round_storage(Qj * scale, w.dtype))
    return out + (extra,)


def make_inputs_np(w: Workload, heads: Optional[list] = None):
    """Stacked fp64 [len(heads), N, d] arrays of the stored values (small workloads); with
    G > 1 (all heads only) Q is [H, N, d] and K, V are [H/G, N, d]."""
    if w.G > 1:
        assert heads is None
        groups = [make_kv_group(w, hk) for hk in range(w.H_kv)]
        return (np.stack([q for g in groups for q in g[0]]), np.stack([g[1] for g in groups]),
                np.stack([g[2] for g in groups]))
    heads = list(range(w.H)) if heads is None else list(heads)
    qs, ks, vs = zip(*(make_head(w, h) for h in heads))
    return np.stack(qs), np.stack(ks), np.stack(vs)


def torch_dtype(dtype: str):
    import torch
    return {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]


def make_inputs_torch(w: Workload, device="cpu", pin: bool = False):
    """Q, K, V as [H, N, d] torch tensors in the storage dtype (exact copies of make_head)."""
    import torch
    td = torch_dtype(w.dtype)
    out = []
    for i in range(3):
        t = torch.empty((w.H if i == 0 else w.H_kv, w.N, w.d), dtype=td, pin_memory=pin and device == "cpu")
        out.append(t)
    # the fp64 values are exactly representable in the storage dtype
    conv = lambda a: torch.from_numpy(a.astype(np.float32)).to(td)
    if w.G > 1:
        for hk in range(w.H_kv):
            qs, k, v = make_kv_group(w, hk)
            for j, q in enumerate(qs):
                out[0][hk * w.G + j].copy_(conv(q))
            out[1][hk].copy_(conv(k))
            out[2][hk].copy_(conv(v))
    else:
        for h in range(w.H):
            for t, a in zip(out, make_head(w, h)):
                t[h].copy_(conv(a))
    if device != "cpu":
        out = [t.to(device) for t in out]
    return tuple(out)
