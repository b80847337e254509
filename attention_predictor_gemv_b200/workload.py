"""Seeded synthetic inputs shared by the tests, the bench and the oracle callers.

This module draws random numbers and shapes them into the layouts the library
takes; it holds none of the method's arithmetic (no predictor evaluation, no
selection, no MLP or attention). It imports neither the CUDA binding nor the
oracle.

Workload recipe (OPT-shaped layers; the models and datasets the pages measure
on are not used, these stand in for them):

* W1, W2 ~ N(0, 1/d), stored neuron-major (row i is column W1_i / W2_i).
* b1 is shifted so a fraction p of the preactivations y W1_i + b1_i is positive
  for y ~ N(0, 1): b1_i = -Phi^{-1}(1 - p) ||W1_i||_2.
* MLP predictor: the rank-r truncated SVD of W1 (of its stored values),
  A = U_r Sigma_r (stored transposed, At[r][d]) and B = V_r (Bm[N][r]).
* Head predictor P_A[h][d] ~ N(0, 1/d).
* Wqkv[h][3][dh][d], WOt[h][dh][d] ~ N(0, 1/d); attention biases zero (absent).
* KV caches [B][h][cap][dh] ~ N(0, 1), every slot pre-filled.
* Layer input x ~ N(0, 1).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, replace
from statistics import NormalDist
from typing import Dict, Optional

import torch


@dataclass(frozen=True)
class LayerShape:
    d: int  # model dim
    N: int  # MLP neurons (4d)
    r: int  # predictor rank
    h: int  # heads
    dh: int  # head dim
    L: int  # KV entries before the decode step
    cap: int  # KV slots allocated
    B: int = 1  # batch rows
    wdtype: str = "bf16"  # weights: 'bf16' or 'f32'
    kvdtype: str = "bf16"
    p_active: float = 0.10  # fraction of positive preactivations
    layers: int = 1

    def with_(self, **kw) -> "LayerShape":
        return replace(self, **kw)


def round_half_up(x: float) -> int:
    return int(math.floor(x + 0.5))


def k_for(fraction: float, n: int) -> int:
    return max(0, min(n, round_half_up(fraction * n)))


# Shapes of the synthetic workloads (OPT-shaped; random init).
CONFIGS: Dict[str, LayerShape] = {
    "tiny": LayerShape(d=256, N=1024, r=32, h=4, dh=64, L=64, cap=65, wdtype="f32", kvdtype="f32", p_active=0.10),
    "opt-1.3b": LayerShape(d=2048, N=8192, r=256, h=32, dh=64, L=512, cap=520, p_active=0.10, layers=24),
    "opt-6.7b": LayerShape(d=4096, N=16384, r=512, h=32, dh=128, L=2048, cap=2176, p_active=0.08, layers=32),
    "opt-66b": LayerShape(d=9216, N=36864, r=1024, h=72, dh=128, L=1024, cap=1032, p_active=0.06, layers=64),
    "opt-175b": LayerShape(d=12288, N=49152, r=1024, h=96, dh=128, L=2048, cap=2056, p_active=0.05, layers=24),
}

# Selection sizes per workload (k neurons, k_h heads) at the default operating point.
DEFAULT_SELECTION = {
    "tiny": (128, 2),
    "opt-1.3b": (k_for(0.10, 8192), k_for(0.25, 32)),
    "opt-6.7b": (k_for(0.08, 16384), k_for(0.20, 32)),
    "opt-66b": (k_for(0.06, 36864), k_for(0.20, 72)),
    "opt-175b": (k_for(0.15, 49152), k_for(0.15, 96)),
}


def _dt(name: str):
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(shape, g, device, std=1.0, dtype=torch.float32):
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def make_layer(shape: LayerShape, seed: int, device="cpu", with_predictor=True) -> Dict[str, torch.Tensor]:
    """All tensors of one layer (weights, predictors, KV caches)."""
    g = _gen(seed, device)
    wdt, kvdt = _dt(shape.wdtype), _dt(shape.kvdtype)
    d, N, r, h, dh = shape.d, shape.N, shape.r, shape.h, shape.dh
    s = 1.0 / math.sqrt(d)
    t: Dict[str, torch.Tensor] = {}
    t["W1t"] = _randn((N, d), g, device, s, wdt)
    t["W2t"] = _randn((N, d), g, device, s, wdt)
    t["PA"] = _randn((h, d), g, device, s, wdt)
    t["Wqkv"] = _randn((h, 3, dh, d), g, device, s, wdt)
    t["WOt"] = _randn((h, dh, d), g, device, s, wdt)
    t["K"] = _randn((shape.B, h, shape.cap, dh), g, device, 1.0, kvdt)
    t["V"] = _randn((shape.B, h, shape.cap, dh), g, device, 1.0, kvdt)
    W1f = t["W1t"].float()
    shift = NormalDist().inv_cdf(1.0 - shape.p_active)
    t["b1"] = (-shift * W1f.norm(dim=1)).contiguous()  # fp32 [N]
    if with_predictor:
        devs = [torch.device(device)] if torch.device(device).type == "cuda" else []
        with torch.random.fork_rng(devices=devs):  # the randomized SVD draws from the global generator
            torch.manual_seed(int(seed) + 104729)
            if devs:
                torch.cuda.manual_seed(int(seed) + 104729)
            At, Bm = svd_predictor(W1f, r)
        t["At"] = At.to(wdt).contiguous()
        t["Bm"] = Bm.to(wdt).contiguous()
    return t


def svd_predictor(W1t_f32: torch.Tensor, r: int):
    """Rank-r truncated SVD of W1 = W1t^T (d x N): W1 ~ U_r S_r V_r^T.
    Returns At = (U_r S_r)^T [r][d] and Bm = V_r [N][r]."""
    W1 = W1t_f32.t()  # d x N
    d, N = W1.shape
    if r < min(d, N) // 2:
        U, S, V = torch.svd_lowrank(W1, q=min(r + 32, min(d, N)), niter=3)
        U, S, V = U[:, :r], S[:r], V[:, :r]
    else:
        U, S, Vh = torch.linalg.svd(W1.double(), full_matrices=False)
        U, S, V = U[:, :r].float(), S[:r].float(), Vh[:r].t().float()
    At = (U * S).t()
    return At, V


def make_input(shape: LayerShape, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed + 7919, device)
    return torch.randn(shape.B, shape.d, generator=g, device=device, dtype=torch.float32)


def make_kv(shape: LayerShape, B: int, seed: int, device="cpu"):
    """KV caches [B][h][cap][dh] ~ N(0, 1) for batch B (the same recipe as
    make_layer's caches), for running one set of weights at several batches."""
    g = _gen(seed + 15485863, device)
    kvdt = _dt(shape.kvdtype)
    K = _randn((B, shape.h, shape.cap, shape.dh), g, device, 1.0, kvdt)
    V = _randn((B, shape.h, shape.cap, shape.dh), g, device, 1.0, kvdt)
    return K, V


def quantize_rows(W: torch.Tensor):
    """Weight-only int8 encoding of a weight tensor whose rows run along the
    last axis: one fp32 scale per row, s = max |W_row| / 127 (1 for an all-zero
    row), q = round(W / s) clamped to [-127, 127]. Returns (q int8, s fp32)
    with s shaped like W without its last axis. The decode path reads q and s;
    the real row it stands for is q * s."""
    Wf = W.float()
    s = Wf.abs().amax(dim=-1) / 127.0
    s = torch.where(s > 0, s, torch.ones_like(s))
    q = torch.clamp(torch.round(Wf / s.unsqueeze(-1)), -127, 127).to(torch.int8)
    return q.contiguous(), s.contiguous()


def quantize_layer(t: Dict[str, torch.Tensor]) -> Dict[str, torch.Tensor]:
    """int8 + row-scale versions of a layer's gathered weights (W1t, W2t,
    Wqkv, WOt) under the keys W1q/W1s, W2q/W2s, Wqkvq/Wqkv_s, WOq/WO_s."""
    out = {}
    for name, qn, sn in (("W1t", "W1q", "W1s"), ("W2t", "W2q", "W2s"), ("Wqkv", "Wqkvq", "Wqkv_s"),
                         ("WOt", "WOq", "WO_s")):
        out[qn], out[sn] = quantize_rows(t[name])
    return out
