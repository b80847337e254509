"""Algorithmic byte accounting for one decode step of one layer.

These are the bytes the method must move from HBM, not the dense work it
avoids: the predictors, the selected neurons' rows of W1 (and their b1 entries)
and W2, the selected heads' rows of W^Q, W^K, W^V and W^O, and the selected
heads' KV cache entries (read over slots 0..L, plus the new slot written).
Activations (O(B d) floats) are left out.

The KV term follows the per-token KV-cache size of the survey note ("KV cache"
subsection): 2 (K and V) x hidden x layers x bytes per element, hidden being
h * dh here.
"""

from __future__ import annotations

from dataclasses import dataclass

ELEM = {"bf16": 2, "f32": 4}


@dataclass
class LayerBytes:
    mlp_predictor: int
    head_predictor: int
    w1: int
    w2: int
    qkv: int
    wo: int
    kv: int

    @property
    def total(self) -> int:
        return (self.mlp_predictor + self.head_predictor + self.w1 + self.w2 + self.qkv + self.wo + self.kv)

    @property
    def mlp(self) -> int:
        return self.w1 + self.w2

    @property
    def attention(self) -> int:
        return self.qkv + self.wo + self.kv


def kv_bytes_per_token(hidden: int, layers: int, elem_bytes: int) -> int:
    """Bytes of K and V that one token adds to the cache over all layers."""
    return 2 * hidden * layers * elem_bytes


def layer_bytes(d, N, r, h, dh, k, k_eff, k_h, B, n_keys, wdtype="bf16", kvdtype="bf16",
                predictors=True) -> LayerBytes:
    """Bytes one layer-step moves.

    k      selected neurons (rows of W1 read, b1 entries gathered),
    k_eff  selected neurons with a nonzero activation in some row (rows of W2 read),
    k_h    selected heads, n_keys = L + 1 cache slots attended per head and row."""
    w, kv = ELEM[wdtype], ELEM[kvdtype]
    mlp_pred = (d * r + N * r) * w + N * 4 if predictors else 0
    head_pred = h * d * w if predictors else 0
    return LayerBytes(
        mlp_predictor=mlp_pred,
        head_predictor=head_pred,
        w1=k * d * w + k * 4,
        w2=k_eff * d * w,
        qkv=k_h * 3 * dh * d * w,
        wo=k_h * dh * d * w,
        kv=B * k_h * (n_keys * 2 * dh * kv + 2 * dh * kv),
    )


def dense_layer_param_bytes(d, N, h, dh, wdtype="bf16"):
    """Weight bytes of a dense layer: (MLP, attention)."""
    w = ELEM[wdtype]
    return 2 * N * d * w, 4 * h * dh * d * w
