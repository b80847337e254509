"""The GeLU MLP variant (eq. (1) with sigma = GeLU, "ReLU or GeLU" in §2.3)
vs the oracle, on fixed neuron sets and through the layer call.

GeLU has no exact zeros, so nothing is compacted: every selected neuron's W2
row is read, and the result is compared with the oracle's eq. (1) on the same
set (the positive-set invariant of ReLU does not hold). Each kernel family
that forms the activations is reached: column-owner (d <= 6144), the
shared-memory ring kernels (d = 8192), the row kernels (batch 3-4), the
kernel-per-step path (d not a multiple of 64), and the tensor-core path
(batch 8-16).
"""

import numpy as np
import pytest
import torch

from oracle import dejavu_oracle as O
from tests._helpers import assert_out, f64, oracle_layer, selected

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from attention_predictor_gemv_b200 import binding as bd
    from attention_predictor_gemv_b200 import workload as wl

DEV = "cuda"

SHAPES = {
    "tiny": dict(d=256, N=1024, r=32, h=4, dh=64, L=64, cap=65, wdtype="f32", kvdtype="f32", p_active=0.10),
    "ragged": dict(d=1032, N=1000, r=40, h=6, dh=128, L=99, cap=100, wdtype="bf16", kvdtype="bf16", p_active=0.2),
    "opt-like": dict(d=2048, N=8192, r=256, h=32, dh=64, L=512, cap=520, wdtype="bf16", kvdtype="bf16",
                     p_active=0.10),
    "fused128": dict(d=1024, N=4096, r=64, h=8, dh=128, L=300, cap=310, wdtype="bf16", kvdtype="bf16", p_active=0.15),
    "wide": dict(d=8192, N=12288, r=64, h=8, dh=128, L=200, cap=210, wdtype="bf16", kvdtype="bf16", p_active=0.10),
}


def _shape(name, B):
    return wl.LayerShape(B=B, **SHAPES[name])


@pytest.mark.parametrize("name,B,k", [("tiny", 1, 128), ("ragged", 2, 300), ("opt-like", 1, 819), ("opt-like", 8, 900),
                                      ("ragged", 5, 77), ("opt-like", 16, 2000)])
def test_sparse_mlp_gelu(name, B, k):
    s = _shape(name, B)
    t = wl.make_layer(s, 71, DEV)
    y = wl.make_input(s, 72, DEV)
    S = np.sort(np.random.default_rng(73).choice(s.N, size=k, replace=False)).astype(np.int32)
    idx = torch.from_numpy(S).to(DEV)
    cnt = torch.tensor([k], dtype=torch.int32, device=DEV)
    b2 = torch.randn(s.d, device=DEV) * 0.1
    out = torch.empty(B, s.d, device=DEV)
    ws = bd.workspace(bd.DV_OP_SPARSE_MLP, bd.dims(B=B, d=s.d, N=s.N, k_max=k))
    bd.dv_sparse_mlp(y, t["W1t"], t["b1"], t["W2t"], b2, idx, cnt, k, out, ws, act=bd.DV_ACT_GELU)
    torch.cuda.synchronize()
    ref = O.sparse_mlp(f64(y), f64(t["W1t"]), f64(t["b1"]), f64(t["W2t"]), f64(b2), S, act="gelu")
    assert_out(out.cpu().numpy(), ref)
    # differs from the ReLU result (the activation is really applied)
    relu = O.sparse_mlp(f64(y), f64(t["W1t"]), f64(t["b1"]), f64(t["W2t"]), f64(b2), S)
    assert np.linalg.norm(ref - relu) > 0.05 * np.linalg.norm(ref - f64(b2))
    assert bd.dv_read_device_status(ws) == 0


@pytest.mark.parametrize("name,B", [("fused128", 1), ("fused128", 2), ("opt-like", 4), ("wide", 1), ("ragged", 1),
                                    ("opt-like", 8)])
def test_decode_layer_gelu(name, B):
    s = _shape(name, B)
    t = wl.make_layer(s, 74, DEV)
    x = wl.make_input(s, 75, DEV)
    k, k_h = wl.k_for(0.1, s.N), max(1, s.h // 4)
    L = bd.Layer(t, B, min(s.N, B * k), min(s.h, B * k_h))
    p = bd.params(k, k_h, 1.0 / np.sqrt(s.dh), act=bd.DV_ACT_GELU)
    ws = bd.workspace(bd.DV_OP_DECODE_LAYER, L.dims)
    f = dict(device=DEV, dtype=torch.float32)
    i = dict(device=DEV, dtype=torch.int32)
    tb = dict(yA=torch.empty(B, s.d, **f), scores_h=torch.empty(B, s.h, **f), head_idx=torch.zeros(s.h, **i),
              head_count=torch.zeros(1, **i), yM=torch.empty(B, s.d, **f), scores=torch.empty(B, s.N, **f),
              idx=torch.zeros(s.N, **i), count=torch.zeros(1, **i))
    x0 = x.clone()
    OL = oracle_layer(t)
    bd.dv_decode_layer(L, p, x, s.L, ws, trace=bd.layer_io(**tb))
    torch.cuda.synchronize()
    hsel = O.select(tb["scores_h"].cpu().numpy(), k=k_h)
    msel = O.select(tb["scores"].cpu().numpy(), k=k)
    assert np.array_equal(selected(tb["head_idx"], tb["head_count"]), hsel)
    assert np.array_equal(selected(tb["idx"], tb["count"]), msel)
    P = O.LayerParams(k=k, k_h=k_h, scale=1.0 / np.sqrt(s.dh), act="gelu")
    tr = O.decode_layer(f64(x0), OL, P, s.L, head_idx=hsel, idx=msel)
    assert_out((x - x0).cpu().numpy(), tr.x_out - f64(x0), "x_out - x")
    assert bd.dv_read_device_status(ws) == 0
