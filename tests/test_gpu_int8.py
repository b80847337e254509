"""Weight-only int8 gathered rows (one fp32 scale per row) vs the oracle.

The oracle decodes the same int8 rows and scales exactly (q * s in float64)
and evaluates eq. (1) / eq. (2) on them; the GPU reads half the bytes of the
bf16 rows. Same tolerances as the bf16 paths; KV slots within one bf16
rounding.
"""

import numpy as np
import pytest
import torch

from oracle import dejavu_oracle as O
from tests._helpers import assert_kv_slot, assert_out, f64

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from attention_predictor_gemv_b200 import binding as bd
    from attention_predictor_gemv_b200 import workload as wl

DEV = "cuda"

SHAPES = {
    "d1040": dict(d=1040, N=1000, r=40, h=6, dh=128, L=99, cap=100, p_active=0.2),
    "opt-like": dict(d=2048, N=8192, r=256, h=32, dh=64, L=512, cap=520, p_active=0.10),
    "175b-slice": dict(d=12288, N=4096, r=64, h=8, dh=128, L=2048, cap=2056, p_active=0.05),
}


def _setup(name, B, seed):
    s = wl.LayerShape(B=B, wdtype="bf16", kvdtype="bf16", **SHAPES[name])
    t = wl.make_layer(s, seed, DEV)
    t.update(wl.quantize_layer(t))
    return s, t


def _deq(t, q, sc):
    return O.dequantize_rows(t[q].cpu().numpy(), t[sc].cpu().numpy())


@pytest.mark.parametrize("name,B,k,act", [("d1040", 1, 300, "relu"), ("opt-like", 1, 819, "relu"),
                                          ("opt-like", 2, 1638, "gelu"), ("opt-like", 4, 900, "relu"),
                                          ("175b-slice", 1, 615, "relu"), ("175b-slice", 2, 615, "gelu")])
def test_sparse_mlp_q8(name, B, k, act):
    s, t = _setup(name, B, 91)
    y = wl.make_input(s, 92, DEV)
    S = np.sort(np.random.default_rng(93).choice(s.N, size=k, replace=False)).astype(np.int32)
    idx = torch.from_numpy(S).to(DEV)
    cnt = torch.tensor([k], dtype=torch.int32, device=DEV)
    b2 = torch.randn(s.d, device=DEV) * 0.1
    out = torch.full((B, s.d), 2.0, device=DEV)
    ws = bd.workspace(bd.DV_OP_SPARSE_MLP, bd.dims(B=B, d=s.d, N=s.N, k_max=k))
    a = bd.DV_ACT_GELU if act == "gelu" else bd.DV_ACT_RELU
    bd.dv_sparse_mlp_q8(y, t["W1q"], t["W1s"], t["b1"], t["W2q"], t["W2s"], b2, idx, cnt, k, out, ws, act=a)
    torch.cuda.synchronize()
    ref = O.sparse_mlp(f64(y), _deq(t, "W1q", "W1s"), f64(t["b1"]), _deq(t, "W2q", "W2s"), f64(b2), S, act=act)
    assert_out(out.cpu().numpy(), ref)
    base = torch.randn(B, s.d, device=DEV)
    acc = base.clone()
    bd.dv_sparse_mlp_q8(y, t["W1q"], t["W1s"], t["b1"], t["W2q"], t["W2s"], b2, idx, cnt, k, acc, ws, accumulate=True,
                        act=a)
    torch.cuda.synchronize()
    assert_out((acc - base).cpu().numpy(), ref)
    assert bd.dv_read_device_status(ws) == 0


@pytest.mark.parametrize("name,B,nsel", [("opt-like", 1, 8), ("opt-like", 3, 5), ("175b-slice", 2, 3),
                                          ("d1040", 1, 4)])
def test_sparse_mha_q8(name, B, nsel):
    s, t = _setup(name, B, 94)
    y = wl.make_input(s, 95, DEV)
    heads = np.sort(np.random.default_rng(96).choice(s.h, size=nsel, replace=False)).astype(np.int32)
    hidx = torch.from_numpy(heads).to(DEV)
    hcnt = torch.tensor([nsel], dtype=torch.int32, device=DEV)
    bO = torch.randn(s.d, device=DEV) * 0.05
    K0, V0 = t["K"].clone(), t["V"].clone()
    out = torch.empty(B, s.d, device=DEV)
    ws = bd.workspace(bd.DV_OP_SPARSE_MHA, bd.dims(B=B, d=s.d, N=1, h=s.h, dh=s.dh, cap=s.cap, kh_max=nsel))
    pos, scale = s.L, 1.0 / np.sqrt(s.dh)
    bd.dv_sparse_mha_q8(y, t["Wqkvq"], t["Wqkv_s"], None, t["WOq"], t["WO_s"], bO, t["K"], t["V"], pos, scale, hidx,
                        hcnt, nsel, out, ws)
    torch.cuda.synchronize()
    ref = O.sparse_mha(f64(y), _deq(t, "Wqkvq", "Wqkv_s"), None, _deq(t, "WOq", "WO_s"), f64(bO), f64(K0), f64(V0),
                       pos, scale, heads, "bf16")
    assert_out(out.cpu().numpy(), ref.out)
    for b in range(B):
        for p, i in enumerate(heads):
            for cache, r in ((t["K"], ref.k_new), (t["V"], ref.v_new)):
                got = f64(cache[b, i, pos])
                assert_kv_slot(got, r[b, p])
    assert bd.dv_read_device_status(ws) == 0


def test_q8_rejects_unsupported_shapes():
    s, t = _setup("opt-like", 5, 97)
    y = wl.make_input(s, 98, DEV)
    idx = torch.arange(10, dtype=torch.int32, device=DEV)
    cnt = torch.tensor([10], dtype=torch.int32, device=DEV)
    out = torch.empty(5, s.d, device=DEV)
    ws = bd.workspace(bd.DV_OP_SPARSE_MLP, bd.dims(B=5, d=s.d, N=s.N, k_max=10))
    with pytest.raises(bd.DvError) as e:  # batch 5
        bd.dv_sparse_mlp_q8(y, t["W1q"], t["W1s"], t["b1"], t["W2q"], t["W2s"], None, idx, cnt, 10, out, ws)
    assert e.value.status == bd.DV_ERR_UNSUPPORTED
