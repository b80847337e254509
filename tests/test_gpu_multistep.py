"""Several decode steps with the KV position advancing, and exact KV
maintenance for the unselected heads, vs the oracle.

Each step appends the token's key and value at slot pos (itpub blog on KV
caching, figure (b)); the next step attends over slots 0..pos+1. Without
exact KV only the selected heads' slots are written; with it (layer param
exact_kv) every head's slot is, so a head left out at one step sees the true
key at a later step. Checked after every step: the selected sets bit-exact,
the stack output, and the whole written cache slot of every head.
"""

import numpy as np
import pytest
import torch

from oracle import dejavu_oracle as O
from tests._helpers import assert_kv_slot, assert_out, f64, oracle_layer, selected

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from attention_predictor_gemv_b200 import binding as bd
    from attention_predictor_gemv_b200 import workload as wl
    from attention_predictor_gemv_b200.stack import DecoderStack

DEV = "cuda"

SHAPES = {
    "ragged": dict(d=1032, N=1000, r=40, h=6, dh=128, L=99, cap=104, wdtype="bf16", kvdtype="bf16", p_active=0.2),
    "opt-like": dict(d=2048, N=8192, r=256, h=32, dh=64, L=512, cap=520, wdtype="bf16", kvdtype="bf16",
                     p_active=0.10),
    "fused128": dict(d=1024, N=4096, r=64, h=8, dh=128, L=300, cap=310, wdtype="bf16", kvdtype="bf16", p_active=0.15),
    "wide": dict(d=8192, N=12288, r=64, h=8, dh=128, L=200, cap=210, wdtype="bf16", kvdtype="bf16", p_active=0.10),
}


def _shape(name, B):
    return wl.LayerShape(B=B, **SHAPES[name])


def _assert_slot(cache_gpu, ref_slot):
    """Slot values within one bf16 rounding of the oracle's (assert_kv_slot)."""
    assert_kv_slot(f64(cache_gpu), ref_slot)


@pytest.mark.parametrize("name,B", [("fused128", 1), ("fused128", 2), ("wide", 1), ("ragged", 1), ("opt-like", 8)])
def test_exact_kv_writes_every_heads_slot(name, B):
    s = _shape(name, B)
    t = wl.make_layer(s, 81, DEV)
    x = wl.make_input(s, 82, DEV)
    k, k_h = wl.k_for(0.1, s.N), max(1, s.h // 4)
    L = bd.Layer(t, B, min(s.N, B * k), min(s.h, B * k_h))
    p = bd.params(k, k_h, 1.0 / np.sqrt(s.dh), exact_kv=True)
    ws = bd.workspace(bd.DV_OP_DECODE_LAYER, L.dims)
    f = dict(device=DEV, dtype=torch.float32)
    i = dict(device=DEV, dtype=torch.int32)
    tb = dict(yA=torch.empty(B, s.d, **f), scores_h=torch.empty(B, s.h, **f), head_idx=torch.zeros(s.h, **i),
              head_count=torch.zeros(1, **i), yM=torch.empty(B, s.d, **f), scores=torch.empty(B, s.N, **f),
              idx=torch.zeros(s.N, **i), count=torch.zeros(1, **i))
    x0 = x.clone()
    OL = oracle_layer(t)
    K0 = t["K"].clone()
    bd.dv_decode_layer(L, p, x, s.L, ws, trace=bd.layer_io(**tb))
    torch.cuda.synchronize()
    hsel = O.select(tb["scores_h"].cpu().numpy(), k=k_h)
    msel = O.select(tb["scores"].cpu().numpy(), k=k)
    assert np.array_equal(selected(tb["head_idx"], tb["head_count"]), hsel)
    assert len(hsel) < s.h  # some heads are unselected
    P = O.LayerParams(k=k, k_h=k_h, scale=1.0 / np.sqrt(s.dh), exact_kv=True)
    tr = O.decode_layer(f64(x0), OL, P, s.L, head_idx=hsel, idx=msel)
    assert_out((x - x0).cpu().numpy(), tr.x_out - f64(x0), "x_out - x")
    _assert_slot(t["K"][:, :, s.L], OL.K[:, :, s.L])
    _assert_slot(t["V"][:, :, s.L], OL.V[:, :, s.L])
    mask = torch.ones(s.cap, dtype=torch.bool)
    mask[s.L] = False
    assert torch.equal(t["K"][:, :, mask], K0[:, :, mask])
    assert bd.dv_read_device_status(ws) == 0


@pytest.mark.parametrize("name,B,exact", [("fused128", 1, False), ("fused128", 1, True), ("opt-like", 2, True),
                                          ("wide", 1, True), ("ragged", 1, True), ("opt-like", 8, True),
                                          ("opt-like", 8, False)])
def test_stack_over_several_steps(name, B, exact):
    """Three layers, look-ahead on, four tokens at positions L..L+3."""
    nL, steps = 3, 4
    s = _shape(name, B)
    layers = [wl.make_layer(s, 500 + l, DEV) for l in range(nL)]
    OLs = [oracle_layer(t) for t in layers]
    k, k_h = wl.k_for(0.1, s.N), 2
    stk = DecoderStack(layers, B, k, k_h, 1.0 / np.sqrt(s.dh), lookahead=True, exact_kv=exact)
    P = O.LayerParams(k=k, k_h=k_h, scale=1.0 / np.sqrt(s.dh), exact_kv=exact)
    x = wl.make_input(s, 83, DEV)
    xo = f64(x)
    for step in range(steps):
        pos = s.L + step
        stk.step(x, pos)
        torch.cuda.synchronize()
        sel = []
        for l in range(nL):
            hs = O.select(stk.scores_h[l].cpu().numpy(), k=k_h)
            ms = O.select(stk.scores[l].cpu().numpy(), k=k)
            assert np.array_equal(selected(stk.head_idx[l], stk.head_count[l]), hs), (step, l)
            assert np.array_equal(selected(stk.idx[l], stk.count[l]), ms), (step, l)
            sel.append((hs, ms))
        x_prev = xo
        xo, _ = O.decode_stack(x_prev, OLs, P, pos, lookahead=True, sel_override=sel)
        assert_out(x.cpu().numpy() - x_prev, xo - x_prev, f"step {step}")
        for l, t in enumerate(layers):
            _assert_slot(t["K"][:, :, pos], OLs[l].K[:, :, pos])
            _assert_slot(t["V"][:, :, pos], OLs[l].V[:, :, pos])
        x = torch.from_numpy(xo.astype(np.float32)).to(DEV)  # both sides continue from the oracle's output
    assert bd.dv_read_device_status(stk.ws_main) == 0
    assert bd.dv_read_device_status(stk.ws_side) == 0
