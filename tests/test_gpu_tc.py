"""Tensor-core gathered-row path (batch 5..16, and 3..4 for rows longer than
4096 bf16 elements; bf16 weights) vs the CPU oracle.

From five batch rows on (three for long rows), the layer and block calls run q/k/v, W1 (+ bias,
ReLU, compaction), W2 and W^O as tcgen05 MMAs over the gathered rows, with
the activations split into two bf16 halves. Same bar as every parity test:
index sets bit-exact, block outputs within relative L2 5e-3 and max-abs
2e-2 ||out||_inf, written KV slots within one bf16 rounding.

Shapes cover partial tiles (counts that are not multiples of 128 rows or 64
columns), d not a multiple of 64, empty sets, every neuron and head selected,
dh = 64 and 128, 5..16 batch rows, and the OPT-175B row length with KV 2048.
"""

import numpy as np
import pytest
import torch

from oracle import dejavu_oracle as O
from tests._helpers import assert_kv_slot, assert_out, assert_scores, f64, oracle_layer, selected

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from attention_predictor_gemv_b200 import binding as bd
    from attention_predictor_gemv_b200 import workload as wl
    from attention_predictor_gemv_b200.stack import DecoderStack

DEV = "cuda"

SHAPES = {
    "ragged": dict(d=1032, N=1000, r=40, h=6, dh=128, L=99, cap=100, p_active=0.2),
    "opt-like": dict(d=2048, N=8192, r=256, h=32, dh=64, L=512, cap=520, p_active=0.10),
    "wide": dict(d=8192, N=12288, r=64, h=8, dh=128, L=200, cap=210, p_active=0.10),
    "175b-slice": dict(d=12288, N=4096, r=64, h=8, dh=128, L=2048, cap=2056, p_active=0.05),
}


def _shape(name, B):
    return wl.LayerShape(B=B, wdtype="bf16", kvdtype="bf16", **SHAPES[name])


def _subset(n, k, seed):
    return np.sort(np.random.default_rng(seed).choice(n, size=k, replace=False)).astype(np.int32)


def _no_device_errors(ws):
    assert bd.dv_read_device_status(ws) == 0


@pytest.mark.parametrize("name,B,k", [("ragged", 5, 37), ("ragged", 8, 1000), ("opt-like", 8, 819),
                                      ("opt-like", 16, 4100), ("opt-like", 16, 8192), ("opt-like", 12, 129),
                                      ("wide", 16, 2000), ("175b-slice", 8, 3001), ("wide", 3, 1500),
                                      ("175b-slice", 4, 615)])
@pytest.mark.parametrize("with_b2", [False, True])
def test_tc_sparse_mlp(name, B, k, with_b2):
    s = _shape(name, B)
    t = wl.make_layer(s, 51, DEV)
    y = wl.make_input(s, 52, DEV)
    S = _subset(s.N, k, 53)
    k_max = min(s.N, k + 40)
    idx = torch.zeros(k_max, dtype=torch.int32, device=DEV)
    idx[:k] = torch.from_numpy(S).to(DEV)
    cnt = torch.tensor([k], dtype=torch.int32, device=DEV)
    b2 = torch.randn(s.d, device=DEV) * 0.1 if with_b2 else None
    out = torch.full((B, s.d), 5.0, device=DEV)
    D = bd.dims(B=B, d=s.d, N=s.N, k_max=k_max)
    ws = bd.workspace(bd.DV_OP_SPARSE_MLP, D)
    ref = O.sparse_mlp(f64(y), f64(t["W1t"]), f64(t["b1"]), f64(t["W2t"]), None if b2 is None else f64(b2), S)
    for _ in range(2):  # twice: per-tile counts and compacted rows are rewritten each call
        bd.dv_sparse_mlp(y, t["W1t"], t["b1"], t["W2t"], b2, idx, cnt, k_max, out, ws)
        torch.cuda.synchronize()
        assert_out(out.cpu().numpy(), ref)
    base = torch.randn(B, s.d, device=DEV)
    acc = base.clone()
    bd.dv_sparse_mlp(y, t["W1t"], t["b1"], t["W2t"], b2, idx, cnt, k_max, acc, ws, accumulate=True)
    torch.cuda.synchronize()
    assert_out((acc - base).cpu().numpy(), ref)
    _no_device_errors(ws)


def test_tc_sparse_mlp_empty_set_and_positive_set_equals_dense():
    s = _shape("opt-like", 8)
    t = wl.make_layer(s, 54, DEV)
    y = wl.make_input(s, 55, DEV)
    b2 = torch.randn(s.d, device=DEV)
    idx = torch.zeros(64, dtype=torch.int32, device=DEV)
    cnt = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = torch.full((8, s.d), 3.0, device=DEV)
    ws = bd.workspace(bd.DV_OP_SPARSE_MLP, bd.dims(B=8, d=s.d, N=s.N, k_max=64))
    bd.dv_sparse_mlp(y, t["W1t"], t["b1"], t["W2t"], b2, idx, cnt, 64, out, ws)
    torch.cuda.synchronize()
    assert torch.allclose(out, b2.expand(8, -1))
    # S_M = every neuron positive in some row reproduces the dense MLP (eq. (1) with ReLU)
    pre = O.mlp_preactivations(f64(y), f64(t["W1t"]), f64(t["b1"]))
    S = np.nonzero((pre > 0).any(axis=0))[0].astype(np.int32)
    dense = O.sparse_mlp(f64(y), f64(t["W1t"]), f64(t["b1"]), f64(t["W2t"]), None, np.arange(s.N))
    idx = torch.from_numpy(S).to(DEV)
    cnt = torch.tensor([len(S)], dtype=torch.int32, device=DEV)
    ws = bd.workspace(bd.DV_OP_SPARSE_MLP, bd.dims(B=8, d=s.d, N=s.N, k_max=len(S)))
    bd.dv_sparse_mlp(y, t["W1t"], t["b1"], t["W2t"], None, idx, cnt, len(S), out, ws)
    torch.cuda.synchronize()
    assert_out(out.cpu().numpy(), dense)
    _no_device_errors(ws)


@pytest.mark.parametrize("name,B,nsel", [("ragged", 5, 3), ("opt-like", 8, 8), ("opt-like", 16, 32),
                                          ("wide", 16, 5), ("175b-slice", 8, 7)])
def test_tc_sparse_mha(name, B, nsel):
    s = _shape(name, B)
    t = wl.make_layer(s, 56, DEV)
    y = wl.make_input(s, 57, DEV)
    heads = _subset(s.h, nsel, 58)
    kh_max = min(s.h, nsel + 1)
    hidx = torch.zeros(kh_max, dtype=torch.int32, device=DEV)
    hidx[:nsel] = torch.from_numpy(heads).to(DEV)
    hcnt = torch.tensor([nsel], dtype=torch.int32, device=DEV)
    bO = torch.randn(s.d, device=DEV) * 0.05
    bqkv = torch.randn(s.h, 3, s.dh, device=DEV) * 0.05
    K0, V0 = t["K"].clone(), t["V"].clone()
    out = torch.empty(B, s.d, device=DEV)
    ws = bd.workspace(bd.DV_OP_SPARSE_MHA, bd.dims(B=B, d=s.d, N=1, h=s.h, dh=s.dh, cap=s.cap, kh_max=kh_max))
    pos = s.L
    scale = 1.0 / np.sqrt(s.dh)
    bd.dv_sparse_mha(y, t["Wqkv"], bqkv, t["WOt"], bO, t["K"], t["V"], pos, scale, hidx, hcnt, kh_max, out, ws)
    torch.cuda.synchronize()
    ref = O.sparse_mha(f64(y), f64(t["Wqkv"]), f64(bqkv), f64(t["WOt"]), f64(bO), f64(K0), f64(V0), pos, scale,
                       heads, "bf16")
    assert_out(out.cpu().numpy(), ref.out)
    for b in range(B):
        for p, i in enumerate(heads):
            for cache, r in ((t["K"], ref.k_new), (t["V"], ref.v_new)):
                got = f64(cache[b, i, pos])
                assert_kv_slot(got, r[b, p])
    untouched = [i for i in range(s.h) if i not in set(heads.tolist())]
    assert torch.equal(t["K"][:, untouched], K0[:, untouched])
    _no_device_errors(ws)


def _trace_bufs(s):
    f = dict(device=DEV, dtype=torch.float32)
    i = dict(device=DEV, dtype=torch.int32)
    return dict(yA=torch.empty(s.B, s.d, **f), scores_h=torch.empty(s.B, s.h, **f), head_idx=torch.zeros(s.h, **i),
                head_count=torch.zeros(1, **i), yM=torch.empty(s.B, s.d, **f), scores=torch.empty(s.B, s.N, **f),
                idx=torch.zeros(s.N, **i), count=torch.zeros(1, **i))


@pytest.mark.parametrize("name,B,kf,khf", [("opt-like", 8, 0.10, 0.25), ("opt-like", 16, 0.05, 0.25),
                                          ("ragged", 6, 0.2, 0.34), ("wide", 8, 0.1, 0.25),
                                          ("175b-slice", 16, 0.15, 0.25), ("opt-like", 16, 1.0, 1.0),
                                          ("wide", 4, 0.1, 0.25), ("175b-slice", 3, 0.15, 0.25)])
def test_tc_decode_layer(name, B, kf, khf):
    s = _shape(name, B)
    t = wl.make_layer(s, 61, DEV)
    t["ln1_g"] = 1.0 + 0.1 * torch.randn(s.d, device=DEV)
    t["ln2_b"] = 0.1 * torch.randn(s.d, device=DEV)
    x = wl.make_input(s, 62, DEV) * 1.5 + 0.25
    k, k_h = max(1, wl.k_for(kf, s.N)), max(1, wl.k_for(khf, s.h))
    L = bd.Layer(t, B, min(s.N, B * k), min(s.h, B * k_h))
    p = bd.params(k, k_h, 1.0 / np.sqrt(s.dh))
    ws = bd.workspace(bd.DV_OP_DECODE_LAYER, L.dims)
    tb = _trace_bufs(s)
    x0 = x.clone()
    OL = oracle_layer(t)
    bd.dv_decode_layer(L, p, x, s.L, ws, trace=bd.layer_io(**tb))
    torch.cuda.synchronize()
    P = O.LayerParams(k=k, k_h=k_h, scale=1.0 / np.sqrt(s.dh))
    sh, sm = tb["scores_h"].cpu().numpy(), tb["scores"].cpu().numpy()
    hsel, msel = O.select(sh, k=k_h), O.select(sm, k=k)
    assert np.array_equal(selected(tb["head_idx"], tb["head_count"]), hsel)
    assert np.array_equal(selected(tb["idx"], tb["count"]), msel)
    tr = O.decode_layer(f64(x0), OL, P, s.L, head_idx=hsel, idx=msel)
    assert_out(tb["yA"].cpu().numpy(), tr.yA, "yA")
    assert_scores(sh, O.head_predictor_scores(f64(tb["yA"]), OL.PA))
    assert_out(tb["yM"].cpu().numpy(), tr.yM, "yM")
    assert_scores(sm, O.mlp_predictor_scores(f64(tb["yM"]), OL.At, OL.Bm, OL.b1))
    assert_out((x - x0).cpu().numpy(), tr.x_out - f64(x0), "x_out - x")
    _no_device_errors(ws)


@pytest.mark.parametrize("name,B", [("opt-like", 8), ("opt-like", 16), ("wide", 12)])
def test_tc_lookahead_stack_and_graph_replay(name, B):
    """Three layers with the look-ahead predictor at batch 8-16 (union sets),
    eager, then the same step replayed from a CUDA graph."""
    nL = 3
    s = _shape(name, B)
    layers = [wl.make_layer(s, 400 + l, DEV) for l in range(nL)]
    K0 = [(t["K"].clone(), t["V"].clone()) for t in layers]
    k, k_h = wl.k_for(0.1, s.N), 2
    stk = DecoderStack(layers, B, k, k_h, 1.0 / np.sqrt(s.dh), lookahead=True)
    x = wl.make_input(s, 63, DEV)
    xin = x.clone()
    stk.step(x, s.L)
    torch.cuda.synchronize()
    OLs = []
    for l, t in enumerate(layers):
        OL = oracle_layer(t)
        OL.K, OL.V = f64(K0[l][0]), f64(K0[l][1])
        OLs.append(OL)
    P = O.LayerParams(k=k, k_h=k_h, scale=1.0 / np.sqrt(s.dh))
    sel = []
    for l in range(nL):
        sh, sm = stk.scores_h[l].cpu().numpy(), stk.scores[l].cpu().numpy()
        hs, ms = O.select(sh, k=k_h), O.select(sm, k=k)
        assert np.array_equal(selected(stk.head_idx[l], stk.head_count[l]), hs), l
        assert np.array_equal(selected(stk.idx[l], stk.count[l]), ms), l
        sel.append((hs, ms))
    x0 = f64(xin)
    xo, _ = O.decode_stack(x0, OLs, P, s.L, lookahead=True, sel_override=sel)
    assert_out(x.cpu().numpy() - x0, xo - x0)
    eager = x.clone()
    # the same step from a CUDA graph, from the same start state
    for (Kc, Vc), t in zip(K0, layers):
        t["K"].copy_(Kc)
        t["V"].copy_(Vc)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            stk.step(x, s.L)
    torch.cuda.current_stream().wait_stream(side)
    x.copy_(xin)
    g.replay()
    torch.cuda.synchronize()
    assert_out((x - xin).cpu().numpy(), (eager - xin).cpu().numpy())
    _no_device_errors(stk.ws_main)
    _no_device_errors(stk.ws_side)
    del g


@pytest.mark.parametrize("name,B", [("opt-like", 8), ("opt-like", 16), ("175b-slice", 4)])
def test_tc_stack_is_bitwise_reproducible(name, B):
    """The tensor-core layer path sums its partials in a fixed order (split-K
    parts in part order, W2 / W^O groups as exact fixed-point integers, the
    attention splits in split order), so two runs of the same step from the
    same state give the same bits: outputs, scores, selected sets and the
    appended KV slots. Without that, a score within rounding of the top-k
    boundary could select a different neuron on a rerun."""
    nL = 3
    s = _shape(name, B)
    layers = [wl.make_layer(s, 700 + l, DEV) for l in range(nL)]
    K0 = [(t["K"].clone(), t["V"].clone()) for t in layers]
    k, k_h = wl.k_for(0.1, s.N), 2
    stk = DecoderStack(layers, B, k, k_h, 1.0 / np.sqrt(s.dh), lookahead=True)
    xin = wl.make_input(s, 71, DEV)
    runs = []
    for _ in range(2):
        for (Kc, Vc), t in zip(K0, layers):
            t["K"].copy_(Kc)
            t["V"].copy_(Vc)
        x = xin.clone()
        stk.step(x, s.L)
        torch.cuda.synchronize()
        runs.append(dict(x=x.clone(), sm=[v.clone() for v in stk.scores], sh=[v.clone() for v in stk.scores_h],
                         idx=[selected(stk.idx[l], stk.count[l]) for l in range(nL)],
                         K=[t["K"][:, :, s.L].clone() for t in layers]))
    a, b = runs
    assert torch.equal(a["x"], b["x"])
    for l in range(nL):
        assert torch.equal(a["sm"][l], b["sm"][l]), l
        assert torch.equal(a["sh"][l], b["sh"][l]), l
        assert np.array_equal(a["idx"][l], b["idx"][l]), l
        assert torch.equal(a["K"][l], b["K"][l]), l
    _no_device_errors(stk.ws_main)
