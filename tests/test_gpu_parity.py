"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Index sets must match bit for bit (the oracle's selection applied to the
scores the GPU emitted); predictor scores within 1e-3 (max-abs relative to
||s||_inf and relative L2); block outputs within relative L2 5e-3 and max-abs
2e-2 ||out||_inf. Shapes span several tiles with ragged tails.
"""

import numpy as np
import pytest
import torch

from oracle import dejavu_oracle as O
from tests._helpers import assert_kv_slot, assert_out, assert_scores, f64, oracle_layer, selected, wname

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from attention_predictor_gemv_b200 import binding as bd
    from attention_predictor_gemv_b200 import workload as wl
    from attention_predictor_gemv_b200.stack import DecoderStack

DEV = "cuda"

# small shapes: the tiny fp32 config, a ragged bf16 shape (d not a multiple
# of the 1024-column tile, N not a multiple of 32, r short), dh = 128
SHAPES = {
    "tiny": dict(d=256, N=1024, r=32, h=4, dh=64, L=64, cap=65, wdtype="f32", kvdtype="f32", p_active=0.10),
    "ragged": dict(d=1032, N=1000, r=40, h=6, dh=128, L=99, cap=100, wdtype="bf16", kvdtype="bf16", p_active=0.2),
    "opt-like": dict(d=2048, N=8192, r=256, h=32, dh=64, L=512, cap=520, wdtype="bf16", kvdtype="bf16",
                     p_active=0.10),
    # dh = 128, a key count that does not split evenly over the attention cluster
    "fused128": dict(d=1024, N=4096, r=64, h=8, dh=128, L=300, cap=310, wdtype="bf16", kvdtype="bf16",
                     p_active=0.15),
    # rows of 16 KB (bf16, d = 8192): the shared-memory ring kernels
    "wide": dict(d=8192, N=12288, r=64, h=8, dh=128, L=200, cap=210, wdtype="bf16", kvdtype="bf16",
                 p_active=0.10),
}
# "ragged" runs the kernel-per-step layer path (d is not a multiple of the
# W^O column slices); the other shapes run the fused layer kernels.


def shape(name, B=1, **kw):
    s = wl.LayerShape(B=B, **SHAPES[name])
    return s.with_(**kw) if kw else s


def layer(name, B=1, seed=0, **kw):
    s = shape(name, B, **kw)
    return s, wl.make_layer(s, seed, DEV)


def ws_for(op, s, k_max=None, kh_max=None):
    D = bd.dims(B=s.B, d=s.d, N=s.N, r=s.r, h=s.h, dh=s.dh, cap=s.cap,
                k_max=s.N if k_max is None else k_max, kh_max=s.h if kh_max is None else kh_max)
    return bd.workspace(op, D)


def no_device_errors(ws):
    assert bd.dv_read_device_status(ws) == 0


# ---------------------------------------------------------------------------
# predictors and selection
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("name,B,mode", [("tiny", 1, "topk"), ("ragged", 3, "topk"), ("opt-like", 1, "topk"),
                                         ("ragged", 2, "threshold"), ("opt-like", 4, "topk")])
def test_predict_mlp(name, B, mode):
    s, t = layer(name, B, seed=1)
    y = wl.make_input(s, 11, DEV)
    k = wl.k_for(0.1, s.N)
    scores = torch.empty(B, s.N, device=DEV)
    idx = torch.full((s.N,), -1, dtype=torch.int32, device=DEV)
    count = torch.zeros(1, dtype=torch.int32, device=DEV)
    ws = ws_for(bd.DV_OP_PREDICT_MLP, s)
    m = bd.DV_TOPK if mode == "topk" else bd.DV_THRESHOLD
    bd.dv_predict_mlp(y, t["At"], t["Bm"], t["b1"], k, scores, idx, count, ws, tau=0.0, mode=m)
    torch.cuda.synchronize()
    ref = O.mlp_predictor_scores(f64(y), f64(t["At"]), f64(t["Bm"]), f64(t["b1"]))
    got = scores.cpu().numpy()
    assert_scores(got, ref)
    want = O.select(got, k=k, tau=0.0, mode=mode)
    assert np.array_equal(selected(idx, count), want)
    no_device_errors(ws)


@pytest.mark.parametrize("name,B", [("tiny", 1), ("ragged", 2), ("opt-like", 1)])
def test_predict_heads(name, B):
    s, t = layer(name, B, seed=2)
    y = wl.make_input(s, 12, DEV)
    k_h = max(1, s.h // 4)
    scores = torch.empty(B, s.h, device=DEV)
    hidx = torch.full((s.h,), -1, dtype=torch.int32, device=DEV)
    hcnt = torch.zeros(1, dtype=torch.int32, device=DEV)
    ws = ws_for(bd.DV_OP_PREDICT_HEADS, s)
    bd.dv_predict_heads(y, t["PA"], k_h, scores, hidx, hcnt, ws)
    torch.cuda.synchronize()
    got = scores.cpu().numpy()
    assert_scores(got, O.head_predictor_scores(f64(y), f64(t["PA"])))
    assert np.array_equal(selected(hidx, hcnt), O.select(got, k=k_h))


def _topk_gpu(scores_np, k, mode="topk", tau=0.0):
    B, n = scores_np.shape
    sc = torch.from_numpy(np.ascontiguousarray(scores_np, dtype=np.float32)).to(DEV)
    idx = torch.full((n,), -1, dtype=torch.int32, device=DEV)
    cnt = torch.zeros(1, dtype=torch.int32, device=DEV)
    ws = bd.workspace(bd.DV_OP_TOPK, bd.dims(B=B, N=n, k_max=min(n, max(k, 0))))
    bd.dv_topk(sc, k, idx, cnt, ws, tau=tau, mode=bd.DV_TOPK if mode == "topk" else bd.DV_THRESHOLD)
    torch.cuda.synchronize()
    return selected(idx, cnt)


@pytest.mark.parametrize("case", ["random", "ties", "signed_zeros", "nan", "inf", "constant"])
@pytest.mark.parametrize("n", [1, 31, 1000, 8192, 49152, 60001])
def test_topk_edge_cases(case, n):
    r = np.random.default_rng(n)
    if case == "random":
        s = r.standard_normal((1, n))
    elif case == "ties":
        s = r.integers(-4, 5, size=(1, n)).astype(np.float64)
    elif case == "signed_zeros":
        s = np.where(r.random((1, n)) < 0.5, -0.0, 0.0)
        s[:, ::9] = 0.5
    elif case == "nan":
        s = r.standard_normal((1, n))
        s[r.random((1, n)) < 0.2] = np.nan
    elif case == "inf":
        s = r.standard_normal((1, n))
        s[:, ::7] = -np.inf
        s[:, ::11] = np.inf
    else:
        s = np.full((1, n), 3.0)
    s = s.astype(np.float32)
    for k in sorted({0, 1, n // 3, n - 1, n, n + 5}):
        assert np.array_equal(_topk_gpu(s, k), O.select(s, k=k)), (case, n, k)


def test_topk_batch_union_and_threshold():
    r = np.random.default_rng(5)
    s = r.standard_normal((7, 5000)).astype(np.float32)
    s[3, :100] = np.nan
    for k in (0, 1, 37, 700, 5000):
        assert np.array_equal(_topk_gpu(s, k), O.select(s, k=k))
    for tau in (-0.5, 0.0, 1.3, 10.0):
        assert np.array_equal(_topk_gpu(s, 0, "threshold", tau), O.select(s, mode="threshold", tau=tau))


def test_selection_is_deterministic():
    s, t = layer("opt-like", 2, seed=3)
    y = wl.make_input(s, 13, DEV)
    outs = []
    for _ in range(5):
        scores = torch.empty(2, s.N, device=DEV)
        idx = torch.zeros(s.N, dtype=torch.int32, device=DEV)
        cnt = torch.zeros(1, dtype=torch.int32, device=DEV)
        ws = ws_for(bd.DV_OP_PREDICT_MLP, s)
        bd.dv_predict_mlp(y, t["At"], t["Bm"], t["b1"], 819, scores, idx, cnt, ws)
        torch.cuda.synchronize()
        outs.append((scores.cpu().numpy().tobytes(), selected(idx, cnt).tobytes()))
    assert all(o == outs[0] for o in outs)


# ---------------------------------------------------------------------------
# eq. (1): sparse MLP
# ---------------------------------------------------------------------------


def _subset(N, k, seed):
    r = np.random.default_rng(seed)
    return np.sort(r.choice(N, size=k, replace=False)).astype(np.int32)


@pytest.mark.parametrize("name,B,frac", [("tiny", 1, 0.125), ("tiny", 1, 1.0), ("ragged", 1, 0.3), ("ragged", 5, 0.05),
                                         ("opt-like", 1, 0.1), ("opt-like", 2, 0.2), ("opt-like", 16, 0.05)])
@pytest.mark.parametrize("with_b2", [False, True])
def test_sparse_mlp(name, B, frac, with_b2):
    s, t = layer(name, B, seed=4)
    y = wl.make_input(s, 14, DEV)
    k = max(1, wl.k_for(frac, s.N))
    S = _subset(s.N, k, 7)
    k_max = min(s.N, k + 17)  # count < k_max
    idx = torch.zeros(k_max, dtype=torch.int32, device=DEV)
    idx[:k] = torch.from_numpy(S).to(DEV)
    cnt = torch.tensor([k], dtype=torch.int32, device=DEV)
    b2 = torch.randn(s.d, device=DEV) * 0.1 if with_b2 else None
    out = torch.full((B, s.d), 7.0, device=DEV)
    ws = ws_for(bd.DV_OP_SPARSE_MLP, s, k_max=k_max)
    bd.dv_sparse_mlp(y, t["W1t"], t["b1"], t["W2t"], b2, idx, cnt, k_max, out, ws)
    torch.cuda.synchronize()
    ref = O.sparse_mlp(f64(y), f64(t["W1t"]), f64(t["b1"]), f64(t["W2t"]), None if b2 is None else f64(b2), S)
    assert_out(out.cpu().numpy(), ref)
    # accumulate mode adds to the residual
    base = torch.randn(B, s.d, device=DEV)
    acc = base.clone()
    bd.dv_sparse_mlp(y, t["W1t"], t["b1"], t["W2t"], b2, idx, cnt, k_max, acc, ws, accumulate=True)
    torch.cuda.synchronize()
    assert_out((acc - base).cpu().numpy(), ref)
    no_device_errors(ws)


def test_sparse_mlp_empty_and_all_zero_activations():
    s, t = layer("ragged", 1, seed=5)
    y = wl.make_input(s, 15, DEV)
    idx = torch.zeros(8, dtype=torch.int32, device=DEV)
    cnt = torch.zeros(1, dtype=torch.int32, device=DEV)
    b2 = torch.randn(s.d, device=DEV)
    out = torch.full((1, s.d), 3.0, device=DEV)
    ws = ws_for(bd.DV_OP_SPARSE_MLP, s, k_max=8)
    bd.dv_sparse_mlp(y, t["W1t"], t["b1"], t["W2t"], b2, idx, cnt, 8, out, ws)
    torch.cuda.synchronize()
    assert torch.allclose(out[0], b2)
    # neurons that are all inactive: a large negative b1 makes every activation 0
    b1 = torch.full_like(t["b1"], -1e6)
    cnt.fill_(8)
    idx.copy_(torch.arange(8, dtype=torch.int32, device=DEV))
    bd.dv_sparse_mlp(y, t["W1t"], b1, t["W2t"], None, idx, cnt, 8, out, ws)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0


def test_sparse_mlp_relu_positive_set_equals_dense():
    """§2.3 invariant on the GPU: S_M = exactly the positive preactivations
    gives the dense MLP output."""
    s, t = layer("opt-like", 1, seed=6)
    y = wl.make_input(s, 16, DEV)
    pre = O.mlp_preactivations(f64(y), f64(t["W1t"]), f64(t["b1"]))[0]
    S = np.nonzero(pre > 0)[0].astype(np.int32)
    dense = O.sparse_mlp(f64(y), f64(t["W1t"]), f64(t["b1"]), f64(t["W2t"]), None, np.arange(s.N))
    idx = torch.from_numpy(S).to(DEV)
    cnt = torch.tensor([len(S)], dtype=torch.int32, device=DEV)
    out = torch.empty(1, s.d, device=DEV)
    ws = ws_for(bd.DV_OP_SPARSE_MLP, s, k_max=len(S))
    bd.dv_sparse_mlp(y, t["W1t"], t["b1"], t["W2t"], None, idx, cnt, len(S), out, ws)
    torch.cuda.synchronize()
    assert_out(out.cpu().numpy(), dense)


def test_device_status_on_bad_count_and_index():
    """A count above k_max is clamped and an out-of-range index skipped; both
    set bits of the device status word (no out-of-bounds access happens)."""
    s, t = layer("ragged", 1, seed=7)
    y = wl.make_input(s, 17, DEV)
    idx = torch.tensor([3, 9, s.N + 5, 40], dtype=torch.int32, device=DEV)
    cnt = torch.tensor([4], dtype=torch.int32, device=DEV)
    out = torch.empty(1, s.d, device=DEV)
    ws = ws_for(bd.DV_OP_SPARSE_MLP, s, k_max=4)
    bd.dv_sparse_mlp(y, t["W1t"], t["b1"], t["W2t"], None, idx, cnt, 4, out, ws)
    st = bd.dv_read_device_status(ws)
    assert st & 2
    ref = O.sparse_mlp(f64(y), f64(t["W1t"]), f64(t["b1"]), f64(t["W2t"]), None, [3, 9, 40])
    assert_out(out.cpu().numpy(), ref)
    cnt.fill_(1000)
    idx2 = torch.tensor([3, 9, 11, 40], dtype=torch.int32, device=DEV)
    bd.dv_sparse_mlp(y, t["W1t"], t["b1"], t["W2t"], None, idx2, cnt, 4, out, ws)
    assert bd.dv_read_device_status(ws) & 1
    assert bd.dv_read_device_status(ws) == 0  # cleared by the read


# ---------------------------------------------------------------------------
# eq. (2): sparse MHA over the KV cache
# ---------------------------------------------------------------------------


def _assert_kv_slot(cache_gpu, ref_vals, b, head, pos, is_bf16):
    got = f64(cache_gpu[b, head, pos])
    if is_bf16:
        assert_kv_slot(got, ref_vals)
    else:
        assert np.all(np.abs(got - ref_vals) <= np.abs(ref_vals) * 1e-5 + 1e-6)


@pytest.mark.parametrize("name,B,pos,nsel", [("tiny", 1, 64, 2), ("tiny", 1, 0, 4), ("ragged", 2, 99, 3),
                                              ("ragged", 1, 37, 6), ("opt-like", 1, 512, 8), ("opt-like", 3, 300, 5)])
def test_sparse_mha(name, B, pos, nsel):
    s, t = layer(name, B, seed=8)
    y = wl.make_input(s, 18, DEV)
    heads = _subset(s.h, nsel, 9)
    kh_max = min(s.h, nsel + 1)
    hidx = torch.zeros(kh_max, dtype=torch.int32, device=DEV)
    hidx[:nsel] = torch.from_numpy(heads).to(DEV)
    hcnt = torch.tensor([nsel], dtype=torch.int32, device=DEV)
    bO = torch.randn(s.d, device=DEV) * 0.05
    bqkv = torch.randn(s.h, 3, s.dh, device=DEV) * 0.05
    K0, V0 = t["K"].clone(), t["V"].clone()
    out = torch.empty(B, s.d, device=DEV)
    ws = ws_for(bd.DV_OP_SPARSE_MHA, s, kh_max=kh_max)
    scale = 1.0 / np.sqrt(s.dh)
    bd.dv_sparse_mha(y, t["Wqkv"], bqkv, t["WOt"], bO, t["K"], t["V"], pos, scale, hidx, hcnt, kh_max, out, ws)
    torch.cuda.synchronize()
    Kr, Vr = f64(K0), f64(V0)
    kv_round = "bf16" if s.kvdtype == "bf16" else None
    ref = O.sparse_mha(f64(y), f64(t["Wqkv"]), f64(bqkv), f64(t["WOt"]), f64(bO), Kr, Vr, pos, scale, heads, kv_round)
    assert_out(out.cpu().numpy(), ref.out)
    for b in range(B):
        for p, i in enumerate(heads):
            _assert_kv_slot(t["K"], ref.k_new[b, p], b, i, pos, s.kvdtype == "bf16")
            _assert_kv_slot(t["V"], ref.v_new[b, p], b, i, pos, s.kvdtype == "bf16")
    untouched = [i for i in range(s.h) if i not in set(heads.tolist())]
    assert torch.equal(t["K"][:, untouched], K0[:, untouched])
    mask = torch.ones(s.cap, dtype=torch.bool)
    mask[pos] = False
    assert torch.equal(t["K"][:, :, mask], K0[:, :, mask])
    no_device_errors(ws)


def test_sparse_mha_no_heads_gives_bias_only():
    s, t = layer("ragged", 1, seed=10)
    y = wl.make_input(s, 19, DEV)
    hidx = torch.zeros(2, dtype=torch.int32, device=DEV)
    hcnt = torch.zeros(1, dtype=torch.int32, device=DEV)
    bO = torch.randn(s.d, device=DEV)
    out = torch.empty(1, s.d, device=DEV)
    ws = ws_for(bd.DV_OP_SPARSE_MHA, s, kh_max=2)
    bd.dv_sparse_mha(y, t["Wqkv"], None, t["WOt"], bO, t["K"], t["V"], 5, 0.1, hidx, hcnt, 2, out, ws)
    torch.cuda.synchronize()
    assert torch.allclose(out[0], bO)


# ---------------------------------------------------------------------------
# one decoder layer, and the look-ahead stack
# ---------------------------------------------------------------------------


def _trace_bufs(s):
    f = dict(device=DEV, dtype=torch.float32)
    i = dict(device=DEV, dtype=torch.int32)
    return dict(yA=torch.empty(s.B, s.d, **f), scores_h=torch.empty(s.B, s.h, **f), head_idx=torch.zeros(s.h, **i),
                head_count=torch.zeros(1, **i), yM=torch.empty(s.B, s.d, **f), scores=torch.empty(s.B, s.N, **f),
                idx=torch.zeros(s.N, **i), count=torch.zeros(1, **i))


@pytest.mark.parametrize("name,B", [("tiny", 1), ("ragged", 3), ("opt-like", 1), ("opt-like", 4), ("fused128", 1),
                                    ("fused128", 3), ("tiny", 2), ("fused128", 6)])
def test_decode_layer(name, B):
    s, t = layer(name, B, seed=11)
    t["ln1_g"] = 1.0 + 0.1 * torch.randn(s.d, device=DEV)
    t["ln2_b"] = 0.1 * torch.randn(s.d, device=DEV)
    x = wl.make_input(s, 21, DEV) * 2.0 + 0.5
    k = wl.k_for(0.1, s.N)
    k_h = max(1, s.h // 4)
    L = bd.Layer(t, B, min(s.N, B * k), min(s.h, B * k_h))
    p = bd.params(k, k_h, 1.0 / np.sqrt(s.dh))
    ws = bd.workspace(bd.DV_OP_DECODE_LAYER, L.dims)
    tb = _trace_bufs(s)
    x0 = x.clone()
    K0, V0 = f64(t["K"]), f64(t["V"])
    pos = s.L
    bd.dv_decode_layer(L, p, x, pos, ws, trace=bd.layer_io(**tb))
    torch.cuda.synchronize()
    OL = oracle_layer(t)
    OL.K, OL.V = K0, V0
    P = O.LayerParams(k=k, k_h=k_h, scale=1.0 / np.sqrt(s.dh))
    # the GPU's selections are the oracle's selections of the GPU's scores
    sh, sm = tb["scores_h"].cpu().numpy(), tb["scores"].cpu().numpy()
    hsel = O.select(sh, k=k_h)
    msel = O.select(sm, k=k)
    assert np.array_equal(selected(tb["head_idx"], tb["head_count"]), hsel)
    assert np.array_equal(selected(tb["idx"], tb["count"]), msel)
    tr = O.decode_layer(f64(x0), OL, P, pos, head_idx=hsel, idx=msel)
    assert_out(tb["yA"].cpu().numpy(), tr.yA, "yA")
    assert_scores(sh, O.head_predictor_scores(f64(tb["yA"]), OL.PA))
    assert_out(tb["yM"].cpu().numpy(), tr.yM, "yM")
    assert_scores(sm, O.mlp_predictor_scores(f64(tb["yM"]), OL.At, OL.Bm, OL.b1))
    assert_out((x - x0).cpu().numpy(), tr.x_out - f64(x0), "x_out - x")
    no_device_errors(ws)


@pytest.mark.parametrize("name,B,kf,khf", [("wide", 1, 0.1, 0.25), ("wide", 1, 1.0, 1.0), ("wide", 2, 0.05, 0.5),
                                          ("wide", 1, 0.0005, 0.125)])
def test_decode_layer_selected_fractions(name, B, kf, khf):
    """Layer output vs the oracle across selection sizes: from a few rows per
    CTA (most CTAs idle) to every neuron and head (several chunks per CTA)."""
    s, t = layer(name, B, seed=15)
    x = wl.make_input(s, 24, DEV)
    k = max(1, wl.k_for(kf, s.N))
    k_h = max(1, wl.k_for(khf, s.h))
    L = bd.Layer(t, B, min(s.N, B * k), min(s.h, B * k_h))
    p = bd.params(k, k_h, 1.0 / np.sqrt(s.dh))
    ws = bd.workspace(bd.DV_OP_DECODE_LAYER, L.dims)
    tb = _trace_bufs(s)
    x0 = x.clone()
    OL = oracle_layer(t)
    OL.K, OL.V = f64(t["K"]), f64(t["V"])
    bd.dv_decode_layer(L, p, x, s.L, ws, trace=bd.layer_io(**tb))
    torch.cuda.synchronize()
    P = O.LayerParams(k=k, k_h=k_h, scale=1.0 / np.sqrt(s.dh))
    sh, sm = tb["scores_h"].cpu().numpy(), tb["scores"].cpu().numpy()
    hsel, msel = O.select(sh, k=k_h), O.select(sm, k=k)
    assert np.array_equal(selected(tb["head_idx"], tb["head_count"]), hsel)
    assert np.array_equal(selected(tb["idx"], tb["count"]), msel)
    tr = O.decode_layer(f64(x0), OL, P, s.L, head_idx=hsel, idx=msel)
    assert_out(tb["yA"].cpu().numpy(), tr.yA, "yA")
    assert_out(tb["yM"].cpu().numpy(), tr.yM, "yM")
    assert_out((x - x0).cpu().numpy(), tr.x_out - f64(x0), "x_out - x")
    no_device_errors(ws)


@pytest.mark.parametrize("name,lookahead,B,fuse", [("ragged", True, 1, True), ("ragged", False, 1, True),
                                                   ("fused128", True, 1, True), ("fused128", False, 2, True),
                                                   ("opt-like", True, 1, True), ("opt-like", True, 1, False),
                                                   ("ragged", True, 2, False), ("fused128", True, 2, True)])
def test_lookahead_stack(name, lookahead, B, fuse):
    """fuse: the next layer's predictor first stage inside the q/k/v kernel
    (begin_ahead + predict_layer_tail) rather than dv_predict_layer."""
    nL = 3
    s = shape(name, B)
    layers = [wl.make_layer(s, 100 + l, DEV) for l in range(nL)]
    K0 = [(f64(t["K"]), f64(t["V"])) for t in layers]
    k, k_h = wl.k_for(0.1, s.N), 2
    stk = DecoderStack(layers, B, k, k_h, 1.0 / np.sqrt(s.dh), lookahead=lookahead, fuse_ahead=fuse)
    x = wl.make_input(s, 31, DEV)
    x0 = f64(x)
    pos = s.L
    stk.step(x, pos)
    torch.cuda.synchronize()
    OLs = []
    for l, t in enumerate(layers):
        OL = oracle_layer(t)
        OL.K, OL.V = K0[l]
        OLs.append(OL)
    P = O.LayerParams(k=k, k_h=k_h, scale=1.0 / np.sqrt(s.dh))
    sel = []
    for l in range(nL):
        sh, sm = stk.scores_h[l].cpu().numpy(), stk.scores[l].cpu().numpy()
        hs, ms = O.select(sh, k=k_h), O.select(sm, k=k)
        assert np.array_equal(selected(stk.head_idx[l], stk.head_count[l]), hs), l
        assert np.array_equal(selected(stk.idx[l], stk.count[l]), ms), l
        if lookahead and l > 0:
            # layer l's scores come from layer l-1's normalised input
            yprev = f64(stk.yA[l - 1])
            assert_scores(sh, O.head_predictor_scores(yprev, OLs[l].PA))
            assert_scores(sm, O.mlp_predictor_scores(yprev, OLs[l].At, OLs[l].Bm, OLs[l].b1))
        sel.append((hs, ms))
    xo, _ = O.decode_stack(x0, OLs, P, pos, lookahead=lookahead, sel_override=sel)
    assert_out((x.cpu().numpy() - x0), xo - x0)
    no_device_errors(stk.ws_main)
    no_device_errors(stk.ws_side)


@pytest.mark.parametrize("name", ["ragged", "fused128"])
def test_stack_step_in_cuda_graph_matches_eager(name):
    nL, B = 3, 2
    s = shape(name, B)
    layers_a = [wl.make_layer(s, 200 + l, DEV) for l in range(nL)]
    layers_b = [{kk: v.clone() for kk, v in t.items()} for t in layers_a]
    k, k_h = wl.k_for(0.1, s.N), 2
    sa = DecoderStack(layers_a, B, k, k_h, 0.09)
    sb = DecoderStack(layers_b, B, k, k_h, 0.09)
    x = wl.make_input(s, 41, DEV)
    xa, xb = x.clone(), x.clone()
    sa.step(xa, s.L)
    g = torch.cuda.CUDAGraph()
    cap_stream = torch.cuda.Stream()
    cap_stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap_stream):
        with torch.cuda.graph(g, stream=cap_stream):
            sb.step(xb, s.L)
    torch.cuda.current_stream().wait_stream(cap_stream)
    xb.copy_(x)
    g.replay()
    torch.cuda.synchronize()
    assert_out((xb - x).cpu().numpy(), (xa - x).cpu().numpy())


@pytest.mark.parametrize("name", ["fused128", "ragged"])
def test_decode_layer_with_empty_sets(name):
    """k = 0 and k_h = 0: the layer adds only the output biases."""
    s, t = layer(name, 1, seed=12)
    t["bO"] = torch.randn(s.d, device=DEV) * 0.1
    t["b2"] = torch.randn(s.d, device=DEV) * 0.1
    x = wl.make_input(s, 22, DEV)
    x0 = x.clone()
    L = bd.Layer(t, 1, 0, 0)
    p = bd.params(0, 0, 0.1)
    ws = bd.workspace(bd.DV_OP_DECODE_LAYER, L.dims)
    bd.dv_decode_layer(L, p, x, s.L, ws)
    torch.cuda.synchronize()
    assert torch.allclose(x, x0 + t["bO"] + t["b2"], rtol=1e-6, atol=1e-6)
    no_device_errors(ws)


@pytest.mark.parametrize("name", ["fused128", "opt-like", "tiny", "wide"])
def test_predict_layer_matches_oracle(name):
    """The look-ahead call (both sets from one input) on the fused predictor."""
    B = 2
    s, t = layer(name, B, seed=13)
    k, k_h = wl.k_for(0.1, s.N), 2
    L = bd.Layer(t, B, min(s.N, B * k), min(s.h, B * k_h))
    p = bd.params(k, k_h, 0.1)
    ws = bd.workspace(bd.DV_OP_DECODE_LAYER, L.dims)
    y = wl.make_input(s, 23, DEV)
    tb = _trace_bufs(s)
    out = bd.layer_io(scores_h=tb["scores_h"], head_idx=tb["head_idx"], head_count=tb["head_count"],
                      scores=tb["scores"], idx=tb["idx"], count=tb["count"])
    for _ in range(2):  # twice: the in-kernel histogram and tickets must be left clean
        bd.dv_predict_layer(L, p, y, out, ws)
        torch.cuda.synchronize()
        sh, sm = tb["scores_h"].cpu().numpy(), tb["scores"].cpu().numpy()
        assert_scores(sh, O.head_predictor_scores(f64(y), f64(t["PA"])))
        assert_scores(sm, O.mlp_predictor_scores(f64(y), f64(t["At"]), f64(t["Bm"]), f64(t["b1"])))
        assert np.array_equal(selected(tb["head_idx"], tb["head_count"]), O.select(sh, k=k_h))
        assert np.array_equal(selected(tb["idx"], tb["count"]), O.select(sm, k=k))
    no_device_errors(ws)


@pytest.mark.parametrize("kf,equal", [(0.15, False), (0.05, False), (0.15, True)])
def test_predict_layer_at_the_largest_neuron_count(kf, equal):
    """The fused selection at N = 49152 (the OPT-175B neuron count, the most
    the selection keeps in shared memory), batch 1: exact top-k of the
    emitted scores, including all-equal scores (every key in one bin)."""
    s = wl.LayerShape(B=1, d=256, N=49152, r=32, h=4, dh=64, L=64, cap=65, wdtype="bf16", kvdtype="bf16",
                      p_active=0.1)
    t = wl.make_layer(s, 19, DEV)
    if equal:
        t["Bm"] = torch.zeros_like(t["Bm"])
        t["b1"] = torch.full_like(t["b1"], 0.25)
    k, k_h = wl.k_for(kf, s.N), 1
    L = bd.Layer(t, 1, k, k_h)
    p = bd.params(k, k_h, 0.1)
    ws = bd.workspace(bd.DV_OP_DECODE_LAYER, L.dims)
    y = wl.make_input(s, 27, DEV)
    tb = _trace_bufs(s)
    out = bd.layer_io(scores_h=tb["scores_h"], head_idx=tb["head_idx"], head_count=tb["head_count"],
                      scores=tb["scores"], idx=tb["idx"], count=tb["count"])
    bd.dv_predict_layer(L, p, y, out, ws)
    torch.cuda.synchronize()
    sm = tb["scores"].cpu().numpy()
    assert_scores(sm, O.mlp_predictor_scores(f64(y), f64(t["At"]), f64(t["Bm"]), f64(t["b1"])))
    assert np.array_equal(selected(tb["idx"], tb["count"]), O.select(sm, k=k))
    no_device_errors(ws)


@pytest.mark.parametrize("name,group", [("opt-like", 8), ("opt-like", 2), ("opt-like", 0), ("ragged", 0), ("wide", 7)])
def test_predict_layer_ties_at_threshold(name, group):
    """Neuron scores with many exact ties at the k-th value (Bm rows and b1
    repeated in groups; group 0: every score equal): the selection takes the
    keys above the threshold and the lowest-index copies of the threshold."""
    B = 1
    s, t = layer(name, B, seed=16)
    if group:
        rep = torch.arange(s.N, device=DEV) // group * group
        t["Bm"] = t["Bm"][rep].contiguous()
        t["b1"] = t["b1"][rep].contiguous()
    else:
        t["Bm"] = torch.zeros_like(t["Bm"])
        t["b1"] = torch.full_like(t["b1"], -0.5)
    k, k_h = wl.k_for(0.1, s.N) + 1, 1
    L = bd.Layer(t, B, min(s.N, B * k), min(s.h, B * k_h))
    p = bd.params(k, k_h, 0.1)
    ws = bd.workspace(bd.DV_OP_DECODE_LAYER, L.dims)
    y = wl.make_input(s, 25, DEV)
    tb = _trace_bufs(s)
    out = bd.layer_io(scores_h=tb["scores_h"], head_idx=tb["head_idx"], head_count=tb["head_count"],
                      scores=tb["scores"], idx=tb["idx"], count=tb["count"])
    bd.dv_predict_layer(L, p, y, out, ws)
    torch.cuda.synchronize()
    sm = tb["scores"].cpu().numpy()
    kth = np.sort(sm[0])[::-1][k - 1]
    assert (sm[0] == kth).sum() > 1  # the threshold value is tied
    assert np.array_equal(selected(tb["idx"], tb["count"]), O.select(sm, k=k))
    no_device_errors(ws)


@pytest.mark.parametrize("name,B,split", [("opt-like", 1, True), ("opt-like", 1, False), ("fused128", 2, True),
                                          ("ragged", 1, True), ("wide", 1, True), ("tiny", 3, False)])
def test_begin_ahead_and_tail_predict_next_layer(name, B, split):
    """The next layer's predictor split over begin_ahead (its first stage in
    this layer's q/k/v kernel) and predict_layer_tail: scores of layer 2 from
    layer 1's yA, sets = the oracle's selection of those scores, and layer 1's
    own q/k/v work unchanged (the KV slot it writes)."""
    s, t = layer(name, B, seed=17)
    t2 = wl.make_layer(s, 18, DEV)
    k, k_h = wl.k_for(0.1, s.N), 2
    L1 = bd.Layer(t, B, min(s.N, B * k), min(s.h, B * k_h))
    L2 = bd.Layer(t2, B, min(s.N, B * k), min(s.h, B * k_h))
    p = bd.params(k, k_h, 0.1)
    ws1 = bd.workspace(bd.DV_OP_DECODE_LAYER, L1.dims)
    ws2 = bd.workspace(bd.DV_OP_DECODE_LAYER, L1.dims)
    x = wl.make_input(s, 26, DEV)
    tb1, tb2 = _trace_bufs(s), _trace_bufs(s)
    Kref, Vref = t["K"].clone(), t["V"].clone()
    x_ref = x.clone()
    ws_ref = bd.workspace(bd.DV_OP_DECODE_LAYER, L1.dims)
    tr_ref = _trace_bufs(s)
    t_ref = {kk: v for kk, v in t.items()}
    t_ref["K"], t_ref["V"] = Kref, Vref
    bd.dv_decode_layer_begin(bd.Layer(t_ref, B, L1.dims.k_max, L1.dims.kh_max), p, x_ref, s.L, ws_ref,
                             trace=bd.layer_io(**tr_ref))
    bd.dv_decode_layer_begin_ahead(L1, p, x, s.L, ws1, L2, tb2["scores_h"], ws2, trace=bd.layer_io(**tb1))
    out2 = bd.layer_io(scores_h=tb2["scores_h"], head_idx=tb2["head_idx"], head_count=tb2["head_count"],
                       scores=tb2["scores"], idx=tb2["idx"], count=tb2["count"])
    if split:  # the head part and the neuron part on two streams, as the stack runs them
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        bd.dv_predict_layer_tail(L2, p, out2, ws2, sets=bd.DV_SET_HEADS)
        bd.dv_predict_layer_tail(L2, p, out2, ws2, sets=bd.DV_SET_NEURONS, stream=side)
        torch.cuda.current_stream().wait_stream(side)
    else:
        bd.dv_predict_layer_tail(L2, p, out2, ws2)
    torch.cuda.synchronize()
    yA = f64(tb1["yA"])
    sh, sm = tb2["scores_h"].cpu().numpy(), tb2["scores"].cpu().numpy()
    assert_scores(sh, O.head_predictor_scores(yA, f64(t2["PA"])))
    assert_scores(sm, O.mlp_predictor_scores(yA, f64(t2["At"]), f64(t2["Bm"]), f64(t2["b1"])))
    assert np.array_equal(selected(tb2["head_idx"], tb2["head_count"]), O.select(sh, k=k_h))
    assert np.array_equal(selected(tb2["idx"], tb2["count"]), O.select(sm, k=k))
    # layer 1's own begin: same sets and the same KV slot as the plain call
    assert np.array_equal(selected(tb1["head_idx"], tb1["head_count"]),
                          selected(tr_ref["head_idx"], tr_ref["head_count"]))
    assert torch.equal(t["K"][:, :, s.L], Kref[:, :, s.L]) and torch.equal(t["V"][:, :, s.L], Vref[:, :, s.L])
    no_device_errors(ws1)
    no_device_errors(ws2)


@pytest.mark.parametrize("name", ["fused128", "ragged", "wide"])
def test_layer_in_three_calls_equals_one(name):
    """begin + attn + mlp (look-ahead sets given) == dv_decode_layer with the same sets."""
    B = 2
    s, t = layer(name, B, seed=14)
    t2 = {kk: v.clone() for kk, v in t.items()}
    k, k_h = wl.k_for(0.1, s.N), 2
    hidx = torch.from_numpy(_subset(s.h, 3, 5)).to(DEV)
    hcnt = torch.tensor([3], dtype=torch.int32, device=DEV)
    midx = torch.from_numpy(_subset(s.N, 2 * k, 6)).to(DEV)
    mcnt = torch.tensor([2 * k], dtype=torch.int32, device=DEV)
    sel = bd.layer_io(head_idx=hidx, head_count=hcnt, idx=midx, count=mcnt)
    x = wl.make_input(s, 24, DEV)
    xa, xb = x.clone(), x.clone()
    La, Lb = bd.Layer(t, B, 2 * k, 3), bd.Layer(t2, B, 2 * k, 3)
    p = bd.params(k, 1, 0.1)  # the sets are given; k and k_h only bound them
    wsa, wsb = bd.workspace(bd.DV_OP_DECODE_LAYER, La.dims), bd.workspace(bd.DV_OP_DECODE_LAYER, Lb.dims)
    bd.dv_decode_layer(La, p, xa, s.L, wsa, sel=sel)
    bd.dv_decode_layer_begin(Lb, p, xb, s.L, wsb, sel=sel)
    bd.dv_decode_layer_attn(Lb, p, xb, s.L, wsb, sel=sel)
    bd.dv_decode_layer_mlp(Lb, p, xb, wsb, sel=sel)
    torch.cuda.synchronize()
    assert_out((xb - x).cpu().numpy(), (xa - x).cpu().numpy())
    no_device_errors(wsa)
    no_device_errors(wsb)
