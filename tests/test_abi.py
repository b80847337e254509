"""The C-ABI library loads, exports every function include/dejavu.h declares,
and rejects bad arguments on the host before touching the GPU (CPU only)."""

import ctypes
import subprocess

import pytest

from attention_predictor_gemv_b200 import binding as bd

A = 0x10000  # a 16-byte aligned fake device address (never dereferenced)


def test_every_declared_function_is_exported():
    names = bd.exported_symbols_declared_in_header()
    assert {"dv_predict_mlp", "dv_predict_heads", "dv_topk", "dv_sparse_mlp", "dv_sparse_mha",
            "dv_decode_layer"} <= set(names)
    out = subprocess.run(["nm", "-D", "--defined-only", bd.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(bd.library(), n)


def test_only_c_abi_symbols_are_exported():
    out = subprocess.run(["nm", "-D", "--defined-only", bd.LIB_PATH], capture_output=True, text=True).stdout
    funcs = [l.split()[-1] for l in out.splitlines() if " T " in l]
    assert funcs and all(f.startswith("dv_") for f in funcs), funcs


def test_status_strings():
    assert bd.status_string(0) == "ok"
    assert "aligned" in bd.status_string(bd.DV_ERR_ALIGN)
    assert bd.status_string(99) == "unknown status"


def test_workspace_size_host_only():
    D = bd.dims(B=1, d=2048, N=8192, r=256, h=32, dh=64, cap=520, k_max=819, kh_max=8)
    n = bd.dv_workspace_size(bd.DV_OP_DECODE_LAYER, D)
    assert n > 64 * 1024
    assert bd.dv_workspace_size(bd.DV_OP_DECODE_LAYER, bd.dims(B=17, d=2048, N=8)) == 0  # B > 16
    assert bd.dv_workspace_size(bd.DV_OP_DECODE_LAYER, bd.dims(B=1, d=12, N=8)) == 0  # d % 8
    assert bd.dv_workspace_size(bd.DV_OP_TOPK, bd.dims(B=2, N=1000, k_max=10)) > 0
    assert bd.dv_workspace_size(99, D) == 0
    # more batch rows never need less workspace
    D4 = bd.dims(B=4, d=2048, N=8192, r=256, h=32, dh=64, cap=520, k_max=819 * 4, kh_max=32)
    assert bd.dv_workspace_size(bd.DV_OP_DECODE_LAYER, D4) > n


def _mlp(**kw):
    a = dict(y=A, B=1, d=64, N=256, W1t=A, b1=A, W2t=A, b2=None, dt=bd.DV_BF16, idx=A, count=A, k_max=16,
             out=A, acc=0, ws=A, wsb=1 << 30, st=None)
    a.update(kw)
    return bd._lib_dv_sparse_mlp(a["y"], a["B"], a["d"], a["N"], a["W1t"], a["b1"], a["W2t"], a["b2"], a["dt"],
                                 a["idx"], a["count"], a["k_max"], a["out"], a["acc"], a["ws"], a["wsb"], a["st"])


def test_sparse_mlp_argument_checks():
    assert _mlp(y=None) == bd.DV_ERR_ARG
    assert _mlp(W1t=A + 8) == bd.DV_ERR_ALIGN
    assert _mlp(b2=A + 4) == bd.DV_ERR_ALIGN
    assert _mlp(d=60) == bd.DV_ERR_ARG  # d % 8
    assert _mlp(B=0) == bd.DV_ERR_ARG
    assert _mlp(B=17) == bd.DV_ERR_ARG
    assert _mlp(k_max=257) == bd.DV_ERR_ARG  # k_max > N
    assert _mlp(dt=7) == bd.DV_ERR_ARG
    assert _mlp(wsb=16) == bd.DV_ERR_WORKSPACE
    assert _mlp(ws=None) == bd.DV_ERR_ARG


def _mha(**kw):
    a = dict(y=A, B=1, d=64, h=4, dh=64, Wqkv=A, bqkv=None, WOt=A, bO=None, dt=bd.DV_BF16, K=A, V=A,
             kvdt=bd.DV_BF16, cap=10, pos=3, scale=0.125, hidx=A, hcnt=A, kh_max=2, out=A, acc=0, ws=A, wsb=1 << 30,
             st=None)
    a.update(kw)
    return bd._lib_dv_sparse_mha(a["y"], a["B"], a["d"], a["h"], a["dh"], a["Wqkv"], a["bqkv"], a["WOt"], a["bO"],
                                 a["dt"], a["K"], a["V"], a["kvdt"], a["cap"], a["pos"], a["scale"], a["hidx"],
                                 a["hcnt"], a["kh_max"], a["out"], a["acc"], a["ws"], a["wsb"], a["st"])


def test_sparse_mha_argument_checks():
    assert _mha(pos=10) == bd.DV_ERR_ARG  # pos >= cap
    assert _mha(pos=-1) == bd.DV_ERR_ARG
    assert _mha(dh=96) == bd.DV_ERR_UNSUPPORTED
    assert _mha(kvdt=bd.DV_F32) == bd.DV_ERR_UNSUPPORTED
    assert _mha(kh_max=5) == bd.DV_ERR_ARG  # > h
    assert _mha(K=A + 2) == bd.DV_ERR_ALIGN
    assert _mha(hidx=None) == bd.DV_ERR_ARG


def test_topk_and_predict_argument_checks():
    assert bd._lib_dv_topk(A, 1, 0, 1, 0.0, 0, A, A, A, 1 << 20, None) == bd.DV_ERR_ARG  # n = 0
    assert bd._lib_dv_topk(A, 1, 100, 1, 0.0, 5, A, A, A, 1 << 20, None) == bd.DV_ERR_ARG  # mode
    assert bd._lib_dv_topk(A + 4, 1, 100, 1, 0.0, 0, A, A, A, 1 << 20, None) == bd.DV_ERR_ALIGN
    assert bd._lib_dv_predict_mlp(A, 1, 64, 4, 256, A, A, A, bd.DV_BF16, 8, 0.0, 0, A, A, A, A, 1 << 20,
                                  None) == bd.DV_ERR_ARG  # r < 8
    assert bd._lib_dv_predict_heads(A, 1, 64, 0, A, bd.DV_BF16, 1, 0.0, 0, A, A, A, A, 1 << 20,
                                    None) == bd.DV_ERR_ARG  # h = 0


def test_decode_layer_argument_checks():
    w = bd.LayerWeightsC(bd.DV_BF16, bd.DV_BF16, None, None, A, A, None, A, None, A, A, None, None, A, A, A, A, A,
                         None)
    D = bd.dims(B=1, d=64, N=256, r=16, h=4, dh=64, cap=8, k_max=32, kh_max=2)
    p = bd.params(32, 2, 0.125)
    f = bd._lib_dv_decode_layer
    assert f(ctypes.byref(w), ctypes.byref(D), ctypes.byref(p), A, 8, None, None, A, 1 << 30, None) == bd.DV_ERR_ARG
    p_bad = bd.params(33, 2, 0.125)  # k > k_max
    assert f(ctypes.byref(w), ctypes.byref(D), ctypes.byref(p_bad), A, 0, None, None, A, 1 << 30,
             None) == bd.DV_ERR_ARG
    w.W1t = A + 8
    assert f(ctypes.byref(w), ctypes.byref(D), ctypes.byref(p), A, 0, None, None, A, 1 << 30,
             None) == bd.DV_ERR_ALIGN


def test_lookahead_split_argument_checks():
    """dv_decode_layer_begin_ahead / dv_predict_layer_tail reject bad
    arguments on the host (no GPU is touched: every pointer is fake)."""
    w = bd.LayerWeightsC(bd.DV_BF16, bd.DV_BF16, None, None, A, A, None, A, None, A, A, None, None, A, A, A, A, A,
                         None)
    D = bd.dims(B=1, d=64, N=256, r=16, h=4, dh=64, cap=8, k_max=32, kh_max=2)
    p = bd.params(32, 2, 0.125)
    ws_bytes = bd.dv_workspace_size(bd.DV_OP_DECODE_LAYER, D)
    W1 = 0x20000  # another fake aligned workspace
    ahead = bd._lib_dv_decode_layer_begin_ahead
    args = lambda **kw: dict(dict(x=A, pos=0, ws=A, nxt=ctypes.byref(w), sh=A, nws=W1), **kw)  # noqa: E731

    def call(**kw):
        a = args(**kw)
        return ahead(ctypes.byref(w), ctypes.byref(D), ctypes.byref(p), a["x"], a["pos"], None, None, a["ws"],
                     ws_bytes, a["nxt"], a["sh"], a["nws"], ws_bytes, None)

    assert call(nws=A) == bd.DV_ERR_ARG  # the look-ahead workspace must not be the layer's
    assert call(sh=None) == bd.DV_ERR_ARG
    assert call(sh=A + 4) == bd.DV_ERR_ALIGN
    assert call(pos=8) == bd.DV_ERR_ARG  # pos >= cap
    assert call(nxt=None) == bd.DV_ERR_ARG
    w16 = bd.LayerWeightsC(bd.DV_F32, bd.DV_F32, None, None, A, A, None, A, None, A, A, None, None, A, A, A, A, A,
                           None)
    assert call(nxt=ctypes.byref(w16)) == bd.DV_ERR_UNSUPPORTED  # next layer's dtype differs
    tail = bd._lib_dv_predict_layer_tail
    io = bd.LayerIOC(None, A, A, A, None, A, A, A)
    for sets in (0, 4, -1):
        assert tail(ctypes.byref(w), ctypes.byref(D), ctypes.byref(p), ctypes.byref(io), sets, W1, ws_bytes,
                    None) == bd.DV_ERR_ARG
    io_no_heads = bd.LayerIOC(None, None, None, None, None, A, A, A)
    assert tail(ctypes.byref(w), ctypes.byref(D), ctypes.byref(p), ctypes.byref(io_no_heads), bd.DV_SET_HEADS, W1,
                ws_bytes, None) == bd.DV_ERR_ARG
    io_bad = bd.LayerIOC(None, A, A, A, None, A + 4, A, A)
    assert tail(ctypes.byref(w), ctypes.byref(D), ctypes.byref(p), ctypes.byref(io_bad), bd.DV_SET_NEURONS, W1,
                ws_bytes, None) == bd.DV_ERR_ALIGN
    assert tail(ctypes.byref(w), ctypes.byref(D), ctypes.byref(p), ctypes.byref(io), bd.DV_SET_HEADS, W1, 16,
                None) == bd.DV_ERR_WORKSPACE


def test_sparse_mlp_act_rejects_unknown_activation():
    f = bd._lib_dv_sparse_mlp_act
    args = [A, 1, 64, 256, A, A, A, None, bd.DV_BF16, A, A, 16, A, 0]
    assert f(*args, 2, A, 1 << 30, None) == bd.DV_ERR_ARG
    assert f(*args, -1, A, 1 << 30, None) == bd.DV_ERR_ARG


def test_q8_block_calls_check_arguments_on_the_host():
    f = bd._lib_dv_sparse_mlp_q8
    base = dict(y=A, B=1, d=64, N=256, W1q=A, W1s=A, b1=A, W2q=A, W2s=A, b2=None, idx=A, count=A, k_max=16, out=A,
                acc=0, act=0, ws=A, wsb=1 << 30, st=None)

    def call(**kw):
        a = dict(base, **kw)
        return f(*a.values())

    assert call(W1s=None) == bd.DV_ERR_ARG
    assert call(W2q=A + 8) == bd.DV_ERR_ALIGN
    assert call(B=5) == bd.DV_ERR_UNSUPPORTED
    assert call(d=72) == bd.DV_ERR_UNSUPPORTED  # d % 16
    assert call(act=3) == bd.DV_ERR_ARG
    assert call(wsb=16) == bd.DV_ERR_WORKSPACE
    g = bd._lib_dv_sparse_mha_q8
    args = [A, 1, 64, 4, 64, A, A, None, A, A, None, A, A, 8, 3, 0.125, A, A, 2, A, 0, A, 1 << 30, None]
    assert g(*args[:5], None, *args[6:]) == bd.DV_ERR_ARG
    bad = list(args)
    bad[4] = 96
    assert g(*bad) == bd.DV_ERR_UNSUPPORTED  # dh
    bad = list(args)
    bad[14] = 8
    assert g(*bad) == bd.DV_ERR_ARG  # pos >= cap


def test_layer_rejects_tensors_shorter_than_the_dims():
    """The binding checks every tensor's extent against the dims the library
    indexes with: a KV cache made for batch 1 cannot back a batch-2 layer."""
    from attention_predictor_gemv_b200 import binding as bd
    from attention_predictor_gemv_b200 import workload as wl

    s = wl.LayerShape(B=1, d=256, N=1024, r=32, h=4, dh=64, L=64, cap=65, wdtype="f32", kvdtype="f32",
                      p_active=0.1)
    t = wl.make_layer(s, 0, "cpu")
    # shapes that match pass the check and stop at the device check (CPU tensors here)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        bd.Layer(t, 1, 64, 2)
    with pytest.raises(ValueError, match="^K: shape"):
        bd.Layer(t, 2, 64, 2)
    K3, V3 = wl.make_kv(s, 3, 1, "cpu")
    with pytest.raises(ValueError, match="must be a CUDA tensor"):  # more cache rows than B is fine
        bd.Layer(dict(t, K=K3, V=V3), 2, 64, 2)
    with pytest.raises(ValueError, match="^Bm: shape"):
        bd.Layer(dict(t, Bm=t["Bm"][:, :16].contiguous()), 1, 64, 2)
