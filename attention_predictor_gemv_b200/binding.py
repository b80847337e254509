"""Thin Python binding of libdejavu.so (include/dejavu.h).

Argument marshalling only: every function takes torch tensors, checks their
dtype / device / contiguity, and passes raw device pointers, sizes and the
current CUDA stream to the C entry point of the same name. No step of the
decode path runs here. Importing this module loads the library and fails
loudly if it is missing.
"""

from __future__ import annotations

import ctypes
import os
import re
from typing import Dict, List, Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdejavu.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "dejavu.h")

DV_OK, DV_ERR_ARG, DV_ERR_ALIGN, DV_ERR_UNSUPPORTED, DV_ERR_CUDA, DV_ERR_DEVICE, DV_ERR_WORKSPACE = range(7)
DV_F32, DV_BF16 = 0, 1
DV_TOPK, DV_THRESHOLD = 0, 1
DV_ACT_RELU, DV_ACT_GELU = 0, 1
(DV_OP_PREDICT_MLP, DV_OP_PREDICT_HEADS, DV_OP_TOPK, DV_OP_SPARSE_MLP, DV_OP_SPARSE_MHA,
 DV_OP_DECODE_LAYER) = range(6)


class DvError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m attention_predictor_gemv_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

_c_int, _c_float, _c_size, _p = ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p


class Dims(ctypes.Structure):
    _fields_ = [(n, _c_int) for n in ("B", "d", "N", "r", "h", "dh", "cap", "k_max", "kh_max")]


class LayerWeightsC(ctypes.Structure):
    _fields_ = [("wdtype", _c_int), ("kvdtype", _c_int), ("ln1_g", _p), ("ln1_b", _p), ("PA", _p), ("Wqkv", _p),
                ("bqkv", _p), ("WOt", _p), ("bO", _p), ("Kc", _p), ("Vc", _p), ("ln2_g", _p), ("ln2_b", _p),
                ("At", _p), ("Bm", _p), ("b1", _p), ("W1t", _p), ("W2t", _p), ("b2", _p)]


class LayerParamsC(ctypes.Structure):
    _fields_ = [("k", _c_int), ("tau", _c_float), ("mode", _c_int), ("k_h", _c_int), ("tau_h", _c_float),
                ("mode_h", _c_int), ("scale", _c_float), ("eps", _c_float), ("act", _c_int), ("exact_kv", _c_int)]


class LayerIOC(ctypes.Structure):
    _fields_ = [("yA", _p), ("scores_h", _p), ("head_idx", _p), ("head_count", _p), ("yM", _p), ("scores", _p),
                ("idx", _p), ("count", _p)]


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


_lib_dv_workspace_size = _sig("dv_workspace_size", _c_size, [_c_int, ctypes.POINTER(Dims)])
_lib_dv_status_string = _sig("dv_status_string", ctypes.c_char_p, [_c_int])
_lib_dv_read_device_status = _sig("dv_read_device_status", _c_int, [_p, _p, ctypes.POINTER(_c_int)])
_lib_dv_predict_mlp = _sig("dv_predict_mlp", _c_int,
                           [_p, _c_int, _c_int, _c_int, _c_int, _p, _p, _p, _c_int, _c_int, _c_float, _c_int, _p, _p,
                            _p, _p, _c_size, _p])
_lib_dv_predict_heads = _sig("dv_predict_heads", _c_int,
                             [_p, _c_int, _c_int, _c_int, _p, _c_int, _c_int, _c_float, _c_int, _p, _p, _p, _p,
                              _c_size, _p])
_lib_dv_topk = _sig("dv_topk", _c_int, [_p, _c_int, _c_int, _c_int, _c_float, _c_int, _p, _p, _p, _c_size, _p])
_lib_dv_sparse_mlp = _sig("dv_sparse_mlp", _c_int,
                          [_p, _c_int, _c_int, _c_int, _p, _p, _p, _p, _c_int, _p, _p, _c_int, _p, _c_int, _p, _c_size,
                           _p])
_lib_dv_sparse_mlp_act = _sig("dv_sparse_mlp_act", _c_int,
                              [_p, _c_int, _c_int, _c_int, _p, _p, _p, _p, _c_int, _p, _p, _c_int, _p, _c_int, _c_int,
                               _p, _c_size, _p])
_lib_dv_sparse_mlp_q8 = _sig("dv_sparse_mlp_q8", _c_int,
                             [_p, _c_int, _c_int, _c_int, _p, _p, _p, _p, _p, _p, _p, _p, _c_int, _p, _c_int, _c_int,
                              _p, _c_size, _p])
_lib_dv_sparse_mha_q8 = _sig("dv_sparse_mha_q8", _c_int,
                             [_p, _c_int, _c_int, _c_int, _c_int, _p, _p, _p, _p, _p, _p, _p, _p, _c_int, _c_int,
                              _c_float, _p, _p, _c_int, _p, _c_int, _p, _c_size, _p])
_lib_dv_sparse_mha = _sig("dv_sparse_mha", _c_int,
                          [_p, _c_int, _c_int, _c_int, _c_int, _p, _p, _p, _p, _c_int, _p, _p, _c_int, _c_int, _c_int,
                           _c_float, _p, _p, _c_int, _p, _c_int, _p, _c_size, _p])
_lib_dv_decode_layer = _sig("dv_decode_layer", _c_int,
                            [ctypes.POINTER(LayerWeightsC), ctypes.POINTER(Dims), ctypes.POINTER(LayerParamsC), _p,
                             _c_int, ctypes.POINTER(LayerIOC), ctypes.POINTER(LayerIOC), _p, _c_size, _p])
_lib_dv_decode_layer_begin = _sig("dv_decode_layer_begin", _c_int,
                                  [ctypes.POINTER(LayerWeightsC), ctypes.POINTER(Dims), ctypes.POINTER(LayerParamsC),
                                   _p, _c_int, ctypes.POINTER(LayerIOC), ctypes.POINTER(LayerIOC), _p, _c_size, _p])
_lib_dv_decode_layer_end = _sig("dv_decode_layer_end", _c_int,
                                [ctypes.POINTER(LayerWeightsC), ctypes.POINTER(Dims), ctypes.POINTER(LayerParamsC),
                                 _p, _c_int, ctypes.POINTER(LayerIOC), ctypes.POINTER(LayerIOC), _p, _c_size, _p])
_lib_dv_decode_layer_attn = _sig("dv_decode_layer_attn", _c_int,
                                 [ctypes.POINTER(LayerWeightsC), ctypes.POINTER(Dims), ctypes.POINTER(LayerParamsC),
                                  _p, _c_int, ctypes.POINTER(LayerIOC), ctypes.POINTER(LayerIOC), _p, _c_size, _p])
_lib_dv_decode_layer_mlp = _sig("dv_decode_layer_mlp", _c_int,
                                [ctypes.POINTER(LayerWeightsC), ctypes.POINTER(Dims), ctypes.POINTER(LayerParamsC),
                                 _p, ctypes.POINTER(LayerIOC), ctypes.POINTER(LayerIOC), _p, _c_size, _p])
_lib_dv_predict_layer = _sig("dv_predict_layer", _c_int,
                             [ctypes.POINTER(LayerWeightsC), ctypes.POINTER(Dims), ctypes.POINTER(LayerParamsC), _p,
                              ctypes.POINTER(LayerIOC), _p, _c_size, _p])
_lib_dv_decode_layer_begin_ahead = _sig("dv_decode_layer_begin_ahead", _c_int,
                                        [ctypes.POINTER(LayerWeightsC), ctypes.POINTER(Dims),
                                         ctypes.POINTER(LayerParamsC), _p, _c_int, ctypes.POINTER(LayerIOC),
                                         ctypes.POINTER(LayerIOC), _p, _c_size, ctypes.POINTER(LayerWeightsC), _p, _p,
                                         _c_size, _p])
_lib_dv_predict_layer_tail = _sig("dv_predict_layer_tail", _c_int,
                                  [ctypes.POINTER(LayerWeightsC), ctypes.POINTER(Dims), ctypes.POINTER(LayerParamsC),
                                   ctypes.POINTER(LayerIOC), _c_int, _p, _c_size, _p])
DV_SET_HEADS, DV_SET_NEURONS = 1, 2
_lib_dv_layernorm = _sig("dv_layernorm", _c_int, [_p, _c_int, _c_int, _p, _p, _c_float, _p, _p])
_lib_dv_topk_static = _sig("dv_topk_static", _c_int, [_p, _c_int, _c_int, _c_int, _c_float, _c_int, _p, _p, _p])
_lib_dv_prefetch_layer = _sig("dv_prefetch_layer", _c_int,
                              [ctypes.POINTER(LayerWeightsC), ctypes.POINTER(Dims), ctypes.POINTER(LayerIOC), _c_int,
                               _c_int, _p])
_lib_dv_launch_count = _sig("dv_launch_count", ctypes.c_uint64, [])


def exported_symbols_declared_in_header() -> List[str]:
    """Function names include/dejavu.h declares (for the export check)."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:[\w\s\*]+?)\b(dv_\w+)\s*\(", text, flags=re.M)))


def library():
    return _lib


def status_string(s: int) -> str:
    return _lib_dv_status_string(int(s)).decode()


def _check(s: int, what: str):
    if s != DV_OK:
        raise DvError(s, what)


# ---------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------

_WDT = {torch.bfloat16: DV_BF16, torch.float32: DV_F32}


def _ptr(t: Optional[torch.Tensor], dtype=None, name="tensor") -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return t.data_ptr()


def _wdt(t: torch.Tensor) -> int:
    if t.dtype not in _WDT:
        raise ValueError(f"weights must be bf16 or fp32, got {t.dtype}")
    return _WDT[t.dtype]


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def dims(B=1, d=8, N=1, r=0, h=0, dh=0, cap=0, k_max=0, kh_max=0) -> Dims:
    return Dims(B, d, N, r, h, dh, cap, k_max, kh_max)


def dv_workspace_size(op: int, D: Dims) -> int:
    return int(_lib_dv_workspace_size(op, ctypes.byref(D)))


def workspace(op: int, D: Dims, device="cuda") -> torch.Tensor:
    n = dv_workspace_size(op, D)
    if n == 0:
        raise DvError(DV_ERR_ARG, "dv_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def dv_launch_count() -> int:
    return int(_lib_dv_launch_count())


def dv_read_device_status(ws: torch.Tensor, stream=None) -> int:
    out = _c_int(0)
    _check(_lib_dv_read_device_status(_ptr(ws, torch.uint8, "ws"), _stream(stream), ctypes.byref(out)),
           "dv_read_device_status")
    return out.value


# ---------------------------------------------------------------------------
# entry points
# ---------------------------------------------------------------------------


def dv_predict_mlp(y, At, Bm, b1, k, scores, idx, count, ws, tau=0.0, mode=DV_TOPK, stream=None):
    B, d = y.shape
    r, N = At.shape[0], Bm.shape[0]
    _check(_lib_dv_predict_mlp(_ptr(y, torch.float32, "y"), B, d, r, N, _ptr(At, None, "At"), _ptr(Bm, At.dtype, "Bm"),
                               _ptr(b1, torch.float32, "b1"), _wdt(At), int(k), float(tau), int(mode),
                               _ptr(scores, torch.float32, "scores"), _ptr(idx, torch.int32, "idx"),
                               _ptr(count, torch.int32, "count"), _ptr(ws, torch.uint8, "ws"), ws.numel(),
                               _stream(stream)), "dv_predict_mlp")


def dv_predict_heads(y, PA, k_h, scores, head_idx, head_count, ws, tau=0.0, mode=DV_TOPK, stream=None):
    B, d = y.shape
    h = PA.shape[0]
    _check(_lib_dv_predict_heads(_ptr(y, torch.float32, "y"), B, d, h, _ptr(PA, None, "PA"), _wdt(PA), int(k_h),
                                 float(tau), int(mode), _ptr(scores, torch.float32, "scores"),
                                 _ptr(head_idx, torch.int32, "head_idx"), _ptr(head_count, torch.int32, "head_count"),
                                 _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)), "dv_predict_heads")


def dv_topk(scores, k, idx, count, ws, tau=0.0, mode=DV_TOPK, stream=None):
    B, n = scores.shape
    _check(_lib_dv_topk(_ptr(scores, torch.float32, "scores"), B, n, int(k), float(tau), int(mode),
                        _ptr(idx, torch.int32, "idx"), _ptr(count, torch.int32, "count"), _ptr(ws, torch.uint8, "ws"),
                        ws.numel(), _stream(stream)), "dv_topk")


def dv_topk_static(scores, k, idx, count, tau=0.0, mode=DV_TOPK, stream=None):
    """dv_topk without a workspace: the scratch is the library's file-scope
    device array (at most 16 rows of 65536 scores)."""
    B, n = scores.shape
    _check(_lib_dv_topk_static(_ptr(scores, torch.float32, "scores"), B, n, int(k), float(tau), int(mode),
                               _ptr(idx, torch.int32, "idx"), _ptr(count, torch.int32, "count"), _stream(stream)),
           "dv_topk_static")


def dv_sparse_mlp(y, W1t, b1, W2t, b2, idx, count, k_max, out, ws, accumulate=False, stream=None, act=DV_ACT_RELU):
    """dv_sparse_mlp (ReLU), or dv_sparse_mlp_act with another activation."""
    B, d = y.shape
    N = W1t.shape[0]
    args = [_ptr(y, torch.float32, "y"), B, d, N, _ptr(W1t, None, "W1t"), _ptr(b1, torch.float32, "b1"),
            _ptr(W2t, W1t.dtype, "W2t"), _ptr(b2, torch.float32, "b2"), _wdt(W1t), _ptr(idx, torch.int32, "idx"),
            _ptr(count, torch.int32, "count"), int(k_max), _ptr(out, torch.float32, "out"), int(bool(accumulate))]
    tail = [_ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)]
    if act == DV_ACT_RELU:
        _check(_lib_dv_sparse_mlp(*args, *tail), "dv_sparse_mlp")
    else:
        _check(_lib_dv_sparse_mlp_act(*args, int(act), *tail), "dv_sparse_mlp_act")


def dv_sparse_mlp_q8(y, W1q, W1s, b1, W2q, W2s, b2, idx, count, k_max, out, ws, accumulate=False, act=DV_ACT_RELU,
                     stream=None):
    """dv_sparse_mlp_q8: int8 rows W1q, W2q [N][d] with fp32 row scales W1s, W2s [N]."""
    B, d = y.shape
    N = W1q.shape[0]
    _check(_lib_dv_sparse_mlp_q8(_ptr(y, torch.float32, "y"), B, d, N, _ptr(W1q, torch.int8, "W1q"),
                                 _ptr(W1s, torch.float32, "W1s"), _ptr(b1, torch.float32, "b1"),
                                 _ptr(W2q, torch.int8, "W2q"), _ptr(W2s, torch.float32, "W2s"),
                                 _ptr(b2, torch.float32, "b2"), _ptr(idx, torch.int32, "idx"),
                                 _ptr(count, torch.int32, "count"), int(k_max), _ptr(out, torch.float32, "out"),
                                 int(bool(accumulate)), int(act), _ptr(ws, torch.uint8, "ws"), ws.numel(),
                                 _stream(stream)), "dv_sparse_mlp_q8")


def dv_sparse_mha_q8(y, Wqkvq, Wqkv_s, bqkv, WOq, WO_s, bO, Kc, Vc, pos, scale, head_idx, head_count, kh_max, out, ws,
                     accumulate=False, stream=None):
    """dv_sparse_mha_q8: int8 rows Wqkvq [h][3][dh][d], WOq [h][dh][d] with fp32 row scales
    Wqkv_s [h][3][dh], WO_s [h][dh]; bf16 KV caches [B][h][cap][dh]."""
    B, d = y.shape
    h, _, dh, _ = Wqkvq.shape
    cap = Kc.shape[2]
    _check(_lib_dv_sparse_mha_q8(_ptr(y, torch.float32, "y"), B, d, h, dh, _ptr(Wqkvq, torch.int8, "Wqkvq"),
                                 _ptr(Wqkv_s, torch.float32, "Wqkv_s"), _ptr(bqkv, torch.float32, "bqkv"),
                                 _ptr(WOq, torch.int8, "WOq"), _ptr(WO_s, torch.float32, "WO_s"),
                                 _ptr(bO, torch.float32, "bO"), _ptr(Kc, torch.bfloat16, "Kc"),
                                 _ptr(Vc, torch.bfloat16, "Vc"), int(cap), int(pos), float(scale),
                                 _ptr(head_idx, torch.int32, "head_idx"), _ptr(head_count, torch.int32, "head_count"),
                                 int(kh_max), _ptr(out, torch.float32, "out"), int(bool(accumulate)),
                                 _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)), "dv_sparse_mha_q8")


def dv_sparse_mha(y, Wqkv, bqkv, WOt, bO, Kc, Vc, pos, scale, head_idx, head_count, kh_max, out, ws,
                  accumulate=False, stream=None):
    B, d = y.shape
    h, _, dh, _ = Wqkv.shape
    cap = Kc.shape[2]
    _check(_lib_dv_sparse_mha(_ptr(y, torch.float32, "y"), B, d, h, dh, _ptr(Wqkv, None, "Wqkv"),
                              _ptr(bqkv, torch.float32, "bqkv"), _ptr(WOt, Wqkv.dtype, "WOt"),
                              _ptr(bO, torch.float32, "bO"), _wdt(Wqkv), _ptr(Kc, None, "Kc"),
                              _ptr(Vc, Kc.dtype, "Vc"), _wdt(Kc), cap, int(pos), float(scale),
                              _ptr(head_idx, torch.int32, "head_idx"), _ptr(head_count, torch.int32, "head_count"),
                              int(kh_max), _ptr(out, torch.float32, "out"), int(bool(accumulate)),
                              _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)), "dv_sparse_mha")


def dv_layernorm(x, y, g=None, beta=None, eps=1e-5, stream=None):
    B, d = x.shape
    _check(_lib_dv_layernorm(_ptr(x, torch.float32, "x"), B, d, _ptr(g, torch.float32, "g"),
                             _ptr(beta, torch.float32, "beta"), float(eps), _ptr(y, torch.float32, "y"),
                             _stream(stream)), "dv_layernorm")


class Layer:
    """Marshals one layer's tensors (workload.make_layer layout) into the
    dv_layer_weights struct, keeping the tensors alive."""

    def __init__(self, t: Dict[str, torch.Tensor], B: int, k_max: int, kh_max: int):
        self.t = t
        W1t, Wqkv, K = t["W1t"], t["Wqkv"], t["K"]
        N, d = W1t.shape
        h, _, dh, _ = Wqkv.shape
        r, cap = t["At"].shape[0], K.shape[2]
        # every tensor's extent against the dims the library will index with
        # (the C ABI sees pointers only, so a short tensor would be read past
        # its end)
        want = {"W1t": (N, d), "W2t": (N, d), "PA": (h, d), "Wqkv": (h, 3, dh, d), "WOt": (h, dh, d),
                "K": (B, h, cap, dh), "V": (B, h, cap, dh), "At": (r, d), "Bm": (N, r), "b1": (N,), "b2": (d,),
                "bqkv": (h, 3, dh), "bO": (d,), "ln1_g": (d,), "ln1_b": (d,), "ln2_g": (d,), "ln2_b": (d,)}
        for n, shp in want.items():
            v = t.get(n)
            if v is None:
                continue
            got = tuple(v.shape)
            if n in ("K", "V"):  # a cache with more batch rows than B: its first B rows are used
                ok = len(got) == 4 and got[0] >= B and got[1:] == shp[1:]
            else:
                ok = got == shp
            if not ok or not v.is_contiguous():
                raise ValueError(f"{n}: shape {got}, expected {shp} (contiguous) for batch {B}")
        self.dims = Dims(B, d, N, r, h, dh, cap, k_max, kh_max)
        g = lambda n, dt=None: _ptr(t.get(n), dt, n)  # noqa: E731
        self.c = LayerWeightsC(_wdt(W1t), _wdt(K), g("ln1_g", torch.float32), g("ln1_b", torch.float32), g("PA"),
                               g("Wqkv"), g("bqkv", torch.float32), g("WOt"), g("bO", torch.float32), g("K"), g("V"),
                               g("ln2_g", torch.float32), g("ln2_b", torch.float32), g("At"), g("Bm"),
                               g("b1", torch.float32), g("W1t"), g("W2t"), g("b2", torch.float32))


def params(k, k_h, scale, eps=1e-5, tau=0.0, mode=DV_TOPK, tau_h=0.0, mode_h=DV_TOPK, act=DV_ACT_RELU,
           exact_kv=False) -> LayerParamsC:
    return LayerParamsC(int(k), float(tau), int(mode), int(k_h), float(tau_h), int(mode_h), float(scale), float(eps),
                        int(act), int(bool(exact_kv)))


def layer_io(yA=None, scores_h=None, head_idx=None, head_count=None, yM=None, scores=None, idx=None,
             count=None) -> LayerIOC:
    return LayerIOC(_ptr(yA, torch.float32, "yA"), _ptr(scores_h, torch.float32, "scores_h"),
                    _ptr(head_idx, torch.int32, "head_idx"), _ptr(head_count, torch.int32, "head_count"),
                    _ptr(yM, torch.float32, "yM"), _ptr(scores, torch.float32, "scores"),
                    _ptr(idx, torch.int32, "idx"), _ptr(count, torch.int32, "count"))


def dv_decode_layer(layer: Layer, p: LayerParamsC, x, pos, ws, sel: Optional[LayerIOC] = None,
                    trace: Optional[LayerIOC] = None, stream=None):
    _check(_lib_dv_decode_layer(ctypes.byref(layer.c), ctypes.byref(layer.dims), ctypes.byref(p),
                                _ptr(x, torch.float32, "x"), int(pos), ctypes.byref(sel) if sel is not None else None,
                                ctypes.byref(trace) if trace is not None else None, _ptr(ws, torch.uint8, "ws"),
                                ws.numel(), _stream(stream)), "dv_decode_layer")


def _layer_call(fn, name, layer, p, x, pos, ws, sel, trace, stream):
    _check(fn(ctypes.byref(layer.c), ctypes.byref(layer.dims), ctypes.byref(p), _ptr(x, torch.float32, "x"), int(pos),
              ctypes.byref(sel) if sel is not None else None, ctypes.byref(trace) if trace is not None else None,
              _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)), name)


def dv_decode_layer_begin(layer: Layer, p: LayerParamsC, x, pos, ws, sel: Optional[LayerIOC] = None,
                          trace: Optional[LayerIOC] = None, stream=None):
    _layer_call(_lib_dv_decode_layer_begin, "dv_decode_layer_begin", layer, p, x, pos, ws, sel, trace, stream)


def dv_decode_layer_end(layer: Layer, p: LayerParamsC, x, pos, ws, sel: Optional[LayerIOC] = None,
                        trace: Optional[LayerIOC] = None, stream=None):
    _layer_call(_lib_dv_decode_layer_end, "dv_decode_layer_end", layer, p, x, pos, ws, sel, trace, stream)


def dv_decode_layer_attn(layer: Layer, p: LayerParamsC, x, pos, ws, sel: Optional[LayerIOC] = None,
                         trace: Optional[LayerIOC] = None, stream=None):
    _layer_call(_lib_dv_decode_layer_attn, "dv_decode_layer_attn", layer, p, x, pos, ws, sel, trace, stream)


def dv_decode_layer_mlp(layer: Layer, p: LayerParamsC, x, ws, sel: Optional[LayerIOC] = None,
                        trace: Optional[LayerIOC] = None, stream=None):
    _check(_lib_dv_decode_layer_mlp(ctypes.byref(layer.c), ctypes.byref(layer.dims), ctypes.byref(p),
                                    _ptr(x, torch.float32, "x"), ctypes.byref(sel) if sel is not None else None,
                                    ctypes.byref(trace) if trace is not None else None, _ptr(ws, torch.uint8, "ws"),
                                    ws.numel(), _stream(stream)), "dv_decode_layer_mlp")


def dv_predict_layer(layer: Layer, p: LayerParamsC, y, out: LayerIOC, ws, stream=None):
    _check(_lib_dv_predict_layer(ctypes.byref(layer.c), ctypes.byref(layer.dims), ctypes.byref(p),
                                 _ptr(y, torch.float32, "y"), ctypes.byref(out), _ptr(ws, torch.uint8, "ws"),
                                 ws.numel(), _stream(stream)), "dv_predict_layer")


def dv_decode_layer_begin_ahead(layer: Layer, p: LayerParamsC, x, pos, ws, nxt: Layer, next_scores_h, next_ws,
                                sel: Optional[LayerIOC] = None, trace: Optional[LayerIOC] = None, stream=None):
    _check(_lib_dv_decode_layer_begin_ahead(
        ctypes.byref(layer.c), ctypes.byref(layer.dims), ctypes.byref(p), _ptr(x, torch.float32, "x"), int(pos),
        ctypes.byref(sel) if sel is not None else None, ctypes.byref(trace) if trace is not None else None,
        _ptr(ws, torch.uint8, "ws"), ws.numel(), ctypes.byref(nxt.c), _ptr(next_scores_h, torch.float32, "scores_h"),
        _ptr(next_ws, torch.uint8, "next_ws"), next_ws.numel(), _stream(stream)), "dv_decode_layer_begin_ahead")


def dv_predict_layer_tail(layer: Layer, p: LayerParamsC, out: LayerIOC, ws, sets=DV_SET_HEADS | DV_SET_NEURONS,
                          stream=None):
    _check(_lib_dv_predict_layer_tail(ctypes.byref(layer.c), ctypes.byref(layer.dims), ctypes.byref(p),
                                      ctypes.byref(out), int(sets), _ptr(ws, torch.uint8, "ws"), ws.numel(),
                                      _stream(stream)), "dv_predict_layer_tail")


def dv_prefetch_layer(layer: Layer, sel: LayerIOC, pos, with_w2=True, stream=None):
    _check(_lib_dv_prefetch_layer(ctypes.byref(layer.c), ctypes.byref(layer.dims), ctypes.byref(sel), int(pos),
                                  int(bool(with_w2)), _stream(stream)), "dv_prefetch_layer")
