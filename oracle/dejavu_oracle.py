"""Plain, slow CPU oracle for the Deja Vu contextual-sparsity decode step.

TEST INFRASTRUCTURE ONLY. This module is imported by ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs
of ``bench.py``, and by nothing else. The product path (the CUDA library and
its Python binding) never imports it, and it imports nothing from the product.

Everything is computed in float64 with numpy. Weights arrive either as float32
arrays or as bfloat16 bit patterns (``uint16`` arrays) and are decoded exactly.
There is no blocking, fusion or reordering beyond what the definitions state.

Sources (page title, then section / equation):

* "Deja Vu: 利用上下文稀疏性提升大语言模型推理效率" (dtcms.com translation of the
  Deja Vu paper), referred to below as [DejaVu]:
    - §2.3 eq. (1): the sparsified MLP, sigma(y W1_{S_M}) (W2_{S_M})^T, with
      W1, W2 in R^{d x 4d} and neuron i being column i of each;
    - §2.3 eq. (2): the sparsified MHA, sum_{i in S_A} H_i(y) W_i^O with
      H_i(y) = D_i(y)^{-1} exp(y W_i^Q (W_i^K)^T X^T) X W_i^V and
      D_i(y) = exp(...) 1_n;
    - §2.3, last paragraph: S_M and S_A are chosen under a compute budget;
    - §1 (list of contributions): a cheap learned predictor per layer, and an
      asynchronous look-ahead predictor that, from one layer's input, predicts
      the sets of the next layer;
    - §3.2: the mean-shift form of one head, m_i(y), and Normalize(y + y~).
* itpub blog on KV caching, figure (b): at decode time the new K and V are
  concatenated with the stored ones before the softmax, and then stored.
* "A Survey on Efficient Inference for Large Language Models" (reading note),
  Transformer section: head outputs are concatenated and projected by W^O.

Readings where the pages are silent or garbled:

* predictor: rank-r factors, s = (y A) B^T + b1, with A = At^T (the pages' §4.1
  is not part of the extraction); head predictor: one linear map P_A [h][d];
* softmax scale is an argument (eq. (2) literally has scale 1); the softmax is
  max-subtracted, which is the same function;
* the current token's k and v are appended at slot ``pos`` before attending
  over slots 0..pos; they are stored rounded to the cache dtype and read back
  rounded;
* selection ties go to the lower index, -0.0 equals +0.0, NaN ranks below
  -inf; threshold mode keeps s > tau (strict); for batch > 1 the selected set
  is the union over rows;
* decoder layer: pre-LayerNorm, attention block then MLP block, each added to
  the residual stream.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np

# ----------------------------------------------------------------------------
# bfloat16 decoding / encoding (plain definitions of the number format)
# ----------------------------------------------------------------------------


def bf16_bits_to_f64(u16) -> np.ndarray:
    """Decode bfloat16 bit patterns exactly: they are the top 16 bits of an
    IEEE-754 binary32 whose low 16 bits are zero."""
    u = np.asarray(u16).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def round_to_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value, ties to even, and
    return them as float64. bfloat16 keeps 8 significant bits, exponent range
    of binary32 (smallest subnormal 2^-133, largest finite (2 - 2^-7) 2^127)."""
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, copy=True)
    finite = np.isfinite(x) & (x != 0)
    m, e = np.frexp(x[finite])  # x = m 2^e, 0.5 <= |m| < 1
    # 8 significant bits: the unit in the last place is 2^(e-8), but never
    # below the subnormal spacing 2^-133 (= 2^(-125-8)).
    ulp_exp = np.maximum(e, -125) - 8
    q = np.ldexp(np.ones_like(m), ulp_exp)
    r = np.rint(x[finite] / q) * q  # np.rint rounds half to even
    big = (2.0 - 2.0 ** -7) * 2.0 ** 127
    r = np.where(np.abs(r) > big, np.copysign(np.inf, r), r)
    out[finite] = r
    return out


def f64_to_bf16_bits(x) -> np.ndarray:
    """bfloat16 bit patterns of round_to_bf16(x)."""
    r = round_to_bf16(x).astype(np.float32)  # exact: r is a bfloat16 value
    return (r.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def dequantize_rows(q, scale) -> np.ndarray:
    """Weight-only int8 rows with one scale per row: the real weight row i is
    q[i] * scale[i], rows running along the last axis of q (so scale has q's
    shape without that axis). Exact in float64 (an int8 times a binary32)."""
    q = np.asarray(q).astype(np.float64)
    s = np.asarray(scale, dtype=np.float32).astype(np.float64)
    return q * s[..., None]


def as_f64(a, dtype: str) -> np.ndarray:
    """Decode a weight array given as float32 ('f32') or bf16 bits ('bf16')."""
    if dtype == "bf16":
        return bf16_bits_to_f64(a)
    if dtype == "f32":
        return np.asarray(a, dtype=np.float32).astype(np.float64)
    raise ValueError(dtype)


# ----------------------------------------------------------------------------
# LayerNorm and residual ([DejaVu] §3.2: Normalize(y + y~); §1: residual
# connections make consecutive layers' inputs similar)
# ----------------------------------------------------------------------------


def layernorm(x, eps: float = 1e-5, gamma=None, beta=None) -> np.ndarray:
    """y = (x - mean(x)) / sqrt(var(x) + eps) * gamma + beta over the last
    axis, with the biased variance (divide by d)."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    y = (x - mu) / np.sqrt(var + eps)
    if gamma is not None:
        y = y * np.asarray(gamma, dtype=np.float64)
    if beta is not None:
        y = y + np.asarray(beta, dtype=np.float64)
    return y


# ----------------------------------------------------------------------------
# Predictors ([DejaVu] §1: the sets are predicted from the similarity between
# the layer's parameters and its input; the predictor's architecture is not in
# the extracted text, so it is a rank-r linear map here)
# ----------------------------------------------------------------------------


def mlp_predictor_scores(y, At, Bm, b1) -> np.ndarray:
    """Neuron scores s = (y A) B^T + b1, where A = At^T is d x r and
    B = Bm is N x r. y: [B][d]; returns [B][N]."""
    y = np.atleast_2d(np.asarray(y, dtype=np.float64))
    z = y @ np.asarray(At, dtype=np.float64).T  # [B][r]
    return z @ np.asarray(Bm, dtype=np.float64).T + np.asarray(b1, dtype=np.float64)


def head_predictor_scores(y, PA) -> np.ndarray:
    """Head scores s_A = y P_A^T, P_A is h x d. y: [B][d]; returns [B][h]."""
    y = np.atleast_2d(np.asarray(y, dtype=np.float64))
    return y @ np.asarray(PA, dtype=np.float64).T


# ----------------------------------------------------------------------------
# Selection ([DejaVu] §2.3: choose S_M / S_A under a budget)
# ----------------------------------------------------------------------------


def topk_row(scores, k: int) -> np.ndarray:
    """Indices of the k largest scores of one row, returned in ascending index
    order. Order: larger score first; equal scores by lower index; -0.0 and
    +0.0 are equal; NaN is below every number (including -inf)."""
    s = np.asarray(scores, dtype=np.float64).ravel()
    n = s.shape[0]
    k = max(0, min(int(k), n))
    isnan = np.isnan(s)
    clean = np.where(isnan, 0.0, s)
    clean = np.where(clean == 0.0, 0.0, clean)  # -0.0 -> +0.0
    order = np.lexsort((np.arange(n), -clean, isnan.astype(np.int8)))
    return np.sort(order[:k]).astype(np.int64)


def threshold_row(scores, tau: float) -> np.ndarray:
    """Indices i with s_i > tau (strict; NaN never passes), ascending."""
    s = np.asarray(scores, dtype=np.float64).ravel()
    return np.nonzero(s > float(tau))[0].astype(np.int64)


def select(scores, k: int = 0, tau: float = 0.0, mode: str = "topk") -> np.ndarray:
    """Selected index set for a batch of score rows: the per-row top-k (or
    threshold) sets, united over the rows, sorted ascending, unique."""
    S = np.atleast_2d(np.asarray(scores))
    sets = []
    for row in S:
        sets.append(topk_row(row, k) if mode == "topk" else threshold_row(row, tau))
    out = np.zeros(0, dtype=np.int64)
    for st in sets:
        out = np.union1d(out, st)
    return out.astype(np.int64)


# ----------------------------------------------------------------------------
# Sparsified MLP, [DejaVu] §2.3 eq. (1)
# ----------------------------------------------------------------------------


def relu(v):
    return np.maximum(v, 0.0)


def gelu(v):
    """GeLU, the exact (erf) form: v * Phi(v)."""
    from math import erf, sqrt

    f = np.vectorize(lambda t: 0.5 * t * (1.0 + erf(t / sqrt(2.0))))
    return f(np.asarray(v, dtype=np.float64)) if np.size(v) else np.asarray(v, dtype=np.float64)


def sparse_mlp(y, W1t, b1, W2t, b2, idx, act: str = "relu") -> np.ndarray:
    """MLP_{S_M}(y) = sigma(y W1_{S_M} + b1_{S_M}) (W2_{S_M})^T (+ b2).

    W1t, W2t are neuron-major: row i holds column W1_i (resp. W2_i), so
    W1_{S_M} = W1t[S_M]^T. b1 is gathered with the selected neurons; b2 is
    added once. y: [B][d]; returns [B][d]."""
    y = np.atleast_2d(np.asarray(y, dtype=np.float64))
    idx = np.asarray(idx, dtype=np.int64)
    W1S = np.asarray(W1t, dtype=np.float64)[idx]  # [k][d]
    W2S = np.asarray(W2t, dtype=np.float64)[idx]  # [k][d]
    pre = y @ W1S.T
    if b1 is not None:
        pre = pre + np.asarray(b1, dtype=np.float64)[idx]
    a = relu(pre) if act == "relu" else gelu(pre)
    out = a @ W2S
    if b2 is not None:
        out = out + np.asarray(b2, dtype=np.float64)
    return out


def mlp_preactivations(y, W1t, b1) -> np.ndarray:
    """y W1 + b1 over all neurons ([B][N]); used by diagnostics and pins."""
    y = np.atleast_2d(np.asarray(y, dtype=np.float64))
    pre = y @ np.asarray(W1t, dtype=np.float64).T
    if b1 is not None:
        pre = pre + np.asarray(b1, dtype=np.float64)
    return pre


# ----------------------------------------------------------------------------
# Sparsified MHA with a KV cache, [DejaVu] §2.3 eq. (2)
# ----------------------------------------------------------------------------


@dataclass
class MHAResult:
    out: np.ndarray  # [B][d]
    H: np.ndarray  # [B][len(head_idx)][dh], per selected head, in head_idx order
    q: np.ndarray  # [B][len(head_idx)][dh]
    k_new: np.ndarray  # [B][len(head_idx)][dh], as stored (rounded)
    v_new: np.ndarray  # [B][len(head_idx)][dh], as stored (rounded)


def head_attention(q, Kh, Vh, scale: float) -> np.ndarray:
    """H = D^{-1} exp(scale q K^T) V with D = exp(scale q K^T) 1, computed with
    the maximum subtracted inside exp (the same function). q: [dh];
    Kh, Vh: [n][dh]; returns [dh]."""
    e = scale * (Kh @ q)
    p = np.exp(e - e.max())
    return (p @ Vh) / p.sum()


def sparse_mha(y, Wqkv, bqkv, WOt, bO, Kc, Vc, pos: int, scale: float, head_idx,
               kv_round: Optional[str] = "bf16") -> MHAResult:
    """MHA_{S_A}(y) = sum_{i in S_A} H_i(y) W_i^O (+ bO) over a KV cache.

    Layouts: Wqkv[h][3][dh][d] holds (W_i^Q)^T, (W_i^K)^T, (W_i^V)^T (rows are
    output channels); WOt[h][dh][d] holds W_i^O; Kc, Vc[B][h][cap][dh] hold
    the keys x_j W_i^K and values x_j W_i^V of the earlier tokens.

    For each selected head the current token's k and v are computed, rounded
    to the cache dtype (kv_round: 'bf16' or None for float32 caches, which
    round to binary32), written at slot ``pos`` of the given cache arrays (in
    place), and the head attends over slots 0..pos. Unselected heads compute
    nothing and their slot ``pos`` is left as it was."""
    y = np.atleast_2d(np.asarray(y, dtype=np.float64))
    B, d = y.shape
    head_idx = [int(i) for i in np.asarray(head_idx).ravel()]
    W = np.asarray(Wqkv, dtype=np.float64)
    WO = np.asarray(WOt, dtype=np.float64)
    dh = W.shape[2]
    out = np.zeros((B, d))
    H = np.zeros((B, len(head_idx), dh))
    Q = np.zeros_like(H)
    KN = np.zeros_like(H)
    VN = np.zeros_like(H)
    for b in range(B):
        for p, i in enumerate(head_idx):
            q = W[i, 0] @ y[b]
            k = W[i, 1] @ y[b]
            v = W[i, 2] @ y[b]
            if bqkv is not None:
                bb = np.asarray(bqkv, dtype=np.float64)
                q, k, v = q + bb[i, 0], k + bb[i, 1], v + bb[i, 2]
            if kv_round == "bf16":
                k, v = round_to_bf16(k), round_to_bf16(v)
            else:
                k = k.astype(np.float32).astype(np.float64)
                v = v.astype(np.float32).astype(np.float64)
            Kc[b, i, pos] = k
            Vc[b, i, pos] = v
            Hh = head_attention(q, Kc[b, i, : pos + 1], Vc[b, i, : pos + 1], scale)
            out[b] += Hh @ WO[i]
            H[b, p], Q[b, p], KN[b, p], VN[b, p] = Hh, q, k, v
    if bO is not None:
        out += np.asarray(bO, dtype=np.float64)
    return MHAResult(out=out, H=H, q=Q, k_new=KN, v_new=VN)


def unselected_kv(y, Wqkv, bqkv, Kc, Vc, pos: int, head_idx, kv_round: Optional[str] = "bf16"):
    """Exact KV maintenance: the current token's key and value for every head
    NOT in head_idx, rounded like the selected heads' (itpub blog on KV
    caching, figure (b): each step appends the new token's K and V for every
    head), written at slot ``pos`` of the given caches in place. With it a
    head left out at one step still holds this token when it is selected at a
    later step, as in the dense model."""
    y = np.atleast_2d(np.asarray(y, dtype=np.float64))
    W = np.asarray(Wqkv, dtype=np.float64)
    chosen = set(int(i) for i in np.asarray(head_idx).ravel())
    for i in range(W.shape[0]):
        if i in chosen:
            continue
        for b in range(y.shape[0]):
            k = W[i, 1] @ y[b]
            v = W[i, 2] @ y[b]
            if bqkv is not None:
                bb = np.asarray(bqkv, dtype=np.float64)
                k, v = k + bb[i, 1], v + bb[i, 2]
            if kv_round == "bf16":
                k, v = round_to_bf16(k), round_to_bf16(v)
            else:
                k = k.astype(np.float32).astype(np.float64)
                v = v.astype(np.float32).astype(np.float64)
            Kc[b, i, pos] = k
            Vc[b, i, pos] = v


# ----------------------------------------------------------------------------
# One decoder layer and a stack with the look-ahead predictor
# ----------------------------------------------------------------------------


@dataclass
class LayerF64:
    """One layer's parameters, decoded to float64. Caches are float64 copies
    that sparse_mha updates in place."""

    PA: np.ndarray
    Wqkv: np.ndarray
    bqkv: Optional[np.ndarray]
    WOt: np.ndarray
    bO: Optional[np.ndarray]
    K: np.ndarray
    V: np.ndarray
    At: np.ndarray
    Bm: np.ndarray
    b1: np.ndarray
    W1t: np.ndarray
    W2t: np.ndarray
    b2: Optional[np.ndarray] = None
    ln1_g: Optional[np.ndarray] = None
    ln1_b: Optional[np.ndarray] = None
    ln2_g: Optional[np.ndarray] = None
    ln2_b: Optional[np.ndarray] = None
    kv_round: Optional[str] = "bf16"


@dataclass
class LayerParams:
    k: int
    k_h: int
    tau: float = 0.0
    tau_h: float = 0.0
    mode: str = "topk"
    mode_h: str = "topk"
    scale: float = 0.125
    eps: float = 1e-5
    act: str = "relu"
    exact_kv: bool = False


@dataclass
class LayerTrace:
    yA: np.ndarray = None
    scores_h: np.ndarray = None
    head_idx: np.ndarray = None
    out_A: np.ndarray = None
    yM: np.ndarray = None
    scores: np.ndarray = None
    idx: np.ndarray = None
    out_M: np.ndarray = None
    x_out: np.ndarray = None
    mha: MHAResult = None


def decode_layer(x, L: LayerF64, P: LayerParams, pos: int, head_idx=None, idx=None) -> LayerTrace:
    """One decode step of one pre-LN decoder layer with contextual sparsity:

        yA = LN1(x);  S_A = select(y_A P_A^T)       (unless head_idx is given)
        x1 = x + MHA_{S_A}(yA)                       (eq. (2), appends k, v at pos;
                                                      with P.exact_kv every head's k, v)
        yM = LN2(x1); S_M = select((yM A) B^T + b1)  (unless idx is given)
        x2 = x1 + MLP_{S_M}(yM)                      (eq. (1))
    """
    t = LayerTrace()
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    t.yA = layernorm(x, P.eps, L.ln1_g, L.ln1_b)
    t.scores_h = head_predictor_scores(t.yA, L.PA)
    t.head_idx = (select(t.scores_h, P.k_h, P.tau_h, P.mode_h) if head_idx is None
                  else np.asarray(head_idx, dtype=np.int64))
    t.mha = sparse_mha(t.yA, L.Wqkv, L.bqkv, L.WOt, L.bO, L.K, L.V, pos, P.scale,
                       t.head_idx, L.kv_round)
    if P.exact_kv:
        unselected_kv(t.yA, L.Wqkv, L.bqkv, L.K, L.V, pos, t.head_idx, L.kv_round)
    t.out_A = t.mha.out
    x1 = x + t.out_A
    t.yM = layernorm(x1, P.eps, L.ln2_g, L.ln2_b)
    t.scores = mlp_predictor_scores(t.yM, L.At, L.Bm, L.b1)
    t.idx = (select(t.scores, P.k, P.tau, P.mode) if idx is None
             else np.asarray(idx, dtype=np.int64))
    t.out_M = sparse_mlp(t.yM, L.W1t, L.b1, L.W2t, L.b2, t.idx, P.act)
    t.x_out = x1 + t.out_M
    return t


def lookahead_selection(yA_prev, L_next: LayerF64, P: LayerParams):
    """[DejaVu] §1: from one layer's (normalised) input, predict the head set
    and the neuron set of the next layer. Returns (head_idx, idx)."""
    sh = head_predictor_scores(yA_prev, L_next.PA)
    sm = mlp_predictor_scores(yA_prev, L_next.At, L_next.Bm, L_next.b1)
    return (select(sh, P.k_h, P.tau_h, P.mode_h), select(sm, P.k, P.tau, P.mode), sh, sm)


def decode_stack(x, layers: Sequence[LayerF64], P: LayerParams, pos: int,
                 lookahead: bool = True, sel_override=None):
    """One token through a stack of layers. With look-ahead, layer 0 selects
    from its own block inputs and every later layer l uses the sets predicted
    from layer l-1's attention input yA_{l-1}. ``sel_override[l]`` (optional)
    supplies (head_idx, idx) per layer instead, for parity against sets a GPU
    emitted. Returns (x_out, traces)."""
    traces = []
    pending = None
    for l, L in enumerate(layers):
        if sel_override is not None and sel_override[l] is not None:
            hi, ii = sel_override[l]
        elif lookahead and pending is not None:
            hi, ii = pending
        else:
            hi, ii = None, None
        t = decode_layer(x, L, P, pos, head_idx=hi, idx=ii)
        if lookahead and l + 1 < len(layers):
            h2, i2, _, _ = lookahead_selection(t.yA, layers[l + 1], P)
            pending = (h2, i2)
        traces.append(t)
        x = t.x_out
    return x, traces


# ----------------------------------------------------------------------------
# Diagnostics (not parity): predictor recall, ground-truth selection by norm
# ([DejaVu] §3.1: first pass records heads / neurons with large output norm)
# ----------------------------------------------------------------------------


def neuron_recall(idx, pre_row) -> float:
    """Fraction of truly active neurons (preactivation > 0) that idx contains."""
    active = set(np.nonzero(np.asarray(pre_row) > 0)[0].tolist())
    if not active:
        return 1.0
    return len(active & set(np.asarray(idx).tolist())) / len(active)


def heads_by_output_norm(y, Wqkv, bqkv, WOt, Kc, Vc, pos, scale, k_h, kv_round="bf16"):
    """The k_h heads whose contribution H_i(y) W_i^O has the largest L2 norm
    (all heads evaluated densely on copies of the caches)."""
    h = np.asarray(Wqkv).shape[0]
    Kx, Vx = np.array(Kc, copy=True), np.array(Vc, copy=True)
    r = sparse_mha(y, Wqkv, bqkv, WOt, None, Kx, Vx, pos, scale, list(range(h)), kv_round)
    WO = np.asarray(WOt, dtype=np.float64)
    norms = np.array([np.linalg.norm(r.H[0, i] @ WO[i]) for i in range(h)])
    return topk_row(norms, k_h)
