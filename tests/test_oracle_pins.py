"""Pins of the CPU oracle against things other than itself.

Each test checks one oracle function against a library routine, a closed
form, an invariant the pages state, or brute force on tiny inputs, chosen so
that a dropped term, a wrong sign or index, or a transposed operand fails.
CPU only.
"""

from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import dejavu_oracle as O


def rng(seed=0):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------------
# number formats and LayerNorm vs library routines
# --------------------------------------------------------------------------


def test_bf16_round_matches_torch_on_binary32_values():
    r = rng(1)
    x = np.concatenate([
        r.standard_normal(20000).astype(np.float32),
        (r.standard_normal(2000) * 1e-38).astype(np.float32),  # subnormal range
        (r.standard_normal(2000) * 1e38).astype(np.float32),  # near overflow
        np.array([0.0, -0.0, 1.0, -1.0, 3.3895314e38, 1.00390625, 1.01171875], np.float32),
    ])
    # values exactly half-way between two bf16 numbers (ties to even)
    ties = (np.arange(1, 200, dtype=np.uint32) << 16) | 0x8000
    x = np.concatenate([x, (ties | 0x3F800000).view(np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.f64_to_bf16_bits(x.astype(np.float64))
    assert np.array_equal(got, ref)
    back = O.bf16_bits_to_f64(ref)
    assert np.array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_layernorm_matches_torch():
    r = rng(2)
    x = r.standard_normal((3, 96)) * 3 + 1.5
    g, b = r.standard_normal(96), r.standard_normal(96)
    ref = F.layer_norm(torch.from_numpy(x), (96,), torch.from_numpy(g), torch.from_numpy(b), 1e-5).numpy()
    assert np.allclose(O.layernorm(x, 1e-5, g, b), ref, rtol=1e-12, atol=1e-12)
    ref0 = F.layer_norm(torch.from_numpy(x), (96,), eps=1e-5).numpy()
    assert np.allclose(O.layernorm(x), ref0, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# eq. (1): sparsified MLP
# --------------------------------------------------------------------------


def _mlp_weights(r, d, N):
    W1t = r.standard_normal((N, d)) / np.sqrt(d)
    W2t = r.standard_normal((N, d)) / np.sqrt(d)
    b1 = r.standard_normal(N) * 0.5
    b2 = r.standard_normal(d) * 0.1
    return W1t, b1, W2t, b2


def _torch_ffn(y, W1t, b1, W2t, b2):
    """Dense FFN as in the survey note's FeedForwardNetwork: Linear -> ReLU ->
    Linear, built from torch.nn.Linear (weights d_model->d_ff and back)."""
    d, N = W1t.shape[1], W1t.shape[0]
    lin1 = torch.nn.Linear(d, N, dtype=torch.float64)
    lin2 = torch.nn.Linear(N, d, dtype=torch.float64)
    with torch.no_grad():
        lin1.weight.copy_(torch.from_numpy(W1t))  # [N][d]: row i = W1_i
        lin1.bias.copy_(torch.from_numpy(b1))
        lin2.weight.copy_(torch.from_numpy(W2t.T.copy()))  # [d][N]
        lin2.bias.copy_(torch.from_numpy(b2))
        return lin2(torch.relu(lin1(torch.from_numpy(y)))).numpy()


def test_sparse_mlp_all_neurons_is_dense_ffn():
    r = rng(3)
    d, N = 32, 128
    W1t, b1, W2t, b2 = _mlp_weights(r, d, N)
    y = r.standard_normal((2, d))
    got = O.sparse_mlp(y, W1t, b1, W2t, b2, np.arange(N))
    assert np.allclose(got, _torch_ffn(y, W1t, b1, W2t, b2), rtol=1e-12, atol=1e-12)


def test_relu_positive_set_reproduces_dense_exactly():
    """§2.3: with ReLU the first layer's activations are sparse, so the set of
    positive preactivations gives the dense output."""
    r = rng(4)
    d, N = 48, 192
    W1t, b1, W2t, b2 = _mlp_weights(r, d, N)
    b1 = b1 - 1.0
    y = r.standard_normal((1, d))
    pre = y @ W1t.T + b1
    S = np.nonzero(pre[0] > 0)[0]
    assert 0 < len(S) < N // 2
    got = O.sparse_mlp(y, W1t, b1, W2t, b2, S)
    assert np.allclose(got, _torch_ffn(y, W1t, b1, W2t, b2), rtol=1e-12, atol=1e-12)
    # dropping one positive neuron must change the output
    assert not np.allclose(O.sparse_mlp(y, W1t, b1, W2t, b2, S[1:]), got, rtol=1e-9, atol=1e-12)


def test_sparse_mlp_brute_force_fractions():
    """Exact rational evaluation of sigma(y W1_S + b1_S)(W2_S)^T + b2 with
    explicit loops over the columns W1_i, W2_i (tiny d)."""
    r = rng(5)
    d, N = 6, 24
    W1 = [[Fraction(int(v), 16) for v in r.integers(-16, 17, size=N)] for _ in range(d)]  # d x N
    W2 = [[Fraction(int(v), 16) for v in r.integers(-16, 17, size=N)] for _ in range(d)]
    b1 = [Fraction(int(v), 8) for v in r.integers(-8, 9, size=N)]
    y = [Fraction(int(v), 4) for v in r.integers(-8, 9, size=d)]
    S = [1, 4, 5, 9, 13, 17, 22]
    expect = [Fraction(0)] * d
    for i in S:
        pre = sum(y[j] * W1[j][i] for j in range(d)) + b1[i]
        a = pre if pre > 0 else Fraction(0)
        for c in range(d):
            expect[c] += a * W2[c][i]
    W1t = np.array([[float(W1[j][i]) for j in range(d)] for i in range(N)])
    W2t = np.array([[float(W2[c][i]) for c in range(d)] for i in range(N)])
    got = O.sparse_mlp(np.array([[float(v) for v in y]]), W1t, np.array([float(v) for v in b1]),
                       W2t, None, np.array(S))
    assert np.array_equal(got[0], np.array([float(v) for v in expect]))


def test_full_rank_predictor_equals_preactivations_and_threshold_zero_is_dense():
    """With rank r = d, the SVD factors reproduce y W1 exactly, so the scores
    equal the preactivations and tau = 0 selects exactly the positive set."""
    r = rng(6)
    d, N = 16, 64
    W1t, b1, W2t, b2 = _mlp_weights(r, d, N)
    U, s, Vt = np.linalg.svd(W1t.T, full_matrices=False)  # W1 = U diag(s) Vt
    At = (U * s).T  # [r][d]
    Bm = Vt.T  # [N][r]
    y = r.standard_normal((2, d))
    sc = O.mlp_predictor_scores(y, At, Bm, b1)
    assert np.allclose(sc, y @ W1t.T + b1, rtol=1e-10, atol=1e-10)
    S = O.select(sc, mode="threshold", tau=0.0)
    got = O.sparse_mlp(y, W1t, b1, W2t, b2, S)
    assert np.allclose(got, _torch_ffn(y, W1t, b1, W2t, b2), rtol=1e-10, atol=1e-10)


# --------------------------------------------------------------------------
# eq. (2): sparsified MHA with a KV cache
# --------------------------------------------------------------------------


def _mha_setup(r, B, d, h, dh, n_prev, cap):
    Wqkv = r.standard_normal((h, 3, dh, d)) / np.sqrt(d)
    WOt = r.standard_normal((h, dh, d)) / np.sqrt(d)
    bqkv = r.standard_normal((h, 3, dh)) * 0.1
    bO = r.standard_normal(d) * 0.1
    K = O.round_to_bf16(r.standard_normal((B, h, cap, dh)))
    V = O.round_to_bf16(r.standard_normal((B, h, cap, dh)))
    y = r.standard_normal((B, d))
    return Wqkv, bqkv, WOt, bO, K, V, y


def test_sparse_mha_all_heads_is_torch_mha_concat_then_project():
    """All heads selected == dense attention over the cache plus the new token,
    heads concatenated and projected by W^O (survey note, Transformer section),
    with torch's scaled_dot_product_attention as the library routine."""
    r = rng(7)
    B, d, h, dh, pos, cap = 2, 32, 4, 8, 9, 12
    Wqkv, bqkv, WOt, bO, K, V, y = _mha_setup(r, B, d, h, dh, pos, cap)
    K0, V0 = K.copy(), V.copy()
    res = O.sparse_mha(y, Wqkv, bqkv, WOt, bO, K, V, pos, 0.37, np.arange(h))
    yt = torch.from_numpy(y)
    q = F.linear(yt, torch.from_numpy(Wqkv[:, 0].reshape(h * dh, d)), torch.from_numpy(bqkv[:, 0].reshape(-1)))
    k = F.linear(yt, torch.from_numpy(Wqkv[:, 1].reshape(h * dh, d)), torch.from_numpy(bqkv[:, 1].reshape(-1)))
    v = F.linear(yt, torch.from_numpy(Wqkv[:, 2].reshape(h * dh, d)), torch.from_numpy(bqkv[:, 2].reshape(-1)))
    k = torch.from_numpy(O.round_to_bf16(k.numpy())).view(B, h, 1, dh)
    v = torch.from_numpy(O.round_to_bf16(v.numpy())).view(B, h, 1, dh)
    Kall = torch.cat([torch.from_numpy(K0[:, :, :pos]), k], dim=2)  # [B][h][pos+1][dh]
    Vall = torch.cat([torch.from_numpy(V0[:, :, :pos]), v], dim=2)
    Hs = F.scaled_dot_product_attention(q.view(B, h, 1, dh), Kall, Vall, scale=0.37)  # [B][h][1][dh]
    Z = Hs.reshape(B, h * dh)  # concat heads
    proj = torch.nn.Linear(h * dh, d, dtype=torch.float64)
    with torch.no_grad():
        proj.weight.copy_(torch.from_numpy(WOt.reshape(h * dh, d).T.copy()))
        proj.bias.copy_(torch.from_numpy(bO))
        ref = proj(Z).numpy()
    assert np.allclose(res.out, ref, rtol=1e-11, atol=1e-11)
    # the cache slot pos now holds the rounded new k, v of every selected head
    assert np.array_equal(K[:, :, pos], k[:, :, 0].numpy())
    assert np.array_equal(V[:, :, pos], v[:, :, 0].numpy())


def test_sparse_mha_subset_and_unselected_slots_untouched():
    r = rng(8)
    B, d, h, dh, pos, cap = 1, 24, 6, 4, 5, 8
    Wqkv, bqkv, WOt, bO, K, V, y = _mha_setup(r, B, d, h, dh, pos, cap)
    K0 = K.copy()
    S = [1, 4]
    res = O.sparse_mha(y, Wqkv, None, WOt, None, K, V, pos, 0.5, S)
    # the sum over S of per-head dense contributions (each computed alone)
    acc = np.zeros(d)
    for i in S:
        Kx, Vx = K0.copy(), V.copy()
        acc += O.sparse_mha(y, Wqkv, None, WOt, None, Kx, Vx, pos, 0.5, [i]).out[0]
    assert np.allclose(res.out[0], acc, rtol=1e-12, atol=1e-12)
    for i in range(h):
        if i not in S:
            assert np.array_equal(K[:, i], K0[:, i])


def test_single_key_gives_v_and_identical_keys_give_mean_of_v():
    """D_i normalisation: one key -> H = v; all keys equal -> H = mean(V)."""
    r = rng(9)
    d, h, dh = 16, 2, 4
    Wqkv, _, WOt, _, K, V, y = _mha_setup(r, 1, d, h, dh, 0, 6)
    res = O.sparse_mha(y, Wqkv, None, WOt, None, K, V, 0, 1.0, [1])
    assert np.allclose(res.H[0, 0], res.v_new[0, 0], rtol=1e-14, atol=1e-14)
    # identical keys: make Wk zero and the cached keys zero -> all scores 0
    Wz = Wqkv.copy()
    Wz[:, 1] = 0.0
    K[:] = 0.0
    res = O.sparse_mha(y, Wz, None, WOt, None, K, V, 4, 1.0, [0])
    assert np.allclose(res.H[0, 0], V[0, 0, :5].mean(axis=0), rtol=1e-13, atol=1e-13)


def test_mean_shift_identity():
    """§3.2: with W^V = I the head output is m(y) = sum_j K(x_j,y) x_j / sum_j
    K(x_j,y) with K(x_j,y) = exp(y W^Q (W^K)^T x_j), X holding every token
    (the current one included)."""
    r = rng(10)
    d, n = 8, 7
    WQ = r.standard_normal((d, d)) / np.sqrt(d)
    WK = r.standard_normal((d, d)) / np.sqrt(d)
    X = r.standard_normal((n, d))  # earlier tokens
    y = r.standard_normal(d)  # current token (also x_{n+1})
    Wqkv = np.stack([WQ.T, WK.T, np.eye(d)])[None]  # [1][3][dh=d][d]
    K = np.zeros((1, 1, n + 1, d))
    V = np.zeros((1, 1, n + 1, d))
    K[0, 0, :n] = (X @ WK).astype(np.float32)
    V[0, 0, :n] = X.astype(np.float32)
    res = O.sparse_mha(y[None], Wqkv, None, np.eye(d)[None], None, K, V, n, 1.0, [0], kv_round=None)
    Xall = np.vstack([X, y]).astype(np.float32).astype(np.float64)
    w = np.array([np.exp(y @ WQ @ WK.T @ xj) for xj in Xall])
    m = (w[:, None] * Xall).sum(0) / w.sum()
    assert np.allclose(res.out[0], m, rtol=1e-6, atol=1e-6)


# --------------------------------------------------------------------------
# selection
# --------------------------------------------------------------------------


def _brute_topk(s, k):
    def key(i):
        v = s[i]
        if np.isnan(v):
            return (1, 0.0, i)
        return (0, -(v + 0.0), i)  # v + 0.0 turns -0.0 into +0.0

    return sorted(sorted(range(len(s)), key=key)[:k])


@pytest.mark.parametrize("case", ["random", "ties", "zeros", "nan", "inf"])
def test_topk_against_brute_force(case):
    r = rng(11)
    n = 300
    if case == "random":
        s = r.standard_normal(n).astype(np.float32)
    elif case == "ties":
        s = r.integers(-3, 4, size=n).astype(np.float32)
    elif case == "zeros":
        s = np.where(r.random(n) < 0.5, -0.0, 0.0).astype(np.float32)
        s[::7] = 1.0
    elif case == "nan":
        s = r.standard_normal(n).astype(np.float32)
        s[r.random(n) < 0.3] = np.nan
    else:
        s = r.standard_normal(n).astype(np.float32)
        s[::5] = -np.inf
        s[::11] = np.inf
        s[::13] = np.nan
    for k in [0, 1, 7, 100, 299, 300, 400]:
        assert O.topk_row(s, k).tolist() == _brute_topk(s, min(k, n)), (case, k)


def test_constant_scores_take_lowest_indices():
    assert O.topk_row(np.full(50, 2.5, np.float32), 9).tolist() == list(range(9))


def test_threshold_strict_and_union():
    s = np.array([[0.0, 1.0, -1.0, 0.5, np.nan], [0.6, 0.4, 0.5, 0.5, 2.0]], np.float32)
    assert O.threshold_row(s[0], 0.5).tolist() == [1]
    assert O.select(s, mode="threshold", tau=0.5).tolist() == [0, 1, 4]
    assert O.select(s, k=1).tolist() == [1, 4]
    assert O.select(s, k=2).tolist() == [0, 1, 3, 4]


# --------------------------------------------------------------------------
# the layer and the look-ahead stack
# --------------------------------------------------------------------------


def _layer(r, d, N, h, dh, r_rank, cap, B):
    W1t, b1, W2t, b2 = _mlp_weights(r, d, N)
    Wqkv, bqkv, WOt, bO, K, V, _ = _mha_setup(r, B, d, h, dh, 0, cap)
    return O.LayerF64(PA=r.standard_normal((h, d)) / np.sqrt(d), Wqkv=Wqkv, bqkv=bqkv, WOt=WOt, bO=bO,
                      K=K, V=V, At=r.standard_normal((r_rank, d)) / np.sqrt(d),
                      Bm=r.standard_normal((N, r_rank)) / np.sqrt(r_rank), b1=b1, W1t=W1t, W2t=W2t, b2=b2)


def test_dense_layer_matches_torch_pre_ln_decoder_layer():
    """All heads and all neurons: the layer equals a pre-LN decoder layer
    built from torch's layer_norm, scaled_dot_product_attention and Linear."""
    r = rng(12)
    B, d, N, h, dh, pos, cap = 2, 32, 128, 4, 8, 6, 8
    L = _layer(r, d, N, h, dh, 8, cap, B)
    K0, V0 = L.K.copy(), L.V.copy()
    x = r.standard_normal((B, d)) * 2
    P = O.LayerParams(k=N, k_h=h, scale=0.3)
    t = O.decode_layer(x, L, P, pos)
    xt = torch.from_numpy(x)
    yA = F.layer_norm(xt, (d,), eps=1e-5)
    qkv = [F.linear(yA, torch.from_numpy(L.Wqkv[:, m].reshape(h * dh, d)),
                    torch.from_numpy(L.bqkv[:, m].reshape(-1))) for m in range(3)]
    kn = torch.from_numpy(O.round_to_bf16(qkv[1].numpy())).view(B, h, 1, dh)
    vn = torch.from_numpy(O.round_to_bf16(qkv[2].numpy())).view(B, h, 1, dh)
    Kall = torch.cat([torch.from_numpy(K0[:, :, :pos]), kn], 2)
    Vall = torch.cat([torch.from_numpy(V0[:, :, :pos]), vn], 2)
    Hs = F.scaled_dot_product_attention(qkv[0].view(B, h, 1, dh), Kall, Vall, scale=0.3).reshape(B, h * dh)
    x1 = xt + F.linear(Hs, torch.from_numpy(L.WOt.reshape(h * dh, d).T.copy()), torch.from_numpy(L.bO))
    yM = F.layer_norm(x1, (d,), eps=1e-5).numpy()
    ref = x1.numpy() + _torch_ffn(yM, L.W1t, L.b1, L.W2t, L.b2)
    assert np.allclose(t.x_out, ref, rtol=1e-11, atol=1e-11)


def test_lookahead_is_exact_when_consecutive_inputs_are_equal():
    """§1: the next layer's sets are predicted from this layer's input. When a
    layer leaves the residual stream unchanged (W^O = 0, W2 = 0, no biases)
    and the next layer has the same predictors, the look-ahead sets equal the
    sets predicted from the next layer's own inputs."""
    r = rng(13)
    B, d, N, h, dh, pos, cap = 1, 32, 128, 4, 8, 3, 4
    L0 = _layer(r, d, N, h, dh, 8, cap, B)
    L0.WOt[:] = 0.0
    L0.W2t[:] = 0.0
    L0.bO = None
    L0.b2 = None
    L1 = _layer(r, d, N, h, dh, 8, cap, B)
    L1.PA, L1.At, L1.Bm, L1.b1 = L0.PA, L0.At, L0.Bm, L0.b1
    L1.WOt[:] = 0.0  # layer 1's MLP input then equals its attention input
    L1.bO = None
    x = r.standard_normal((B, d))
    P = O.LayerParams(k=20, k_h=2)
    _, tr = O.decode_stack(x, [L0, L1], P, pos, lookahead=True)
    # layer 1 used the sets predicted from layer 0's attention input
    hA, iM, _, _ = O.lookahead_selection(tr[0].yA, L1, P)
    assert tr[1].head_idx.tolist() == hA.tolist() and tr[1].idx.tolist() == iM.tolist()
    # and, inputs being equal, they are the sets layer 1 would pick itself
    assert tr[1].head_idx.tolist() == O.select(O.head_predictor_scores(tr[1].yA, L1.PA), 2).tolist()
    assert tr[1].idx.tolist() == O.select(O.mlp_predictor_scores(tr[1].yM, L1.At, L1.Bm, L1.b1), 20).tolist()


def test_lookahead_with_full_sets_equals_synchronous():
    r = rng(14)
    B, d, N, h, dh, pos, cap = 1, 16, 64, 2, 8, 2, 3
    layers = [_layer(r, d, N, h, dh, 4, cap, B) for _ in range(3)]
    import copy
    la = copy.deepcopy(layers)
    x = r.standard_normal((B, d))
    P = O.LayerParams(k=N, k_h=h)
    xs, _ = O.decode_stack(x, layers, P, pos, lookahead=False)
    xl, _ = O.decode_stack(x, la, P, pos, lookahead=True)
    assert np.allclose(xs, xl, rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------------
# head predictor and GeLU (pins independent of the oracle's own expressions)
# --------------------------------------------------------------------------


def test_head_predictor_scores_against_library_and_closed_forms():
    """s_A = y P_A^T, pinned four ways: torch's F.linear (another library's
    matrix product), unit rows of P_A that pick single coordinates of y, a row
    equal to y (its squared norm) and a row orthogonal to y (zero), and exact
    rational brute force. h != d, so a transposed P_A cannot pass."""
    r = rng(21)
    B, d, h = 3, 10, 7
    y = r.standard_normal((B, d))
    PA = r.standard_normal((h, d))
    got = O.head_predictor_scores(y, PA)
    assert got.shape == (B, h)
    want = F.linear(torch.from_numpy(y), torch.from_numpy(PA)).numpy()
    assert np.allclose(got, want, rtol=1e-13, atol=1e-13)
    # unit rows: head i scores coordinate j_i of y
    cols = [4, 0, 9, 2, 2, 7, 5]
    E = np.zeros((h, d))
    E[np.arange(h), cols] = 1.0
    assert np.array_equal(O.head_predictor_scores(y, E), y[:, cols])
    # a row equal to y[0] scores ||y[0]||^2; a row orthogonal to it scores 0
    u = y[0] / np.linalg.norm(y[0])
    v = r.standard_normal(d)
    v -= (v @ u) * u
    P2 = np.stack([y[0], v])
    s = O.head_predictor_scores(y[:1], P2)[0]
    assert np.isclose(s[0], float(np.sum(y[0] ** 2)), rtol=1e-13)
    assert abs(s[1]) <= 1e-12 * np.linalg.norm(v) * np.linalg.norm(y[0])
    # permuting the heads permutes the scores
    perm = r.permutation(h)
    assert np.array_equal(O.head_predictor_scores(y, PA[perm]), got[:, perm])
    # exact rationals on small integers / powers of two: the float64 result is exact
    yi = r.integers(-8, 9, size=(2, d))
    Pi = r.integers(-8, 9, size=(h, d))
    exact = [[float(sum(Fraction(int(yi[b, j]), 4) * Fraction(int(Pi[i, j]), 8) for j in range(d)))
              for i in range(h)] for b in range(2)]
    assert np.array_equal(O.head_predictor_scores(yi / 4.0, Pi / 8.0), np.array(exact))


def test_gelu_against_torch_and_limits():
    """GeLU in the exact erf form v * Phi(v): torch's F.gelu (approximate='none'),
    GeLU(0) = 0, GeLU(v) - GeLU(-v) = v (odd part), and the limits v -> +inf
    (identity) and v -> -inf (zero)."""
    v = np.concatenate([np.linspace(-8.0, 8.0, 401), rng(22).standard_normal(200) * 3.0])
    got = O.gelu(v)
    want = F.gelu(torch.from_numpy(v), approximate="none").numpy()
    assert np.allclose(got, want, rtol=1e-12, atol=1e-15)
    assert O.gelu(np.array([0.0]))[0] == 0.0
    assert np.allclose(O.gelu(v) - O.gelu(-v), v, rtol=1e-12, atol=1e-14)
    assert np.isclose(O.gelu(np.array([40.0]))[0], 40.0) and abs(O.gelu(np.array([-40.0]))[0]) < 1e-300
    # the tanh approximation differs: the oracle is the erf form
    tanh_form = F.gelu(torch.from_numpy(v), approximate="tanh").numpy()
    assert np.max(np.abs(got - tanh_form)) > 1e-6


def test_sparse_mlp_gelu_all_neurons_is_dense_gelu_ffn():
    """eq. (1) with sigma = GeLU: with S_M = every neuron the sparse MLP equals a
    torch Linear -> GeLU -> Linear FFN; dropping a neuron changes it (GeLU has
    no exact zeros, so no set smaller than all neurons is exact)."""
    r = rng(23)
    B, d, N = 2, 12, 40
    y = r.standard_normal((B, d))
    W1t = r.standard_normal((N, d)) / np.sqrt(d)
    W2t = r.standard_normal((N, d)) / np.sqrt(d)
    b1 = r.standard_normal(N) * 0.3
    b2 = r.standard_normal(d) * 0.1
    got = O.sparse_mlp(y, W1t, b1, W2t, b2, np.arange(N), act="gelu")
    ty = torch.from_numpy(y)
    hid = F.gelu(F.linear(ty, torch.from_numpy(W1t), torch.from_numpy(b1)), approximate="none")
    want = F.linear(hid, torch.from_numpy(W2t).t().contiguous(), torch.from_numpy(b2)).numpy()
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)
    assert not np.allclose(O.sparse_mlp(y, W1t, b1, W2t, b2, np.arange(1, N), act="gelu"), got, rtol=1e-9)


# --------------------------------------------------------------------------
# exact KV maintenance for unselected heads
# --------------------------------------------------------------------------


def test_unselected_kv_against_torch_projection_and_bf16_rounding():
    """Slot pos of every unselected head holds bf16(y W_i^K) and bf16(y W_i^V)
    as torch's F.linear and its bfloat16 conversion (round to nearest even)
    give them; selected heads and other slots are untouched."""
    r = rng(31)
    B, d, h, dh, cap, pos = 2, 24, 5, 8, 6, 3
    y = r.standard_normal((B, d))
    Wqkv = r.standard_normal((h, 3, dh, d)) / np.sqrt(d)
    bqkv = r.standard_normal((h, 3, dh)) * 0.1
    K0 = r.standard_normal((B, h, cap, dh))
    V0 = r.standard_normal((B, h, cap, dh))
    K, V = K0.copy(), V0.copy()
    S = [1, 3]
    O.unselected_kv(y, Wqkv, bqkv, K, V, pos, S, "bf16")
    ty = torch.from_numpy(y)
    for i in range(h):
        if i in S:
            assert np.array_equal(K[:, i], K0[:, i]) and np.array_equal(V[:, i], V0[:, i])
            continue
        for m, cache in ((1, K), (2, V)):
            want = F.linear(ty, torch.from_numpy(Wqkv[i, m]), torch.from_numpy(bqkv[i, m]))
            want = want.to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
            # float64 -> bf16 directly vs via float32 can differ only where a
            # double rounding lands on a tie; allow one bf16 ulp there
            assert np.all(np.abs(cache[:, i, pos] - want) <= np.abs(want) * 2.0 ** -7 + 1e-12)
        mask = np.ones(cap, bool)
        mask[pos] = False
        assert np.array_equal(K[:, i][:, mask], K0[:, i][:, mask])


def test_exact_kv_completes_the_dense_cache_and_leaves_outputs_unchanged():
    """sparse_mha on S followed by unselected_kv writes at slot pos exactly
    what sparse_mha over all heads writes (the dense cache), and the layer's
    output is the same with and without exact KV at that step."""
    r = rng(32)
    B, d, h, dh, cap, pos = 2, 32, 6, 8, 9, 5
    L = O.LayerF64(PA=r.standard_normal((h, d)), Wqkv=r.standard_normal((h, 3, dh, d)) / np.sqrt(d), bqkv=None,
                   WOt=r.standard_normal((h, dh, d)) / np.sqrt(dh), bO=None, K=r.standard_normal((B, h, cap, dh)),
                   V=r.standard_normal((B, h, cap, dh)), At=r.standard_normal((8, d)),
                   Bm=r.standard_normal((64, 8)), b1=r.standard_normal(64) * 0.1,
                   W1t=r.standard_normal((64, d)) / np.sqrt(d), W2t=r.standard_normal((64, d)) / np.sqrt(d))
    x = r.standard_normal((B, d))
    dense_K, dense_V = L.K.copy(), L.V.copy()
    y = O.layernorm(x)
    O.sparse_mha(y, L.Wqkv, None, L.WOt, None, dense_K, dense_V, pos, 0.3, list(range(h)), "bf16")
    import copy
    La, Lb = copy.deepcopy(L), copy.deepcopy(L)
    ta = O.decode_layer(x, La, O.LayerParams(k=10, k_h=2, scale=0.3), pos)
    tb = O.decode_layer(x, Lb, O.LayerParams(k=10, k_h=2, scale=0.3, exact_kv=True), pos)
    assert np.array_equal(ta.x_out, tb.x_out)
    assert np.array_equal(Lb.K[:, :, pos], dense_K[:, :, pos]) and np.array_equal(Lb.V[:, :, pos], dense_V[:, :, pos])
    unsel = [i for i in range(h) if i not in set(ta.head_idx.tolist())]
    assert unsel and np.array_equal(La.K[:, unsel, pos], L.K[:, unsel, pos])  # without: the old slot stays


def test_dequantize_rows_is_q_times_row_scale():
    """int8 rows with one scale per row, rows along the last axis: checked
    element by element with explicit loops and exact rationals (power-of-two
    scales), a scale of 1 giving the integers back, and a transposed scale
    shape failing."""
    r = rng(41)
    q = r.integers(-127, 128, size=(2, 3, 4, 5)).astype(np.int8)
    s = (2.0 ** r.integers(-8, 3, size=(2, 3, 4))).astype(np.float32)
    W = O.dequantize_rows(q, s)
    assert W.shape == q.shape
    for a in range(2):
        for b in range(3):
            for c in range(4):
                for e in range(5):
                    assert W[a, b, c, e] == float(Fraction(int(q[a, b, c, e])) * Fraction(float(s[a, b, c])))
    assert np.array_equal(O.dequantize_rows(q, np.ones((2, 3, 4), np.float32)), q.astype(np.float64))
    with pytest.raises(ValueError):
        O.dequantize_rows(q, np.ones((5, 4, 3, 2), np.float32)[..., 0])
