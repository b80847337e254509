"""Glue between torch tensors, the oracle and the tolerances the tests use."""

from __future__ import annotations

import numpy as np
import torch

from oracle import dejavu_oracle as O

# Tolerances (fp32 accumulation over bf16 / fp32 inputs vs the float64 oracle)
SCORE_MAX_REL = 1e-3  # max |ds| <= 1e-3 * ||s_ref||_inf
SCORE_L2_REL = 1e-3  # ||ds||_2 <= 1e-3 * ||s_ref||_2
OUT_L2_REL = 5e-3  # ||dout||_2 <= 5e-3 * ||out_ref||_2
OUT_MAX_REL = 2e-2  # max |dout| <= 2e-2 * ||out_ref||_inf


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a bf16 / fp32 tensor (bf16 decoded by the oracle)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return O.bf16_bits_to_f64(t.view(torch.int16).numpy().view(np.uint16))
    return t.double().numpy()


def wname(t: torch.Tensor) -> str:
    return "bf16" if t.dtype == torch.bfloat16 else "f32"


def assert_scores(got, ref, what="scores"):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    dmax = np.max(np.abs(got - ref)) if ref.size else 0.0
    assert dmax <= SCORE_MAX_REL * max(np.max(np.abs(ref)), 1e-30), (what, dmax, np.max(np.abs(ref)))
    l2 = np.linalg.norm(got - ref)
    assert l2 <= SCORE_L2_REL * max(np.linalg.norm(ref), 1e-30), (what, l2, np.linalg.norm(ref))


def assert_out(got, ref, what="out"):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    l2 = np.linalg.norm(got - ref)
    nref = np.linalg.norm(ref)
    assert l2 <= OUT_L2_REL * max(nref, 1e-30), (what, "rel-L2", l2 / max(nref, 1e-30))
    dmax = np.max(np.abs(got - ref)) if ref.size else 0.0
    inf = np.max(np.abs(ref)) if ref.size else 0.0
    assert dmax <= OUT_MAX_REL * max(inf, 1e-30), (what, "max-abs", dmax, inf)


def assert_kv_slot(got, ref, what="KV slot"):
    """A written K or V slot (last axis = dh channels) against the oracle's:
    every element within one bf16 rounding of the oracle's value
    (2^-7 |ref|) plus 2^-12 of the largest magnitude in its dh-vector. The
    second term is the accumulation difference of a d-term fp32 dot product
    (its absolute error scales with the vector's magnitude, not with one
    small element); both stay far inside the layer-output bar (max-abs
    2e-2 ||out||_inf)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = np.max(np.abs(ref), axis=-1, keepdims=True)
    bad = np.abs(got - ref) > np.abs(ref) * 2.0 ** -7 + scale * 2.0 ** -12
    assert not bad.any(), (what, int(bad.sum()), np.argwhere(bad)[:4].tolist())


def oracle_layer(t, kv_round="bf16") -> O.LayerF64:
    g = lambda n: f64(t[n]) if n in t and t[n] is not None else None  # noqa: E731
    return O.LayerF64(PA=g("PA"), Wqkv=g("Wqkv"), bqkv=g("bqkv"), WOt=g("WOt"), bO=g("bO"), K=g("K"), V=g("V"),
                      At=g("At"), Bm=g("Bm"), b1=g("b1"), W1t=g("W1t"), W2t=g("W2t"), b2=g("b2"), ln1_g=g("ln1_g"),
                      ln1_b=g("ln1_b"), ln2_g=g("ln2_g"), ln2_b=g("ln2_b"),
                      kv_round=kv_round if t["K"].dtype == torch.bfloat16 else None)


def selected(idx: torch.Tensor, count: torch.Tensor) -> np.ndarray:
    c = int(count.item())
    return idx[:c].cpu().numpy().astype(np.int64)
