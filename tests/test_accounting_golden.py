"""Byte accounting pinned to the worked numbers the pages print."""

import json
import os

from attention_predictor_gemv_b200 import accounting as A

G = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(G, name)) as f:
        return json.load(f)


def test_kv_bytes_per_token_llama13b():
    g = load("kv_cache_llama13b.json")
    per_tok = A.kv_bytes_per_token(g["hidden"], g["layers"], g["elem_bytes"])
    assert per_tok == g["bytes_per_token"]
    assert per_tok * g["tokens"] == g["bytes_total"]
    # the layer accounting's KV write of one new slot, all heads, over all layers
    h, dh = 40, 128  # 40 x 128 = 5120
    one = A.layer_bytes(5120, 4 * 5120, 8, h, dh, 0, 0, h, 1, 0, predictors=False)
    assert one.kv * g["layers"] == g["bytes_per_token"]


def test_mlp_is_two_thirds_of_dense_weight_io():
    g = load("param_io_split.json")
    c = g["opt175b"]
    mlp, attn = A.dense_layer_param_bytes(c["d"], c["N"], c["h"], c["dh"])
    assert mlp / attn == g["mlp_over_attention"]
    assert abs(mlp / (mlp + attn) - g["mlp_share"]) < 1e-15
    full = A.layer_bytes(c["d"], c["N"], 1024, c["h"], c["dh"], c["N"], c["N"], c["h"], 1, 0, predictors=False)
    assert full.w1 + full.w2 - 4 * c["N"] == mlp
    assert full.qkv + full.wo == attn
