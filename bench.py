"""Benchmark: decode steps of OPT-shaped decoder stacks with contextual
sparsity (the look-ahead predictors, top-k selection, sparse MHA over the
selected heads and sparse MLP over the selected neurons), through the C ABI,
bf16 weights and KV cache, fp32 arithmetic.

Headline: 24 OPT-175B-shaped layers (d=12288, N=49152, r=1024, h=96, dh=128,
KV length 2048; 87 GB of weights), batch 1, 85% sparsity on neurons and heads
(k = 7373, k_h = 14), look-ahead on; one step = one token through the 24
layers. Metric: microseconds per decode step per layer (lower is better), with
the effective HBM bandwidth on the selected bytes.

Also measured in the same run (each in the JSON line):
  * the OPT-175B sweep: sparsity 50/75/85/95% x batch 1/2/4/8/16, plus the
    dense path of the same kernels at each batch (sparse/dense crossover);
  * OPT-6.7B-shaped stack, 32 layers, 128 generated tokens with the KV
    position advancing, look-ahead on and off;
  * OPT-66B-shaped stack, 64 layers, batch 1/2/4/8 (union sets);
  * OPT-1.3B-shaped stack, 24 layers, neuron x head fraction sweep; the tiny
    layer (latency only, L2-resident);
  * the CPU oracle on the host cores (single thread and all cores).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

For N > 1 (torchrun) every rank runs an independent replica of the headline
stack (the path has no exchange step); the time is the maximum over ranks.
"""

from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from attention_predictor_gemv_b200 import accounting as acct  # noqa: E402
from attention_predictor_gemv_b200 import workload as wl  # noqa: E402

METRIC = "us/decode-step/layer"
HEADLINE = "opt-175b"
HEADLINE_SPARSITY = 0.85


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=HEADLINE, choices=sorted(wl.CONFIGS))
    ap.add_argument("--layers", type=int, default=0, help="0: the workload's own layer count")
    ap.add_argument("--sparsity", type=float, default=HEADLINE_SPARSITY,
                    help="fraction of neurons and heads skipped at the headline point")
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--no-lookahead", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="skip the sparsity x batch sweep")
    ap.add_argument("--no-extra", action="store_true", help="skip the OPT-6.7B/66B/1.3B/tiny measurements")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=2.0, help="seconds per CPU oracle timing")
    ap.add_argument("--neurons", type=int, default=0,
                    help="0: the workload's neuron count; else fewer neurons per layer, for profiler captures of a "
                         "small case (k stays the headline's)")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# distributed plumbing (replicas only: barrier and max-over-ranks timing)
# ---------------------------------------------------------------------------


def dist_init():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws <= 1:
        return 0, 1, None
    import datetime

    import torch.distributed as dist

    rank = int(os.environ["RANK"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:  # host-only ranks (the reference arm, tests): gloo
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=300))
    return rank, ws, dist


def barrier(dist):
    if dist is not None:
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def max_over_ranks(v, dist):
    """The largest of the ranks' values (every rank gets it)."""
    if dist is None:
        return v
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------


class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_index: int):
        self.dev = dev_index
        self.p = None
        self.out = ""

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "100"], stdout=subprocess.PIPE,
                                      stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.p = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        time.sleep(0.15)
        if self.p is not None:
            self.p.terminate()
            try:
                self.out, _ = self.p.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.p.kill()
                self.out = ""

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# stacks, graphs and timing
# ---------------------------------------------------------------------------


def make_layers(shape, n, seed0):
    """n layers of `shape` (weights, predictors, batch-1 KV caches) on the GPU."""
    return [wl.make_layer(shape.with_(B=1), seed0 + l, "cuda") for l in range(n)]


def with_kv(layers, shape, B, seed):
    """The layers with fresh KV caches for batch B (weights shared)."""
    out = []
    for l, t in enumerate(layers):
        K, V = wl.make_kv(shape, B, seed + l, "cuda")
        out.append(dict(t, K=K, V=V))
    return out


def build_stack(layers, shape, B, k, k_h, lookahead):
    from attention_predictor_gemv_b200.stack import DecoderStack

    return DecoderStack(layers, B, k, k_h, 1.0 / float(np.sqrt(shape.dh)), lookahead=lookahead)


def graph_of(fn):
    """Captures fn (library launches on the current stream) into a CUDA graph
    after one eager call (kernel set-up stays outside the capture)."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    return g


def capture(stk, x, pos):
    """The decode step as a CUDA graph, and how many library kernels it holds."""
    from attention_predictor_gemv_b200 import binding as bd

    stk.step(x, pos)
    torch.cuda.synchronize()
    n0 = bd.dv_launch_count()
    g = graph_of(lambda: stk.step(x, pos))
    n1 = bd.dv_launch_count()
    return g, (n1 - n0) // 2  # graph_of calls fn twice (eager, then captured)


def time_graph(g, steps, warmup, dist):
    for _ in range(warmup):
        g.replay()
    barrier(dist)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    e1.synchronize()
    barrier(dist)
    return e0.elapsed_time(e1) / steps  # ms per step


def selected_counts(stk):
    """Mean k (selected neurons) and k_h over the layers."""
    ks = [int(stk.count[l].item()) for l in range(len(stk.layers))]
    khs = [int(stk.head_count[l].item()) for l in range(len(stk.layers))]
    return float(np.mean(ks)), float(np.mean(khs))


def nonzero_neurons(stk):
    """k' per layer: selected neurons with a nonzero activation in some batch
    row, recomputed from the layer's y_M on the device (torch, reporting only)."""
    kp = []
    for l, L in enumerate(stk.layers):
        c = int(stk.count[l].item())
        idx = stk.idx[l][:c].long()
        pre = stk.yM[l] @ L.t["W1t"][idx].float().t() + L.t["b1"][idx]
        kp.append(int((pre > 0).any(dim=0).sum().item()))
    return float(np.mean(kp))


def layer_bytes(shape, k, kp, kh, B):
    return acct.layer_bytes(shape.d, shape.N, shape.r, shape.h, shape.dh, int(round(k)), int(round(kp)),
                            int(round(kh)), B, shape.L + 1, wdtype=shape.wdtype, kvdtype=shape.kvdtype)


def point(layers, shape, B, sparsity, steps, warmup, dist, lookahead=True, kv_seed=None):
    """One (batch, sparsity) point: the step of the whole stack as a CUDA
    graph, timed; returns the measurement and the stack (for more timing)."""
    keep = 1.0 - sparsity
    k, k_h = wl.k_for(keep, shape.N), wl.k_for(keep, shape.h)
    ls = with_kv(layers, shape, B, kv_seed) if kv_seed is not None else layers
    stk = build_stack(ls, shape, B, k, k_h, lookahead)
    x = wl.make_input(shape.with_(B=B), 7 + B, "cuda")
    g, launches = capture(stk, x, shape.L)
    ms = time_graph(g, steps, warmup, dist)
    km, kh = selected_counts(stk)
    kp = nonzero_neurons(stk)
    lb = layer_bytes(shape, km, kp, kh, B)
    n = len(layers)
    us = ms * 1e3 / n
    res = {"batch": B, "sparsity": sparsity, "k": k, "k_h": k_h, "k_union": km, "k_eff": kp, "k_h_union": kh,
           "us_per_layer": us, "tokens_per_s": B * 1e3 / ms, "bytes_per_layer": lb.total,
           "gbs": lb.total / us / 1e3, "launches_per_step": launches}
    return res, stk, g, x, lb


# Source headers of each main-path kernel, for matching a committed ncu
# capture to the code that runs now.
KERNEL_HEADERS = {
    "attn_in": ("dv_common.cuh", "dv_fused.cuh", "dv_colowner.cuh", "dv_stream.cuh"),
    "mlp_block": ("dv_common.cuh", "dv_fused.cuh", "dv_colowner.cuh", "dv_stream.cuh"),
    "attn_out": ("dv_common.cuh", "dv_kernels.cuh", "dv_fused.cuh", "dv_stream.cuh"),
    "predict_neurons": ("dv_common.cuh", "dv_fused.cuh", "dv_api_kernels.cuh"),
}


def kernel_sources_digest(op):
    """SHA-256 prefix of `op`'s kernel source headers with comments and
    blank lines removed (so an edited comment keeps a capture valid)."""
    import hashlib
    import re

    csrc = os.path.join(ROOT, "attention_predictor_gemv_b200", "csrc")
    h = hashlib.sha256()
    for f in KERNEL_HEADERS.get(op, ()):
        with open(os.path.join(csrc, f)) as fh:
            text = re.sub(r"/\*.*?\*/", "", fh.read(), flags=re.S)
        for line in text.splitlines():
            code = re.sub(r"//.*", "", line).rstrip()
            if code.strip():
                h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def measured_traffic(op, profiles_dir=None, workload=None):
    """Per-launch DRAM bytes (read + write) of `op`'s kernel from the ncu
    summaries under profiles/ (lines `traffic <op> <bytes> <sha256 prefix>
    [workload]`), or None when no capture exists or the kernel's headers
    changed since. With `workload`, only lines naming it count."""
    import glob

    digest = kernel_sources_digest(op)
    pdir = profiles_dir or os.path.join(ROOT, "profiles")
    for path in sorted(glob.glob(os.path.join(pdir, "*.md"))):
        with open(path) as fh:
            for line in fh:
                parts = line.split()
                if len(parts) in (4, 5) and parts[0] == "traffic" and parts[1] == op and parts[3] == digest:
                    if workload is not None and (len(parts) < 5 or parts[4] != workload):
                        continue
                    return {"bytes": int(parts[2]), "source": os.path.relpath(path, ROOT)}
    return None


def kernel_roofline(stk, shape, B, pos, peak_gbs, reps=20):
    """Average duration of each kernel of the step in the look-ahead steady
    state (sets given): one CUDA graph per kernel with that kernel's call for
    every layer, timed with CUDA events on the launching stream; each
    kernel's algorithmic bytes per launch divided by its average duration.
    The residual state and caches are restored afterwards."""
    from attention_predictor_gemv_b200 import binding as bd

    nL = len(stk.layers)
    x = torch.randn(B, shape.d, device="cuda")
    snap = [(t["K"].clone(), t["V"].clone()) for t in (L.t for L in stk.layers)]
    kp = nonzero_neurons(stk)
    k, kh = selected_counts(stk)
    lb = layer_bytes(shape, k, kp, kh, B)
    w = acct.ELEM[shape.wdtype]
    p, ws = stk.p, stk.ws_main
    pred_bytes = shape.N * shape.r * w + 4 * shape.N + 2 * 4 * B * shape.N + 4 * int(round(k))
    calls = {
        "attn_in": (lambda l: bd.dv_decode_layer_begin(stk.layers[l], p, x, pos, ws, sel=stk.io_given[l],
                                                       trace=stk.io_trace_y[l]), lb.qkv, range(nL)),
        "attn_out": (lambda l: bd.dv_decode_layer_attn(stk.layers[l], p, x, pos, ws, sel=stk.io_given[l],
                                                       trace=stk.io_trace_y[l]), lb.kv + lb.wo, range(nL)),
        "mlp_block": (lambda l: bd.dv_decode_layer_mlp(stk.layers[l], p, x, ws, sel=stk.io_given[l],
                                                       trace=stk.io_trace_y[l]), lb.w1 + lb.w2, range(nL)),
    }
    if stk.fuse_ahead and nL > 1:
        # the look-ahead tails on the main stream: neuron scores z B^T + b1 and
        # their selection; the head selection
        calls["predict_neurons"] = (
            lambda l: bd.dv_predict_layer_tail(stk.layers[l], p, stk.io_sets[l], stk.ws_ahead[l % 2],
                                               sets=bd.DV_SET_NEURONS), pred_bytes, range(1, nL))
        calls["select_heads"] = (
            lambda l: bd.dv_predict_layer_tail(stk.layers[l], p, stk.io_sets[l], stk.ws_ahead[l % 2],
                                               sets=bd.DV_SET_HEADS), 2 * 4 * B * shape.h, range(1, nL))
    res = {}
    for name, (fn, nbytes, ls) in calls.items():
        ls = list(ls)
        g = graph_of(lambda: [fn(l) for l in ls])
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        e1.synchronize()
        us = e0.elapsed_time(e1) * 1000.0 / (reps * len(ls))
        res[name] = {"us": us, "bytes": nbytes, "gbs": nbytes / us / 1e3, "frac": nbytes / us / 1e3 / peak_gbs}
        del g
    for t, (K, V) in zip((L.t for L in stk.layers), snap):
        t["K"].copy_(K)
        t["V"].copy_(V)
    return res, lb, k, kp, kh


def int8_blocks(stk, shape, pos, peak_gbs, reps=20):
    """The sparse MLP and MHA blocks of the headline layer 0 (its own selected
    sets, batch 1) through the block calls, bf16 rows (dv_sparse_mlp /
    dv_sparse_mha) against weight-only int8 rows with per-row scales
    (dv_sparse_mlp_q8 / dv_sparse_mha_q8): CUDA graph of one call, replayed;
    the selected rows (0.2-0.4 GB) exceed L2, so each replay reads HBM."""
    from attention_predictor_gemv_b200 import binding as bd

    t = stk.layers[0].t
    q = wl.quantize_layer(t)
    yM, yA = stk.yM[0], stk.yA[0]
    idx, cnt, hidx, hcnt = stk.idx[0], stk.count[0], stk.head_idx[0], stk.head_count[0]
    k, kh = int(cnt.item()), int(hcnt.item())
    rows = idx[:k].long()
    kp = int((yM @ t["W1t"][rows].float().t() + t["b1"][rows] > 0).any(dim=0).sum().item())
    d, dh = shape.d, shape.dh
    out = torch.empty(1, d, device="cuda")
    ws_m = bd.workspace(bd.DV_OP_SPARSE_MLP, bd.dims(B=1, d=d, N=shape.N, k_max=k))
    ws_a = bd.workspace(bd.DV_OP_SPARSE_MHA, bd.dims(B=1, d=d, N=1, h=shape.h, dh=dh, cap=shape.cap, kh_max=kh))
    K, V = t["K"].clone(), t["V"].clone()
    sc = 1.0 / float(np.sqrt(dh))
    kv = kh * (pos + 2) * 2 * dh * 2
    calls = {
        "mlp_bf16": (lambda: bd.dv_sparse_mlp(yM, t["W1t"], t["b1"], t["W2t"], None, idx, cnt, k, out, ws_m),
                     k * (2 * d + 4) + kp * 2 * d),
        "mlp_int8": (lambda: bd.dv_sparse_mlp_q8(yM, q["W1q"], q["W1s"], t["b1"], q["W2q"], q["W2s"], None, idx, cnt,
                                                 k, out, ws_m), k * (d + 8) + kp * (d + 4)),
        "mha_bf16": (lambda: bd.dv_sparse_mha(yA, t["Wqkv"], None, t["WOt"], None, K, V, pos, sc, hidx, hcnt, kh, out,
                                              ws_a), kh * 4 * dh * d * 2 + kv),
        "mha_int8": (lambda: bd.dv_sparse_mha_q8(yA, q["Wqkvq"], q["Wqkv_s"], None, q["WOq"], q["WO_s"], None, K, V,
                                                 pos, sc, hidx, hcnt, kh, out, ws_a), kh * 4 * dh * (d + 4) + kv),
    }
    res = {}
    for name, (fn, nbytes) in calls.items():
        g = graph_of(fn)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        e1.synchronize()
        us = e0.elapsed_time(e1) * 1000.0 / reps
        res[name] = {"us": us, "bytes": nbytes, "gbs": nbytes / us / 1e3, "frac": nbytes / us / 1e3 / peak_gbs}
        del g
    del q
    free_gpu()
    return {"workload": f"one OPT-175B-shaped layer's sparse MLP (k={k}, k'={kp}) and MHA (k_h={kh}, KV {pos + 1}) "
                        "blocks, batch 1, block calls (kernel per step)", **res}


def free_gpu():
    import gc

    gc.collect()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# secondary workloads
# ---------------------------------------------------------------------------


def sweep_175b(layers, shape, args, dist):
    """Sparsity 50/75/85/95% x batch 1/2/4/8/16 on the headline stack's
    weights, and the dense path (every neuron and head) at each batch."""
    out = []
    for B in (1, 2, 4, 8, 16):
        ls = with_kv(layers, shape, B, 9000 + 100 * B) if B > 1 else layers  # one set of caches per batch
        for s in (0.50, 0.75, 0.85, 0.95, 0.0):
            res, stk, g, x, _ = point(ls, shape, B, s, 6, 2, dist)
            res["dense"] = s == 0.0
            out.append(res)
            del stk, g, x
        del ls
        free_gpu()
    return out


def generation(shape, nL, lookahead, tokens, dist):
    """OPT-6.7B-shaped stack: `tokens` decode steps with the KV position
    advancing (one CUDA graph per position), timed as one generation."""
    layers = make_layers(shape, nL, 3000)
    k, k_h = wl.DEFAULT_SELECTION["opt-6.7b"]
    res = {}
    for la in ((True, False) if lookahead else (False,)):
        stk = build_stack(layers, shape, 1, k, k_h, la)
        x = wl.make_input(shape, 3, "cuda")
        graphs = [graph_of(lambda p=shape.L + i: stk.step(x, p)) for i in range(tokens)]
        for g in graphs:  # warm-up generation
            g.replay()
        barrier(dist)
        times = []
        for _ in range(2):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for g in graphs:
                g.replay()
            e1.record()
            e1.synchronize()
            times.append(e0.elapsed_time(e1))
        barrier(dist)
        ms = float(np.mean(times))
        km, kh = selected_counts(stk)
        kp = nonzero_neurons(stk)
        lb = layer_bytes(shape, km, kp, kh, 1)  # bytes at the first position; KV grows by one slot per token
        us = ms * 1e3 / (tokens * nL)
        res["lookahead" if la else "synchronous"] = {
            "us_per_layer": us, "tokens_per_s": tokens * 1e3 / ms, "ms_per_token": ms / tokens,
            "k": k, "k_h": k_h, "k_eff": kp, "bytes_per_layer": lb.total, "gbs": lb.total / us / 1e3}
        del graphs, stk, x
        free_gpu()
    del layers
    free_gpu()
    return {"workload": f"{nL} OPT-6.7B-shaped layers: d={shape.d}, N={shape.N}, r={shape.r}, h={shape.h}, "
                        f"dh={shape.dh}, KV positions {shape.L}..{shape.L + tokens - 1}, batch 1, k={k} (8%), "
                        f"k_h={k_h} (20%); {tokens} generated tokens, one graph per position", **res}


def opt66b(shape, nL, dist):
    """OPT-66B-shaped stack, 64 layers (about 139 GB of weights), batch
    1/2/4/8 with union sets, 6% of neurons and 20% of heads per row."""
    layers = make_layers(shape, nL, 4000)
    k, k_h = wl.DEFAULT_SELECTION["opt-66b"]
    out = []
    for B in (1, 2, 4, 8):
        ls = with_kv(layers, shape, B, 4500 + B) if B > 1 else layers
        stk = build_stack(ls, shape, B, k, k_h, True)
        x = wl.make_input(shape.with_(B=B), 5, "cuda")
        g, launches = capture(stk, x, shape.L)
        ms = time_graph(g, 6, 2, dist)
        km, kh = selected_counts(stk)
        kp = nonzero_neurons(stk)
        lb = layer_bytes(shape, km, kp, kh, B)
        us = ms * 1e3 / nL
        out.append({"batch": B, "k": k, "k_h": k_h, "k_union": km, "k_eff": kp, "k_h_union": kh, "us_per_layer": us,
                    "tokens_per_s": B * 1e3 / ms, "bytes_per_layer": lb.total, "gbs": lb.total / us / 1e3})
        del g, stk, x, ls
        free_gpu()
    del layers
    free_gpu()
    return {"workload": f"{nL} OPT-66B-shaped layers: d={shape.d}, N={shape.N}, r={shape.r}, h={shape.h}, "
                        f"dh={shape.dh}, KV length {shape.L}, k={k} (6%), k_h={k_h} (20%) per row, look-ahead",
            "points": out}


def opt13b(dist):
    """OPT-1.3B-shaped stack (24 layers, 2.6 GB of weights), batch 1: the
    neuron x head fraction sweep of the configuration."""
    shape = wl.CONFIGS["opt-1.3b"]
    layers = make_layers(shape, 24, 1000)
    out = []
    for kf in (0.05, 0.10, 0.20, 1.00):
        for hf in (0.25, 0.50, 1.00):
            k, k_h = wl.k_for(kf, shape.N), wl.k_for(hf, shape.h)
            stk = build_stack(layers, shape, 1, k, k_h, True)
            x = wl.make_input(shape, 7, "cuda")
            g, _ = capture(stk, x, shape.L)
            ms = time_graph(g, 20, 3, dist)
            km, kh = selected_counts(stk)
            lb = layer_bytes(shape, km, nonzero_neurons(stk), kh, 1)
            us = ms * 1e3 / 24
            out.append({"k_frac": kf, "kh_frac": hf, "k": k, "k_h": k_h, "us_per_layer": us,
                        "bytes_per_layer": lb.total, "gbs": lb.total / us / 1e3})
            del g, stk, x
    del layers
    free_gpu()
    return {"workload": "24 OPT-1.3B-shaped layers: d=2048, N=8192, r=256, h=32, dh=64, KV length 512, batch 1, "
                        "look-ahead; 2.6 GB of weights streamed per step", "points": out}


def tiny_latency(dist):
    """The tiny fp32 layer (L2-resident): latency of one layer-step."""
    shape = wl.CONFIGS["tiny"]
    layers = make_layers(shape, 1, 0)
    k, k_h = wl.DEFAULT_SELECTION["tiny"]
    stk = build_stack(layers, shape, 1, k, k_h, False)
    x = wl.make_input(shape, 0, "cuda")
    g, launches = capture(stk, x, shape.L)
    ms = time_graph(g, 200, 20, dist)
    del g, stk
    return {"workload": "1 tiny fp32 layer: d=256, N=1024, r=32, h=4, dh=64, KV length 64, k=128, k_h=2, "
                        "synchronous prediction (L2-resident: latency only)", "us_per_layer": ms * 1e3,
            "launches_per_step": launches}


# ---------------------------------------------------------------------------
# the CPU oracle (reported baseline; also the reference arm)
# ---------------------------------------------------------------------------


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_layer_from(t):
    """The oracle's float64 layer from a layer's tensors (device or host)."""
    from oracle import dejavu_oracle as O

    def f(a):
        a = a.detach().cpu().contiguous()
        if a.dtype == torch.bfloat16:
            return O.bf16_bits_to_f64(a.view(torch.int16).numpy().view(np.uint16))
        return a.double().numpy()

    return O.LayerF64(PA=f(t["PA"]), Wqkv=f(t["Wqkv"]), bqkv=None, WOt=f(t["WOt"]), bO=None, K=f(t["K"]),
                      V=f(t["V"]), At=f(t["At"]), Bm=f(t["Bm"]), b1=f(t["b1"]), W1t=f(t["W1t"]), W2t=f(t["W2t"]),
                      kv_round="bf16" if t["K"].dtype == torch.bfloat16 else None)


def time_oracle(OL, shape, k, k_h, seconds, threads=None, max_steps=None):
    """Repeated oracle layer-steps (float64 numpy: LN, predictors, selection,
    sparse MHA, sparse MLP) for about `seconds`; `threads` limits the BLAS
    threads (None: all). Returns (us per layer-step, steps)."""
    from threadpoolctl import threadpool_limits

    from oracle import dejavu_oracle as O

    P = O.LayerParams(k=k, k_h=k_h, scale=1.0 / float(np.sqrt(shape.dh)))
    x = wl.make_input(shape.with_(B=1), 0, "cpu").double().numpy()
    n, t0 = 0, time.perf_counter()
    with threadpool_limits(limits=threads):
        while True:
            O.decode_layer(x, OL, P, shape.L)
            n += 1
            el = time.perf_counter() - t0
            if el >= seconds or (max_steps and n >= max_steps):
                break
    return el * 1e6 / n, n


def cpu_baseline(headline_layer, shape, k, k_h, seconds):
    """The oracle on the host cores: one headline-shaped layer-step (sparse),
    single-threaded and on all cores; and configs tiny, OPT-1.3B and one
    OPT-6.7B layer, sparse and dense, single-threaded and on all cores."""
    cores = host_cores()
    OL = oracle_layer_from(headline_layer)
    v_all, n_all = time_oracle(OL, shape, k, k_h, 3 * seconds)
    v_one, n_one = time_oracle(OL, shape, k, k_h, 3 * seconds, threads=1)
    del OL
    table = []
    for name in ("tiny", "opt-1.3b", "opt-6.7b"):
        s = wl.CONFIGS[name].with_(B=1)
        t = wl.make_layer(s, 1000, "cpu")
        OLs = oracle_layer_from(t)
        ks, khs = wl.DEFAULT_SELECTION[name]
        for mode, kk, hh in (("sparse", ks, khs), ("dense", s.N, s.h)):
            for thr in (1, None):
                us, n = time_oracle(OLs, s, kk, hh, seconds, threads=thr)
                table.append({"workload": name, "mode": mode, "k": kk, "k_h": hh,
                              "threads": 1 if thr == 1 else cores, "us_per_layer_step": us, "steps": n})
        del OLs, t
    return {"value": v_all, "unit": "us/layer-step", "cores": cores, "kind": "oracle",
            "sample": f"{n_all} layer-steps of one OPT-175B-shaped layer (d={shape.d}, N={shape.N}, r={shape.r}, "
                      f"h={shape.h}, dh={shape.dh}, KV {shape.L}+1, B=1, k={k}, k_h={k_h}), float64 numpy, full "
                      f"layer (LN, predictors, selection, sparse MHA, sparse MLP), all {cores} host cores",
            "single_thread": {"value": v_one, "steps": n_one}, "table": table}


def run_reference(args, rank, dist):
    """The reference arm: the oracle (float64 numpy, host cores) on the
    headline workload, one layer-step per timed step (the layer built on the
    host; the GPU is not used)."""
    if rank != 0:
        return
    shape = wl.CONFIGS[args.config]
    keep = 1.0 - args.sparsity
    k, k_h = wl.k_for(keep, shape.N), wl.k_for(keep, shape.h)
    # the inputs are drawn on the GPU when there is one (faster; the same
    # seeded recipe), then decoded to float64 on the host for the oracle
    t = wl.make_layer(shape.with_(B=1), 5000, "cuda" if torch.cuda.is_available() else "cpu")
    OL = oracle_layer_from(t)
    del t
    time_oracle(OL, shape, k, k_h, 0.0, max_steps=max(1, args.warmup))
    v, n = time_oracle(OL, shape, k, k_h, 1e9, max_steps=max(1, args.steps))
    cores = host_cores()
    nL = args.layers or shape.layers
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "us", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": v * nL / 1e3, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(args.config, shape, nL, args.batch, k, k_h, not args.no_lookahead),
            "cpu_baseline": {"value": v, "unit": "us/layer-step", "cores": cores, "kind": "oracle",
                             "sample": f"{n} layer-steps of one {args.config}-shaped layer (B=1, k={k}, k_h={k_h}), "
                                       f"float64 numpy on {cores} host cores, one layer-step per timed step"},
            "e2e": {"value": v, "unit": "us", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(key, shape, nL, B, k, k_h, lookahead):
    name = {"opt-175b": "OPT-175B", "opt-66b": "OPT-66B", "opt-6.7b": "OPT-6.7B", "opt-1.3b": "OPT-1.3B",
            "tiny": "tiny"}
    return {"workload": f"{nL} {name[key]}-shaped decoder layers (bf16 weights and KV cache, fp32 arithmetic): "
                        f"d={shape.d}, N={shape.N}, r={shape.r}, h={shape.h}, dh={shape.dh}, KV length {shape.L}, "
                        f"batch {B}, k={k} ({k / shape.N:.0%}), k_h={k_h} ({k_h / shape.h:.0%}), "
                        f"{'look-ahead' if lookahead else 'synchronous'} prediction",
            "global_batch": B, "seq_len": shape.L + 1}


# ---------------------------------------------------------------------------
# main
# ---------------------------------------------------------------------------


def main():
    args = parse()
    rank, world, dist = dist_init()
    if args.impl == "reference":
        run_reference(args, rank, dist)
        if dist is not None:
            dist.destroy_process_group()
        return
    from attention_predictor_gemv_b200 import binding as bd

    dev = torch.cuda.current_device()
    peaks = {}
    pk = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pk):
        with open(pk) as f:
            peaks = json.load(f)
    peak_gbs = float(peaks.get("hbm_gbs", 6650.0))
    peak_src = "measured" if "hbm_gbs" in peaks else "fallback"

    B = args.batch
    shape = wl.CONFIGS[args.config].with_(B=B)
    nL = args.layers or shape.layers
    keep = 1.0 - args.sparsity
    k, k_h = wl.k_for(keep, shape.N), wl.k_for(keep, shape.h)
    if args.neurons:  # a small case for profiler captures: fewer neurons, the same k
        shape = shape.with_(N=args.neurons)
        k = min(k, args.neurons)
    pos = shape.L
    torch.manual_seed(rank)
    layers = make_layers(shape, nL, 5000 + 100 * rank)
    ls = with_kv(layers, shape, B, 6000 + rank) if B > 1 else layers
    stk = build_stack(ls, shape, B, k, k_h, not args.no_lookahead)
    x0 = wl.make_input(shape, 7 + rank, "cuda")
    x = x0.clone()
    g, launches_per_step = capture(stk, x, pos)

    with Clocks(dev) as clk:
        ms = time_graph(g, args.steps, args.warmup, dist)
    ms = max_over_ranks(ms, dist)
    clocks = clk.summary()

    # end to end: pinned host input -> device, step, device -> host result
    xh = torch.empty(B, shape.d, dtype=torch.float32, pin_memory=True)
    xh.copy_(x0.cpu())
    oh = torch.empty_like(xh).pin_memory()
    for _ in range(max(1, args.warmup)):
        x.copy_(xh, non_blocking=True)
        g.replay()
        oh.copy_(x, non_blocking=True)
    barrier(dist)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        x.copy_(xh, non_blocking=True)
        g.replay()
        oh.copy_(x, non_blocking=True)
    e1.record()
    e1.synchronize()
    barrier(dist)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dist)

    ops, lb, kmean, kp, kh = kernel_roofline(stk, shape, B, pos, peak_gbs)
    main_ops = [n for n in ("attn_in", "attn_out", "mlp_block") if n in ops]
    dom = max(main_ops, key=lambda n: ops[n]["us"])
    wl_tag = f"{args.config}-b{B}-s{int(round(args.sparsity * 100))}"
    traffic = measured_traffic(dom, workload=wl_tag)
    us_layer = ms * 1e3 / nL
    value = ms * 1e3 / (nL * world)  # whole job: all ranks' layer-steps in the max-over-ranks time
    del g
    side = {}
    if world == 1:
        headline_layer0 = layers[0]
        if not args.no_extra:
            side["int8_blocks"] = int8_blocks(stk, shape, pos, peak_gbs)
        del stk
        free_gpu()
        if not args.no_sweep:
            side["opt175b_sweep"] = sweep_175b(layers, shape.with_(B=1), args, dist)
        cpu = None
        if rank == 0 and not args.no_cpu_baseline:
            cpu = cpu_baseline(headline_layer0, shape.with_(B=1), k, k_h, args.cpu_seconds)
        del layers, ls, headline_layer0
        free_gpu()
        if not args.no_extra:
            side["opt6.7b_generation"] = generation(wl.CONFIGS["opt-6.7b"], 32, True, 128, dist)
            side["opt66b"] = opt66b(wl.CONFIGS["opt-66b"], 64, dist)
            side["opt1.3b"] = opt13b(dist)
            side["tiny"] = tiny_latency(dist)
    else:
        cpu = None

    line = {
        "metric": METRIC, "value": value, "unit": "us", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": dict(config_of(args.config, shape, nL, B, k, k_h, not args.no_lookahead),
                       parallelism=f"replicas x{world}",
                       l2=f"inputs larger than L2: {nL} layers, {weight_bytes(shape) * nL / 1e9:.0f} GB of "
                          "weights streamed per step"),
        "tokens_per_s": B * world * 1e3 / ms,
        "us_per_layer_step": us_layer,
        "selected": {"k": kmean, "k_eff": kp, "k_h": kh},
        "bytes_per_layer": lb.total,
        "effective_gbs": lb.total / us_layer / 1e3,
        "effective_frac": lb.total / us_layer / 1e3 / peak_gbs,
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": ops[dom]["gbs"], "peak": peak_gbs, "unit": "GB/s",
                     "frac": ops[dom]["frac"], "traffic": traffic["bytes"] if traffic else None,
                     "traffic_source": traffic["source"] if traffic else None,
                     "algorithmic_bytes": ops[dom]["bytes"], "peak_source": peak_src, "per_op": ops},
        "e2e": {"value": e2e_ms * 1e3 / (nL * world), "unit": "us", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": xh.numel() * 4, "d2h_bytes_per_step": oh.numel() * 4},
        "gpu_launches": int(launches_per_step * args.steps),
        "launches_per_step": int(launches_per_step),
        "clocks": clocks,
        **side,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def weight_bytes(shape):
    """Bytes of one layer's weights and predictors (bf16 / fp32)."""
    w = acct.ELEM[shape.wdtype]
    return (2 * shape.N * shape.d + 4 * shape.h * shape.dh * shape.d + shape.h * shape.d + shape.r * shape.d
            + shape.N * shape.r) * w


if __name__ == "__main__":
    main()
