"""Benchmark: one decode step of an OPT-1.3B-shaped decoder (24 layers of the
d=2048, N=8192, h=32, dh=64 layer, KV length 512, batch 1, bf16 weights,
fp32 accumulation) with contextual sparsity: the look-ahead predictors, top-k
selection, sparse MHA over the selected heads and sparse MLP over the
selected neurons, through the C ABI.

Metric: microseconds per decode step per layer (lower is better), with the
effective HBM bandwidth on the selected bytes. The 24 layers hold 2.6 GB of
weights, more than L2 (126 MB), so every step streams its selected bytes
from HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

For N > 1 (torchrun) every rank runs an independent replica (the path has
no exchange step); the time is the maximum over ranks.
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
CONFIG = "opt-1.3b"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=24)
    ap.add_argument("--k-frac", type=float, default=0.10)
    ap.add_argument("--kh-frac", type=float, default=0.25)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--no-lookahead", action="store_true")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-big", action="store_true", help="skip the OPT-175B-shaped measurement")
    ap.add_argument("--big-layers", type=int, default=4)
    ap.add_argument("--prefetch", action="store_true", help="L2-prefetch each layer's selected rows on the side stream")
    ap.add_argument("--no-prefetch-w2", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    return ap.parse_args()


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
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:  # host-only ranks (the reference arm, tests): gloo
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
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

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "100"], stdout=subprocess.PIPE,
                                      stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.p = None
        time.sleep(0.25)
        return self

    def __exit__(self, *a):
        time.sleep(0.15)
        self.out = ""
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
# the GPU arm
# ---------------------------------------------------------------------------


def build_stack(shape, nlayers, B, k, k_h, lookahead, seed0=1000, layers=None, prefetch=False, prefetch_w2=True):
    from attention_predictor_gemv_b200.stack import DecoderStack

    if layers is None:
        layers = [wl.make_layer(shape, seed0 + l, "cuda") for l in range(nlayers)]
    stk = DecoderStack(layers, B, k, k_h, 1.0 / float(np.sqrt(shape.dh)), lookahead=lookahead, prefetch=prefetch,
                       prefetch_w2=prefetch_w2)
    return stk, layers


def capture(stk, x, pos):
    """The decode step as a CUDA graph, and how many library kernels it holds."""
    from attention_predictor_gemv_b200 import binding as bd

    stk.step(x, pos)  # eager warm-up
    torch.cuda.synchronize()
    n0 = bd.dv_launch_count()
    g = graph_of(lambda: stk.step(x, pos))
    n1 = bd.dv_launch_count()
    return g, (n1 - n0) // 2  # graph_of runs fn once eagerly, then captures it


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
    """Mean k (selected neurons), k' (nonzero activations) and k_h over layers."""
    ks, khs = [], []
    for l in range(len(stk.layers)):
        ks.append(int(stk.count[l].item()))
        khs.append(int(stk.head_count[l].item()))
    return float(np.mean(ks)), float(np.mean(khs))


def nonzero_neurons(stk):
    """k' per layer: selected neurons with a nonzero activation, read from the
    workspace-independent recomputation y_M . W1 + b1 on the device (torch)."""
    kp = []
    for l, L in enumerate(stk.layers):
        c = int(stk.count[l].item())
        idx = stk.idx[l][:c].long()
        pre = stk.yM[l] @ L.t["W1t"][idx].float().t() + L.t["b1"][idx]
        kp.append(int((pre > 0).any(dim=0).sum().item()))
    return float(np.mean(kp))


def layer_bytes(shape, k, kp, kh, B):
    return acct.layer_bytes(shape.d, shape.N, shape.r, shape.h, shape.dh, int(round(k)), int(round(kp)),
                            int(round(kh)), B, shape.L + 1)


def graph_of(fn):
    """Captures fn (library launches on the current stream) into a CUDA graph."""
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


# Source headers of each main-path kernel, for matching a committed ncu
# capture to the code that runs now.
KERNEL_HEADERS = {
    "attn_in": ("dv_common.cuh", "dv_fused.cuh", "dv_colowner.cuh"),
    "mlp_block": ("dv_common.cuh", "dv_fused.cuh", "dv_colowner.cuh"),
    "attn_out": ("dv_common.cuh", "dv_kernels.cuh", "dv_fused.cuh"),
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


def measured_traffic(op, profiles_dir=None):
    """Per-launch DRAM bytes (read + write) of `op`'s kernel from the ncu
    summary under profiles/ (lines `traffic <op> <bytes> <sha256 prefix>`),
    or None when no capture exists or the kernel's headers changed since."""
    import glob

    digest = kernel_sources_digest(op)
    pdir = profiles_dir or os.path.join(ROOT, "profiles")
    for path in sorted(glob.glob(os.path.join(pdir, "*.md"))):
        with open(path) as fh:
            for line in fh:
                parts = line.split()
                if len(parts) == 4 and parts[0] == "traffic" and parts[1] == op and parts[3] == digest:
                    return {"bytes": int(parts[2]), "source": os.path.relpath(path, ROOT)}
    return None


def kernel_roofline(stk, shape, B, pos, peak_gbs, reps=20):
    """Average duration of each main-path kernel in the look-ahead steady
    state (sets given): one CUDA graph per kernel with that kernel's call for
    every layer, timed with CUDA events on the launching stream; each
    kernel's algorithmic bytes per launch divided by its average duration.
    The residual state is restored afterwards."""
    from attention_predictor_gemv_b200 import binding as bd

    nL = len(stk.layers)
    x = torch.randn(B, shape.d, device="cuda")
    snap = [(t["K"].clone(), t["V"].clone()) for t in (L.t for L in stk.layers)]
    kp = nonzero_neurons(stk)
    k, kh = selected_counts(stk)
    lb = layer_bytes(shape, k, kp, kh, B)
    p, ws = stk.p, stk.ws_main
    calls = {
        "attn_in": (lambda l: bd.dv_decode_layer_begin(stk.layers[l], p, x, pos, ws, sel=stk.io_given[l],
                                                       trace=stk.io_trace_y[l]), lb.qkv),
        "attn_out": (lambda l: bd.dv_decode_layer_attn(stk.layers[l], p, x, pos, ws, sel=stk.io_given[l],
                                                       trace=stk.io_trace_y[l]), lb.kv + lb.wo),
        "mlp_block": (lambda l: bd.dv_decode_layer_mlp(stk.layers[l], p, x, ws, sel=stk.io_given[l],
                                                       trace=stk.io_trace_y[l]), lb.w1 + lb.w2),
    }
    res = {}
    for name, (fn, nbytes) in calls.items():
        g = graph_of(lambda: [fn(l) for l in range(nL)])
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        e1.synchronize()
        us = e0.elapsed_time(e1) * 1000.0 / (reps * nL)
        res[name] = {"us": us, "bytes": nbytes, "gbs": nbytes / us / 1e3, "frac": nbytes / us / 1e3 / peak_gbs}
        del g
    for t, (K, V) in zip((L.t for L in stk.layers), snap):
        t["K"].copy_(K)
        t["V"].copy_(V)
    return res, lb, k, kp, kh


def big_config(args, peak_gbs, dist):
    """OPT-175B-shaped layers (d=12288, N=49152, h=96, dh=128, KV 2048) at
    85% sparsity on neurons and heads, batch 1: the regime where the selected
    bytes (about 0.65 GB per layer) rather than latency bound the step."""
    shape = wl.CONFIGS["opt-175b"].with_(B=1)
    k, k_h = wl.k_for(0.15, shape.N), wl.k_for(0.15, shape.h)
    stk, layers = build_stack(shape, args.big_layers, 1, k, k_h, True, seed0=5000)
    x = wl.make_input(shape, 11, "cuda")
    g, _ = capture(stk, x, shape.L)
    ms = time_graph(g, 10, 3, dist)
    kern, lb, km, kp, kh = kernel_roofline(stk, shape, 1, shape.L, peak_gbs, reps=5)
    us_layer = ms * 1e3 / args.big_layers
    out = {"workload": f"{args.big_layers} OPT-175B-shaped layers: d={shape.d}, N={shape.N}, r={shape.r}, "
                       f"h={shape.h}, dh={shape.dh}, KV length {shape.L}, batch 1, k={k} (15%), k_h={k_h} (15%), "
                       "look-ahead", "us_per_layer_step": us_layer, "bytes_per_layer": lb.total,
           "effective_gbs": lb.total / us_layer / 1e3, "effective_frac": lb.total / us_layer / 1e3 / peak_gbs,
           "selected": {"k": km, "k_eff": kp, "k_h": kh}, "kernels": kern}
    del g, stk, layers
    torch.cuda.empty_cache()
    return out


def cpu_baseline(shape, B, k, k_h, seconds, seed=1000):
    """The oracle (float64 numpy) on a bounded sample: repeated layer-steps of
    one layer of the same shape, on the host cores."""
    from threadpoolctl import threadpool_info

    from oracle import dejavu_oracle as O

    t = wl.make_layer(shape, seed, "cpu")
    f = lambda a: O.bf16_bits_to_f64(a.contiguous().view(torch.int16).numpy().view(np.uint16)) \
        if a.dtype == torch.bfloat16 else a.double().numpy()  # noqa: E731
    L = O.LayerF64(PA=f(t["PA"]), Wqkv=f(t["Wqkv"]), bqkv=None, WOt=f(t["WOt"]), bO=None, K=f(t["K"]), V=f(t["V"]),
                   At=f(t["At"]), Bm=f(t["Bm"]), b1=f(t["b1"]), W1t=f(t["W1t"]), W2t=f(t["W2t"]))
    P = O.LayerParams(k=k, k_h=k_h, scale=1.0 / float(np.sqrt(shape.dh)))
    x = wl.make_input(shape, 0, "cpu").double().numpy()
    n, t0 = 0, time.perf_counter()
    while True:
        O.decode_layer(x, L, P, shape.L)
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return {"value": el * 1e6 / n, "unit": "us/layer-step", "cores": int(threads), "kind": "oracle",
            "sample": f"{n} layer-steps of one {CONFIG}-shaped layer (d={shape.d}, N={shape.N}, h={shape.h}, "
                      f"dh={shape.dh}, KV {shape.L}+1, B={B}, k={k}, k_h={k_h}), float64 numpy, full layer "
                      f"(LN, predictors, selection, sparse MHA, sparse MLP)"}


def run_reference(args, rank, dist):
    shape = wl.CONFIGS[CONFIG].with_(B=args.batch)
    k, k_h = wl.k_for(args.k_frac, shape.N), wl.k_for(args.kh_frac, shape.h)
    if rank != 0:
        return
    per_step = max(1.0, 60.0 / max(1, args.steps + args.warmup))
    cb = cpu_baseline(shape, args.batch, k, k_h, min(per_step, args.cpu_seconds))
    v = cb["value"]
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "us", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": v * args.layers / 1e3,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{CONFIG}-shaped decoder layer, batch {args.batch}, KV {shape.L}, "
                                   f"k={k}/{shape.N}, k_h={k_h}/{shape.h}", "layers": args.layers},
            "cpu_baseline": cb, "e2e": {"value": v, "unit": "us", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


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
    shape = wl.CONFIGS[CONFIG].with_(B=B)
    k, k_h = wl.k_for(args.k_frac, shape.N), wl.k_for(args.kh_frac, shape.h)
    pos = shape.L
    torch.manual_seed(rank)
    pf = dict(prefetch=args.prefetch, prefetch_w2=not args.no_prefetch_w2)
    stk, layers = build_stack(shape, args.layers, B, k, k_h, not args.no_lookahead, seed0=1000 + 100 * rank, **pf)
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
    dom = max(ops, key=lambda n: ops[n]["us"])
    traffic = measured_traffic(dom)
    total_layer_bytes = lb.total
    us_layer = ms * 1e3 / args.layers
    value = ms * 1e3 / (args.layers * world)  # whole job: all ranks' layer-steps in the max-over-ranks time

    sweep = []
    if not args.no_sweep:
        for kf in (0.05, 0.10, 0.20, 1.00):
            for hf in (0.25, 0.50, 1.00):
                kk, hh = wl.k_for(kf, shape.N), wl.k_for(hf, shape.h)
                s2, _ = build_stack(shape, args.layers, B, kk, hh, not args.no_lookahead, layers=layers, **pf)
                g2, _ = capture(s2, x, pos)
                m2 = time_graph(g2, max(10, args.steps // 2), 3, dist)
                kk_m, hh_m = selected_counts(s2)
                b2 = layer_bytes(shape, kk_m, nonzero_neurons(s2), hh_m, B).total
                sweep.append({"k_frac": kf, "kh_frac": hf, "k": kk, "k_h": hh, "us_per_layer": m2 * 1e3 / args.layers,
                              "bytes_per_layer": b2, "gbs": b2 / (m2 * 1e3 / args.layers) / 1e3})
                del g2, s2

    big = None
    if not args.no_big:
        big = big_config(args, peak_gbs, dist)

    line = {
        "metric": METRIC, "value": value, "unit": "us", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": f"{CONFIG}-shaped decoder (bf16 weights and KV cache, fp32 arithmetic): "
                               f"{args.layers} layers of d={shape.d}, N={shape.N}, "
                               f"r={shape.r}, h={shape.h}, dh={shape.dh}, KV length {shape.L}, batch {B}, "
                               f"k={k} ({args.k_frac:.0%}), k_h={k_h} ({args.kh_frac:.0%}), "
                               f"{'look-ahead' if not args.no_lookahead else 'synchronous'} prediction",
                   "global_batch": B * world, "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2: 24 layers, 2.6 GB of weights streamed per step"},
        "tokens_per_s": B * world * 1e3 / ms,
        "us_per_layer_step": us_layer,
        "selected": {"k": kmean, "k_eff": kp, "k_h": kh},
        "bytes_per_layer": total_layer_bytes,
        "effective_gbs": total_layer_bytes / us_layer / 1e3,
        "effective_frac": total_layer_bytes / us_layer / 1e3 / peak_gbs,
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": ops[dom]["gbs"], "peak": peak_gbs, "unit": "GB/s",
                     "frac": ops[dom]["frac"], "traffic": traffic["bytes"] if traffic else None,
                     "traffic_source": traffic["source"] if traffic else None,
                     "algorithmic_bytes": ops[dom]["bytes"], "peak_source": peak_src, "per_op": ops},
        "e2e": {"value": e2e_ms * 1e3 / (args.layers * world), "unit": "us", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": xh.numel() * 4, "d2h_bytes_per_step": oh.numel() * 4},
        "gpu_launches": int(launches_per_step * args.steps),
        "launches_per_step": int(launches_per_step),
        "clocks": clocks,
        "sweep": sweep,
        "opt175b_shaped": big,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(shape, B, k, k_h, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
