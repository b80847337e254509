"""Decoder stack driver with the asynchronous look-ahead predictor.

"Deja Vu: 利用上下文稀疏性提升大语言模型推理效率", §1: consecutive layers see
similar inputs (residual connections), so the sets of layer l+1 are predicted
from layer l's input, asynchronously, off the critical path. Here the
predictor of layer l+1 reads layer l's normalised attention input yA_l: its
first stage (head scores and z = yA_l A) runs inside layer l's q/k/v kernel,
the head selection on one side stream and the neuron scores and selection on
another, while the main stream runs layer l's sparse blocks; layer l+1 waits
on one event for its head set before its q/k/v and on another for its neuron
set before its MLP. Layer 0 predicts its own sets.

This module only orders library calls on streams (events, waits); every
arithmetic step runs in libdejavu's kernels. A step can be captured into a
CUDA graph (both streams fork and join inside the step).
"""

from __future__ import annotations

from typing import Dict, List, Optional

import torch

from . import binding as bd


class DecoderStack:
    def __init__(self, layers: List[Dict[str, torch.Tensor]], B: int, k: int, k_h: int, scale: float,
                 lookahead: bool = True, eps: float = 1e-5, mode: int = bd.DV_TOPK, tau: float = 0.0,
                 mode_h: int = bd.DV_TOPK, tau_h: float = 0.0, k_max: Optional[int] = None,
                 kh_max: Optional[int] = None, prefetch: bool = False, prefetch_w2: bool = True,
                 fuse_ahead: bool = True, act: int = bd.DV_ACT_RELU, exact_kv: bool = False):
        t0 = layers[0]
        N, d = t0["W1t"].shape
        h = t0["Wqkv"].shape[0]
        dev = t0["W1t"].device
        self.B, self.d, self.N, self.h = B, d, N, h
        self.k_max = k_max if k_max is not None else (N if mode == bd.DV_THRESHOLD else min(N, B * k))
        self.kh_max = kh_max if kh_max is not None else (h if mode_h == bd.DV_THRESHOLD else min(h, B * k_h))
        self.layers = [bd.Layer(t, B, self.k_max, self.kh_max) for t in layers]
        self.p = bd.params(k, k_h, scale, eps, tau, mode, tau_h, mode_h, act=act, exact_kv=exact_kv)
        self.lookahead = lookahead
        self.prefetch = prefetch and lookahead
        self.prefetch_w2 = prefetch_w2
        # the predictor's first stage for layer l+1 inside layer l's q/k/v kernel
        # (the L2 prefetch option keeps the one-call predictor on one side stream)
        self.fuse_ahead = fuse_ahead and not self.prefetch
        D = self.layers[0].dims
        self.ws_main = bd.workspace(bd.DV_OP_DECODE_LAYER, D, dev)
        self.ws_side = bd.workspace(bd.DV_OP_DECODE_LAYER, D, dev)
        # fused look-ahead: layer l+1's z and selection scratch live in the
        # side workspace of l+1's parity, so layer l+1's q/k/v kernel (which
        # writes z for l+2) never overwrites a z that is still being read
        self.ws_ahead = [self.ws_side, bd.workspace(bd.DV_OP_DECODE_LAYER, D, dev)] if self.fuse_ahead else []
        nL = len(layers)
        i32 = dict(dtype=torch.int32, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        # per-layer buffers: the layer's normalised input and its selected sets
        self.yA = [torch.empty(B, d, **f32) for _ in range(nL)]
        self.scores_h = [torch.empty(B, h, **f32) for _ in range(nL)]
        self.head_idx = [torch.zeros(h, **i32) for _ in range(nL)]
        self.head_count = [torch.zeros(1, **i32) for _ in range(nL)]
        self.scores = [torch.empty(B, N, **f32) for _ in range(nL)]
        self.idx = [torch.zeros(N, **i32) for _ in range(nL)]
        self.count = [torch.zeros(1, **i32) for _ in range(nL)]
        self.yM = [torch.empty(B, d, **f32) for _ in range(nL)]
        # the side stream writes a layer's sets here
        self.io_sets = [bd.layer_io(scores_h=self.scores_h[l], head_idx=self.head_idx[l],
                                    head_count=self.head_count[l], scores=self.scores[l], idx=self.idx[l],
                                    count=self.count[l]) for l in range(nL)]
        # a layer that predicts its own sets writes them (and yA, yM) here
        self.io_trace = [bd.layer_io(yA=self.yA[l], scores_h=self.scores_h[l], head_idx=self.head_idx[l],
                                     head_count=self.head_count[l], yM=self.yM[l], scores=self.scores[l],
                                     idx=self.idx[l], count=self.count[l]) for l in range(nL)]
        # a layer whose sets were predicted ahead reads them from here ...
        self.io_given = [bd.layer_io(head_idx=self.head_idx[l], head_count=self.head_count[l], idx=self.idx[l],
                                     count=self.count[l]) for l in range(nL)]
        # ... and writes its normalised block inputs here
        self.io_trace_y = [bd.layer_io(yA=self.yA[l], yM=self.yM[l]) for l in range(nL)]
        self.side = torch.cuda.Stream(device=dev)
        self.side_m = torch.cuda.Stream(device=dev)  # fused look-ahead: the neuron sets
        self.ev_heads = [torch.cuda.Event() for _ in range(nL)]
        self.ev_neurons = [torch.cuda.Event() for _ in range(nL)]
        self.ev_join_m = torch.cuda.Event()
        self.ev_yA = [torch.cuda.Event() for _ in range(nL)]
        self.ev_sel = [torch.cuda.Event() for _ in range(nL)]
        self.ev_join = torch.cuda.Event()

    def step(self, x: torch.Tensor, pos: int):
        """One token through every layer, in place on the residual x [B][d]."""
        if self.lookahead and self.fuse_ahead and len(self.layers) > 1:
            return self._step_fused(x, pos)
        main = torch.cuda.current_stream()
        nL = len(self.layers)
        la = self.lookahead and nL > 1
        for l, L in enumerate(self.layers):
            if la and l > 0:
                main.wait_event(self.ev_sel[l])  # sets of layer l, predicted from layer l-1
                sel, trace = self.io_given[l], self.io_trace_y[l]
            else:
                sel, trace = None, self.io_trace[l]
            bd.dv_decode_layer_begin(L, self.p, x, pos, self.ws_main, sel=sel, trace=trace)
            if la and l + 1 < nL:
                self.ev_yA[l].record(main)  # yA[l] is written by the work just issued
                self._predict_next(l, pos)
            bd.dv_decode_layer_end(L, self.p, x, pos, self.ws_main, sel=sel, trace=trace)
        if la:
            # join the side stream back into the main stream
            self.ev_join.record(self.side)
            main.wait_event(self.ev_join)

    def _step_fused(self, x: torch.Tensor, pos: int):
        """Look-ahead with the predictor's first stage for layer l+1 inside
        layer l's q/k/v kernel. The head selection runs on one side stream and
        the neuron scores and selection on another. Both waits of the main
        stream sit just before layer l's MLP kernel: the neuron set of layer l
        is read there, and the head set of layer l+1 is read by layer l+1's
        q/k/v kernel, which follows the MLP kernel with programmatic launch
        (a kernel after a cross-stream wait cannot launch early, so no wait
        sits in front of the q/k/v or attention kernels)."""
        main = torch.cuda.current_stream()
        nL = len(self.layers)
        for l, L in enumerate(self.layers):
            if l > 0:
                sel, trace = self.io_given[l], self.io_trace_y[l]
            else:
                sel, trace = None, self.io_trace[l]
            if l + 1 < nL:
                ws_next = self.ws_ahead[(l + 1) % 2]
                bd.dv_decode_layer_begin_ahead(L, self.p, x, pos, self.ws_main, self.layers[l + 1],
                                               self.scores_h[l + 1], ws_next, sel=sel, trace=trace)
                self.ev_yA[l].record(main)  # the first stage for l+1 is written by the work just issued
                self.side.wait_event(self.ev_yA[l])
                bd.dv_predict_layer_tail(self.layers[l + 1], self.p, self.io_sets[l + 1], ws_next,
                                         sets=bd.DV_SET_HEADS, stream=self.side)
                self.ev_heads[l + 1].record(self.side)
                self.side_m.wait_event(self.ev_yA[l])
                bd.dv_predict_layer_tail(self.layers[l + 1], self.p, self.io_sets[l + 1], ws_next,
                                         sets=bd.DV_SET_NEURONS, stream=self.side_m)
                self.ev_neurons[l + 1].record(self.side_m)
            else:
                bd.dv_decode_layer_begin(L, self.p, x, pos, self.ws_main, sel=sel, trace=trace)
            bd.dv_decode_layer_attn(L, self.p, x, pos, self.ws_main, sel=sel, trace=trace)
            if l > 0:
                main.wait_event(self.ev_neurons[l])
            if l + 1 < nL:
                main.wait_event(self.ev_heads[l + 1])
            bd.dv_decode_layer_mlp(L, self.p, x, self.ws_main, sel=sel, trace=trace)
        self.ev_join.record(self.side)
        main.wait_event(self.ev_join)
        self.ev_join_m.record(self.side_m)
        main.wait_event(self.ev_join_m)

    def _predict_next(self, l: int, pos: int):
        """Side stream: the sets of layer l+1 from layer l's yA, then an L2
        prefetch of the parameters those sets select (layer l+1 runs after
        layer l on the main stream, and finds them in L2)."""
        self.side.wait_event(self.ev_yA[l])
        bd.dv_predict_layer(self.layers[l + 1], self.p, self.yA[l], self.io_sets[l + 1], self.ws_side,
                            stream=self.side)
        self.ev_sel[l + 1].record(self.side)
        if self.prefetch:
            bd.dv_prefetch_layer(self.layers[l + 1], self.io_sets[l + 1], pos, with_w2=self.prefetch_w2,
                                 stream=self.side)
