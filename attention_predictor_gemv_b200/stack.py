"""Decoder stack driver with the asynchronous look-ahead predictor.

"Deja Vu: 利用上下文稀疏性提升大语言模型推理效率", §1: consecutive layers see
similar inputs (residual connections), so the sets of layer l+1 are predicted
from layer l's input, asynchronously, off the critical path. Here the
predictor of layer l+1 runs on a side CUDA stream from layer l's normalised
attention input yA_l while the main stream runs layer l's sparse blocks; layer
l+1 waits on an event for its sets. Layer 0 predicts its own sets.

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
                 fuse_ahead: bool = True):
        t0 = layers[0]
        N, d = t0["W1t"].shape
        h = t0["Wqkv"].shape[0]
        dev = t0["W1t"].device
        self.B, self.d, self.N, self.h = B, d, N, h
        self.k_max = k_max if k_max is not None else (N if mode == bd.DV_THRESHOLD else min(N, B * k))
        self.kh_max = kh_max if kh_max is not None else (h if mode_h == bd.DV_THRESHOLD else min(h, B * k_h))
        self.layers = [bd.Layer(t, B, self.k_max, self.kh_max) for t in layers]
        self.p = bd.params(k, k_h, scale, eps, tau, mode, tau_h, mode_h)
        self.lookahead = lookahead
        self.prefetch = prefetch and lookahead
        self.prefetch_w2 = prefetch_w2
        # the predictor's first stage for layer l+1 inside layer l's q/k/v kernel
        self.fuse_ahead = fuse_ahead
        D = self.layers[0].dims
        self.ws_main = bd.workspace(bd.DV_OP_DECODE_LAYER, D, dev)
        self.ws_side = bd.workspace(bd.DV_OP_DECODE_LAYER, D, dev)
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
        self.ev_yA = [torch.cuda.Event() for _ in range(nL)]
        self.ev_sel = [torch.cuda.Event() for _ in range(nL)]
        self.ev_join = torch.cuda.Event()

    def step(self, x: torch.Tensor, pos: int):
        """One token through every layer, in place on the residual x [B][d]."""
        main = torch.cuda.current_stream()
        nL = len(self.layers)
        la = self.lookahead and nL > 1
        for l, L in enumerate(self.layers):
            if la and l > 0:
                main.wait_event(self.ev_sel[l])  # sets of layer l, predicted from layer l-1
                sel, trace = self.io_given[l], self.io_trace_y[l]
            else:
                sel, trace = None, self.io_trace[l]
            ahead = la and l + 1 < nL
            if ahead and self.fuse_ahead:
                bd.dv_decode_layer_begin_ahead(L, self.p, x, pos, self.ws_main, self.layers[l + 1],
                                               self.scores_h[l + 1], self.ws_side, sel=sel, trace=trace)
            else:
                bd.dv_decode_layer_begin(L, self.p, x, pos, self.ws_main, sel=sel, trace=trace)
            if ahead:
                self.ev_yA[l].record(main)  # yA[l] (and the first stage for l+1) written by the work just issued
                self._predict_next(l, pos)
            bd.dv_decode_layer_end(L, self.p, x, pos, self.ws_main, sel=sel, trace=trace)
        if la:
            # join the side stream back into the main stream
            self.ev_join.record(self.side)
            main.wait_event(self.ev_join)

    def _predict_next(self, l: int, pos: int):
        """Side stream: the sets of layer l+1 from layer l's yA, then an L2
        prefetch of the parameters those sets select (layer l+1 runs after
        layer l on the main stream, and finds them in L2)."""
        self.side.wait_event(self.ev_yA[l])
        if self.fuse_ahead:
            bd.dv_predict_layer_tail(self.layers[l + 1], self.p, self.io_sets[l + 1], self.ws_side,
                                     stream=self.side)
        else:
            bd.dv_predict_layer(self.layers[l + 1], self.p, self.yA[l], self.io_sets[l + 1], self.ws_side,
                                stream=self.side)
        self.ev_sel[l + 1].record(self.side)
        if self.prefetch:
            bd.dv_prefetch_layer(self.layers[l + 1], self.io_sets[l + 1], pos, with_w2=self.prefetch_w2,
                                 stream=self.side)
