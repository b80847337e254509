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
                 kh_max: Optional[int] = None):
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
        self.io_sets = [bd.layer_io(yA=self.yA[l], scores_h=self.scores_h[l], head_idx=self.head_idx[l],
                                    head_count=self.head_count[l], scores=self.scores[l], idx=self.idx[l],
                                    count=self.count[l]) for l in range(nL)]
        self.io_trace = [bd.layer_io(yA=self.yA[l], scores_h=self.scores_h[l], head_idx=self.head_idx[l],
                                     head_count=self.head_count[l], yM=self.yM[l], scores=self.scores[l],
                                     idx=self.idx[l], count=self.count[l]) for l in range(nL)]
        self.io_given = [bd.layer_io(yA=self.yA[l], head_idx=self.head_idx[l], head_count=self.head_count[l],
                                     idx=self.idx[l], count=self.count[l]) for l in range(nL)]
        self.io_trace_yM = [bd.layer_io(yM=self.yM[l]) for l in range(nL)]
        # layer 0 under look-ahead: the side stream reads yA[0] while layer 0
        # runs, so layer 0 keeps its own LN1 output in the workspace
        self.io_trace_no_yA = [bd.layer_io(scores_h=self.scores_h[l], head_idx=self.head_idx[l],
                                           head_count=self.head_count[l], yM=self.yM[l], scores=self.scores[l],
                                           idx=self.idx[l], count=self.count[l]) for l in range(nL)]
        self.side = torch.cuda.Stream(device=dev)
        self.ev_yA = [torch.cuda.Event() for _ in range(nL)]
        self.ev_sel = [torch.cuda.Event() for _ in range(nL)]

    def step(self, x: torch.Tensor, pos: int):
        """One token through every layer, in place on the residual x [B][d]."""
        main = torch.cuda.current_stream()
        nL = len(self.layers)
        for l, L in enumerate(self.layers):
            if not self.lookahead or l == 0:
                if self.lookahead and nL > 1:
                    bd.dv_layernorm(x, self.yA[l], L.t.get("ln1_g"), L.t.get("ln1_b"), self.p.eps)
                    self.ev_yA[l].record(main)
                    self._predict_next(l)
                    bd.dv_decode_layer(L, self.p, x, pos, self.ws_main, trace=self.io_trace_no_yA[l])
                else:
                    bd.dv_decode_layer(L, self.p, x, pos, self.ws_main, trace=self.io_trace[l])
            else:
                bd.dv_layernorm(x, self.yA[l], L.t.get("ln1_g"), L.t.get("ln1_b"), self.p.eps)
                if l + 1 < nL:
                    self.ev_yA[l].record(main)
                    self._predict_next(l)
                main.wait_event(self.ev_sel[l])
                bd.dv_decode_layer(L, self.p, x, pos, self.ws_main, sel=self.io_given[l],
                                   trace=self.io_trace_yM[l])

    def _predict_next(self, l: int):
        """Side stream: the sets of layer l+1 from layer l's yA."""
        self.side.wait_event(self.ev_yA[l])
        bd.dv_predict_layer(self.layers[l + 1], self.p, self.yA[l], self.io_sets[l + 1], self.ws_side,
                            stream=self.side)
        self.ev_sel[l + 1].record(self.side)
