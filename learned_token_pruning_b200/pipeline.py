"""One gated prefill step on the device: gate score -> top-K select -> gather ->
one token-gated decoder layer above the gate (the three-stage forward of
"TokenGate and T2Quant: a close reading", §4.1, for the gate layer and the
first pruned layer).

This module only owns device buffers and calls the C-ABI entry points in
order on one stream; it never computes anything itself.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

from . import synth
from . import tokengate as tg


def to_device(a: np.ndarray, dtype: torch.dtype, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device=device, dtype=dtype)


class GatedPrefillStep:
    """Device-resident buffers of one workload plus the four library calls."""

    def __init__(self, w: synth.Workload, device="cuda", gate: Optional[Dict] = None, layer: Optional[Dict] = None,
                 head: Optional[Dict] = None, norm_eps: float = 1e-6, eps_s: float = 1e-6,
                 pass_norm_weight: bool = False):
        self.w = w
        self.device = torch.device(device)
        dt = synth.torch_dtype(w.dtype)
        self.dt = dt
        gate = synth.gate_inputs(w) if gate is None else gate
        layer = synth.layer_weights(w) if layer is None else layer
        head = synth.head_params(w) if head is None else head
        dev = self.device
        self.norm_eps, self.eps_s = norm_eps, eps_s
        self.hidden = to_device(gate["hidden"], dt, dev)
        self.prunable = to_device(gate["prunable"], torch.uint8, dev)
        self.n_prunable = int(gate["prunable"].sum())
        self.norm_w = to_device(gate["norm_w"], torch.float32, dev) if pass_norm_weight else None
        self.w1 = to_device(gate["w1"], dt, dev)
        self.b1 = to_device(gate["b1"], torch.float32, dev)
        self.w2 = to_device(gate["w2"], torch.float32, dev)
        self.b2 = float(gate["b2"])
        self.scores = torch.empty(w.n, dtype=torch.float32, device=dev)
        self.sumsq = torch.empty(1, dtype=torch.float32, device=dev)
        gws = tg.tg_workspace_bytes(tg.TG_OP_GATE_SCORE, n=w.n, d_model=w.d_model, h=w.gate_hidden)
        self.ws_gate = torch.empty(max(gws, 16), dtype=torch.uint8, device=dev)
        self.m = min(w.k, self.n_prunable) + (w.n - self.n_prunable)
        self.kept = torch.empty(self.m, dtype=torch.int32, device=dev)
        self.hidden_kept = torch.empty(self.m, w.d_model, dtype=dt, device=dev)
        self.pos = torch.empty(self.m, dtype=torch.int32, device=dev)
        self.bias = torch.empty(self.m, dtype=torch.float32, device=dev)
        self.ratio = torch.empty(self.m, dtype=torch.float32, device=dev)
        self.layer = {k: to_device(v, torch.float32 if k.endswith("norm") else dt, dev) for k, v in layer.items()}
        self.layer["head_gain"] = to_device(head["head_gain"], torch.float32, dev)
        self.layer["head_temp"] = to_device(head["head_temp"], torch.float32, dev)
        self.W, self.S = tg.layer_structs(self.layer, dtype=dt, d_model=w.d_model, hq=w.hq, hkv=w.hkv,
                                          head_dim=w.head_dim, d_ff=w.d_ff, qk_norm=w.qk_norm,
                                          rope_theta=w.rope_theta, norm_eps=norm_eps)
        lws = tg.tg_workspace_bytes(tg.TG_OP_LAYER, m=self.m, shape=self.S)
        self.ws_layer = torch.empty(lws, dtype=torch.uint8, device=dev)

    def gate_score(self, stream=None):
        tg.tg_gate_score(self.hidden, self.norm_w, self.norm_eps, self.w1, self.b1, self.w2, self.b2, self.prunable,
                         self.scores, self.sumsq, self.ws_gate, stream)

    def select(self, stream=None):
        tg.tg_topk_select(self.scores, self.prunable, self.n_prunable, self.w.k, self.kept, stream)

    def gather(self, stream=None):
        tg.tg_gather(self.hidden, self.kept, self.scores, self.sumsq, self.n_prunable, self.eps_s, self.hidden_kept,
                     self.pos, self.bias, self.ratio, stream)

    def layer_above(self, stream=None):
        tg.tg_pruned_prefill_layer(self.W, self.S, self.hidden_kept, self.pos, self.bias, self.ratio, self.ws_layer,
                                   stream)

    def run(self, stream=None):
        """One whole step; the result is left in self.hidden_kept ([m, d_model])."""
        self.gate_score(stream)
        self.select(stream)
        self.gather(stream)
        self.layer_above(stream)
        return self.hidden_kept

    def capture(self):
        """Record run() once into a CUDA graph, so a step costs one graph launch
        (the TMA descriptors and launch parameters are baked into the graph).
        One eager step runs first to set the kernels' attributes up."""
        self.run()
        torch.cuda.synchronize(self.device)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self.run()
        self._graph = graph
        return graph

    def replay(self):
        """One step by replaying the captured graph on the current stream."""
        if getattr(self, "_graph", None) is None:
            self.capture()
        self._graph.replay()
        return self.hidden_kept
