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
        gws = tg.tg_workspace_bytes(tg.TG_OP_GATE_SELECT, n=w.n, d_model=w.d_model, h=w.gate_hidden)
        self.ws_gate = torch.empty(max(gws, 16), dtype=torch.uint8, device=dev)  # tg_gate_score alone
        # the fused call's own workspace, zero-filled once: each call leaves its
        # counters at zero again, so no memset precedes the gate kernel
        self.ws_gate_sel = torch.zeros(max(gws, 16), dtype=torch.uint8, device=dev)
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

    def gate_select(self, stream=None):
        """Gate scores and the top-K selection, the selection's first radix pass
        folded into the scoring kernel."""
        tg.tg_gate_score_select(self.hidden, self.norm_w, self.norm_eps, self.w1, self.b1, self.w2, self.b2,
                                self.prunable, self.n_prunable, self.w.k, self.scores, self.sumsq, self.kept,
                                self.ws_gate_sel, stream, flags=tg.TG_WS_KEPT_ZERO)

    def gather(self, stream=None):
        tg.tg_gather(self.hidden, self.kept, self.scores, self.sumsq, self.n_prunable, self.eps_s, self.hidden_kept,
                     self.pos, self.bias, self.ratio, stream)

    def layer_above(self, stream=None):
        tg.tg_pruned_prefill_layer(self.W, self.S, self.hidden_kept, self.pos, self.bias, self.ratio, self.ws_layer,
                                   stream)

    def gather_layer(self, stream=None):
        """The gather folded into the layer above: one pass gathers the kept rows
        (and pos, bias, ratio) and normalises them for the QKV projection."""
        tg.tg_gather_prefill_layer(self.W, self.S, tg.TG_LAYER_FULL, self.hidden, self.kept, self.scores, self.sumsq,
                                   self.n_prunable, self.eps_s, self.hidden_kept, self.pos, self.bias, self.ratio,
                                   self.ws_layer, stream)

    def run(self, stream=None):
        """One whole step; the result is left in self.hidden_kept ([m, d_model])."""
        self.gate_select(stream)
        self.gather_layer(stream)
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


class BatchedPrefillStep:
    """Several requests through the gated step at once (varlen batching).  Per
    request: gate score -> top-K select -> gather, into one buffer of kept rows
    in which request r owns rows seg_rows[r] .. seg_rows[r+1]-1; then one
    tg_pruned_prefill_layer_varlen call over all rows (every step row-wise,
    attention per request).  The requests share the model: the gate and layer
    weights are those of the first workload; each request brings its own
    hidden states, prunable mask and budget K."""

    def __init__(self, ws, device="cuda", norm_eps: float = 1e-6, eps_s: float = 1e-6):
        w0 = ws[0]
        self.w = w0
        self.device = torch.device(device)
        dev, dt = self.device, synth.torch_dtype(w0.dtype)
        self.dt, self.norm_eps, self.eps_s = dt, norm_eps, eps_s
        gate0 = synth.gate_inputs(w0)
        self.gate_weights = {k: gate0[k] for k in ("norm_w", "w1", "b1", "w2", "b2")}
        self.w1 = to_device(gate0["w1"], dt, dev)
        self.b1 = to_device(gate0["b1"], torch.float32, dev)
        self.w2 = to_device(gate0["w2"], torch.float32, dev)
        self.b2 = float(gate0["b2"])
        self.reqs = []
        seg = [0]
        for w in ws:
            g = synth.gate_inputs(w)
            n_prunable = int(g["prunable"].sum())
            m = min(w.k, n_prunable) + (w.n - n_prunable)
            gws = tg.tg_workspace_bytes(tg.TG_OP_GATE_SCORE, n=w.n, d_model=w.d_model, h=w.gate_hidden)
            self.reqs.append({
                "w": w, "k": w.k, "n_prunable": n_prunable, "m": m,
                "hidden": to_device(g["hidden"], dt, dev), "prunable": to_device(g["prunable"], torch.uint8, dev),
                "scores": torch.empty(w.n, dtype=torch.float32, device=dev),
                "sumsq": torch.empty(1, dtype=torch.float32, device=dev),
                "ws_gate": torch.empty(max(gws, 16), dtype=torch.uint8, device=dev)})
            seg.append(seg[-1] + m)
        self.seg_rows = seg
        total = seg[-1]
        self.kept = torch.empty(total, dtype=torch.int32, device=dev)
        self.hidden_kept = torch.empty(total, w0.d_model, dtype=dt, device=dev)
        self.pos = torch.empty(total, dtype=torch.int32, device=dev)
        self.bias = torch.empty(total, dtype=torch.float32, device=dev)
        self.ratio = torch.empty(total, dtype=torch.float32, device=dev)
        layer = synth.layer_weights(w0)
        head = synth.head_params(w0)
        self.layer = {k: to_device(v, torch.float32 if k.endswith("norm") else dt, dev) for k, v in layer.items()}
        self.layer["head_gain"] = to_device(head["head_gain"], torch.float32, dev)
        self.layer["head_temp"] = to_device(head["head_temp"], torch.float32, dev)
        self.W, self.S = tg.layer_structs(self.layer, dtype=dt, d_model=w0.d_model, hq=w0.hq, hkv=w0.hkv,
                                          head_dim=w0.head_dim, d_ff=w0.d_ff, qk_norm=w0.qk_norm,
                                          rope_theta=w0.rope_theta, norm_eps=norm_eps)
        self.ws_layer = torch.empty(tg.tg_layer_varlen_workspace_bytes(self.S, seg), dtype=torch.uint8, device=dev)

    def rows(self, r: int) -> slice:
        return slice(self.seg_rows[r], self.seg_rows[r + 1])

    def front(self, stream=None):
        """Gate, select and gather of every request."""
        for r, q in enumerate(self.reqs):
            sl = self.rows(r)
            tg.tg_gate_score(q["hidden"], None, self.norm_eps, self.w1, self.b1, self.w2, self.b2, q["prunable"],
                             q["scores"], q["sumsq"], q["ws_gate"], stream)
            tg.tg_topk_select(q["scores"], q["prunable"], q["n_prunable"], q["k"], self.kept[sl], stream)
            tg.tg_gather(q["hidden"], self.kept[sl], q["scores"], q["sumsq"], q["n_prunable"], self.eps_s,
                         self.hidden_kept[sl], self.pos[sl], self.bias[sl], self.ratio[sl], stream)

    def layer_above(self, stream=None):
        tg.tg_pruned_prefill_layer_varlen(self.W, self.S, self.hidden_kept, self.pos, self.bias, self.ratio,
                                          self.seg_rows, self.ws_layer, stream)

    def run(self, stream=None):
        self.front(stream)
        self.layer_above(stream)
        return self.hidden_kept

    def capture(self):
        self.run()
        torch.cuda.synchronize(self.device)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self.run()
        self._graph = graph
        return graph

    def replay(self):
        if getattr(self, "_graph", None) is None:
            self.capture()
        self._graph.replay()
        return self.hidden_kept


class PrunedPrefillStack:
    """Prefill of one prompt through a decoder stack, the three-stage forward of
    "TokenGate and T2Quant: a close reading", §4.1 (Gate module; [K] "tying the
    mechanism together" and [M] "how does learned token pruning work" put the
    scoring in the same place):
      layers 0 .. L-1      all N rows;
      layer L, attention   all N rows -> the post-attention residual;
      gate                 scores that residual normalised by layer L's own
                           post-attention RMSNorm; top-K document tokens plus
                           every question token are selected;
      layer L, MLP         on the kept rows only, with the gather folded into
                           its RMSNorm;
      layers L+1 ..        on the kept rows with token-gated attention.
    `unpruned()` runs every layer on all rows with no gate.  Every step is a
    library call on the current stream.

    layers: per layer a dict of device tensors (tg_layer_weights names, without
    head_gain / head_temp); heads: per layer a dict with device tensors
    head_gain and head_temp (used by the layers above the gate; the layers on
    all rows run with no gate bias and unit temperature)."""

    def __init__(self, w: synth.Workload, hidden, prunable, gate: Dict, layers, heads, gate_layer: int,
                 norm_eps: float = 1e-6, eps_s: float = 1e-6):
        self.w, self.gate_layer, self.norm_eps, self.eps_s = w, gate_layer, norm_eps, eps_s
        dev = hidden.device
        self.dt = hidden.dtype
        self.hidden0 = hidden
        self.h = torch.empty_like(hidden)
        self.prunable = prunable
        self.n_prunable = int(prunable.sum().item())
        self.gate = gate
        self.m = min(w.k, self.n_prunable) + (w.n - self.n_prunable)
        self.pos_all = torch.arange(w.n, dtype=torch.int32, device=dev)
        self.scores = torch.empty(w.n, dtype=torch.float32, device=dev)
        self.sumsq = torch.empty(1, dtype=torch.float32, device=dev)
        # zero-filled once: each fused call leaves its counters at zero again
        self.ws_gate = torch.zeros(max(tg.tg_workspace_bytes(tg.TG_OP_GATE_SELECT, n=w.n, d_model=w.d_model,
                                                             h=gate["w1"].shape[0]), 16), dtype=torch.uint8,
                                   device=dev)
        self.kept = torch.empty(self.m, dtype=torch.int32, device=dev)
        self.hk = torch.empty(self.m, w.d_model, dtype=self.dt, device=dev)
        self.pos = torch.empty(self.m, dtype=torch.int32, device=dev)
        self.bias = torch.empty(self.m, dtype=torch.float32, device=dev)
        self.ratio = torch.empty(self.m, dtype=torch.float32, device=dev)
        ones = torch.ones(w.hq, dtype=torch.float32, device=dev)
        zeros = torch.zeros(w.hq, dtype=torch.float32, device=dev)
        # the gate normalises with layer L's post-attention RMSNorm weight
        self.gate_norm_w = layers[gate_layer]["w_post_norm"]
        self._keep = []  # device tensors the structs point to
        self.full_layers, self.pruned_layers = [], []
        for l, lw in enumerate(layers):
            for gated in (False, True):
                d = dict(lw)
                d["head_gain"], d["head_temp"] = (heads[l]["head_gain"], heads[l]["head_temp"]) if gated else (zeros, ones)
                W, S = tg.layer_structs(d, dtype=self.dt, d_model=w.d_model, hq=w.hq, hkv=w.hkv, head_dim=w.head_dim,
                                        d_ff=w.d_ff, qk_norm=w.qk_norm, rope_theta=w.rope_theta, norm_eps=norm_eps)
                self._keep.append(d)
                (self.pruned_layers if gated else self.full_layers).append((W, S))
        S0 = self.full_layers[0][1]
        ws = max(tg.tg_workspace_bytes(tg.TG_OP_LAYER, m=w.n, shape=S0),
                 tg.tg_workspace_bytes(tg.TG_OP_LAYER, m=self.m, shape=S0))
        self.ws_layer = torch.empty(ws, dtype=torch.uint8, device=dev)

    def reset(self):
        """Load the layer-0 input (kept out of the timed region by the caller)."""
        self.h.copy_(self.hidden0)

    def full_part(self):
        """Layers 0 .. L-1 and layer L's attention half on all rows: self.h ends
        as layer L's post-attention residual, the gate's input."""
        for W, S in self.full_layers[: self.gate_layer]:
            tg.tg_pruned_prefill_layer(W, S, self.h, self.pos_all, None, None, self.ws_layer)
        W, S = self.full_layers[self.gate_layer]
        tg.tg_layer_attention_block(W, S, self.h, self.pos_all, None, None, self.ws_layer)

    def gate_select(self):
        g = self.gate
        tg.tg_gate_score_select(self.h, self.gate_norm_w, self.norm_eps, g["w1"], g["b1"], g["w2"], g["b2"],
                                self.prunable, self.n_prunable, self.w.k, self.scores, self.sumsq, self.kept,
                                self.ws_gate, flags=tg.TG_WS_KEPT_ZERO)

    def gather_mlp(self):
        """Gather the kept rows of the residual into self.hk and run layer L's
        MLP half on them (the gather folded into its RMSNorm)."""
        W, S = self.full_layers[self.gate_layer]
        tg.tg_gather_prefill_layer(W, S, tg.TG_LAYER_MLP, self.h, self.kept, self.scores, self.sumsq, self.n_prunable,
                                   self.eps_s, self.hk, self.pos, self.bias, self.ratio, self.ws_layer)

    def pruned_part(self):
        for W, S in self.pruned_layers[self.gate_layer + 1:]:
            tg.tg_pruned_prefill_layer(W, S, self.hk, self.pos, self.bias, self.ratio, self.ws_layer)

    def run(self):
        """Layer-0 input in self.h -> kept-row output of the last layer in self.hk."""
        self.full_part()
        self.gate_select()
        self.gather_mlp()
        self.pruned_part()
        return self.hk

    def unpruned(self):
        """Every layer on all rows (self.h), no gate."""
        for W, S in self.full_layers:
            tg.tg_pruned_prefill_layer(W, S, self.h, self.pos_all, None, None, self.ws_layer)
        return self.h


def stack_weights_from_synth(w: synth.Workload, n_layers: int, device="cuda"):
    """Layer and head parameters of synth.py (the oracle reads the same arrays)."""
    dt = synth.torch_dtype(w.dtype)
    layers, heads = [], []
    for l in range(n_layers):
        lw = synth.layer_weights(w, layer=l)
        layers.append({k: to_device(v, torch.float32 if k.endswith("norm") else dt, device) for k, v in lw.items()})
        hp = synth.head_params(w, seed_offset=100 + l)
        heads.append({k: to_device(v, torch.float32, device) for k, v in hp.items()})
    return layers, heads


def stack_weights_on_device(w: synth.Workload, n_layers: int, device="cuda"):
    """The same distributions drawn by a seeded generator on the device (weights
    N(0, 0.02), norm weights 1, gain U(0.5, 2), temperature U(0.8, 1.2)), for
    stacks too large to draw on the host."""
    dt = synth.torch_dtype(w.dtype)
    d, D, hq, hkv, dff = w.d_model, w.head_dim, w.hq, w.hkv, w.d_ff
    layers, heads = [], []
    for l in range(n_layers):
        g = torch.Generator(device=device)
        g.manual_seed(w.seed * 1000 + 200 + l)
        rnd = lambda *shape: (torch.randn(*shape, generator=g, device=device) * 0.02).to(dt)
        layers.append({
            "w_in_norm": torch.ones(d, device=device), "w_qkv": rnd((hq + 2 * hkv) * D, d),
            "w_q_norm": torch.ones(D, device=device), "w_k_norm": torch.ones(D, device=device),
            "w_o": rnd(d, hq * D), "w_post_norm": torch.ones(d, device=device),
            "w_gate_up": rnd(2 * dff, d), "w_down": rnd(d, dff)})
        heads.append({"head_gain": torch.rand(hq, generator=g, device=device) * 1.5 + 0.5,
                      "head_temp": torch.rand(hq, generator=g, device=device) * 0.4 + 0.8})
    return layers, heads
