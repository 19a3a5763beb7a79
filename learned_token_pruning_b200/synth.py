"""Seeded synthetic inputs for the TokenGate pruned-prefill workloads.

This module only draws inputs: hidden states, gate and layer weights, the
prunable mask, per-head gains and temperatures, and (for the selector-only
long-context case) directly injected score arrays.  It contains none of the
method's arithmetic, so the CUDA path and the CPU oracle can both consume
exactly the same bytes.

Every array is returned as float32 numpy data whose values are already
representable in the workload dtype (bf16 workloads are rounded to bf16 once,
here), so a bf16 device tensor built from it is exact and an fp64 upcast for the
oracle is exact too.

Workload shapes follow the TokenGate setting: a document of N tokens followed by
a short question (the request/document split of the problem definition in the
TokenGate/T2Quant close reading, §3.1), a Qwen3-1.7B-shaped layer (the
experiments of §5.1 of the same page) and a budget K of kept document tokens.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and seed of one synthetic pruned-prefill problem."""

    name: str
    seed: int
    n: int                 # tokens in the prompt
    n_question: int        # non-prunable tokens (question), placed last unless question_first
    d_model: int
    hq: int
    hkv: int
    head_dim: int
    gate_hidden: int       # gate MLP hidden width (d_model -> gate_hidden -> 1)
    k: int                 # budget of kept document tokens
    dtype: str             # "f32" or "bf16"
    d_ff: int
    rope_theta: float = 1.0e6
    qk_norm: bool = True
    plant_len: int = 0     # planted high-score block length (0 = none)
    plant_shift: float = 3.0
    question_first: bool = False
    score_mixture: bool = False   # inject Gaussian-mixture scores for the selector
    n_layers: int = 1             # decoder layers of a whole-stack workload
    gate_layer: int = 0           # the gate scores this layer's post-attention residual

    @property
    def n_prunable(self) -> int:
        return self.n - self.n_question

    @property
    def m(self) -> int:
        return min(self.k, self.n_prunable) + self.n_question

    @property
    def plant_start(self) -> int:
        # midpoint of the document span
        doc0 = self.n_question if self.question_first else 0
        return doc0 + (self.n_prunable - self.plant_len) // 2

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def tiny_f32(**kw) -> Workload:
    """Tiny single gated layer in fp32 (N=512, last 32 question, K=128)."""
    w = Workload(name="tiny_f32_n512", seed=1, n=512, n_question=32, d_model=256, hq=4, hkv=2,
                 head_dim=64, gate_hidden=64, k=128, dtype="f32", d_ff=512, qk_norm=False,
                 plant_len=16)
    return w.replace(**kw) if kw else w


def qwen3_1p7b_16k(**kw) -> Workload:
    """Qwen3-1.7B-shaped single layer, bf16, N=16384 with 64 question tokens, K=2000."""
    w = Workload(name="qwen3_1.7b_layer_n16384_k2000", seed=2, n=16384, n_question=64,
                 d_model=2048, hq=16, hkv=8, head_dim=128, gate_hidden=256, k=2000, dtype="bf16",
                 d_ff=6144, plant_len=32)
    return w.replace(**kw) if kw else w


def budget_sweep_32k(k: int, **kw) -> Workload:
    """Same layer shape at N=32768, K in {1024, 4096, 8192}."""
    w = Workload(name=f"qwen3_1.7b_layer_n32768_k{k}", seed=3, n=32768, n_question=64,
                 d_model=2048, hq=16, hkv=8, head_dim=128, gate_hidden=256, k=k, dtype="bf16",
                 d_ff=6144)
    return w.replace(**kw) if kw else w


def long_128k(**kw) -> Workload:
    """Long context: N=131072, K=8192, selector scores from a 3-component mixture."""
    w = Workload(name="qwen3_1.7b_layer_n131072_k8192", seed=4, n=131072, n_question=64,
                 d_model=2048, hq=16, hkv=8, head_dim=128, gate_hidden=256, k=8192, dtype="bf16",
                 d_ff=6144, score_mixture=True)
    return w.replace(**kw) if kw else w


def full_stack_64k(**kw) -> Workload:
    """Random-init 28-layer Qwen3-1.7B-shaped stack, gate after layer 13,
    N=65536 with 64 question tokens, K=4096 (TTFT against the unpruned stack)."""
    w = Workload(name="qwen3_1.7b_stack28_n65536_k4096", seed=5, n=65536, n_question=64,
                 d_model=2048, hq=16, hkv=8, head_dim=128, gate_hidden=256, k=4096, dtype="bf16",
                 d_ff=6144, n_layers=28, gate_layer=13)
    return w.replace(**kw) if kw else w


def round_to(a: np.ndarray, dtype: str) -> np.ndarray:
    """Round float data to the workload dtype (round-to-nearest-even), keep it as float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    if dtype == "f32":
        return a
    if dtype == "bf16":
        return torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    raise ValueError(dtype)


def torch_dtype(dtype: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]


def prunable_mask(w: Workload) -> np.ndarray:
    """uint8[N]; 1 marks a document (prunable) token, 0 a question token."""
    mask = np.ones(w.n, dtype=np.uint8)
    if w.n_question:
        if w.question_first:
            mask[: w.n_question] = 0
        else:
            mask[w.n - w.n_question:] = 0
    return mask


def _normal(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    return (rng.standard_normal(shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


def gate_inputs(w: Workload) -> Dict[str, np.ndarray]:
    """Hidden states at the gate layer and the gate MLP weights.

    hidden ~ N(0,1) [N, d]; W1 [h, d] and w2 [h] ~ N(0, 0.02); b1 = 0, b2 = 0,
    norm weight = 1.  When a planted block is requested, its rows are moved
    by plant_shift (in units of the hidden std) along the unit vector
    W1^T w2 / |W1^T w2|, the direction in which the gate MLP, linearised at 0,
    rises fastest.
    """
    rng = np.random.Generator(np.random.PCG64(w.seed))
    w1 = round_to(_normal(rng, (w.gate_hidden, w.d_model), 0.02), w.dtype)
    w2 = round_to(_normal(rng, (w.gate_hidden,), 0.02), w.dtype)
    hidden = rng.standard_normal((w.n, w.d_model), dtype=np.float32)
    if w.plant_len:
        u = w1.astype(np.float64).T @ w2.astype(np.float64)
        u /= np.linalg.norm(u)
        s0 = w.plant_start
        hidden[s0:s0 + w.plant_len] += (w.plant_shift * u).astype(np.float32)
    hidden = round_to(hidden, w.dtype)
    return {
        "hidden": hidden,
        "norm_w": np.ones(w.d_model, dtype=np.float32),
        "w1": w1,
        "b1": np.zeros(w.gate_hidden, dtype=np.float32),
        "w2": w2,
        "b2": np.float32(0.0),
        "prunable": prunable_mask(w),
    }


def head_params(w: Workload, seed_offset: int = 100) -> Dict[str, np.ndarray]:
    """Per-head gain ~ U(0.5, 2) and temperature ~ U(0.8, 1.2) (post-softplus values)."""
    rng = np.random.Generator(np.random.PCG64(w.seed + seed_offset))
    gain = rng.uniform(0.5, 2.0, size=w.hq).astype(np.float32)
    temp = rng.uniform(0.8, 1.2, size=w.hq).astype(np.float32)
    return {"head_gain": gain, "head_temp": temp}


def layer_weights(w: Workload, seed_offset: int = 200, layer: int = 0) -> Dict[str, np.ndarray]:
    """Random-init Qwen3-style decoder layer: weights ~ N(0, 0.02), norm weights = 1.

    Linear weights use the [out_features, in_features] layout.
    """
    rng = np.random.Generator(np.random.PCG64(w.seed * 1000 + seed_offset + layer))
    d, D = w.d_model, w.head_dim
    out = {
        "w_in_norm": np.ones(d, dtype=np.float32),
        "w_qkv": round_to(_normal(rng, ((w.hq + 2 * w.hkv) * D, d), 0.02), w.dtype),
        "w_q_norm": np.ones(D, dtype=np.float32),
        "w_k_norm": np.ones(D, dtype=np.float32),
        "w_o": round_to(_normal(rng, (d, w.hq * D), 0.02), w.dtype),
        "w_post_norm": np.ones(d, dtype=np.float32),
        # gate and up projections interleaved in blocks: rows [gate(d_ff); up(d_ff)]
        "w_gate_up": round_to(_normal(rng, (2 * w.d_ff, d), 0.02), w.dtype),
        "w_down": round_to(_normal(rng, (d, w.d_ff), 0.02), w.dtype),
    }
    return out


def attention_inputs(w: Workload, m: Optional[int] = None, seed_offset: int = 300) -> Dict[str, np.ndarray]:
    """Standalone q/k/v for the gated-attention kernel: q [m,hq,D], k/v [m,hkv,D] ~ N(0,1)."""
    m = w.m if m is None else m
    rng = np.random.Generator(np.random.PCG64(w.seed * 1000 + seed_offset))
    q = round_to(rng.standard_normal((m, w.hq, w.head_dim), dtype=np.float32), w.dtype)
    k = round_to(rng.standard_normal((m, w.hkv, w.head_dim), dtype=np.float32), w.dtype)
    v = round_to(rng.standard_normal((m, w.hkv, w.head_dim), dtype=np.float32), w.dtype)
    bias = rng.standard_normal(m).astype(np.float32)
    # ratios in (0, 1], first row 0, as a kept set drawn from a longer prompt would give
    ratio = rng.uniform(0.6, 1.0, size=m).astype(np.float32)
    ratio[0] = 0.0
    return {"q": q, "k": k, "v": v, "bias": bias, "ratio": ratio}


def mixture_scores(n: int, seed: int, exact_ties: bool = False) -> np.ndarray:
    """Selector-level scores from a 3-component Gaussian mixture.

    Weights (0.85, 0.05, 0.10), means (0, 1.5, 3.0), stds (1.0, 0.3, 0.01): the
    narrow top component holds the top 10% of tokens, so a budget of 6.25% cuts
    through a cluster of near-ties.  With exact_ties the values are rounded to
    bf16 precision (kept as float32), which creates many exactly equal scores.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    comp = rng.choice(3, size=n, p=[0.85, 0.05, 0.10])
    means = np.array([0.0, 1.5, 3.0], dtype=np.float32)
    stds = np.array([1.0, 0.3, 0.01], dtype=np.float32)
    s = (means[comp] + stds[comp] * rng.standard_normal(n, dtype=np.float32)).astype(np.float32)
    if exact_ties:
        s = round_to(s, "bf16")
    return s
