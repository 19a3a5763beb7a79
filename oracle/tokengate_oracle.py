"""CPU oracle for the TokenGate pruned-prefill hot path -- TEST INFRASTRUCTURE.

This is a plain, slow, deliberately unoptimised restatement of what the method
computes, in float64 numpy.  It exists to check the CUDA library, never to stand
in for it: only the test suite, the smoke check in __graft_entry__ and the CPU
baseline leg of bench.py may import it.  It shares no code with the CUDA path;
the only module both sides use is the seeded input generator.

Sources (the TokenGate pages):
  [R]  "TokenGate and T2Quant: a close reading" (MessageDaily blog), §3.1
       (problem definition) and §4.1 (three-stage forward; Gate module; token-
       gated attention; head-wise gain; temperature scaling; engineering notes).
  [K]  "Stanford-Berkeley TokenGate" explainer (kg.zhiyong.dev), "putting the
       mechanism together".
  [M]  MarkTechPost TokenGate article (farwalk translation), "how does learned
       token pruning work" / "what is token-gated attention".

Readings where the pages leave a step open are marked READING below.  Every
function has a pin in tests/test_oracle_pins.py (brute force, closed forms,
invariants, or an independent library routine).
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence

import numpy as np

F64 = np.float64


# ---------------------------------------------------------------------------
# Gate scoring  ([R] §4.1 "Gate module"; [M] "how does ... work"; [K])
# ---------------------------------------------------------------------------

def rms_norm(x: np.ndarray, weight: Optional[np.ndarray], eps: float) -> np.ndarray:
    """Row-wise RMSNorm: x / sqrt(mean(x^2) + eps) * weight."""
    x = np.asarray(x, dtype=F64)
    r = np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    y = x / r
    if weight is not None:
        y = y * np.asarray(weight, dtype=F64)
    return y


def silu(u: np.ndarray) -> np.ndarray:
    """SiLU(u) = u * sigmoid(u) = u / (1 + exp(-u))."""
    u = np.asarray(u, dtype=F64)
    return u / (1.0 + np.exp(-u))


def gate_scores(hidden, norm_w, norm_eps, w1, b1, w2, b2, prunable) -> np.ndarray:
    """Raw gate scores s_j for every token.

    The gate reads the normalised post-attention residual of the gate layer
    (READING: RMSNorm with the layer's weight norm_w, eps norm_eps), runs the
    small MLP  s_j = w2 . SiLU(W1 x_j + b1) + b2  (W1 is [h, d], the
    nn.Linear layout), and fixes the score of every non-prunable token
    (instruction/question) to 0 ([R] §4.1 Gate module).
    Returns float64 [N].
    """
    x = rms_norm(hidden, norm_w, norm_eps)
    u = x @ np.asarray(w1, dtype=F64).T
    if b1 is not None:
        u = u + np.asarray(b1, dtype=F64)
    s = silu(u) @ np.asarray(w2, dtype=F64) + float(b2)
    s = np.where(np.asarray(prunable) != 0, s, 0.0)
    return s


def seq_rms(scores, prunable, eps_s: float) -> float:
    """r = sqrt(mean_{j in P} s_j^2 + eps_s), the sequence-wise RMS of the scores.

    [R] §4.1: the MLP scalars are RMS-normalised along the sequence into the
    importance scores b_j = s_j / r.  READING: the mean runs over the prunable
    set P only (non-prunable scores are fixed at 0 and are not part of the
    normalisation), there is no learnable scale, eps_s = 1e-6.
    """
    s = np.asarray(scores, dtype=F64)
    p = np.asarray(prunable) != 0
    n_p = int(p.sum())
    if n_p == 0:
        return math.sqrt(eps_s)
    return math.sqrt(float(np.sum(s[p] * s[p])) / n_p + eps_s)


def importance(scores, prunable, eps_s: float) -> np.ndarray:
    """b_j = s_j / r on P, 0 elsewhere ([R] §4.1)."""
    s = np.asarray(scores, dtype=F64)
    r = seq_rms(s, prunable, eps_s)
    return np.where(np.asarray(prunable) != 0, s / r, 0.0)


# ---------------------------------------------------------------------------
# Top-K selection  ([R] §4.1 "Top-K selector": S = top-K(b) U N)
# ---------------------------------------------------------------------------

def select_kept(scores, prunable, k: int) -> np.ndarray:
    """Kept token indices, ascending (int64).

    S = top-K(b_j) over the prunable set, united with every non-prunable token
    ([R] §4.1).  b is a positive multiple of s, so ranking by s ranks by b.
    READING (the pages fix no tie rule): rank by value, larger first; equal
    values (-0 == +0) go to the lower index; NaN ranks below every number.
    Done as a full stable sort of the prunable set, then a sort of the union.
    """
    s = np.asarray(scores, dtype=np.float32).astype(F64)
    p = np.flatnonzero(np.asarray(prunable) != 0)
    if k < 0:
        raise ValueError("k must be >= 0")
    kp = min(k, p.size)
    vals = s[p]
    nan = np.isnan(vals)
    primary = nan.astype(np.int64)                  # numbers first, NaN last
    secondary = np.where(nan, 0.0, -vals)           # larger value first
    order = np.lexsort((p, secondary, primary))     # last key is the primary key
    chosen = p[order[:kp]]
    keep = np.concatenate([chosen, np.flatnonzero(np.asarray(prunable) == 0)])
    return np.sort(keep).astype(np.int64)


# ---------------------------------------------------------------------------
# Compaction / gather  ([R] §4.1 three-stage forward, temperature scaling)
# ---------------------------------------------------------------------------

def temperature_ratio(kept_idx) -> np.ndarray:
    """log m_i / log max(2, p_i) for each kept row i ([R] §4.1 temperature scaling).

    READING: m_i = i + 1 is the number of kept keys query i sees (1-based rank
    in the compacted, causally ordered kept set) and p_i = idx_i + 1 the number
    of keys it would see in the unpruned prompt.
    """
    idx = np.asarray(kept_idx, dtype=F64)
    m_i = np.arange(1, idx.size + 1, dtype=F64)
    p_i = idx + 1.0
    return np.log(m_i) / np.log(np.maximum(2.0, p_i))


def gather(hidden, kept_idx, scores, prunable, eps_s: float) -> Dict[str, np.ndarray]:
    """Compacted rows of the kept tokens in original order, with their
    original positions, importance bias b and temperature ratio ([R] §4.1:
    pruned tokens never enter the layers above the gate)."""
    idx = np.asarray(kept_idx, dtype=np.int64)
    b = importance(scores, prunable, eps_s)
    return {
        "hidden_kept": np.asarray(hidden)[idx],
        "pos": idx.copy(),
        "bias": b[idx],
        "ratio": temperature_ratio(idx),
    }


# ---------------------------------------------------------------------------
# Token-gated attention  ([R] §4.1 token-gated attention, head gain, temperature)
# ---------------------------------------------------------------------------

def gated_attention(q, k, v, bias, head_gain, head_temp, ratio, sm_scale: float,
                    rows: Optional[Sequence[int]] = None, return_lse: bool = False):
    """Causal token-gated GQA attention over the kept rows.

    [R] §4.1: alpha_ij = exp(z_ij) g_j / sum_j' exp(z_ij') g_j' with
    g_j = softmax(b_j).  The softmax normaliser of g is common to every key and
    cancels, so alpha is a softmax over z_ij + b_j ([K] and [M] describe the
    score acting as a bias on the attention logits).  READINGS: the head-wise gain
    softplus(gamma_h) acts in log space, i.e. the bias term is gain_h * b_j (a
    plain multiplier on g_j would cancel); the temperature
    tau_i = softplus(sigma_h) * log m_i / log max(2, p_i) multiplies the content
    logit z_ij = (q_i . k_j) * sm_scale only.  So for head h with KV head
    g = h // (Hq/Hkv) and key c <= row r:
        l_rc = temp_h * ratio_r * sm_scale * (q_r . k_c) + gain_h * bias_c
        o_r  = sum_c softmax_c(l_r.) v_c
    q [M, Hq, D], k/v [M, Hkv, D]; bias/ratio [M] (None = 0 / 1).
    Returns o [M or len(rows), Hq, D] float64 (and lse [Hq, rows] natural log).
    """
    q = np.asarray(q, dtype=F64)
    k = np.asarray(k, dtype=F64)
    v = np.asarray(v, dtype=F64)
    m, hq, dh = q.shape
    hkv = k.shape[1]
    group = hq // hkv
    bias = np.zeros(m) if bias is None else np.asarray(bias, dtype=F64)
    ratio = np.ones(m) if ratio is None else np.asarray(ratio, dtype=F64)
    gain = np.asarray(head_gain, dtype=F64)
    temp = np.asarray(head_temp, dtype=F64)
    rows = np.arange(m) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.zeros((rows.size, hq, dh))
    lse = np.zeros((hq, rows.size))
    cols = np.arange(m)
    for h in range(hq):
        g = h // group
        z = (q[rows, h, :] @ k[:, g, :].T) * sm_scale              # [R, M]
        logits = (temp[h] * ratio[rows])[:, None] * z + gain[h] * bias[None, :]
        logits = np.where(cols[None, :] <= rows[:, None], logits, -np.inf)
        mx = logits.max(axis=1, keepdims=True)
        e = np.exp(logits - mx)
        den = e.sum(axis=1, keepdims=True)
        out[:, h, :] = (e / den) @ v[:, g, :]
        lse[h] = (mx + np.log(den))[:, 0]
    return (out, lse) if return_lse else out


def gated_attention_backward(q, k, v, bias, head_gain, head_temp, ratio, sm_scale: float, dout):
    """Gradients of token-gated attention ([R] §4.1 engineering notes: the same
    attention kernel accumulates the bias gradient back into the scorer; the
    gate value multiplies exp(z), i.e. the bias adds to the logits).

    With l_rc = temp_h * ratio_r * sm_scale * (q_r . k_c) + gain_h * bias_c for
    c <= r, P = softmax_c(l), o_r = sum_c P_rc v_c and upstream dO:
        dP_rc = dO_r . v_c,   dl_rc = P_rc * (dP_rc - dO_r . o_r)
        dq_r  = sum_c dl_rc * temp_h ratio_r sm_scale * k_c
        dk_c  = sum over the group's heads and rows of dl_rc * temp_h ratio_r sm_scale * q_r
        dv_c  = sum over the group's heads and rows of P_rc * dO_r
        dbias_c = sum over all heads h of gain_h * sum_r dl_rc
        dgain_h = sum_{r,c} dl_rc * bias_c
        dtemp_h = sum_{r,c} dl_rc * ratio_r * sm_scale * (q_r . k_c)
    Shapes as gated_attention; dout [M, Hq, D].  Returns a dict of float64
    arrays dq [M, Hq, D], dk/dv [M, Hkv, D], dbias [M], dgain/dtemp [Hq].
    """
    q = np.asarray(q, dtype=F64)
    k = np.asarray(k, dtype=F64)
    v = np.asarray(v, dtype=F64)
    do = np.asarray(dout, dtype=F64)
    m, hq, dh = q.shape
    hkv = k.shape[1]
    group = hq // hkv
    bias = np.zeros(m) if bias is None else np.asarray(bias, dtype=F64)
    ratio = np.ones(m) if ratio is None else np.asarray(ratio, dtype=F64)
    gain = np.asarray(head_gain, dtype=F64)
    temp = np.asarray(head_temp, dtype=F64)
    causal = np.tril(np.ones((m, m), dtype=bool))
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dbias = np.zeros(m)
    dgain = np.zeros(hq)
    dtemp = np.zeros(hq)
    for h in range(hq):
        g = h // group
        z = (q[:, h, :] @ k[:, g, :].T) * sm_scale                  # [M, M]
        a = temp[h] * ratio                                          # content scale per row
        logits = np.where(causal, a[:, None] * z + gain[h] * bias[None, :], -np.inf)
        p = np.exp(logits - logits.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        o = p @ v[:, g, :]
        dp = do[:, h, :] @ v[:, g, :].T
        dl = p * (dp - np.sum(do[:, h, :] * o, axis=1, keepdims=True))
        dq[:, h, :] = (dl * (a * sm_scale)[:, None]) @ k[:, g, :]
        dk[:, g, :] += (dl * (a * sm_scale)[:, None]).T @ q[:, h, :]
        dv[:, g, :] += p.T @ do[:, h, :]
        dbias += gain[h] * dl.sum(axis=0)
        dgain[h] = np.sum(dl * bias[None, :])
        dtemp[h] = np.sum(dl * ratio[:, None] * z)
    return {"dq": dq, "dk": dk, "dv": dv, "dbias": dbias, "dgain": dgain, "dtemp": dtemp}


# ---------------------------------------------------------------------------
# Decode over the gated KV cache  ([R] §4.1 Gate module, temperature scaling,
# engineering notes)
# ---------------------------------------------------------------------------

def decode_temperature_ratio(m_kept: int, n_prompt: int, t: int) -> float:
    """Temperature ratio of the query generated at decode step t (0-based).

    [R] §4.1: tokens produced while decoding are not prunable (their score is
    fixed at 0), and tau = softplus(sigma) * log m / log max(2, p) with m the
    number of keys the query sees after pruning and p the number it would see
    without.  READING: the step-t query is kept row M + t of the cache (after
    the M kept prompt rows and the t tokens generated before it) and original
    position N + t, so, as for a kept prompt row i with m_i = i + 1 and
    p_i = idx_i + 1: m = M + t + 1, p = N + t + 1.
    """
    m = float(m_kept + t + 1)
    p = float(n_prompt + t + 1)
    return math.log(m) / math.log(max(2.0, p))


def gated_decode_attention(q, k_cache, v_cache, bias, head_gain, head_temp, ratio: float, sm_scale: float,
                           return_lse: bool = False):
    """Attention of one new query token over the gated KV cache.

    [R] §4.1 engineering notes: at decode time the gate term becomes an
    additive attention mask, i.e. the same logits as token-gated attention for
    the newest row, which sees every cached key:
        l_c = temp_h * ratio * sm_scale * (q_h . k_c) + gain_h * bias_c
        o_h = sum_c softmax_c(l) v_c,   c = 0 .. L-1 (the cache ends with the
    query token's own key).  bias_c is the kept prompt token's importance b_c
    and 0 for generated tokens (the caller passes it that way).
    q [Hq, D], k/v cache [L, Hkv, D], bias [L] (None = 0).
    Returns o [Hq, D] float64 (and lse [Hq], natural log).
    """
    q = np.asarray(q, dtype=F64)
    k = np.asarray(k_cache, dtype=F64)
    v = np.asarray(v_cache, dtype=F64)
    hq, dh = q.shape
    length, hkv, _ = k.shape
    group = hq // hkv
    bias = np.zeros(length) if bias is None else np.asarray(bias, dtype=F64)
    gain = np.asarray(head_gain, dtype=F64)
    temp = np.asarray(head_temp, dtype=F64)
    out = np.zeros((hq, dh))
    lse = np.zeros(hq)
    for h in range(hq):
        g = h // group
        logits = temp[h] * ratio * sm_scale * (k[:, g, :] @ q[h]) + gain[h] * bias
        mx = logits.max()
        e = np.exp(logits - mx)
        den = e.sum()
        out[h] = (e / den) @ v[:, g, :]
        lse[h] = mx + math.log(den)
    return (out, lse) if return_lse else out


# ---------------------------------------------------------------------------
# Decoder layer above the gate  ([R] §4.1 three-stage forward; [M])
# ---------------------------------------------------------------------------

def rope(x, pos, theta: float) -> np.ndarray:
    """Rotary embedding, rotate-half convention, at positions pos.

    x [M, H, D]; frequencies theta^(-2i/D), i < D/2; the first and second
    halves of each head vector form the rotated pairs.  READING: the layers
    above the gate rotate kept tokens at their ORIGINAL positions.
    """
    x = np.asarray(x, dtype=F64)
    dh = x.shape[-1]
    half = dh // 2
    inv_freq = theta ** (-np.arange(half, dtype=F64) * 2.0 / dh)
    ang = np.asarray(pos, dtype=F64)[:, None] * inv_freq[None, :]      # [M, half]
    cos = np.cos(ang)[:, None, :]
    sin = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def attention_block(hidden, weights: Dict[str, np.ndarray], *, hq: int, hkv: int, head_dim: int,
                    pos, bias, ratio, head_gain, head_temp, rope_theta: float, qk_norm: bool,
                    norm_eps: float = 1e-6, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """The attention half of a Qwen3-shaped decoder layer: the post-attention
    residual h + Attn(RMSNorm(h)) Wo^T.

    RMSNorm -> QKV projection -> (per-head q/k RMSNorm) -> RoPE at the original
    positions -> token-gated attention -> O projection + residual.  Linear
    weights are [out, in].  All float64.  With `rows`, only those output rows
    are produced (keys and values still come from every row).
    """
    h = np.asarray(hidden, dtype=F64)
    mrows = h.shape[0]
    sel = np.arange(mrows) if rows is None else np.asarray(rows, dtype=np.int64)
    x = rms_norm(h, weights["w_in_norm"], norm_eps)
    qkv = x @ np.asarray(weights["w_qkv"], dtype=F64).T
    q = qkv[:, : hq * head_dim].reshape(mrows, hq, head_dim)
    k = qkv[:, hq * head_dim:(hq + hkv) * head_dim].reshape(mrows, hkv, head_dim)
    v = qkv[:, (hq + hkv) * head_dim:].reshape(mrows, hkv, head_dim)
    if qk_norm:
        q = rms_norm(q, weights["w_q_norm"], norm_eps)
        k = rms_norm(k, weights["w_k_norm"], norm_eps)
    q = rope(q, pos, rope_theta)
    k = rope(k, pos, rope_theta)
    a = gated_attention(q, k, v, bias, head_gain, head_temp, ratio, 1.0 / math.sqrt(head_dim), rows=sel)
    return h[sel] + a.reshape(sel.size, hq * head_dim) @ np.asarray(weights["w_o"], dtype=F64).T


def mlp_block(hidden, weights: Dict[str, np.ndarray], *, norm_eps: float = 1e-6) -> np.ndarray:
    """The MLP half of a Qwen3-shaped decoder layer, row by row:
    h + (SiLU(y Wg^T) * (y Wu^T)) Wd^T with y = RMSNorm(h) (post-attention
    norm); w_gate_up stacks the gate rows over the up rows.  float64."""
    h1 = np.asarray(hidden, dtype=F64)
    y = rms_norm(h1, weights["w_post_norm"], norm_eps)
    gu = y @ np.asarray(weights["w_gate_up"], dtype=F64).T
    d_ff = gu.shape[1] // 2
    act = silu(gu[:, :d_ff]) * gu[:, d_ff:]
    return h1 + act @ np.asarray(weights["w_down"], dtype=F64).T


def decoder_layer(hidden, weights: Dict[str, np.ndarray], *, hq: int, hkv: int, head_dim: int,
                  pos, bias, ratio, head_gain, head_temp, rope_theta: float, qk_norm: bool,
                  norm_eps: float = 1e-6, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """One Qwen3-shaped decoder layer run on the kept rows only: the attention
    half (attention_block) followed by the MLP half (mlp_block).

    RMSNorm -> QKV projection -> (per-head q/k RMSNorm) -> RoPE at the original
    positions -> token-gated attention -> O projection + residual -> RMSNorm ->
    SwiGLU MLP + residual.  All float64.  With `rows`, only those output rows
    are produced (keys and values still come from every row).
    """
    h1 = attention_block(hidden, weights, hq=hq, hkv=hkv, head_dim=head_dim, pos=pos, bias=bias, ratio=ratio,
                         head_gain=head_gain, head_temp=head_temp, rope_theta=rope_theta, qk_norm=qk_norm,
                         norm_eps=norm_eps, rows=rows)
    return mlp_block(h1, weights, norm_eps=norm_eps)


def pruned_prefill_step(hidden, gate: Dict[str, np.ndarray], k: int, layer: Dict[str, np.ndarray], *,
                        hq: int, hkv: int, head_dim: int, head_gain, head_temp, rope_theta: float,
                        qk_norm: bool, norm_eps: float = 1e-6, eps_s: float = 1e-6,
                        scores_override=None) -> Dict[str, np.ndarray]:
    """Gate layer -> select -> compact -> one gated layer above the gate.

    The three-stage forward of [R] §4.1 restricted to the gate and the first
    pruned layer.  Scores are rounded to float32 (the precision the selector
    ranks in) before selection.
    """
    prunable = gate["prunable"]
    if scores_override is None:
        s = gate_scores(hidden, gate["norm_w"], norm_eps, gate["w1"], gate["b1"], gate["w2"],
                        gate["b2"], prunable)
    else:
        s = np.asarray(scores_override, dtype=F64)
    s32 = s.astype(np.float32)
    idx = select_kept(s32, prunable, k)
    g = gather(hidden, idx, s32, prunable, eps_s)
    out = decoder_layer(g["hidden_kept"], layer, hq=hq, hkv=hkv, head_dim=head_dim, pos=g["pos"],
                        bias=g["bias"], ratio=g["ratio"], head_gain=head_gain, head_temp=head_temp,
                        rope_theta=rope_theta, qk_norm=qk_norm, norm_eps=norm_eps)
    return {"scores": s, "kept_idx": idx, **g, "out": out}


# ---------------------------------------------------------------------------
# A whole decoder stack  ([R] §4.1 three-stage forward and Gate module; [K]
# "tying the mechanism together"; [M] "how does learned token pruning work")
# ---------------------------------------------------------------------------
def pruned_prefill_stack(hidden, layers: Sequence[Dict[str, np.ndarray]], heads: Sequence[Dict[str, np.ndarray]],
                         gate: Dict[str, np.ndarray], k: int, gate_layer: int, *, hq: int, hkv: int,
                         head_dim: int, rope_theta: float, qk_norm: bool, norm_eps: float = 1e-6,
                         eps_s: float = 1e-6, pruned: bool = True) -> Dict[str, np.ndarray]:
    """Prefill of one prompt through len(layers) decoder layers.

    [R] §4.1 splits the forward in three: below the gate every token is
    processed; at gate layer L the gate scores each prunable token from that
    layer's normalised post-attention residual, the top-K document tokens
    plus every question token are kept and compacted in order; everything
    after runs on the kept tokens only, with token-gated attention in the
    layers above L ([K] and [M] place the scoring in the same spot: after
    layer L's attention).  So here:
      layers 0 .. L-1        all N rows (positions 0..N-1, no gate bias,
                             ratio 1, temperature 1);
      layer L, attention     all N rows, the same way -> residual h1 (N rows);
      gate                   scores RMSNorm(h1) * w_post_norm of layer L (READING:
                             the gate's normalisation is layer L's own
                             post-attention RMSNorm, the vector layer L's MLP
                             reads), select, gather the kept rows of h1;
      layer L, MLP           the kept rows only (row-wise, so the same rows as
                             running it on all N and gathering afterwards);
      layers L+1 ..          the kept rows with each layer's head gain and
                             temperature (heads[l]).
    With pruned=False every layer runs on all rows with no gate: the unpruned
    stack.  gate["norm_w"] is not used here (the layer's weight takes its place).
    """
    h = np.asarray(hidden, dtype=F64)
    n = h.shape[0]
    pos = np.arange(n)
    n_layers = len(layers)
    common = dict(hq=hq, hkv=hkv, head_dim=head_dim, rope_theta=rope_theta, qk_norm=qk_norm, norm_eps=norm_eps)
    flat = dict(pos=pos, bias=None, ratio=None, head_gain=np.zeros(hq), head_temp=np.ones(hq))
    if not pruned:
        for l in range(n_layers):
            h = decoder_layer(h, layers[l], **flat, **common)
        return {"out": h}
    for l in range(gate_layer):
        h = decoder_layer(h, layers[l], **flat, **common)
    h1 = attention_block(h, layers[gate_layer], **flat, **common)
    prunable = gate["prunable"]
    s = gate_scores(h1, layers[gate_layer]["w_post_norm"], norm_eps, gate["w1"], gate["b1"], gate["w2"], gate["b2"],
                    prunable)
    s32 = s.astype(np.float32)
    idx = select_kept(s32, prunable, k)
    g = gather(h1, idx, s32, prunable, eps_s)
    hk = mlp_block(g["hidden_kept"], layers[gate_layer], norm_eps=norm_eps)
    for l in range(gate_layer + 1, n_layers):
        hk = decoder_layer(hk, layers[l], pos=g["pos"], bias=g["bias"], ratio=g["ratio"],
                           head_gain=heads[l]["head_gain"], head_temp=heads[l]["head_temp"], **common)
    return {"gate_input": h1, "scores": s, "kept_idx": idx, **g, "out": hk}
