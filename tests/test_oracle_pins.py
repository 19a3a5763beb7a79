"""Pins for the CPU oracle: each oracle function is checked against something
other than itself -- brute force, closed forms, invariants, hand-worked
fixtures, or an independent library routine (torch / transformers fp64)."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import tokengate_oracle as O
from learned_token_pruning_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f(x):
    return float(x) if not isinstance(x, str) else float(x.replace("nan", "nan"))


# ----------------------------------------------------------------------------- gate scores

def test_gate_scores_match_torch_library_routines():
    rng = np.random.default_rng(11)
    n, d, h = 37, 48, 12
    hidden = rng.standard_normal((n, d))
    norm_w = rng.uniform(0.5, 1.5, d)
    w1 = rng.standard_normal((h, d)) * 0.1
    b1 = rng.standard_normal(h) * 0.1
    w2 = rng.standard_normal(h)
    b2 = 0.37
    prunable = (rng.random(n) < 0.8).astype(np.uint8)
    s = O.gate_scores(hidden, norm_w, 1e-6, w1, b1, w2, b2, prunable)

    t = torch.from_numpy
    x = F.rms_norm(t(hidden), (d,), weight=t(norm_w), eps=1e-6)
    ref = F.linear(F.silu(F.linear(x, t(w1), t(b1))), t(w2)[None, :])[:, 0] + b2
    ref = torch.where(t(prunable).bool(), ref, torch.zeros_like(ref)).numpy()
    np.testing.assert_allclose(s, ref, rtol=1e-12, atol=1e-12)


def test_gate_zero_mlp_gives_zero_scores_and_keeps_first_k():
    # zero-output MLP init: the gate starts as the identity (keeps everything);
    # with all scores equal the tie rule keeps the first K prunable tokens
    rng = np.random.default_rng(3)
    n, d, h = 20, 16, 4
    hidden = rng.standard_normal((n, d))
    s = O.gate_scores(hidden, None, 1e-6, rng.standard_normal((h, d)), None, np.zeros(h), 0.0,
                      np.ones(n, np.uint8))
    assert np.all(s == 0.0)
    mask = np.ones(n, np.uint8)
    mask[-3:] = 0
    assert list(O.select_kept(s, mask, 5)) == [0, 1, 2, 3, 4, 17, 18, 19]
    assert list(O.select_kept(s, mask, 1000)) == list(range(n))


def test_gate_single_unit_closed_form():
    # hidden row = c * e_i  => RMSNorm gives sqrt(d) e_i exactly (eps -> 0);
    # W1 = e_i^T, b1 = 0  => u = sqrt(d); s = w2 * u / (1 + exp(-u)) + b2
    d = 9
    for i, c in [(0, 2.5), (4, -0.3), (8, 7.0)]:
        hidden = np.zeros((1, d))
        hidden[0, i] = c
        w1 = np.zeros((1, d))
        w1[0, i] = 1.0
        s = O.gate_scores(hidden, None, 0.0, w1, None, np.array([1.7]), -0.2, np.ones(1, np.uint8))
        u = math.copysign(math.sqrt(d), c)
        assert s[0] == pytest.approx(1.7 * u / (1.0 + math.exp(-u)) - 0.2, rel=1e-14)


def test_gate_score_rms_scale_invariance_and_question_zero():
    rng = np.random.default_rng(5)
    n, d, h = 10, 32, 6
    hidden = rng.standard_normal((n, d))
    w1, w2 = rng.standard_normal((h, d)), rng.standard_normal(h)
    mask = np.array([1, 1, 1, 1, 1, 1, 1, 0, 0, 1], np.uint8)
    s1 = O.gate_scores(hidden, None, 0.0, w1, None, w2, 0.1, mask)
    s2 = O.gate_scores(hidden * 13.0, None, 0.0, w1, None, w2, 0.1, mask)
    np.testing.assert_allclose(s1, s2, rtol=1e-12)
    assert s1[7] == 0.0 and s1[8] == 0.0


# ----------------------------------------------------------------------------- sequence RMS

def test_seq_rms_normalises_prunable_scores_to_unit_rms():
    rng = np.random.default_rng(8)
    s = rng.standard_normal(50) * 3.0
    mask = (rng.random(50) < 0.7).astype(np.uint8)
    b = O.importance(s, mask, 0.0)
    p = mask != 0
    assert math.sqrt(np.mean(b[p] ** 2)) == pytest.approx(1.0, rel=1e-13)
    assert np.all(b[~p] == 0.0)
    # a positive rescaling of the scores leaves b (and therefore the selection) unchanged
    np.testing.assert_allclose(O.importance(s * 0.01, mask, 0.0), b, rtol=1e-12)
    # non-prunable entries never enter r
    s2 = s.copy()
    s2[~p] = 1e6
    assert O.seq_rms(s2, mask, 0.0) == pytest.approx(O.seq_rms(s, mask, 0.0), rel=1e-15)


# ----------------------------------------------------------------------------- selector

def _value_rank_key(v):
    # larger first; NaN below everything
    return (1, 0.0) if math.isnan(v) else (0, -v)


def _brute_force_select(scores, prunable, k):
    """Enumerate every subset of the prunable set of size min(k, |P|) and keep
    the one that (a) never drops a strictly better value than one it keeps and
    (b) among equal values keeps the lower indices.  Exactly one subset passes."""
    p = [j for j in range(len(scores)) if prunable[j]]
    kp = min(k, len(p))
    winners = []
    for sub in itertools.combinations(p, kp):
        kept = set(sub)
        ok = True
        for a in kept:
            for b in p:
                if b in kept:
                    continue
                ka, kb = _value_rank_key(scores[a]), _value_rank_key(scores[b])
                if kb < ka or (kb == ka and b < a):
                    ok = False
                    break
            if not ok:
                break
        if ok:
            winners.append(sorted(kept | {j for j in range(len(scores)) if not prunable[j]}))
    assert len(winners) == 1
    return winners[0]


@pytest.mark.parametrize("seed", range(6))
def test_select_matches_brute_force_on_tie_heavy_inputs(seed):
    rng = np.random.default_rng(100 + seed)
    n = 9
    pool = np.array([2.0, 1.0, 1.0, 0.0, -0.0, -3.0, np.inf, -np.inf, np.nan], np.float32)
    scores = rng.choice(pool, size=n).astype(np.float32)
    prunable = (rng.random(n) < 0.75).astype(np.uint8)
    for k in range(0, n + 2):
        got = list(O.select_kept(scores, prunable, k))
        assert got == _brute_force_select([float(x) for x in scores], prunable, k), (scores, prunable, k)


def test_select_golden_hand_worked_cases():
    data = json.load(open(os.path.join(GOLDEN, "select_cases.json")))
    for c in data["cases"]:
        scores = np.array([float(x) for x in c["scores"]], np.float32)
        got = list(O.select_kept(scores, np.array(c["prunable"], np.uint8), c["k"]))
        assert got == c["kept"], c["name"]


def test_select_planted_block_always_kept():
    rng = np.random.default_rng(21)
    n = 400
    s = rng.standard_normal(n).astype(np.float32)
    s[150:166] = 10.0 + rng.random(16).astype(np.float32)
    mask = np.ones(n, np.uint8)
    mask[-20:] = 0
    for k in (16, 17, 50, 379, 380):
        kept = set(O.select_kept(s, mask, k).tolist())
        assert set(range(150, 166)) <= kept
        assert set(range(380, 400)) <= kept
        assert len(kept) == min(k, 380) + 20


def test_select_count_and_threshold_property_random():
    rng = np.random.default_rng(9)
    n = 5000
    s = np.round(rng.standard_normal(n), 1).astype(np.float32)   # many exact ties
    mask = (rng.random(n) < 0.9).astype(np.uint8)
    for k in (0, 1, 777, int(mask.sum()) - 1, int(mask.sum())):
        idx = O.select_kept(s, mask, k)
        kp = min(k, int(mask.sum()))
        assert len(idx) == kp + int((mask == 0).sum())
        kept = np.zeros(n, bool)
        kept[idx] = True
        kp_mask = kept & (mask != 0)
        dropped = (~kept) & (mask != 0)
        if kp and dropped.any():
            assert s[kp_mask].min() >= s[dropped].max()
            t = s[kp_mask].min()
            # among ties at the threshold the kept ones precede the dropped ones
            tk = np.flatnonzero(kp_mask & (s == t))
            td = np.flatnonzero(dropped & (s == t))
            if td.size:
                assert tk.max() < td.min()


# ----------------------------------------------------------------------------- gather / ratio

def test_temperature_ratio_closed_forms():
    cases = [
        ([0, 3, 7], [0.0, math.log(2) / math.log(4), math.log(3) / math.log(8)]),
        ([0, 1, 2, 3], [0.0, 1.0, 1.0, 1.0]),
        ([5, 9], [0.0, math.log(2) / math.log(10)]),
        ([1, 2], [0.0, math.log(2) / math.log(3)]),
    ]
    for idx, want in cases:
        np.testing.assert_allclose(O.temperature_ratio(idx), want, rtol=1e-15, atol=0)


def test_gather_copies_rows_and_positions():
    rng = np.random.default_rng(4)
    n, d = 30, 8
    hidden = rng.standard_normal((n, d))
    s = rng.standard_normal(n).astype(np.float32)
    mask = np.ones(n, np.uint8)
    mask[-4:] = 0
    idx = O.select_kept(s, mask, 7)
    g = O.gather(hidden, idx, s, mask, 1e-6)
    for r, j in enumerate(idx):
        assert np.array_equal(g["hidden_kept"][r], hidden[j])
        assert g["pos"][r] == j
    r_s = math.sqrt(sum(float(s[j]) ** 2 for j in range(n) if mask[j]) / mask.sum() + 1e-6)
    for r, j in enumerate(idx):
        assert g["bias"][r] == pytest.approx(float(s[j]) / r_s if mask[j] else 0.0, rel=1e-12)


# ----------------------------------------------------------------------------- attention

def _rand_attn(m, hq, hkv, dh, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((m, hq, dh)), rng.standard_normal((m, hkv, dh)),
            rng.standard_normal((m, hkv, dh)), rng.standard_normal(m), rng.uniform(0.5, 2, hq),
            rng.uniform(0.8, 1.2, hq), rng.uniform(0.0, 1.0, m))


def test_attention_matches_torch_sdpa_with_additive_mask():
    m, hq, hkv, dh = 23, 4, 2, 16
    q, k, v, bias, gain, temp, ratio = _rand_attn(m, hq, hkv, dh, 1)
    scale = 1.0 / math.sqrt(dh)
    out, lse = O.gated_attention(q, k, v, bias, gain, temp, ratio, scale, return_lse=True)

    t = torch.from_numpy
    qs = t(q) * (t(temp)[None, :, None] * t(ratio)[:, None, None])        # row/head content scale
    mask = t(gain)[:, None, None] * t(bias)[None, None, :]                 # [hq, 1, m]
    causal = torch.ones(m, m, dtype=torch.bool).tril()
    mask = mask.expand(hq, m, m).masked_fill(~causal, float("-inf"))
    ref = F.scaled_dot_product_attention(qs.transpose(0, 1)[None], t(k).transpose(0, 1)[None],
                                         t(v).transpose(0, 1)[None], attn_mask=mask[None],
                                         scale=scale, enable_gqa=True)[0].transpose(0, 1)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-10, atol=1e-12)
    logits = torch.einsum("rhd,chd->hrc", qs, t(k).repeat_interleave(hq // hkv, 1)) * scale + mask
    np.testing.assert_allclose(lse, torch.logsumexp(logits, -1).numpy(), rtol=1e-12)


def test_attention_zero_bias_unit_temperature_is_plain_causal_attention():
    m, hq, hkv, dh = 17, 6, 3, 8
    q, k, v, _, gain, _, _ = _rand_attn(m, hq, hkv, dh, 2)
    out = O.gated_attention(q, k, v, np.zeros(m), gain, np.ones(hq), np.ones(m), 0.3)
    t = torch.from_numpy
    ref = F.scaled_dot_product_attention(t(q).transpose(0, 1)[None], t(k).transpose(0, 1)[None],
                                         t(v).transpose(0, 1)[None], is_causal=True, scale=0.3,
                                         enable_gqa=True)[0].transpose(0, 1)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-10, atol=1e-12)


def test_attention_closed_forms():
    m, hq, hkv, dh = 12, 2, 1, 4
    q, k, v, bias, gain, temp, ratio = _rand_attn(m, hq, hkv, dh, 3)
    out = O.gated_attention(q, k, v, bias, gain, temp, ratio, 0.5)
    # row 0 sees only itself
    for h in range(hq):
        np.testing.assert_allclose(out[0, h], v[0, 0], rtol=1e-14)
    # zero content scale: weights are softmax(gain * bias) over the visible prefix
    out0 = O.gated_attention(q, k, v, bias, gain, np.zeros(hq), ratio, 0.5)
    for r in range(m):
        for h in range(hq):
            w = [math.exp(gain[h] * bias[c]) for c in range(r + 1)]
            z = sum(w)
            want = sum(w[c] / z * v[c, 0] for c in range(r + 1))
            np.testing.assert_allclose(out0[r, h], want, rtol=1e-12)
    # a constant added to every bias changes nothing
    out_shift = O.gated_attention(q, k, v, bias + 4.0, gain, temp, ratio, 0.5)
    np.testing.assert_allclose(out_shift, out, rtol=1e-11, atol=1e-13)


def test_attention_sampled_rows_match_full():
    m, hq, hkv, dh = 40, 4, 2, 8
    q, k, v, bias, gain, temp, ratio = _rand_attn(m, hq, hkv, dh, 4)
    full = O.gated_attention(q, k, v, bias, gain, temp, ratio, 0.25)
    rows = [0, 7, 39]
    part = O.gated_attention(q, k, v, bias, gain, temp, ratio, 0.25, rows=rows)
    np.testing.assert_allclose(part, full[rows], rtol=1e-14)


# ----------------------------------------------------------------------------- decode over the gated cache

def test_decode_ratio_closed_forms_and_prefill_continuation():
    # M = 3 kept rows out of N = 10 prompt tokens; step 0 is kept row 3 at position 10
    assert O.decode_temperature_ratio(3, 10, 0) == pytest.approx(math.log(4) / math.log(11), rel=1e-15)
    assert O.decode_temperature_ratio(3, 10, 5) == pytest.approx(math.log(9) / math.log(16), rel=1e-15)
    # nothing pruned (M = N): the ratio is 1 from the second token on
    assert O.decode_temperature_ratio(7, 7, 2) == pytest.approx(1.0, rel=1e-15)
    # the first token of an empty prompt sees only itself: log 1 / log 2 = 0
    assert O.decode_temperature_ratio(0, 0, 0) == 0.0
    # the decode query continues the kept rows: its ratio is the prefill formula
    # applied to a kept set extended by the generated positions N .. N + t
    idx = [0, 4, 9]                 # kept prompt rows of a 10-token prompt
    ext = idx + [10, 11, 12]        # then three generated tokens
    pre = O.temperature_ratio(ext)
    for t in range(3):
        assert O.decode_temperature_ratio(len(idx), 10, t) == pytest.approx(pre[len(idx) + t], rel=1e-14)


def test_decode_attention_is_the_last_row_of_gated_attention():
    # the query of a decode step is the newest row of the cache: the prefill
    # attention's last row over the same rows, with the same ratio
    m, hq, hkv, dh = 19, 4, 2, 8
    q, k, v, bias, gain, temp, ratio = _rand_attn(m, hq, hkv, dh, 11)
    full, lse_full = O.gated_attention(q, k, v, bias, gain, temp, ratio, 0.35, return_lse=True)
    out, lse = O.gated_decode_attention(q[-1], k, v, bias, gain, temp, float(ratio[-1]), 0.35, return_lse=True)
    np.testing.assert_allclose(out, full[-1], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse, lse_full[:, -1], rtol=1e-13)


def test_decode_attention_matches_torch_sdpa_and_closed_forms():
    rng = np.random.default_rng(12)
    length, hq, hkv, dh = 33, 6, 2, 16
    q = rng.standard_normal((hq, dh))
    k, v = rng.standard_normal((length, hkv, dh)), rng.standard_normal((length, hkv, dh))
    bias = rng.standard_normal(length)
    bias[-5:] = 0.0                  # generated tokens carry no gate bias
    gain, temp = rng.uniform(0.5, 2, hq), rng.uniform(0.8, 1.2, hq)
    ratio, scale = 0.83, 1.0 / math.sqrt(dh)
    out = O.gated_decode_attention(q, k, v, bias, gain, temp, ratio, scale)
    t = torch.from_numpy
    qs = (t(q) * (t(temp) * ratio)[:, None])[None, :, None, :]              # [1, hq, 1, dh]
    kk = t(k).transpose(0, 1)[None]                                         # [1, hkv, L, dh]
    vv = t(v).transpose(0, 1)[None]
    mask = (t(gain)[:, None] * t(bias)[None, :])[None, :, None, :]          # [1, hq, 1, L]
    ref = F.scaled_dot_product_attention(qs, kk, vv, attn_mask=mask, scale=scale, enable_gqa=True)[0, :, 0]
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-10, atol=1e-12)
    # zero content scale: the weights are softmax(gain * bias), written out
    out0 = O.gated_decode_attention(q, k, v, bias, gain, np.zeros(hq), ratio, scale)
    for h in range(hq):
        g = h // (hq // hkv)
        w = np.exp(gain[h] * bias - np.max(gain[h] * bias))
        np.testing.assert_allclose(out0[h], (w / w.sum()) @ v[:, g], rtol=1e-12)
    # a one-row cache returns its value row
    one = O.gated_decode_attention(q, k[:1], v[:1], bias[:1], gain, temp, ratio, scale)
    for h in range(hq):
        np.testing.assert_allclose(one[h], v[0, h // (hq // hkv)], rtol=1e-15)


# ----------------------------------------------------------------------------- attention backward

def _loss(q, k, v, bias, gain, temp, ratio, scale, w):
    return float(np.sum(O.gated_attention(q, k, v, bias, gain, temp, ratio, scale) * w))


def test_attention_backward_matches_finite_differences():
    # central differences of the forward oracle, every input, in fp64
    m, hq, hkv, dh = 7, 4, 2, 3
    q, k, v, bias, gain, temp, ratio = _rand_attn(m, hq, hkv, dh, 21)
    scale = 0.6
    w = np.random.default_rng(22).standard_normal((m, hq, dh))      # dL/do
    g = O.gated_attention_backward(q, k, v, bias, gain, temp, ratio, scale, w)
    eps = 1e-6
    for name, arr in (("dq", q), ("dk", k), ("dv", v), ("dbias", bias), ("dgain", gain), ("dtemp", temp)):
        num = np.zeros_like(arr)
        for i in np.ndindex(arr.shape):
            old = arr[i]
            arr[i] = old + eps
            lp = _loss(q, k, v, bias, gain, temp, ratio, scale, w)
            arr[i] = old - eps
            lm = _loss(q, k, v, bias, gain, temp, ratio, scale, w)
            arr[i] = old
            num[i] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(g[name], num, rtol=1e-6, atol=1e-8, err_msg=name)


def test_attention_backward_matches_torch_autograd():
    m, hq, hkv, dh = 19, 4, 2, 8
    q, k, v, bias, gain, temp, ratio = _rand_attn(m, hq, hkv, dh, 23)
    scale = 1.0 / math.sqrt(dh)
    w = np.random.default_rng(24).standard_normal((m, hq, dh))
    g = O.gated_attention_backward(q, k, v, bias, gain, temp, ratio, scale, w)
    t = lambda a: torch.tensor(a, dtype=torch.float64, requires_grad=True)
    tq, tk, tv, tb, tgn, ttp = t(q), t(k), t(v), t(bias), t(gain), t(temp)
    tr = torch.tensor(ratio, dtype=torch.float64)
    qs = tq * (ttp[None, :, None] * tr[:, None, None])
    mask = (tgn[:, None, None] * tb[None, None, :]).expand(hq, m, m)
    mask = mask.masked_fill(~torch.ones(m, m, dtype=torch.bool).tril(), float("-inf"))
    out = F.scaled_dot_product_attention(qs.transpose(0, 1)[None], tk.transpose(0, 1)[None], tv.transpose(0, 1)[None],
                                         attn_mask=mask[None], scale=scale, enable_gqa=True)[0].transpose(0, 1)
    (out * torch.tensor(w)).sum().backward()
    for name, tt in (("dq", tq), ("dk", tk), ("dv", tv), ("dbias", tb), ("dgain", tgn), ("dtemp", ttp)):
        np.testing.assert_allclose(g[name], tt.grad.numpy(), rtol=1e-10, atol=1e-12, err_msg=name)


# ----------------------------------------------------------------------------- decoder layer

def _hf_layer(w, lw, n_rows):
    from transformers import Qwen3Config
    from transformers.models.qwen3.modeling_qwen3 import Qwen3DecoderLayer, Qwen3RotaryEmbedding
    cfg = Qwen3Config(hidden_size=w.d_model, intermediate_size=w.d_ff, num_attention_heads=w.hq,
                      num_key_value_heads=w.hkv, head_dim=w.head_dim, rms_norm_eps=1e-6,
                      rope_theta=w.rope_theta, max_position_embeddings=1 << 20,
                      attention_bias=False)
    cfg._attn_implementation = "eager"
    layer = Qwen3DecoderLayer(cfg, 0).double()
    t = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))
    D, hq, hkv = w.head_dim, w.hq, w.hkv
    with torch.no_grad():
        layer.input_layernorm.weight.copy_(t(lw["w_in_norm"]))
        layer.self_attn.q_proj.weight.copy_(t(lw["w_qkv"][: hq * D]))
        layer.self_attn.k_proj.weight.copy_(t(lw["w_qkv"][hq * D:(hq + hkv) * D]))
        layer.self_attn.v_proj.weight.copy_(t(lw["w_qkv"][(hq + hkv) * D:]))
        layer.self_attn.q_norm.weight.copy_(t(lw["w_q_norm"]))
        layer.self_attn.k_norm.weight.copy_(t(lw["w_k_norm"]))
        layer.self_attn.o_proj.weight.copy_(t(lw["w_o"]))
        layer.post_attention_layernorm.weight.copy_(t(lw["w_post_norm"]))
        layer.mlp.gate_proj.weight.copy_(t(lw["w_gate_up"][: w.d_ff]))
        layer.mlp.up_proj.weight.copy_(t(lw["w_gate_up"][w.d_ff:]))
        layer.mlp.down_proj.weight.copy_(t(lw["w_down"]))
    rot = Qwen3RotaryEmbedding(cfg).double()
    return layer, rot


def _small_layer_workload():
    return synth.Workload(name="t", seed=7, n=24, n_question=4, d_model=64, hq=4, hkv=2,
                          head_dim=16, gate_hidden=8, k=10, dtype="f32", d_ff=96)


@pytest.mark.parametrize("gain_scale", [0.0, 1.0])
def test_decoder_layer_matches_transformers_qwen3_layer(gain_scale):
    """Unit temperature / ratio: the gated layer equals the transformers Qwen3
    layer fed an additive per-head key-bias mask, at non-contiguous original
    positions (the RoPE of kept tokens)."""
    w = _small_layer_workload()
    lw = synth.layer_weights(w)
    rng = np.random.default_rng(0)
    for key in ("w_in_norm", "w_q_norm", "w_k_norm", "w_post_norm"):
        lw[key] = rng.uniform(0.5, 1.5, lw[key].shape)
    m = 11
    hidden = rng.standard_normal((m, w.d_model))
    pos = np.sort(rng.choice(5000, m, replace=False))
    bias = rng.standard_normal(m)
    gain = rng.uniform(0.5, 2, w.hq) * gain_scale
    ours = O.decoder_layer(hidden, lw, hq=w.hq, hkv=w.hkv, head_dim=w.head_dim, pos=pos, bias=bias,
                           ratio=np.ones(m), head_gain=gain, head_temp=np.ones(w.hq),
                           rope_theta=w.rope_theta, qk_norm=True)
    layer, rot = _hf_layer(w, lw, m)
    x = torch.from_numpy(hidden)[None]
    pid = torch.from_numpy(pos)[None]
    cos, sin = rot(x, pid)
    mask = torch.from_numpy(gain)[:, None, None] * torch.from_numpy(bias)[None, None, :]
    mask = mask.expand(w.hq, m, m).masked_fill(~torch.ones(m, m, dtype=torch.bool).tril(), float("-inf"))
    with torch.no_grad():
        ref = layer(x, attention_mask=mask[None], position_ids=pid, position_embeddings=(cos, sin))
    ref = ref[0] if isinstance(ref, tuple) else ref
    # the eager softmax of transformers runs in float32, hence the loose-ish tolerance
    np.testing.assert_allclose(ours, ref[0].numpy(), rtol=2e-6, atol=2e-6)


def test_rope_matches_transformers_apply_rotary():
    from transformers.models.qwen3.modeling_qwen3 import apply_rotary_pos_emb
    rng = np.random.default_rng(1)
    m, h, dh, theta = 9, 3, 32, 1.0e6
    x = rng.standard_normal((m, h, dh))
    pos = np.array([0, 1, 5, 17, 100, 1000, 4097, 65535, 131071])
    inv = theta ** (-np.arange(0, dh, 2, dtype=np.float64) / dh)
    ang = pos[:, None] * inv[None, :]
    emb = np.concatenate([ang, ang], -1)
    cos, sin = torch.from_numpy(np.cos(emb))[None], torch.from_numpy(np.sin(emb))[None]
    xt = torch.from_numpy(x).transpose(0, 1)[None]
    ref, _ = apply_rotary_pos_emb(xt, xt, cos, sin)
    np.testing.assert_allclose(O.rope(x, pos, theta), ref[0].transpose(0, 1).numpy(), rtol=1e-12, atol=1e-12)


def test_keep_everything_with_zero_gain_reduces_to_unpruned_layer():
    w = _small_layer_workload()
    g = synth.gate_inputs(w)
    lw = synth.layer_weights(w)
    hp = synth.head_params(w)
    res = O.pruned_prefill_step(g["hidden"], g, w.n, lw, hq=w.hq, hkv=w.hkv, head_dim=w.head_dim,
                                head_gain=np.zeros(w.hq), head_temp=hp["head_temp"] * 0 + 1.0,
                                rope_theta=w.rope_theta, qk_norm=True)
    assert list(res["kept_idx"]) == list(range(w.n))
    full = O.decoder_layer(g["hidden"], lw, hq=w.hq, hkv=w.hkv, head_dim=w.head_dim,
                           pos=np.arange(w.n), bias=None, ratio=None, head_gain=np.zeros(w.hq),
                           head_temp=np.ones(w.hq), rope_theta=w.rope_theta, qk_norm=True)
    np.testing.assert_allclose(res["out"], full, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- a whole stack

def _stack_case(n_layers=4):
    w = _small_layer_workload()
    layers = [synth.layer_weights(w, layer=l) for l in range(n_layers)]
    heads = [synth.head_params(w, seed_offset=100 + l) for l in range(n_layers)]
    return w, synth.gate_inputs(w), layers, heads


def _stack(w, g, layers, heads, k, gate_layer, pruned=True):
    return O.pruned_prefill_stack(g["hidden"], layers, heads, g, k, gate_layer, hq=w.hq, hkv=w.hkv,
                                  head_dim=w.head_dim, rope_theta=w.rope_theta, qk_norm=True, pruned=pruned)


def test_stack_keeping_everything_with_zero_gain_is_the_unpruned_stack():
    w, g, layers, heads = _stack_case()
    flat = [{"head_gain": np.zeros(w.hq), "head_temp": np.ones(w.hq)} for _ in layers]
    res = _stack(w, g, layers, flat, w.n, gate_layer=1)
    assert list(res["kept_idx"]) == list(range(w.n))
    full = _stack(w, g, layers, heads, w.n, gate_layer=1, pruned=False)
    np.testing.assert_allclose(res["out"], full["out"], rtol=1e-12, atol=1e-12)


def test_stack_gate_at_the_top_gathers_the_unpruned_output():
    w, g, layers, heads = _stack_case(3)
    res = _stack(w, g, layers, heads, w.k, gate_layer=2)
    full = _stack(w, g, layers, heads, w.k, gate_layer=2, pruned=False)
    assert len(res["kept_idx"]) == w.k + w.n_question
    # layer 2's MLP runs on the kept rows only, a row-wise step: equal up to
    # the summation order of the matmul over fewer rows
    np.testing.assert_allclose(res["out"], full["out"][res["kept_idx"]], rtol=1e-12, atol=1e-12)


def test_stack_layer_mlp_runs_on_the_kept_rows_only():
    # the gate sits inside layer L (after its attention): with the gate in the
    # middle of the stack, the kept rows entering layer L+1 are layer L's
    # unpruned output at those rows (its MLP is row-wise), and the pruned
    # output differs from the unpruned one (the layers above see fewer keys)
    w, g, layers, heads = _stack_case(3)
    res = _stack(w, g, layers, heads, w.k, gate_layer=1)
    two = _stack(w, g, layers[:2], heads, w.k, gate_layer=1, pruned=False)["out"]
    idx = res["kept_idx"]
    hk = O.mlp_block(res["hidden_kept"], layers[1])
    np.testing.assert_allclose(hk, two[idx], rtol=1e-12, atol=1e-12)
    full = _stack(w, g, layers, heads, w.k, gate_layer=1, pruned=False)["out"]
    assert np.max(np.abs(res["out"] - full[idx])) > 1e-3


def _hf_chain_gate_input(w, g, layers, gate_layer):
    """Run transformers Qwen3DecoderLayers 0..gate_layer and capture, with
    forward hooks, the input and output of layer gate_layer's
    post_attention_layernorm: its post-attention residual and that residual
    normalised by the layer's own RMSNorm."""
    x = torch.from_numpy(np.asarray(g["hidden"], dtype=np.float64))[None]
    pid = torch.arange(w.n)[None]
    mask = torch.zeros(w.n, w.n, dtype=torch.float64).masked_fill(
        ~torch.ones(w.n, w.n, dtype=torch.bool).tril(), float("-inf"))[None, None]
    seen = {}
    with torch.no_grad():
        for l in range(gate_layer + 1):
            layer, rot = _hf_layer(w, layers[l], w.n)
            if l == gate_layer:
                def hook(mod, args, out):
                    seen["in"] = args[0][0].clone()
                    seen["out"] = out[0].clone()
                layer.post_attention_layernorm.register_forward_hook(hook)
            cos, sin = rot(x, pid)
            x = layer(x, attention_mask=mask, position_ids=pid, position_embeddings=(cos, sin))
            x = x[0] if isinstance(x, tuple) else x
    return seen["in"].numpy(), seen["out"].numpy()


@pytest.mark.parametrize("gate_layer", [0, 1, 2])
def test_stack_gate_reads_the_post_attention_residual_of_its_layer(gate_layer):
    # [R] §4.1 Gate module / [K] / [M]: the gate scores layer L's normalised
    # post-attention residual.  Pinned against transformers' Qwen3 layer: the
    # input of layer L's post_attention_layernorm is the oracle's gate input,
    # and that norm's output fed to the gate MLP gives the oracle's scores.
    w, g, layers, heads = _stack_case(3)
    w = w.replace(k=6)
    g = dict(g)
    # a non-trivial post-attention norm weight, so that taking the gate's
    # normalisation from the wrong place shows
    rng = np.random.default_rng(11)
    layers = [dict(lw) for lw in layers]
    layers[gate_layer]["w_post_norm"] = rng.uniform(0.5, 1.5, w.d_model)
    res = _stack(w, g, layers, heads, w.k, gate_layer=gate_layer)
    hf_in, hf_out = _hf_chain_gate_input(w, g, layers, gate_layer)
    np.testing.assert_allclose(res["gate_input"], hf_in, rtol=1e-5, atol=1e-5)
    t = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))
    u = F.linear(t(hf_out), t(g["w1"]), t(g["b1"]))
    s_hf = (F.silu(u) @ t(g["w2"]) + float(g["b2"])).numpy()
    s_hf = np.where(np.asarray(g["prunable"]) != 0, s_hf, 0.0)
    np.testing.assert_allclose(res["scores"], s_hf, rtol=1e-5, atol=1e-7)
    # the residual leaving layer L (after its MLP) is a different vector
    leaving = _stack(w, g, layers[: gate_layer + 1], heads, w.k, gate_layer=0, pruned=False)["out"]
    assert np.max(np.abs(leaving - res["gate_input"])) > 1e-3


def test_unpruned_stack_matches_a_chain_of_transformers_layers():
    w, g, layers, heads = _stack_case(3)
    ours = _stack(w, g, layers, heads, w.k, gate_layer=0, pruned=False)["out"]
    x = torch.from_numpy(np.asarray(g["hidden"], dtype=np.float64))[None]
    pid = torch.arange(w.n)[None]
    mask = torch.zeros(w.n, w.n, dtype=torch.float64).masked_fill(
        ~torch.ones(w.n, w.n, dtype=torch.bool).tril(), float("-inf"))[None, None]
    with torch.no_grad():
        for lw in layers:
            layer, rot = _hf_layer(w, lw, w.n)
            cos, sin = rot(x, pid)
            x = layer(x, attention_mask=mask, position_ids=pid, position_embeddings=(cos, sin))
            x = x[0] if isinstance(x, tuple) else x
    np.testing.assert_allclose(ours, x[0].numpy(), rtol=1e-5, atol=1e-5)


# ----------------------------------------------------------------------------- synthetic inputs

def test_tiny_workload_planted_block_is_kept_by_oracle():
    w = synth.tiny_f32()
    g = synth.gate_inputs(w)
    s = O.gate_scores(g["hidden"], g["norm_w"], 1e-6, g["w1"], g["b1"], g["w2"], g["b2"], g["prunable"])
    idx = set(O.select_kept(s.astype(np.float32), g["prunable"], w.k).tolist())
    block = set(range(w.plant_start, w.plant_start + w.plant_len))
    assert block <= idx
    assert set(range(w.n - w.n_question, w.n)) <= idx
    assert len(idx) == w.m == 160
