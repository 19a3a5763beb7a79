"""GPU parity of a whole pruned-prefill stack (layers on all rows, the gate,
layers on the kept rows) against the oracle's composition of the same steps."""
import numpy as np
import pytest
import torch

from learned_token_pruning_b200 import pipeline, synth
from oracle import tokengate_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _to(a, dt):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV, dt)


def _host(t):
    return t.float().cpu().numpy().astype(np.float64)


def _build(w):
    dt = synth.torch_dtype(w.dtype)
    g = synth.gate_inputs(w)
    gate = {"w1": _to(g["w1"], dt), "b1": _to(g["b1"], torch.float32), "w2": _to(g["w2"], torch.float32),
            "b2": float(g["b2"]), "norm_w": None}
    layers, heads = pipeline.stack_weights_from_synth(w, w.n_layers, DEV)
    st = pipeline.PrunedPrefillStack(w, _to(g["hidden"], dt), _to(g["prunable"], torch.uint8), gate, layers, heads,
                                     w.gate_layer)
    olayers = [synth.layer_weights(w, layer=l) for l in range(w.n_layers)]
    oheads = [synth.head_params(w, seed_offset=100 + l) for l in range(w.n_layers)]
    return st, g, olayers, oheads


def _common(w):
    return dict(hq=w.hq, hkv=w.hkv, head_dim=w.head_dim, rope_theta=w.rope_theta, qk_norm=w.qk_norm)


def test_stack_fp32_matches_oracle():
    w = synth.tiny_f32(n_layers=4, gate_layer=1)
    st, g, ol, oh = _build(w)
    st.reset()
    st.run()
    torch.cuda.synchronize()
    want = O.pruned_prefill_stack(g["hidden"], ol, oh, g, w.k, w.gate_layer, **_common(w))
    np.testing.assert_array_equal(st.kept.cpu().numpy(), want["kept_idx"])
    np.testing.assert_allclose(_host(st.hk), want["out"], atol=2e-3, rtol=2e-3)


def test_stack_bf16_parts_match_oracle():
    # bf16 tensor-core path: each part is checked against the oracle fed the
    # GPU's own input to that part, so bf16 rounding upstream cannot move the
    # kept set of the comparison
    w = synth.tiny_f32(dtype="bf16", qk_norm=True, n_layers=4, gate_layer=1)
    st, g, ol, oh = _build(w)
    common = _common(w)
    flat = dict(pos=np.arange(w.n), bias=None, ratio=None, head_gain=np.zeros(w.hq), head_temp=np.ones(w.hq))
    st.reset()
    st.full_part()
    torch.cuda.synchronize()
    # layers 0 .. L-1 and layer L's attention half: the post-attention residual
    h_gate = _host(st.h)
    h = g["hidden"]
    for l in range(w.gate_layer):
        h = O.decoder_layer(h, ol[l], **flat, **common)
    want_h1 = O.attention_block(h, ol[w.gate_layer], **flat, **common)
    np.testing.assert_allclose(h_gate, want_h1, atol=6e-2, rtol=4e-2)
    st.gate_select()
    torch.cuda.synchronize()
    s_gpu = st.scores.cpu().numpy()
    # the gate normalises with layer L's post-attention RMSNorm weight
    s_or = O.gate_scores(h_gate, ol[w.gate_layer]["w_post_norm"], 1e-6, g["w1"], g["b1"], g["w2"], g["b2"],
                         g["prunable"])
    rms = np.sqrt(np.mean(s_or[g["prunable"] == 1] ** 2))
    assert np.max(np.abs(s_gpu - s_or)) <= 1e-3 * rms
    idx = O.select_kept(s_gpu, g["prunable"], w.k)
    np.testing.assert_array_equal(st.kept.cpu().numpy(), idx)     # bit-exact on the GPU's own scores
    st.gather_mlp()
    torch.cuda.synchronize()
    gat = O.gather(h_gate, idx, s_gpu, g["prunable"], 1e-6)
    np.testing.assert_array_equal(st.pos.cpu().numpy(), gat["pos"])
    np.testing.assert_allclose(st.bias.cpu().numpy(), gat["bias"], atol=1e-6, rtol=2e-6)
    np.testing.assert_allclose(st.ratio.cpu().numpy(), gat["ratio"], atol=1e-6, rtol=2e-6)
    # layer L's MLP half on the kept rows only
    hk0 = _host(st.hk)
    np.testing.assert_allclose(hk0, O.mlp_block(gat["hidden_kept"], ol[w.gate_layer]), atol=6e-2, rtol=4e-2)
    st.pruned_part()
    torch.cuda.synchronize()
    out = hk0
    for l in range(w.gate_layer + 1, w.n_layers):
        out = O.decoder_layer(out, ol[l], pos=gat["pos"], bias=gat["bias"], ratio=gat["ratio"],
                              head_gain=oh[l]["head_gain"], head_temp=oh[l]["head_temp"], **common)
    np.testing.assert_allclose(_host(st.hk), out, atol=6e-2, rtol=4e-2)


def test_stack_keeping_everything_with_zero_gain_is_the_unpruned_stack():
    w = synth.tiny_f32(dtype="bf16", qk_norm=True, n_layers=4, gate_layer=1)
    w = w.replace(k=w.n)
    st, g, ol, oh = _build(w)
    for hp in st._keep:
        if "head_gain" in hp:
            hp["head_gain"].zero_()
            hp["head_temp"].fill_(1.0)
    st.reset()
    pruned = _host(st.run())
    st.reset()
    full = _host(st.unpruned())
    np.testing.assert_array_equal(st.kept.cpu().numpy(), np.arange(w.n))
    np.testing.assert_allclose(pruned, full, atol=1e-2, rtol=1e-2)
