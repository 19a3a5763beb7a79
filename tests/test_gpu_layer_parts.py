"""GPU parity of the layer halves and of the gather folded into a layer's first
RMSNorm: tg_layer_attention_block / tg_layer_mlp_block (the gate layer's two
halves), tg_gather_rmsnorm and tg_gather_prefill_layer, against the oracle and
against the unfused calls they replace."""
import numpy as np
import pytest
import torch

from learned_token_pruning_b200 import synth, tokengate as tg
from oracle import tokengate_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"
LAYER_BF16 = dict(atol=3e-2, rtol=2e-2)
LAYER_F32 = dict(atol=2e-4, rtol=2e-4)


def d(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV, dtype)


def host(t):
    return t.detach().float().cpu().numpy() if t.dtype in (torch.bfloat16, torch.float32) else t.cpu().numpy()


def assert_close(got, want, atol, rtol, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    err = np.abs(got - want) - (atol + rtol * np.abs(want))
    bad = int((err > 0).sum())
    assert bad == 0, f"{what}: {bad} of {got.size} outside tolerance; max |d| = {np.abs(got - want).max():.3g}"


@pytest.fixture(autouse=True)
def _clean_device_error():
    tg.tg_check_device_error()
    yield
    assert tg.tg_check_device_error() == 0


def _case(n, m_keep, dm, hq, hkv, D, dff, dtype, qk_norm, seed, post_norm_random=True):
    w = synth.Workload(name="p", seed=seed, n=n, n_question=4, d_model=dm, hq=hq, hkv=hkv, head_dim=D,
                       gate_hidden=16, k=m_keep - 4, dtype=dtype, d_ff=dff, qk_norm=qk_norm)
    lw = dict(synth.layer_weights(w))
    rng = np.random.default_rng(seed)
    if post_norm_random:   # non-trivial norm weights, so a swapped weight shows
        lw["w_in_norm"] = rng.uniform(0.5, 1.5, dm).astype(np.float32)
        lw["w_post_norm"] = rng.uniform(0.5, 1.5, dm).astype(np.float32)
    hidden = synth.round_to(rng.standard_normal((n, dm)).astype(np.float32), dtype)
    prunable = np.ones(n, np.uint8)
    prunable[-4:] = 0
    scores = np.where(prunable != 0, rng.standard_normal(n), 0.0).astype(np.float32)
    idx = O.select_kept(scores, prunable, w.k)
    hp = synth.head_params(w)
    return w, lw, hidden, prunable, scores, idx, hp


def _structs(w, lw, hp):
    dt = synth.torch_dtype(w.dtype)
    wd = {k: d(v, torch.float32 if k.endswith("norm") else dt) for k, v in lw.items()}
    wd["head_gain"], wd["head_temp"] = d(hp["head_gain"]), d(hp["head_temp"])
    W, S = tg.layer_structs(wd, dtype=dt, d_model=w.d_model, hq=w.hq, hkv=w.hkv, head_dim=w.head_dim, d_ff=w.d_ff,
                            qk_norm=w.qk_norm, rope_theta=w.rope_theta)
    return W, S, wd


CASES = [
    dict(n=700, m_keep=300, dm=512, hq=4, hkv=2, D=128, dff=1024, dtype="bf16", qk_norm=True, seed=3),
    dict(n=400, m_keep=129, dm=256, hq=4, hkv=2, D=64, dff=384, dtype="bf16", qk_norm=True, seed=4),
    dict(n=300, m_keep=160, dm=256, hq=4, hkv=2, D=64, dff=512, dtype="f32", qk_norm=False, seed=5),
]


@pytest.mark.parametrize("case", CASES)
def test_attention_then_mlp_block_is_the_layer(case):
    w, lw, hidden, prunable, scores, idx, hp = _case(**case)
    W, S, _ = _structs(w, lw, hp)
    m = idx.size
    dt = synth.torch_dtype(w.dtype)
    g = O.gather(hidden, idx, scores, prunable, 1e-6)
    pos, bias, ratio = d(g["pos"], torch.int32), d(g["bias"]), d(g["ratio"])
    ws = torch.empty(tg.tg_workspace_bytes(tg.TG_OP_LAYER, m=m, shape=S), dtype=torch.uint8, device=DEV)
    a = d(g["hidden_kept"], dt)
    tg.tg_pruned_prefill_layer(W, S, a, pos, bias, ratio, ws)
    b = d(g["hidden_kept"], dt)
    tg.tg_layer_attention_block(W, S, b, pos, bias, ratio, ws)
    torch.cuda.synchronize()
    tol = LAYER_BF16 if w.dtype == "bf16" else LAYER_F32
    common = dict(hq=w.hq, hkv=w.hkv, head_dim=w.head_dim, rope_theta=w.rope_theta, qk_norm=w.qk_norm)
    h1 = O.attention_block(g["hidden_kept"], lw, pos=g["pos"], bias=g["bias"], ratio=g["ratio"],
                           head_gain=hp["head_gain"], head_temp=hp["head_temp"], **common)
    assert_close(host(b), h1, what="attention half", **tol)
    tg.tg_layer_mlp_block(W, S, b, ws)
    torch.cuda.synchronize()
    # the same kernels in the same order: bit-identical to the whole layer
    assert torch.equal(a, b)
    assert_close(host(b), O.mlp_block(h1, lw), what="layer", **tol)


@pytest.mark.parametrize("case", CASES)
def test_gather_rmsnorm_bit_exact_rows_and_norm(case):
    w, lw, hidden, prunable, scores, idx, hp = _case(**case)
    dt = synth.torch_dtype(w.dtype)
    m = idx.size
    hd, sc = d(hidden, dt), d(scores)
    sumsq = d(np.array([np.sum(scores.astype(np.float64) ** 2)], np.float32))
    kept = d(idx, torch.int32)
    n_p = int(prunable.sum())
    outs = []
    for fused in (False, True):
        hk = torch.full((m, w.d_model), 7.0, dtype=dt, device=DEV)
        pos = torch.full((m,), -1, dtype=torch.int32, device=DEV)
        bias, ratio = torch.full((m,), 9.0, device=DEV), torch.full((m,), 9.0, device=DEV)
        xn = torch.full((m, w.d_model), 7.0, dtype=dt, device=DEV)
        if fused:
            tg.tg_gather_rmsnorm(hd, kept, sc, sumsq, n_p, 1e-6, d(lw["w_in_norm"]), 1e-6, hk, xn, pos, bias, ratio)
        else:
            tg.tg_gather(hd, kept, sc, sumsq, n_p, 1e-6, hk, pos, bias, ratio)
        torch.cuda.synchronize()
        outs.append((hk, pos, bias, ratio, xn))
    (hk0, pos0, b0, r0, _), (hk1, pos1, b1, r1, xn1) = outs
    assert np.array_equal(host(hk1), hidden[idx])          # bit-exact gather
    for x0, x1 in ((hk0, hk1), (pos0, pos1), (b0, b1), (r0, r1)):
        assert torch.equal(x0, x1)                          # the same side outputs as tg_gather
    want = O.rms_norm(hidden[idx], lw["w_in_norm"], 1e-6)
    # one rounding to the row dtype (bf16: 2^-8 relative), fp32 sums
    tol = dict(atol=1e-2, rtol=8e-3) if w.dtype == "bf16" else dict(atol=1e-5, rtol=1e-5)
    assert_close(host(xn1), want, what="x_norm", **tol)


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("part", ["full", "mlp"])
def test_gather_prefill_layer_equals_gather_then_layer(case, part):
    w, lw, hidden, prunable, scores, idx, hp = _case(**case)
    W, S, _ = _structs(w, lw, hp)
    dt = synth.torch_dtype(w.dtype)
    m = idx.size
    hd, sc = d(hidden, dt), d(scores)
    sumsq = d(np.array([np.sum(scores.astype(np.float64) ** 2)], np.float32))
    kept = d(idx, torch.int32)
    n_p = int(prunable.sum())
    ws = torch.empty(tg.tg_workspace_bytes(tg.TG_OP_LAYER, m=m, shape=S), dtype=torch.uint8, device=DEV)
    res = []
    for fused in (False, True):
        hk = torch.empty(m, w.d_model, dtype=dt, device=DEV)
        pos = torch.empty(m, dtype=torch.int32, device=DEV)
        bias, ratio = torch.empty(m, device=DEV), torch.empty(m, device=DEV)
        if fused:
            tg.tg_gather_prefill_layer(W, S, tg.TG_LAYER_FULL if part == "full" else tg.TG_LAYER_MLP, hd, kept, sc,
                                       sumsq, n_p, 1e-6, hk, pos, bias, ratio, ws)
        else:
            tg.tg_gather(hd, kept, sc, sumsq, n_p, 1e-6, hk, pos, bias, ratio)
            if part == "full":
                tg.tg_pruned_prefill_layer(W, S, hk, pos, bias, ratio, ws)
            else:
                tg.tg_layer_mlp_block(W, S, hk, ws)
        torch.cuda.synchronize()
        res.append((hk, pos, bias, ratio))
    for x0, x1 in zip(*res):
        assert torch.equal(x0, x1)       # the fused norm does the arithmetic of the layer's own
    g = O.gather(hidden, idx, scores, prunable, 1e-6)
    common = dict(hq=w.hq, hkv=w.hkv, head_dim=w.head_dim, rope_theta=w.rope_theta, qk_norm=w.qk_norm)
    if part == "full":
        want = O.decoder_layer(g["hidden_kept"], lw, pos=g["pos"], bias=g["bias"], ratio=g["ratio"],
                               head_gain=hp["head_gain"], head_temp=hp["head_temp"], **common)
    else:
        want = O.mlp_block(g["hidden_kept"], lw)
    assert_close(host(res[1][0]), want, what=part, **(LAYER_BF16 if w.dtype == "bf16" else LAYER_F32))


def test_layer_parts_argument_checks():
    w, lw, hidden, prunable, scores, idx, hp = _case(**CASES[1])
    W, S, _ = _structs(w, lw, hp)
    dt = synth.torch_dtype(w.dtype)
    m = idx.size
    hk = torch.empty(m, w.d_model, dtype=dt, device=DEV)
    kept = d(idx, torch.int32)
    ws = torch.empty(tg.tg_workspace_bytes(tg.TG_OP_LAYER, m=m, shape=S), dtype=torch.uint8, device=DEV)
    sc = d(scores)
    sq = torch.ones(1, device=DEV)
    with pytest.raises(tg.TokenGateError) as e:   # a part that is neither the layer nor its MLP half
        tg.tg_gather_prefill_layer(W, S, tg.TG_LAYER_ATTENTION, d(hidden, dt), kept, sc, sq, 1, 1e-6, hk, None, None,
                                   None, ws)
    assert e.value.status == 1
    with pytest.raises(tg.TokenGateError) as e:   # the whole layer needs positions for RoPE
        tg.tg_gather_prefill_layer(W, S, tg.TG_LAYER_FULL, d(hidden, dt), kept, sc, sq, 1, 1e-6, hk, None, None,
                                   None, ws)
    assert e.value.status == 1
    with pytest.raises(tg.TokenGateError) as e:   # workspace too small
        tg.tg_layer_mlp_block(W, S, hk, ws[:16])
    assert e.value.status == 5
