"""GPU parity: every C-ABI entry point against the CPU oracle on the same
seeded inputs.  Integer/index outputs must be bit-exact; floating point within
the tolerances stated next to each check."""
import math

import numpy as np
import pytest
import torch

from learned_token_pruning_b200 import pipeline, synth, tokengate as tg
from oracle import tokengate_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"

# tolerances
ATTN_BF16 = dict(atol=2e-2, rtol=1e-2)     # bf16 operands, bf16 P and output
ATTN_F32 = dict(atol=1e-4, rtol=1e-4)
LAYER_BF16 = dict(atol=3e-2, rtol=2e-2)    # a chain of bf16 roundings between steps
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


# ============================================================================ select

def gpu_select(scores, mask, k):
    n = scores.size
    n_p = int(mask.sum())
    m = min(k, n_p) + n - n_p
    kept = torch.full((max(m, 1),), -7, dtype=torch.int32, device=DEV)
    tg.tg_topk_select(d(scores), d(mask, torch.uint8), n_p, k, kept[:m] if m else kept[:0])
    return host(kept[:m]).astype(np.int64)


def test_select_golden_cases():
    import json, os
    data = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "select_cases.json")))
    for c in data["cases"]:
        s = np.array([float(x) for x in c["scores"]], np.float32)
        got = gpu_select(s, np.array(c["prunable"], np.uint8), c["k"])
        assert got.tolist() == c["kept"], c["name"]


@pytest.mark.parametrize("n", [1, 2, 9, 100, 4099, 50000])
def test_select_random_tie_heavy_bit_exact(n):
    rng = np.random.default_rng(n)
    pool = np.array([2.0, 1.0, 1.0, 0.5, 0.0, -0.0, -3.0, np.inf, -np.inf, np.nan], np.float32)
    s = rng.choice(pool, size=n).astype(np.float32)
    cont = rng.random(n) < 0.3
    s[cont] = rng.standard_normal(int(cont.sum())).astype(np.float32)
    mask = (rng.random(n) < 0.85).astype(np.uint8)
    n_p = int(mask.sum())
    for k in sorted({0, 1, 2, n_p // 3, max(n_p - 1, 0), n_p, n_p + 5}):
        assert np.array_equal(gpu_select(s, mask, k), O.select_kept(s, mask, k)), (n, k)


@pytest.mark.parametrize("n", [777, 16384, 131072])
def test_select_continuous_scores_bit_exact(n):
    rng = np.random.default_rng(7 + n)
    s = rng.standard_normal(n).astype(np.float32)
    mask = np.ones(n, np.uint8)
    mask[-64:] = 0
    n_p = n - 64
    for k in (1, 100, n_p // 8, n_p - 1):
        assert np.array_equal(gpu_select(s, mask, k), O.select_kept(s, mask, k)), (n, k)


@pytest.mark.parametrize("exact_ties", [False, True])
def test_select_gaussian_mixture_128k_near_and_exact_ties(exact_ties):
    w = synth.long_128k()
    s = synth.mixture_scores(w.n, w.seed, exact_ties=exact_ties)
    mask = synth.prunable_mask(w)
    s[mask == 0] = 0.0
    want = O.select_kept(s, mask, w.k)
    got = gpu_select(s, mask, w.k)
    assert got.size == w.m == 8256
    assert np.array_equal(got, want)


def test_select_layouts_and_degenerate_masks():
    rng = np.random.default_rng(3)
    n = 3000
    s = np.round(rng.standard_normal(n), 2).astype(np.float32)
    qf = np.ones(n, np.uint8)
    qf[:40] = 0  # question first
    for mask in (qf, np.ones(n, np.uint8), np.zeros(n, np.uint8)):
        n_p = int(mask.sum())
        for k in (0, 5, n_p, n_p + 1):
            assert np.array_equal(gpu_select(s, mask, k), O.select_kept(s, mask, k))


def test_select_beyond_shared_memory_cache():
    n = (1 << 19) + 5                       # slices larger than the per-CTA key cache
    rng = np.random.default_rng(5)
    s = np.round(rng.standard_normal(n), 3).astype(np.float32)
    mask = (rng.random(n) < 0.99).astype(np.uint8)
    k = 40000
    assert np.array_equal(gpu_select(s, mask, k), O.select_kept(s, mask, k))


@pytest.mark.parametrize("exact_ties", [False, True])
def test_select_threshold_bin_too_full_for_the_candidate_lists(exact_ties):
    # every score in [1, 1.25): all 131008 prunable keys share the first
    # 11-bit digit, more than a CTA can gather, so the low bits are found by
    # cluster-wide passes instead
    n = 131072
    rng = np.random.default_rng(11)
    s = (1.0 + 0.25 * rng.random(n)).astype(np.float32)
    if exact_ties:
        s = (np.floor(s * 4096) / 4096).astype(np.float32)
    mask = np.ones(n, np.uint8)
    mask[-64:] = 0
    n_p = n - 64
    for k in (1, 8192, n_p // 2, n_p - 1):
        assert np.array_equal(gpu_select(s, mask, k), O.select_kept(s, mask, k)), k


def test_select_planted_block_kept():
    rng = np.random.default_rng(9)
    n = 20000
    s = rng.standard_normal(n).astype(np.float32)
    s[9000:9032] = 8.0 + rng.random(32).astype(np.float32)
    mask = np.ones(n, np.uint8)
    mask[-64:] = 0
    got = set(gpu_select(s, mask, 32).tolist())
    assert set(range(9000, 9032)) <= got and len(got) == 96


def test_select_mask_count_mismatch_reports_device_error():
    n = 1000
    s = np.arange(n, dtype=np.float32)
    mask = np.ones(n, np.uint8)
    # caller claims 990 prunable tokens although all 1000 are: m = 10 + 10
    kept = torch.zeros(20, dtype=torch.int32, device=DEV)
    tg.tg_topk_select(d(s), d(mask, torch.uint8), 990, 10, kept)
    with pytest.raises(tg.TokenGateError) as e:
        tg.tg_check_device_error()
    assert e.value.status == 8


def test_select_mask_count_mismatch_reports_device_error_cluster():
    n = 20000                               # the cluster selector
    s = np.arange(n, dtype=np.float32)
    mask = np.ones(n, np.uint8)
    kept = torch.zeros(200, dtype=torch.int32, device=DEV)
    tg.tg_topk_select(d(s), d(mask, torch.uint8), n - 100, 100, kept)
    with pytest.raises(tg.TokenGateError) as e:
        tg.tg_check_device_error()
    assert e.value.status == 8


# ============================================================================ gather

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gather_bit_exact_rows_and_fp32_side_outputs(dtype):
    rng = np.random.default_rng(11)
    n, dm = 3001, 256
    hidden = synth.round_to(rng.standard_normal((n, dm)).astype(np.float32), dtype)
    mask = np.ones(n, np.uint8)
    mask[-33:] = 0
    s = rng.standard_normal(n).astype(np.float32)
    s[mask == 0] = 0.0
    idx = O.select_kept(s, mask, 700)
    m = idx.size
    sumsq = np.float32(np.sum(s.astype(np.float64)[mask != 0] ** 2))
    dt = synth.torch_dtype(dtype)
    hk = torch.empty(m, dm, dtype=dt, device=DEV)
    pos = torch.empty(m, dtype=torch.int32, device=DEV)
    bias = torch.empty(m, dtype=torch.float32, device=DEV)
    ratio = torch.empty(m, dtype=torch.float32, device=DEV)
    tg.tg_gather(d(hidden, dt), d(idx, torch.int32), d(s), d(np.array([sumsq])), int(mask.sum()), 1e-6, hk, pos,
                 bias, ratio)
    want = O.gather(hidden, idx, s, mask, 1e-6)
    assert torch.equal(hk.cpu(), torch.from_numpy(want["hidden_kept"]).to(dt))
    assert np.array_equal(host(pos), want["pos"])
    assert_close(host(bias), want["bias"], 1e-6, 2e-6, "bias")
    assert_close(host(ratio), want["ratio"], 1e-7, 1e-6, "ratio")


# ============================================================================ gate score

def _gate_case(n, dm, h, dtype, seed, norm_w=False):
    w = synth.Workload(name="g", seed=seed, n=n, n_question=17, d_model=dm, hq=2, hkv=1, head_dim=64,
                       gate_hidden=h, k=10, dtype=dtype, d_ff=128, plant_len=8)
    g = synth.gate_inputs(w)
    if norm_w:
        g["norm_w"] = np.random.default_rng(seed).uniform(0.5, 1.5, dm).astype(np.float32)
        g["b1"] = np.random.default_rng(seed + 1).standard_normal(h).astype(np.float32) * 0.1
        g["b2"] = np.float32(0.25)
    return w, g


def _gpu_scores(w, g, pass_norm):
    dt = synth.torch_dtype(w.dtype)
    scores = torch.empty(w.n, dtype=torch.float32, device=DEV)
    sumsq = torch.empty(1, dtype=torch.float32, device=DEV)
    ws = torch.empty(max(tg.tg_workspace_bytes(tg.TG_OP_GATE_SCORE, n=w.n, d_model=w.d_model, h=w.gate_hidden), 16),
                     dtype=torch.uint8, device=DEV)
    tg.tg_gate_score(d(g["hidden"], dt), d(g["norm_w"]) if pass_norm else None, 1e-6, d(g["w1"], dt), d(g["b1"]),
                     d(g["w2"]), float(g["b2"]), d(g["prunable"], torch.uint8), scores, sumsq, ws)
    return host(scores), float(host(sumsq)[0])


@pytest.mark.parametrize("n,dm,h,dtype,tol", [
    (512, 256, 64, "f32", 1e-4),          # tiny fp32 workload shape (CUDA cores)
    (1000, 256, 64, "bf16", 1e-3),         # tensor cores, 64-wide MLP
    (777, 512, 128, "bf16", 1e-3),         # 128-wide MLP, ragged last tile
    (4096 + 77, 2048, 256, "bf16", 1e-3),  # Qwen3-1.7B gate shape
    (300, 200, 48, "bf16", 1e-3),          # K tail (200 = 3*64 + 8) and h padded to 64
    (300, 200, 200, "bf16", 1e-3),         # K tail and h padded to 256
    (16384, 2048, 256, "bf16", 1e-3),      # the 16K-token step's gate: 128 CTAs, one wave
])
def test_gate_score_matches_oracle(n, dm, h, dtype, tol):
    w, g = _gate_case(n, dm, h, dtype, seed=n)
    got, sumsq = _gpu_scores(w, g, pass_norm=False)
    want = O.gate_scores(g["hidden"], None, 1e-6, g["w1"], g["b1"], g["w2"], g["b2"], g["prunable"])
    rms = math.sqrt(np.mean(want ** 2))
    assert np.max(np.abs(got - want)) <= tol * rms
    assert np.all(got[g["prunable"] == 0] == 0.0)
    ref_sumsq = float(np.sum(want[g["prunable"] != 0] ** 2))
    assert abs(sumsq - ref_sumsq) <= 10 * tol * ref_sumsq


def test_gate_score_norm_weight_and_biases():
    # a non-unit norm weight is folded into W1 in bf16 first: one extra bf16 rounding per weight
    w, g = _gate_case(2000, 512, 256, "bf16", seed=5, norm_w=True)
    got, _ = _gpu_scores(w, g, pass_norm=True)
    want = O.gate_scores(g["hidden"], g["norm_w"], 1e-6, g["w1"], g["b1"], g["w2"], g["b2"], g["prunable"])
    rms = math.sqrt(np.mean(want ** 2))
    assert np.max(np.abs(got - want)) <= 1e-2 * rms


def test_gate_score_is_deterministic():
    w, g = _gate_case(4096, 512, 128, "bf16", seed=8)
    a = _gpu_scores(w, g, False)
    b = _gpu_scores(w, g, False)
    assert np.array_equal(a[0], b[0]) and a[1] == b[1]


def _fused_vs_separate(w, g, k):
    dt = synth.torch_dtype(w.dtype)
    n = w.n
    n_p = int(g["prunable"].sum())
    m = min(k, n_p) + n - n_p
    hid, w1 = d(g["hidden"], dt), d(g["w1"], dt)
    b1, w2 = d(g["b1"]), d(g["w2"])
    mask = d(g["prunable"], torch.uint8)
    ws = torch.empty(tg.tg_workspace_bytes(tg.TG_OP_GATE_SELECT, n=n, d_model=w.d_model, h=w.gate_hidden),
                     dtype=torch.uint8, device=DEV)
    out = []
    for fused in (True, False):
        sc = torch.full((n,), float("nan"), device=DEV)
        sq = torch.full((1,), float("nan"), device=DEV)
        kept = torch.full((max(m, 1),), -1, dtype=torch.int32, device=DEV)
        if fused:
            tg.tg_gate_score_select(hid, None, 1e-6, w1, b1, w2, float(g["b2"]), mask, n_p, k, sc, sq, kept[:m], ws)
        else:
            tg.tg_gate_score(hid, None, 1e-6, w1, b1, w2, float(g["b2"]), mask, sc, sq, ws)
            tg.tg_topk_select(sc, mask, n_p, k, kept[:m])
        torch.cuda.synchronize()
        out.append((sc, sq, kept[:m]))
    (sf, qf, kf), (ss, qs, ks) = out
    assert torch.equal(sf, ss) and torch.equal(qf, qs)          # the same scoring kernel
    assert torch.equal(kf, ks)                                   # bit-exact kept indices
    want = O.select_kept(host(sf), g["prunable"], k)
    assert np.array_equal(host(kf).astype(np.int64), want)       # and the oracle's selection on those scores
    return host(sf)


@pytest.mark.parametrize("n,dm,k", [
    (1000, 512, 100),      # one-CTA selector: no histogram
    (5000, 512, 600),      # cluster selector from the gate's histogram
    (16384, 2048, 2000),   # the 16K-token step
    (40000, 512, 3000),
    (16384, 512, 0),       # keep only the question
    (16384, 512, 20000),   # keep everything
])
def test_gate_score_select_equals_separate_calls(n, dm, k):
    w, g = _gate_case(n, dm, 256, "bf16", seed=n + k)
    _fused_vs_separate(w, g, k)


@pytest.mark.parametrize("dtype,dm,h,norm_w", [
    ("f32", 256, 64, False),     # CUDA-core gate: the cluster selector builds its own first digit
    ("bf16", 2048, 256, True),   # the norm weight folded into W1, histogram from the gate
])
def test_gate_score_select_other_gate_paths(dtype, dm, h, norm_w):
    n, k = 9000, 1500
    w, g = _gate_case(n, dm, h, dtype, seed=31, norm_w=norm_w)
    dt = synth.torch_dtype(w.dtype)
    n_p = int(g["prunable"].sum())
    m = min(k, n_p) + n - n_p
    args = [d(g["hidden"], dt), d(g["norm_w"]) if norm_w else None, 1e-6, d(g["w1"], dt), d(g["b1"]), d(g["w2"]),
            float(g["b2"]), d(g["prunable"], torch.uint8)]
    ws = torch.empty(tg.tg_workspace_bytes(tg.TG_OP_GATE_SELECT, n=n, d_model=dm, h=h), dtype=torch.uint8, device=DEV)
    sc, sq = torch.empty(n, device=DEV), torch.empty(1, device=DEV)
    kept = torch.empty(m, dtype=torch.int32, device=DEV)
    tg.tg_gate_score_select(*args, n_p, k, sc, sq, kept, ws)
    sc2, sq2 = torch.empty(n, device=DEV), torch.empty(1, device=DEV)
    kept2 = torch.empty(m, dtype=torch.int32, device=DEV)
    tg.tg_gate_score(*args, sc2, sq2, ws)
    tg.tg_topk_select(sc2, args[-1], n_p, k, kept2)
    torch.cuda.synchronize()
    assert torch.equal(sc, sc2) and torch.equal(sq, sq2) and torch.equal(kept, kept2)
    assert np.array_equal(host(kept).astype(np.int64), O.select_kept(host(sc), g["prunable"], k))
    want = O.gate_scores(g["hidden"], g["norm_w"] if norm_w else None, 1e-6, g["w1"], g["b1"], g["w2"], g["b2"],
                         g["prunable"])
    rms = math.sqrt(np.mean(want ** 2))
    tol = 1e-4 if dtype == "f32" else 1e-2
    assert np.max(np.abs(host(sc) - want)) <= tol * rms


def test_gate_score_select_kept_zero_workspace_across_calls():
    # TG_WS_KEPT_ZERO: no memset; each call must leave the gate's counter and
    # the selector's histogram at zero, so calls on alternating inputs through
    # one zero-filled workspace equal calls without the flag
    n, dm, h, k = 20000, 512, 256, 3000
    cases = [_gate_case(n, dm, h, "bf16", seed=s) for s in (41, 42)]
    n_p = int(cases[0][1]["prunable"].sum())
    m = min(k, n_p) + n - n_p
    nbytes = tg.tg_workspace_bytes(tg.TG_OP_GATE_SELECT, n=n, d_model=dm, h=h)
    ws_kept = torch.zeros(nbytes, dtype=torch.uint8, device=DEV)
    ws_plain = torch.full((nbytes,), 0xA5, dtype=torch.uint8, device=DEV)   # contents do not matter without the flag
    part = (((n + 127) // 128) * 4 + 255) // 256 * 256     # the counter slot, then the histogram
    for rep in range(4):
        w, g = cases[rep % 2]
        args = [d(g["hidden"], torch.bfloat16), None, 1e-6, d(g["w1"], torch.bfloat16), d(g["b1"]), d(g["w2"]),
                float(g["b2"]), d(g["prunable"], torch.uint8), n_p, k]
        out = []
        for ws, flags in ((ws_kept, tg.TG_WS_KEPT_ZERO), (ws_plain, 0)):
            sc, sq = torch.empty(n, device=DEV), torch.empty(1, device=DEV)
            kept = torch.empty(m, dtype=torch.int32, device=DEV)
            tg.tg_gate_score_select(*args, sc, sq, kept, ws, flags=flags)
            out.append((sc, sq, kept))
        torch.cuda.synchronize()
        assert torch.equal(out[0][0], out[1][0]) and torch.equal(out[0][1], out[1][1])
        assert torch.equal(out[0][2], out[1][2])
        assert int(ws_kept[part:part + 256 + 8192].count_nonzero()) == 0
    with pytest.raises(tg.TokenGateError):
        tg.tg_gate_score_select(*args, sc, sq, kept, ws_kept, flags=2)


def test_gate_score_select_exact_ties_at_the_threshold():
    # 400 copies of one hidden row; its entries are 0 or +-1/8, so the row's
    # sum of squares is exact in any summation order and the copies score
    # bit-identically wherever they sit in a tile.  The budget puts the
    # threshold inside that group, so the kept set depends on breaking the
    # ties towards the lower index
    n, dm = 20000, 512
    w, g = _gate_case(n, dm, 256, "bf16", seed=77)
    rng = np.random.default_rng(77)
    dup = rng.choice(np.flatnonzero(g["prunable"]), 400, replace=False)
    g = dict(g)
    g["hidden"] = g["hidden"].copy()
    g["hidden"][dup] = np.round(np.clip(g["hidden"][dup[0]], -1, 1)) * 0.125
    s = _fused_vs_separate(w, g, 1000)              # any budget: scores first
    above = int(np.sum(s[g["prunable"] != 0] > s[dup[0]]))
    assert np.all(s[dup] == s[dup[0]])
    _fused_vs_separate(w, g, above + 150)


def test_gate_score_select_all_scores_tied():
    # every prunable row the same (entries 0 or +-1/8): one score, one bin,
    # more candidates than a CTA can gather; the budget splits the tie
    n, dm = 40000, 512
    w, g = _gate_case(n, dm, 256, "bf16", seed=78)
    g = dict(g)
    row = np.round(np.clip(g["hidden"][0], -1, 1)) * 0.125
    g["hidden"] = np.broadcast_to(row, g["hidden"].shape).astype(g["hidden"].dtype).copy()
    s = _fused_vs_separate(w, g, 3000)
    assert np.unique(s[g["prunable"] != 0]).size == 1


# ============================================================================ attention

def _attn_case(m, hq, hkv, D, dtype, seed):
    rng = np.random.default_rng(seed)
    q = synth.round_to(rng.standard_normal((m, hq * D)).astype(np.float32), dtype)
    k = synth.round_to(rng.standard_normal((m, hkv * D)).astype(np.float32), dtype)
    v = synth.round_to(rng.standard_normal((m, hkv * D)).astype(np.float32), dtype)
    bias = rng.standard_normal(m).astype(np.float32)
    ratio = rng.uniform(0.5, 1.0, m).astype(np.float32)
    ratio[0] = 0.0
    gain = rng.uniform(0.5, 2.0, hq).astype(np.float32)
    temp = rng.uniform(0.8, 1.2, hq).astype(np.float32)
    return q, k, v, bias, ratio, gain, temp


def _attn_ws(m, hq, hkv, D, dt, split=True):
    """Workspace for the key-range split (garbage-filled: the call must not rely on its contents)."""
    nbytes = tg.attention_workspace_bytes(m, hq, hkv, D, dt) if split else 0
    if nbytes == 0:
        return None
    return torch.full((nbytes,), 0xA5, dtype=torch.uint8, device=DEV)


def _gpu_attn(q, k, v, D, bias, ratio, gain, temp, dtype, with_lse=True, split=True):
    dt = synth.torch_dtype(dtype)
    m = q.shape[0]
    hq = q.shape[1] // D
    out = torch.empty(m, q.shape[1], dtype=dt, device=DEV)
    lse = torch.empty(hq, m, dtype=torch.float32, device=DEV) if with_lse else None
    ws = _attn_ws(m, hq, k.shape[1] // D, D, dt, split)
    tg.tg_gated_attention(d(q, dt), d(k, dt), d(v, dt), D, None if bias is None else d(bias), d(gain), d(temp),
                          None if ratio is None else d(ratio), 1.0 / math.sqrt(D), out, lse, ws)
    assert tg.tg_check_device_error() == 0
    return host(out), (host(lse) if with_lse else None)


def _oracle_attn(q, k, v, D, bias, ratio, gain, temp, rows=None):
    m = q.shape[0]
    o, lse = O.gated_attention(q.reshape(m, -1, D), k.reshape(m, -1, D), v.reshape(m, -1, D), bias, gain, temp,
                               ratio, 1.0 / math.sqrt(D), rows=rows, return_lse=True)
    return o.reshape(o.shape[0], -1), lse


@pytest.mark.parametrize("split", [True, False])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("m", [1, 5, 127, 128, 129, 255, 256, 257, 300, 1000])
def test_attention_bf16_tensor_cores(m, D, split):
    q, k, v, bias, ratio, gain, temp = _attn_case(m, 4, 2, D, "bf16", seed=m + D)
    got, lse = _gpu_attn(q, k, v, D, bias, ratio, gain, temp, "bf16", split=split)
    want, wlse = _oracle_attn(q, k, v, D, bias, ratio, gain, temp)
    assert_close(got, want, what="out", **ATTN_BF16)
    assert_close(lse, wlse, 2e-2, 1e-3, "lse")


@pytest.mark.parametrize("m", [1000, 2064])
def test_attention_bf16_split_key_range_bench_shapes(m):
    # about one wave of causal work: the longest row blocks run as two CTAs whose
    # partial results are merged; every 7th row is compared, ragged tail included
    q, k, v, bias, ratio, gain, temp = _attn_case(m, 16, 8, 128, "bf16", seed=m)
    assert tg.attention_workspace_bytes(m, 16, 8, 128, torch.bfloat16) > 0
    got, lse = _gpu_attn(q, k, v, 128, bias, ratio, gain, temp, "bf16")
    rows = list(range(0, m, 7)) + [m - 1]
    want, wlse = _oracle_attn(q, k, v, 128, bias, ratio, gain, temp, rows=rows)
    assert_close(got[rows], want, what="out", **ATTN_BF16)
    assert_close(lse[:, rows], wlse, 2e-2, 1e-3, "lse")
    # a second call with the same (now used) workspace gives the same bits
    again, _ = _gpu_attn(q, k, v, 128, bias, ratio, gain, temp, "bf16")
    assert np.array_equal(got, again)
    # and the unsplit schedule agrees to within the kernel's own rounding
    whole, _ = _gpu_attn(q, k, v, 128, bias, ratio, gain, temp, "bf16", split=False)
    assert_close(got, whole, what="split vs whole", **ATTN_BF16)


def test_attention_bf16_gqa_16_8_and_no_bias_ratio():
    q, k, v, bias, ratio, gain, temp = _attn_case(515, 16, 8, 128, "bf16", seed=3)
    got, _ = _gpu_attn(q, k, v, 128, None, None, gain, temp, "bf16", with_lse=False)
    want, _ = _oracle_attn(q, k, v, 128, None, None, gain, temp)
    assert_close(got, want, what="out", **ATTN_BF16)
    got, _ = _gpu_attn(q, k, v, 128, bias, ratio, gain, temp, "bf16")
    want, _ = _oracle_attn(q, k, v, 128, bias, ratio, gain, temp)
    assert_close(got, want, what="out", **ATTN_BF16)


def test_attention_bf16_strided_qkv_views():
    m, hq, hkv, D = 333, 4, 2, 128
    q, k, v, bias, ratio, gain, temp = _attn_case(m, hq, hkv, D, "bf16", seed=4)
    qkv = torch.cat([d(q, torch.bfloat16), d(k, torch.bfloat16), d(v, torch.bfloat16)], dim=1).contiguous()
    out = torch.empty(m, hq * D, dtype=torch.bfloat16, device=DEV)
    tg.tg_gated_attention(qkv[:, : hq * D], qkv[:, hq * D:(hq + hkv) * D], qkv[:, (hq + hkv) * D:], D, d(bias),
                          d(gain), d(temp), d(ratio), 1.0 / math.sqrt(D), out,
                          ws=_attn_ws(m, hq, hkv, D, torch.bfloat16))
    want, _ = _oracle_attn(q, k, v, D, bias, ratio, gain, temp)
    assert_close(host(out), want, what="out", **ATTN_BF16)


@pytest.mark.parametrize("m,D", [(160, 64), (37, 128)])
def test_attention_fp32_cuda_cores(m, D):
    q, k, v, bias, ratio, gain, temp = _attn_case(m, 4, 2, D, "f32", seed=m)
    got, lse = _gpu_attn(q, k, v, D, bias, ratio, gain, temp, "f32")
    want, wlse = _oracle_attn(q, k, v, D, bias, ratio, gain, temp)
    assert_close(got, want, what="out", **ATTN_F32)
    assert_close(lse, wlse, 1e-4, 1e-5, "lse")


def test_attention_bf16_group_of_one_uses_cuda_cores():
    q, k, v, bias, ratio, gain, temp = _attn_case(200, 3, 3, 64, "bf16", seed=6)
    got, _ = _gpu_attn(q, k, v, 64, bias, ratio, gain, temp, "bf16")
    want, _ = _oracle_attn(q, k, v, 64, bias, ratio, gain, temp)
    assert_close(got, want, what="out", **ATTN_BF16)


def test_attention_bf16_full_size_sampled_rows():
    # the longest attention of the workloads: M = 8256 kept rows, 16/8 heads, head_dim 128
    m = 8256
    q, k, v, bias, ratio, gain, temp = _attn_case(m, 16, 8, 128, "bf16", seed=8)
    got, lse = _gpu_attn(q, k, v, 128, bias, ratio, gain, temp, "bf16")
    rows = [0, 1, 127, 128, 129, 4095, 4096, 6000, 8191, 8192, 8255]
    want, wlse = _oracle_attn(q, k, v, 128, bias, ratio, gain, temp, rows=rows)
    assert_close(got[rows], want, what="out", **ATTN_BF16)
    assert_close(lse[:, rows], wlse, 2e-2, 1e-3, "lse")
    assert np.all(np.isfinite(got))


# ============================================================================ linear / layer

def _linear_case(epilogue, m, n_out, k_in, seed):
    rng = np.random.default_rng(seed)
    w_rows = 2 * n_out if epilogue == tg.TG_EPI_SWIGLU else n_out
    x = synth.round_to(rng.standard_normal((m, k_in)).astype(np.float32), "bf16")
    w = synth.round_to(rng.standard_normal((w_rows, k_in)).astype(np.float32) * 0.05, "bf16")
    y0 = synth.round_to(rng.standard_normal((m, n_out)).astype(np.float32), "bf16")
    return x, w, y0


def _linear_want(epilogue, x, w, y0, n_out):
    xw = x.astype(np.float64) @ w.astype(np.float64).T
    if epilogue == tg.TG_EPI_SWIGLU:
        return O.silu(xw[:, :n_out]) * xw[:, n_out:]
    return xw + (y0 if epilogue == tg.TG_EPI_RESIDUAL else 0.0)


@pytest.mark.parametrize("kernel", ["pair", "single"])
@pytest.mark.parametrize("shape", [(300, 512, 384), (257, 128, 200), (333, 18432, 192), (600, 32768, 128)],
                         ids=["one-wave", "ragged-m-and-k", "ragged-m-wide", "several-tiles-per-cta"])
@pytest.mark.parametrize("epilogue", [tg.TG_EPI_STORE, tg.TG_EPI_RESIDUAL, tg.TG_EPI_SWIGLU])
def test_linear_bf16_tensor_cores(epilogue, shape, kernel, monkeypatch):
    # "pair": two-SM clusters, 256 x 256 tiles, double-buffered accumulators;
    # "single": the one-SM kernel (128- or 256-row tiles).  The wide shapes give
    # each CTA or pair several tiles, so accumulators are handed back and reused;
    # K = 200 ends in a partial 64-column k-step (zero-filled by the copy engine)
    if kernel == "single":
        monkeypatch.setenv("TG_GEMM_SINGLE_SM", "1")
    else:
        monkeypatch.delenv("TG_GEMM_SINGLE_SM", raising=False)
    m, n_out, k_in = shape
    x, w, y0 = _linear_case(epilogue, m, n_out, k_in, 12)
    y = d(y0, torch.bfloat16)
    tg.tg_linear(d(x, torch.bfloat16), d(w, torch.bfloat16), y, epilogue)
    assert_close(host(y), _linear_want(epilogue, x, w, y0, n_out), 2e-2, 1e-2, "linear")


@pytest.mark.parametrize("shape", [(2064, 6144, 2048, tg.TG_EPI_SWIGLU), (2064, 4096, 2048, tg.TG_EPI_STORE),
                                   (2064, 2048, 2048, tg.TG_EPI_RESIDUAL), (2064, 2048, 6144, tg.TG_EPI_RESIDUAL)],
                         ids=["gate-up-swiglu", "qkv", "o-proj", "down-proj"])
def test_linear_bench_shapes_sampled_rows(shape, monkeypatch):
    # the four projections of the 16K-token step (m = 2064 kept rows), in the
    # launch configuration the step uses; the oracle product on sampled rows
    monkeypatch.delenv("TG_GEMM_SINGLE_SM", raising=False)
    m, n_out, k_in, epilogue = shape
    x, w, y0 = _linear_case(epilogue, m, n_out, k_in, 21)
    y = d(y0, torch.bfloat16)
    tg.tg_linear(d(x, torch.bfloat16), d(w, torch.bfloat16), y, epilogue)
    rows = [0, 1, 127, 128, 255, 256, 1000, 1791, 1792, 2047, 2048, 2063]
    got = host(y)[rows]
    assert_close(got, _linear_want(epilogue, x[rows], w, y0[rows], n_out), 2e-2, 1e-2, "linear")
    assert np.all(np.isfinite(host(y)))


def test_linear_fp32_cuda_cores_ragged():
    rng = np.random.default_rng(13)
    m, n_out, k_in = 77, 100, 45
    x = rng.standard_normal((m, k_in)).astype(np.float32)
    w = rng.standard_normal((n_out, k_in)).astype(np.float32)
    y = torch.empty(m, n_out, device=DEV)
    tg.tg_linear(d(x), d(w), y)
    assert_close(host(y), x.astype(np.float64) @ w.astype(np.float64).T, 1e-4, 1e-5, "linear f32")


def _layer_case(m, dm, hq, hkv, D, dff, dtype, qk_norm, seed):
    w = synth.Workload(name="l", seed=seed, n=m, n_question=0, d_model=dm, hq=hq, hkv=hkv, head_dim=D, gate_hidden=16,
                       k=m, dtype=dtype, d_ff=dff, qk_norm=qk_norm)
    lw = synth.layer_weights(w)
    rng = np.random.default_rng(seed)
    hidden = synth.round_to(rng.standard_normal((m, dm)).astype(np.float32), dtype)
    pos = np.sort(rng.choice(40 * m, m, replace=False)).astype(np.int64)
    bias = rng.standard_normal(m).astype(np.float32)
    ratio = O.temperature_ratio(pos).astype(np.float32)
    hp = synth.head_params(w)
    return w, lw, hidden, pos, bias, ratio, hp


def _gpu_layer(w, lw, hidden, pos, bias, ratio, hp):
    dt = synth.torch_dtype(w.dtype)
    wd = {k: d(v, torch.float32 if k.endswith("norm") else dt) for k, v in lw.items()}
    wd["head_gain"], wd["head_temp"] = d(hp["head_gain"]), d(hp["head_temp"])
    W, S = tg.layer_structs(wd, dtype=dt, d_model=w.d_model, hq=w.hq, hkv=w.hkv, head_dim=w.head_dim, d_ff=w.d_ff,
                            qk_norm=w.qk_norm, rope_theta=w.rope_theta)
    ws = torch.empty(tg.tg_workspace_bytes(tg.TG_OP_LAYER, m=hidden.shape[0], shape=S), dtype=torch.uint8, device=DEV)
    h = d(hidden, dt)
    tg.tg_pruned_prefill_layer(W, S, h, d(pos, torch.int32), d(bias), d(ratio), ws)
    return host(h)


@pytest.mark.parametrize("case", [
    dict(m=160, dm=256, hq=4, hkv=2, D=64, dff=512, dtype="f32", qk_norm=False, tol=LAYER_F32),
    dict(m=300, dm=512, hq=4, hkv=2, D=128, dff=1024, dtype="bf16", qk_norm=True, tol=LAYER_BF16),
    dict(m=129, dm=256, hq=4, hkv=2, D=64, dff=384, dtype="bf16", qk_norm=True, tol=LAYER_BF16),
])
def test_pruned_layer_matches_oracle(case):
    tol = case.pop("tol")
    w, lw, hidden, pos, bias, ratio, hp = _layer_case(seed=case["m"], **case)
    got = _gpu_layer(w, lw, hidden, pos, bias, ratio, hp)
    want = O.decoder_layer(hidden, lw, hq=w.hq, hkv=w.hkv, head_dim=w.head_dim, pos=pos, bias=bias, ratio=ratio,
                           head_gain=hp["head_gain"], head_temp=hp["head_temp"], rope_theta=w.rope_theta,
                           qk_norm=w.qk_norm)
    assert_close(got, want, what="layer", **tol)


# ============================================================================ whole step

def _check_step(w, tol, sample_rows=None, graph=False):
    step = pipeline.GatedPrefillStep(w, DEV)
    if graph:
        # the launch configuration bench.py times: one CUDA graph per step,
        # replayed twice (the second replay starts from the first one's buffers)
        step.capture()
        step.replay()
        step.replay()
    else:
        step.run()
    torch.cuda.synchronize()
    gate = synth.gate_inputs(w)
    layer = synth.layer_weights(w)
    hp = synth.head_params(w)
    s_gpu = host(step.scores)
    # scores: against the oracle on sampled rows (the MLP is row-wise)
    rows = np.arange(w.n) if sample_rows is None else np.asarray(sample_rows)
    want_s = O.gate_scores(gate["hidden"][rows], gate["norm_w"], 1e-6, gate["w1"], gate["b1"], gate["w2"],
                           gate["b2"], gate["prunable"][rows])
    rms = math.sqrt(np.mean(want_s ** 2)) if np.any(want_s) else 1.0
    assert np.max(np.abs(s_gpu[rows] - want_s)) <= tol["score"] * rms
    # selection and compaction: bit-exact given the same fp32 scores
    idx = O.select_kept(s_gpu, gate["prunable"], w.k)
    assert np.array_equal(host(step.kept).astype(np.int64), idx)
    g = O.gather(gate["hidden"], idx, s_gpu, gate["prunable"], 1e-6)
    assert np.array_equal(host(step.pos).astype(np.int64), g["pos"])
    assert_close(host(step.bias), g["bias"], 1e-6, 2e-6, "bias")
    assert_close(host(step.ratio), g["ratio"], 1e-7, 1e-6, "ratio")
    # the layer above the gate on every kept row
    out_rows = None
    want = O.decoder_layer(g["hidden_kept"], layer, hq=w.hq, hkv=w.hkv, head_dim=w.head_dim, pos=g["pos"],
                           bias=g["bias"], ratio=g["ratio"], head_gain=hp["head_gain"], head_temp=hp["head_temp"],
                           rope_theta=w.rope_theta, qk_norm=w.qk_norm, rows=out_rows)
    got = host(step.hidden_kept)
    assert_close(got if out_rows is None else got[out_rows], want, what="layer", **tol["layer"])
    return step


def test_step_tiny_fp32_workload():
    w = synth.tiny_f32()
    step = _check_step(w, dict(score=1e-4, layer=LAYER_F32))
    kept = set(host(step.kept).tolist())
    assert set(range(w.plant_start, w.plant_start + w.plant_len)) <= kept


def test_step_qwen3_shape_reduced_n():
    w = synth.qwen3_1p7b_16k(n=4096, k=500, plant_len=16)
    _check_step(w, dict(score=1e-3, layer=LAYER_BF16))


def test_step_qwen3_16k_full_size():
    # the bench workload itself, in the launch configuration bench.py times:
    # scores on sampled rows (the gate MLP is row-wise; its full-size rows are
    # covered by the gate test), the kept set bit-exact, pos / bias / ratio and
    # every one of the 2064 layer-output rows against the oracle
    w = synth.qwen3_1p7b_16k()
    rng = np.random.default_rng(0)
    rows = np.unique(np.r_[0, 1, 8191, 8192, 8200, 16319, 16320, 16383, rng.integers(0, w.n, 200)])
    _check_step(w, dict(score=1e-3, layer=LAYER_BF16), sample_rows=rows, graph=True)


def test_attention_bf16_zero_gain_ignores_bias():
    q, k, v, bias, ratio, gain, temp = _attn_case(260, 4, 2, 128, "bf16", seed=21)
    gain[[0, 3]] = 0.0
    got, lse = _gpu_attn(q, k, v, 128, bias, ratio, gain, temp, "bf16")
    want, wlse = _oracle_attn(q, k, v, 128, bias, ratio, gain, temp)
    assert_close(got, want, what="out", **ATTN_BF16)
    assert_close(lse, wlse, 2e-2, 1e-3, "lse")
