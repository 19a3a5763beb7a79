"""Varlen batching: several requests' kept rows concatenated through one layer
call (every step row-wise, attention per request), and the whole gated step
for a batch of requests of different lengths and budgets, against the oracle
run on each request on its own."""
import math

import numpy as np
import pytest
import torch

from learned_token_pruning_b200 import pipeline, synth, tokengate as tg
from oracle import tokengate_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"
LAYER_BF16 = dict(atol=3e-2, rtol=3e-2)


def _host(t):
    return t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()


def _layer_inputs(w, rows, seed):
    rng = np.random.default_rng(seed)
    hidden = synth.round_to(rng.standard_normal((rows, w.d_model)).astype(np.float32), w.dtype)
    pos = np.sort(rng.choice(4 * rows + 8, size=rows, replace=False)).astype(np.int32)
    bias = rng.standard_normal(rows).astype(np.float32)
    ratio = rng.uniform(0.3, 1.0, rows).astype(np.float32)
    return hidden, pos, bias, ratio


def _structs(w, dev_layer):
    return tg.layer_structs(dev_layer, dtype=synth.torch_dtype(w.dtype), d_model=w.d_model, hq=w.hq, hkv=w.hkv,
                            head_dim=w.head_dim, d_ff=w.d_ff, qk_norm=w.qk_norm, rope_theta=w.rope_theta)


@pytest.mark.parametrize("segs", [(130, 257, 64), (300, 0, 1000, 1)], ids=["three", "with-empty-and-single-row"])
def test_varlen_layer_equals_each_request_alone(segs):
    w = synth.qwen3_1p7b_16k(n=4096, k=500, plant_len=0)
    w = type(w)(**{**w.__dict__, "d_model": 512, "d_ff": 1536})
    dt = synth.torch_dtype(w.dtype)
    lw = synth.layer_weights(w)
    hp = synth.head_params(w)
    dev_layer = {k: torch.from_numpy(v).to(DEV, torch.float32 if k.endswith("norm") else dt) for k, v in lw.items()}
    dev_layer["head_gain"] = torch.from_numpy(hp["head_gain"]).to(DEV)
    dev_layer["head_temp"] = torch.from_numpy(hp["head_temp"]).to(DEV)
    W, S = _structs(w, dev_layer)
    seg = np.r_[0, np.cumsum(segs)].tolist()
    total = seg[-1]
    hidden, pos, bias, ratio = _layer_inputs(w, total, seed=len(segs))
    # pos restarts in every request (original positions of each prompt)
    for r in range(len(segs)):
        pos[seg[r]:seg[r + 1]] = np.sort(np.random.default_rng(r).choice(4 * max(segs[r], 1) + 8, size=segs[r],
                                                                        replace=False))
    h = torch.from_numpy(hidden).to(DEV, dt)
    dpos, dbias, dratio = (torch.from_numpy(a).to(DEV) for a in (pos, bias, ratio))
    ws = torch.empty(tg.tg_layer_varlen_workspace_bytes(S, seg), dtype=torch.uint8, device=DEV)
    tg.tg_pruned_prefill_layer_varlen(W, S, h, dpos, dbias, dratio, seg, ws)
    got = _host(h)
    for r in range(len(segs)):
        a, b = seg[r], seg[r + 1]
        if a == b:
            continue
        # the single-request entry point on the same rows
        hr = torch.from_numpy(hidden[a:b]).to(DEV, dt)
        wsr = torch.empty(tg.tg_workspace_bytes(tg.TG_OP_LAYER, m=b - a, shape=S), dtype=torch.uint8, device=DEV)
        tg.tg_pruned_prefill_layer(W, S, hr, dpos[a:b].contiguous(), dbias[a:b].contiguous(),
                                   dratio[a:b].contiguous(), wsr)
        np.testing.assert_allclose(got[a:b], _host(hr), atol=1e-2, rtol=1e-2)
        # and the oracle
        want = O.decoder_layer(hidden[a:b], lw, hq=w.hq, hkv=w.hkv, head_dim=w.head_dim, pos=pos[a:b],
                               bias=bias[a:b], ratio=ratio[a:b], head_gain=hp["head_gain"], head_temp=hp["head_temp"],
                               rope_theta=w.rope_theta, qk_norm=w.qk_norm)
        np.testing.assert_allclose(got[a:b], want, **LAYER_BF16)
    assert tg.tg_check_device_error() == 0


def test_batched_step_matches_the_oracle_request_by_request():
    base = synth.qwen3_1p7b_16k(n=4096, k=500, plant_len=0)
    ws = [type(base)(**{**base.__dict__, "name": f"r{i}", "seed": base.seed + 17 * i, "n": n, "k": k,
                        "n_question": nq, "d_model": 512, "d_ff": 1536})
          for i, (n, k, nq) in enumerate([(1500, 200, 64), (3000, 700, 32), (700, 1000, 16)])]
    step = pipeline.BatchedPrefillStep(ws, DEV)
    step.capture()
    step.replay()
    torch.cuda.synchronize()
    assert tg.tg_check_device_error() == 0
    w0 = ws[0]
    gate0 = synth.gate_inputs(w0)
    lw = synth.layer_weights(w0)
    hp = synth.head_params(w0)
    out = _host(step.hidden_kept)
    for r, w in enumerate(ws):
        q = step.reqs[r]
        g = synth.gate_inputs(w)
        gate = {**g, **{k: gate0[k] for k in ("norm_w", "w1", "b1", "w2", "b2")}}
        s_gpu = _host(q["scores"])
        want_s = O.gate_scores(g["hidden"], gate["norm_w"], 1e-6, gate["w1"], gate["b1"], gate["w2"], gate["b2"],
                               g["prunable"])
        rms = math.sqrt(np.mean(want_s ** 2))
        assert np.max(np.abs(s_gpu - want_s)) <= 1e-3 * rms
        idx = O.select_kept(s_gpu, g["prunable"], w.k)
        sl = step.rows(r)
        assert np.array_equal(_host(step.kept[sl]).astype(np.int64), idx)   # the budget K >= Np keeps all (r = 2)
        gg = O.gather(g["hidden"], idx, s_gpu, g["prunable"], 1e-6)
        assert np.array_equal(_host(step.pos[sl]).astype(np.int64), gg["pos"])
        want = O.decoder_layer(gg["hidden_kept"], lw, hq=w.hq, hkv=w.hkv, head_dim=w.head_dim, pos=gg["pos"],
                               bias=gg["bias"], ratio=gg["ratio"], head_gain=hp["head_gain"],
                               head_temp=hp["head_temp"], rope_theta=w.rope_theta, qk_norm=w.qk_norm)
        np.testing.assert_allclose(out[sl], want, **LAYER_BF16)
