"""The timeout path of a bounded device wait, made to run out on purpose.

Every wait inside the kernels is bounded; when one expires the kernel records
the site in the device error word, winds down without further waits and
returns, and tg_check_device_error reports TG_ERR_DEVICE_TIMEOUT.  Here the
split-merge wait of the attention kernel -- the second half of a split query
block waiting (in global memory, with no copy or MMA in flight) for the first
half's ready count -- is given a short limit and a target that no CTA reaches
(tg_debug_set_flag_wait), so it runs out.  No other wait is touched, nothing
faults or traps, and the context stays usable: the next call is correct."""
import math

import numpy as np
import pytest
import torch

from learned_token_pruning_b200 import synth, tokengate as tg
from oracle import tokengate_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(m, hq=16, hkv=8, D=128, seed=5):
    rng = np.random.default_rng(seed)
    bf = lambda *s: synth.round_to(rng.standard_normal(s).astype(np.float32), "bf16")
    q, k, v = bf(m, hq * D), bf(m, hkv * D), bf(m, hkv * D)
    bias = rng.standard_normal(m).astype(np.float32)
    ratio = O.temperature_ratio(np.sort(rng.choice(8 * m, m, replace=False))).astype(np.float32)
    gain = rng.uniform(0.5, 2.0, hq).astype(np.float32)
    temp = rng.uniform(0.8, 1.2, hq).astype(np.float32)
    return q, k, v, bias, ratio, gain, temp


def _run(q, k, v, bias, ratio, gain, temp, D, ws):
    d = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(DEV, dt)
    out = torch.full((q.shape[0], q.shape[1]), 3.0, dtype=torch.bfloat16, device=DEV)
    tg.tg_gated_attention(d(q, torch.bfloat16), d(k, torch.bfloat16), d(v, torch.bfloat16), D, d(bias), d(gain),
                          d(temp), d(ratio), 1.0 / math.sqrt(D), out, ws=ws)
    return out


def test_split_merge_wait_runs_out_and_reports_timeout():
    m, hq, hkv, D = 2064, 16, 8, 128
    q, k, v, bias, ratio, gain, temp = _case(m, hq, hkv, D)
    nws = tg.attention_workspace_bytes(m, hq, hkv, D, torch.bfloat16)
    assert nws > 0, "this shape must split its longest query blocks"
    ws = torch.empty(nws, dtype=torch.uint8, device=DEV)
    assert tg.tg_check_device_error() == 0
    tg.tg_debug_set_flag_wait(1_000_000, 1000)     # 1 ms, and a ready count no CTA reaches
    try:
        _run(q, k, v, bias, ratio, gain, temp, D, ws)
        with pytest.raises(tg.TokenGateError) as e:
            tg.tg_check_device_error()
        assert e.value.status == 7                  # TG_ERR_DEVICE_TIMEOUT
        assert "site 9" in str(e)                   # the attention kernel's wait
    finally:
        tg.tg_debug_set_flag_wait(0, 0)
    # the word was read and cleared, and the next call runs normally
    out = _run(q, k, v, bias, ratio, gain, temp, D, ws)
    assert tg.tg_check_device_error() == 0
    rows = np.r_[0, 1, 127, 128, 1000, 2047, 2048, 2063]
    want = O.gated_attention(q.reshape(m, hq, D), k.reshape(m, hkv, D), v.reshape(m, hkv, D), bias, gain, temp,
                             ratio, 1.0 / math.sqrt(D), rows=rows)
    got = out.float().cpu().numpy().reshape(m, hq, D)[rows]
    err = np.abs(got - want) - (2e-2 + 1e-2 * np.abs(want))
    assert np.all(err <= 0)
