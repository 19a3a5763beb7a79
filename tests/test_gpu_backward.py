"""Backward of token-gated attention: the CUDA kernels (fed by the CUDA forward's
output and log-sum-exp) against the oracle's fp64 gradients on the same seeded
inputs, every element of dq, dk, dv, dbias, dgain and dtemp, at sizes with
ragged 32-row tiles, every GQA group the layer shapes use, both head dims and
dtypes, strided views of one fused QKV buffer, and the kept-row count of the
16K-token prompt."""
import math

import numpy as np
import pytest
import torch

from learned_token_pruning_b200 import synth, tokengate as tg
from oracle import tokengate_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"
NAMES = ("dq", "dk", "dv", "dbias", "dgain", "dtemp")
# Both sides take the same rounded q, k, v and dO.  The fp32 path differs from
# fp64 only by fp32 accumulation (a few ulp times sqrt of the terms);  the bf16
# path also reads the forward's output rounded to bf16 (relative 2^-9) when it
# forms dO . o, which shifts every dl of a row by P times that error.
TOL = {"f32": 1e-4, "bf16": 2e-2}
# A one-key softmax has no gradient: at m = 1 the exact dq, dk, dbias, dgain and
# dtemp are 0 and the CUDA path returns the rounding of P (dP - dO . o) there,
# whose terms dO . v and dO . o are of order sqrt(D) for unit-normal inputs; a
# tensor whose exact values all lie below 1 is held to tol * FLOOR.
FLOOR = 1.0


def _case(m, hq, hkv, dh, dtype, seed, with_bias=True, with_ratio=True):
    rng = np.random.default_rng(seed)
    r = lambda *s: synth.round_to(rng.standard_normal(s).astype(np.float32), dtype)
    q, k, v, do = r(m, hq, dh), r(m, hkv, dh), r(m, hkv, dh), r(m, hq, dh)
    bias = rng.standard_normal(m).astype(np.float32) if with_bias else None
    ratio = rng.uniform(0.2, 1.0, m).astype(np.float32) if with_ratio else None
    gain = rng.uniform(0.5, 2.0, hq).astype(np.float32)
    temp = rng.uniform(0.8, 1.2, hq).astype(np.float32)
    return q, k, v, do, bias, ratio, gain, temp


def _gpu(q, k, v, do, bias, ratio, gain, temp, dtype, fused=False, pad=0):
    dt = synth.torch_dtype(dtype)
    m, hq, dh = q.shape
    hkv = k.shape[1]
    t = lambda a: None if a is None else torch.from_numpy(a).to(DEV)
    if fused:
        # q, k, v as column ranges of one [m][(hq + 2 hkv) dh] buffer, as the layer holds them
        buf = torch.from_numpy(np.concatenate([q.reshape(m, -1), k.reshape(m, -1), v.reshape(m, -1)], 1)).to(DEV, dt)
        qd, kd, vd = buf[:, :hq * dh], buf[:, hq * dh:(hq + hkv) * dh], buf[:, (hq + hkv) * dh:]
    elif pad:
        # rows padded by `pad` elements: a row stride TMA cannot take (the CUDA-core path)
        def padded(a):
            buf = torch.zeros(m, a.shape[1] * dh + pad, dtype=dt, device=DEV)
            buf[:, :a.shape[1] * dh] = torch.from_numpy(a.reshape(m, -1)).to(DEV, dt)
            return buf[:, :a.shape[1] * dh]
        qd, kd, vd = (padded(a) for a in (q, k, v))
    else:
        qd, kd, vd = (torch.from_numpy(a.reshape(m, -1)).to(DEV, dt) for a in (q, k, v))
    dod = torch.from_numpy(do.reshape(m, -1)).to(DEV, dt)
    out = torch.empty(m, hq * dh, dtype=dt, device=DEV)
    lse = torch.empty(hq, m, dtype=torch.float32, device=DEV)
    scale = 1.0 / math.sqrt(dh)
    # (the forward needs TMA-aligned rows: it reads dense copies of padded views)
    dense = lambda x: torch.empty(x.shape, dtype=x.dtype, device=DEV).copy_(x)
    tg.tg_gated_attention(dense(qd), dense(kd), dense(vd), dh, t(bias), t(gain), t(temp), t(ratio), scale, out, lse)
    g = {"dq": torch.full((m, hq * dh), float("nan"), device=DEV),
         "dk": torch.full((m, hkv * dh), float("nan"), device=DEV),
         "dv": torch.full((m, hkv * dh), float("nan"), device=DEV),
         "dbias": torch.full((m,), float("nan"), device=DEV),
         "dgain": torch.full((hq,), float("nan"), device=DEV),
         "dtemp": torch.full((hq,), float("nan"), device=DEV)}
    ws = torch.full((tg.attention_backward_workspace_bytes(m, hq, hkv, dh),), 0xA5, dtype=torch.uint8, device=DEV)
    tg.tg_gated_attention_backward(qd, kd, vd, out, dod, dh, t(bias), t(gain), t(temp), t(ratio), scale, lse,
                                   g["dq"], g["dk"], g["dv"], ws, dbias=g["dbias"], dgain=g["dgain"],
                                   dtemp=g["dtemp"])
    torch.cuda.synchronize()
    assert tg.tg_check_device_error() == 0
    return {n: g[n].cpu().numpy() for n in NAMES}


def _compare(got, want, dtype, m, hq, hkv, dh):
    tol = TOL[dtype]
    shapes = {"dq": (m, hq * dh), "dk": (m, hkv * dh), "dv": (m, hkv * dh)}
    for n in NAMES:
        w = want[n].reshape(shapes.get(n, want[n].shape))
        gg = got[n]
        assert np.all(np.isfinite(gg)), n
        scale = max(np.max(np.abs(w)), FLOOR)
        err = np.abs(gg - w)
        assert np.all(err <= tol * scale + tol * np.abs(w)), (n, float(err.max()), float(scale))


def _check(m, hq, hkv, dh, dtype, seed, **kw):
    q, k, v, do, bias, ratio, gain, temp = _case(m, hq, hkv, dh, dtype, seed, **kw)
    got = _gpu(q, k, v, do, bias, ratio, gain, temp, dtype)
    want = O.gated_attention_backward(q, k, v, bias, gain, temp, ratio, 1.0 / math.sqrt(dh), do)
    _compare(got, want, dtype, m, hq, hkv, dh)
    return got


@pytest.mark.parametrize("m", [1, 2, 31, 32, 33, 100, 257])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_backward_small_and_ragged(m, dtype):
    # one row, one partial tile, exact tiles, ragged tails of 32-row tiles
    _check(m, 4, 2, 128, dtype, seed=m)


@pytest.mark.parametrize("hq,hkv", [(2, 2), (4, 1), (6, 2), (16, 8)])
@pytest.mark.parametrize("dh", [64, 128])
def test_backward_groups_and_head_dims(hq, hkv, dh):
    _check(150, hq, hkv, dh, "bf16", seed=hq * 10 + hkv + dh)


@pytest.mark.parametrize("with_bias,with_ratio", [(False, True), (True, False), (False, False)])
def test_backward_without_bias_or_ratio(with_bias, with_ratio):
    # no bias: plain attention with a per-row content scale; no ratio: ratio 1
    _check(90, 4, 2, 64, "f32", seed=3, with_bias=with_bias, with_ratio=with_ratio)


def test_backward_is_deterministic_and_reads_strided_views():
    m, hq, hkv, dh = 300, 16, 8, 128
    q, k, v, do, bias, ratio, gain, temp = _case(m, hq, hkv, dh, "bf16", seed=11)
    a = _gpu(q, k, v, do, bias, ratio, gain, temp, "bf16", fused=True)
    b = _gpu(q, k, v, do, bias, ratio, gain, temp, "bf16", fused=True)
    c = _gpu(q, k, v, do, bias, ratio, gain, temp, "bf16", fused=False)
    for n in NAMES:
        assert np.array_equal(a[n], b[n]), n   # bit-identical reruns
        assert np.array_equal(a[n], c[n]), n   # the view does not change the arithmetic
    want = O.gated_attention_backward(q, k, v, bias, gain, temp, ratio, 1.0 / math.sqrt(dh), do)
    _compare(a, want, "bf16", m, hq, hkv, dh)


def test_backward_bias_gradient_sums_to_zero_over_keys_per_row():
    # sum_c dl_rc = 0 for every row and head (softmax rows sum to 1), so
    # sum_c dbias_c = 0 up to the rounding of the forward output (fp32 path)
    got = _check(200, 4, 2, 64, "f32", seed=21)
    assert abs(got["dbias"].sum()) <= 1e-4 * np.abs(got["dbias"]).sum()


def test_backward_workload_kept_rows():
    # the 2064 kept rows of the 16K-token prompt, Qwen3-1.7B attention heads
    _check(2064, 16, 8, 128, "bf16", seed=2064)


@pytest.mark.parametrize("m", [1, 70, 300])
def test_backward_bf16_unaligned_rows_use_the_cuda_core_kernels(m):
    # a row stride of hq * D + 4 elements is not 16-byte aligned: the CUDA-core
    # kernels take it, and agree with the oracle and with the tensor-core path
    hq, hkv, dh = 4, 2, 64
    q, k, v, do, bias, ratio, gain, temp = _case(m, hq, hkv, dh, "bf16", seed=m + 5)
    got = _gpu(q, k, v, do, bias, ratio, gain, temp, "bf16", pad=4)
    want = O.gated_attention_backward(q, k, v, bias, gain, temp, ratio, 1.0 / math.sqrt(dh), do)
    _compare(got, want, "bf16", m, hq, hkv, dh)
    tc = _gpu(q, k, v, do, bias, ratio, gain, temp, "bf16")
    for n in NAMES:
        scale = max(np.max(np.abs(got[n])), FLOOR)
        assert np.max(np.abs(tc[n] - got[n])) <= 2 * TOL["bf16"] * scale, n


def test_backward_kept_rows_of_the_128k_prompt_properties_and_sampled_rows():
    # 8256 rows (the 128K-token prompt's kept rows) in the bench's configuration:
    # every gradient finite, the bias gradient summing to zero over keys,
    # bit-identical reruns, and sampled query rows r against the oracle run on
    # rows 0 .. r (row r's dq depends only on its causal prefix)
    m, hq, hkv, dh = 8256, 16, 8, 128
    q, k, v, do, bias, ratio, gain, temp = _case(m, hq, hkv, dh, "bf16", seed=8256)
    a = _gpu(q, k, v, do, bias, ratio, gain, temp, "bf16")
    b = _gpu(q, k, v, do, bias, ratio, gain, temp, "bf16")
    for n in NAMES:
        assert np.all(np.isfinite(a[n])), n
        assert np.array_equal(a[n], b[n]), n
    assert abs(a["dbias"].sum()) <= 2e-3 * np.abs(a["dbias"]).sum()
    scale = 1.0 / math.sqrt(dh)
    for r in (0, 63, 64, 127, 128, 255, 383):
        sl = slice(0, r + 1)
        want = O.gated_attention_backward(q[sl], k[sl], v[sl], bias[sl], gain, temp, ratio[sl], scale, do[sl])
        w = want["dq"][r].reshape(-1)
        got = a["dq"][r]
        tol = TOL["bf16"] * max(np.max(np.abs(w)), FLOOR)
        assert np.max(np.abs(got - w)) <= tol, r
