"""Decode over the gated KV cache: the CUDA kernels against the CPU oracle on the
same seeded inputs, element by element (small caches, ragged chunk tails, every
GQA group size the kernels take, both head dims and dtypes), and at the cache
lengths of the workloads (kept rows of the 16K and 128K prompts plus generated
tokens) on every output.  bf16 caches take the kernel that streams the cache
through shared memory by TMA; TG_DECODE_SIMT=1 sends them to the CUDA-core
kernel that fp32 caches use, and a few cases run that way too."""
import math

import numpy as np
import pytest
import torch

from learned_token_pruning_b200 import synth, tokengate as tg
from oracle import tokengate_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"
ATTN_BF16 = dict(atol=2e-2, rtol=1e-2)
ATTN_F32 = dict(atol=1e-4, rtol=1e-4)


def _case(length, hq, hkv, dh, dtype, seed, generated=3):
    rng = np.random.default_rng(seed)
    q = synth.round_to(rng.standard_normal((hq, dh)).astype(np.float32), dtype)
    k = synth.round_to(rng.standard_normal((length, hkv, dh)).astype(np.float32), dtype)
    v = synth.round_to(rng.standard_normal((length, hkv, dh)).astype(np.float32), dtype)
    bias = rng.standard_normal(length).astype(np.float32)
    bias[max(0, length - generated):] = 0.0   # generated rows carry no gate bias
    gain = rng.uniform(0.5, 2.0, hq).astype(np.float32)
    temp = rng.uniform(0.8, 1.2, hq).astype(np.float32)
    return q, k, v, bias, gain, temp


def _gpu(q, k, v, dh, bias, gain, temp, ratio, dtype, kv_buffer=None):
    dt = synth.torch_dtype(dtype)
    length, hkv, _ = k.shape
    hq = q.shape[0]
    if kv_buffer is None:
        kd = torch.from_numpy(k.reshape(length, hkv * dh)).to(DEV, dt)
        vd = torch.from_numpy(v.reshape(length, hkv * dh)).to(DEV, dt)
    else:
        kd, vd = kv_buffer
    qd = torch.from_numpy(q).to(DEV, dt)
    out = torch.empty(hq, dh, dtype=dt, device=DEV)
    lse = torch.empty(hq, dtype=torch.float32, device=DEV)
    ws = torch.full((tg.decode_workspace_bytes(length, hq, hkv, dh),), 0xA5, dtype=torch.uint8, device=DEV)
    tg.tg_gated_decode_attention(qd, kd, vd, dh, None if bias is None else torch.from_numpy(bias).to(DEV),
                                 torch.from_numpy(gain).to(DEV), torch.from_numpy(temp).to(DEV), ratio,
                                 1.0 / math.sqrt(dh), out, ws, lse)
    assert tg.tg_check_device_error() == 0
    return out.float().cpu().numpy(), lse.cpu().numpy()


def _check(length, hq, hkv, dh, dtype, seed, with_bias=True):
    q, k, v, bias, gain, temp = _case(length, hq, hkv, dh, dtype, seed)
    ratio = tg.tg_decode_temperature_ratio(max(length - 3, 0), 4 * length, 2)
    got, lse = _gpu(q, k, v, dh, bias if with_bias else None, gain, temp, ratio, dtype)
    want, wlse = O.gated_decode_attention(q, k, v, bias if with_bias else None, gain, temp, ratio,
                                          1.0 / math.sqrt(dh), return_lse=True)
    tol = ATTN_BF16 if dtype == "bf16" else ATTN_F32
    np.testing.assert_allclose(got, want, **tol)
    np.testing.assert_allclose(lse, wlse, rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("length", [1, 2, 63, 64, 65, 127, 300, 1000])
@pytest.mark.parametrize("dh", [64, 128])
def test_decode_bf16_small_caches(length, dh):
    # a single row, one chunk, ragged last chunk, several chunks (64-key multiples)
    _check(length, 16, 8, dh, "bf16", seed=length + dh)


@pytest.mark.parametrize("hq,hkv", [(4, 4), (4, 2), (6, 2), (8, 1), (16, 8)])
def test_decode_group_sizes(hq, hkv):
    # group 1 .. 8 query heads per KV head (8 is the kernel's limit)
    _check(517, hq, hkv, 128, "bf16", seed=hq * 10 + hkv)


@pytest.mark.parametrize("length,dh", [(1, 64), (200, 64), (777, 128)])
def test_decode_fp32(length, dh):
    _check(length, 8, 2, dh, "f32", seed=length)


def test_decode_no_bias_is_plain_attention_of_the_last_row():
    _check(300, 16, 8, 128, "bf16", seed=7, with_bias=False)


@pytest.mark.parametrize("length", [2064 + 1, 8256 + 17])
def test_decode_workload_cache_lengths(length):
    # the kept rows of the 16K- and 128K-token prompts, then generated tokens;
    # every output compared (one row of attention is cheap for the oracle)
    _check(length, 16, 8, 128, "bf16", seed=length)


def test_decode_strided_cache_views_and_reruns_are_identical():
    # the cache as K and V column ranges of one fused [L][(Hq + 2 Hkv) D] buffer
    length, hq, hkv, dh = 1500, 16, 8, 128
    q, k, v, bias, gain, temp = _case(length, hq, hkv, dh, "bf16", seed=5)
    qkv = np.zeros((length, (hq + 2 * hkv) * dh), np.float32)
    qkv[:, hq * dh:(hq + hkv) * dh] = k.reshape(length, -1)
    qkv[:, (hq + hkv) * dh:] = v.reshape(length, -1)
    buf = torch.from_numpy(qkv).to(DEV, torch.bfloat16)
    views = (buf[:, hq * dh:(hq + hkv) * dh], buf[:, (hq + hkv) * dh:])
    ratio = 0.9
    got, _ = _gpu(q, k, v, dh, bias, gain, temp, ratio, "bf16", kv_buffer=views)
    again, _ = _gpu(q, k, v, dh, bias, gain, temp, ratio, "bf16", kv_buffer=views)
    assert np.array_equal(got, again)
    want = O.gated_decode_attention(q, k, v, bias, gain, temp, ratio, 1.0 / math.sqrt(dh))
    np.testing.assert_allclose(got, want, **ATTN_BF16)


def test_decode_continues_prefill_attention():
    # the decode query is the newest row: decode over the first L rows with the
    # row's ratio equals the prefill kernel's row L - 1 (two CUDA paths agree)
    length, hq, hkv, dh = 700, 16, 8, 128
    rng = np.random.default_rng(9)
    q = synth.round_to(rng.standard_normal((length, hq * dh)).astype(np.float32), "bf16")
    k = synth.round_to(rng.standard_normal((length, hkv * dh)).astype(np.float32), "bf16")
    v = synth.round_to(rng.standard_normal((length, hkv * dh)).astype(np.float32), "bf16")
    bias = rng.standard_normal(length).astype(np.float32)
    ratio = rng.uniform(0.2, 1.0, length).astype(np.float32)
    gain = rng.uniform(0.5, 2.0, hq).astype(np.float32)
    temp = rng.uniform(0.8, 1.2, hq).astype(np.float32)
    t = lambda a, dt=torch.float32: torch.from_numpy(a).to(DEV, dt)
    out = torch.empty(length, hq * dh, dtype=torch.bfloat16, device=DEV)
    tg.tg_gated_attention(t(q, torch.bfloat16), t(k, torch.bfloat16), t(v, torch.bfloat16), dh, t(bias), t(gain),
                          t(temp), t(ratio), 1.0 / math.sqrt(dh), out)
    got, _ = _gpu(q[-1].reshape(hq, dh), k.reshape(length, hkv, dh), v.reshape(length, hkv, dh), dh, bias, gain,
                  temp, float(ratio[-1]), "bf16")
    np.testing.assert_allclose(got.reshape(-1), out[-1].float().cpu().numpy(), atol=1e-2, rtol=1e-2)


def test_decode_maximum_cache_length():
    # 262144 rows: 256 chunks of 1024 keys per KV head, the most one call takes
    _check(262144, 4, 2, 128, "bf16", seed=3)


@pytest.fixture
def cuda_core_decode(monkeypatch):
    monkeypatch.setenv("TG_DECODE_SIMT", "1")


@pytest.mark.parametrize("length,hq,hkv,dh", [(1, 16, 8, 128), (1000, 16, 8, 64), (2065, 16, 8, 128),
                                              (517, 8, 1, 128), (517, 6, 2, 128)])
def test_decode_bf16_through_the_cuda_core_kernel(cuda_core_decode, length, hq, hkv, dh):
    _check(length, hq, hkv, dh, "bf16", seed=length + hq)


@pytest.mark.parametrize("length", [64 * 18 * 3 + 1, 64 * 18 * 3, 64 * 18 * 3 - 1])
def test_decode_chunk_boundaries_of_the_streaming_kernel(length):
    # 8 KV heads share the SMs: chunks of whole 64-row tiles, a last chunk of
    # one row, exactly full, and one row short
    _check(length, 16, 8, 128, "bf16", seed=length)


@pytest.mark.parametrize("hq,hkv,dh", [(8, 1, 64), (12, 2, 64), (14, 2, 128), (10, 2, 128)])
def test_decode_group_sizes_streaming_kernel(hq, hkv, dh):
    # query rows from registers (group x head_dim / 4 <= 64) or from shared memory, slices that leave threads idle
    _check(1333, hq, hkv, dh, "bf16", seed=hq * 100 + hkv * 10 + dh)


def test_decode_unaligned_bias_vector_takes_the_cuda_core_kernel():
    # a bias vector that starts off a 16-byte boundary cannot be a TMA source
    length, hq, hkv, dh = 700, 16, 8, 128
    q, k, v, bias, gain, temp = _case(length, hq, hkv, dh, "bf16", seed=11)
    dt = torch.bfloat16
    kd = torch.from_numpy(k.reshape(length, -1)).to(DEV, dt)
    vd = torch.from_numpy(v.reshape(length, -1)).to(DEV, dt)
    bd = torch.from_numpy(np.concatenate([[0.0], bias]).astype(np.float32)).to(DEV)[1:]
    assert bd.data_ptr() % 16 != 0
    out = torch.empty(hq, dh, dtype=dt, device=DEV)
    ws = torch.empty(tg.decode_workspace_bytes(length, hq, hkv, dh), dtype=torch.uint8, device=DEV)
    tg.tg_gated_decode_attention(torch.from_numpy(q).to(DEV, dt), kd, vd, dh, bd, torch.from_numpy(gain).to(DEV),
                                 torch.from_numpy(temp).to(DEV), 0.8, 1.0 / math.sqrt(dh), out, ws)
    assert tg.tg_check_device_error() == 0
    want = O.gated_decode_attention(q, k, v, bias, gain, temp, 0.8, 1.0 / math.sqrt(dh))
    np.testing.assert_allclose(out.float().cpu().numpy(), want, **ATTN_BF16)


def test_decode_graph_replays_and_a_reused_workspace():
    # the chunk-merge counters: a workspace of garbage, one call replayed from a
    # CUDA graph, and eager calls of another cache length on the same workspace
    # in between
    hq, hkv, dh = 16, 8, 128
    dt = torch.bfloat16
    ws = torch.full((tg.decode_workspace_bytes(5000, hq, hkv, dh),), 0xA5, dtype=torch.uint8, device=DEV)
    cases = []
    for length, seed in ((5000, 21), (1300, 22)):
        q, k, v, bias, gain, temp = _case(length, hq, hkv, dh, "bf16", seed=seed)
        want = O.gated_decode_attention(q, k, v, bias, gain, temp, 0.85, 1.0 / math.sqrt(dh))
        dev = [torch.from_numpy(q).to(DEV, dt), torch.from_numpy(k.reshape(length, -1)).to(DEV, dt),
               torch.from_numpy(v.reshape(length, -1)).to(DEV, dt), torch.from_numpy(bias).to(DEV),
               torch.from_numpy(gain).to(DEV), torch.from_numpy(temp).to(DEV),
               torch.empty(hq, dh, dtype=dt, device=DEV)]
        cases.append((dev, want))

    def call(dev):
        q, k, v, b, g, t, out = dev
        tg.tg_gated_decode_attention(q, k, v, dh, b, g, t, 0.85, 1.0 / math.sqrt(dh), out, ws)

    def check(i):
        torch.cuda.synchronize()
        assert tg.tg_check_device_error() == 0
        np.testing.assert_allclose(cases[i][0][-1].float().cpu().numpy(), cases[i][1], **ATTN_BF16)

    call(cases[0][0])
    check(0)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call(cases[0][0])
    for _ in range(3):
        cases[0][0][-1].zero_()
        graph.replay()
        check(0)
        cases[1][0][-1].zero_()
        call(cases[1][0])
        check(1)
    del graph
