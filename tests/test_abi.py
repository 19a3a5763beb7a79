"""CPU-only checks of the C ABI: the library builds, loads, exports every entry
point the header declares, and rejects bad arguments on the host before any
CUDA call."""
import ctypes
import math
import os
import re

import pytest

from learned_token_pruning_b200 import build, tokengate as tg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return tg.lib()


def header_functions():
    src = open(os.path.join(ROOT, "include", "tg.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tg_\w+)\s*\(", src)))


def test_header_declares_the_hot_path_entry_points():
    names = header_functions()
    for n in ("tg_gate_score", "tg_topk_select", "tg_gather", "tg_gated_attention", "tg_pruned_prefill_layer"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    names = header_functions()
    assert names
    for n in names:
        assert hasattr(L, n), n
        assert n in tg.SIGNATURES, f"binding lacks {n}"


def test_version_and_status_strings(L):
    assert tg.tg_version().startswith("tokengate-b200")
    assert L.tg_status_string(0) == b"ok"
    assert L.tg_status_string(7) == b"device-side wait timed out"


P = ctypes.c_void_p(256)  # a non-null dummy: validation fails before it is ever dereferenced


def test_select_validation(L):
    assert L.tg_topk_select(None, P, 10, 5, 3, P, 8, None) == 1
    assert L.tg_topk_select(P, P, 10, 5, -1, P, 5, None) == 1           # k < 0
    assert L.tg_topk_select(P, P, 10, 11, 3, P, 8, None) == 1           # n_prunable > n
    assert L.tg_topk_select(P, P, 10, 5, 3, P, 7, None) == 2            # m mismatch
    assert b"m = 7" in L.tg_last_error()
    assert L.tg_topk_select(P, P, 1 << 31, 5, 3, P, (1 << 31) - 2, None) == 4


def test_attention_validation(L):
    g = ctypes.c_void_p(256)
    assert L.tg_gated_attention(g, 2048, g, 1024, g, 1024, 1, 100, 16, 8, 96, None, g, g, None, 0.1, g, 2048, None, None, 0, None) == 4
    assert L.tg_gated_attention(g, 2048, g, 1024, g, 1024, 1, 100, 16, 6, 128, None, g, g, None, 0.1, g, 2048, None, None, 0, None) == 1
    assert L.tg_gated_attention(g, 100, g, 1024, g, 1024, 1, 100, 16, 8, 128, None, g, g, None, 0.1, g, 2048, None, None, 0, None) == 2
    assert L.tg_gated_attention(ctypes.c_void_p(258), 2048, g, 1024, g, 1024, 1, 100, 16, 8, 128, None, g, g, None,
                                0.1, g, 2048, None, None, 0, None) == 3


def test_gather_and_gate_validation(L):
    assert L.tg_gather(P, 1, 10, 2048, P, 11, P, P, 5, 1e-6, P, None, None, None, None) == 1   # m > n
    assert L.tg_gather(P, 1, 10, 20, P, 5, P, P, 5, 1e-6, P, None, None, None, None) == 3      # 40-byte rows
    assert L.tg_gate_score(P, 1, 100, 256, None, 1e-6, P, None, P, 0.0, 64, P, P, P, None, 0, None) == 5


def test_workspace_sizes(L):
    S = tg.LayerShape(1, 2048, 16, 8, 128, 6144, 1, 1e6, 1e-6)
    m = 2064
    want = sum((b + 255) // 256 * 256 for b in (m * 2048 * 2, m * 4096 * 2, m * 2048 * 2, m * 2 * 6144 * 2))
    attn = tg.tg_workspace_bytes(tg.TG_OP_ATTENTION, m=m, shape=S)
    assert tg.tg_workspace_bytes(tg.TG_OP_LAYER, m=m, shape=S) == want + attn
    # without a GPU the library plans for 148 SMs: 17 row blocks x 8 head pairs are
    # one wave, so some of the longest blocks are split; each split block keeps two
    # halves of O (fp32) and of (max, sum) for both heads, plus one counter
    al = lambda b: (b + 255) // 256 * 256
    layout = lambda slots: al(slots * 2 * 2 * 128 * 128 * 4) + al(slots * 2 * 2 * 128 * 8) + al(slots * 4)
    splits = [k for k in range(1, 17) if layout(8 * k) == attn]
    assert len(splits) == 1, attn
    # a launch of several waves needs no split and no workspace
    assert tg.tg_workspace_bytes(tg.TG_OP_ATTENTION, m=8256, shape=S) == 0
    S32 = tg.LayerShape(0, 2048, 16, 8, 128, 6144, 1, 1e6, 1e-6)  # fp32 runs on CUDA cores: no split
    assert tg.tg_workspace_bytes(tg.TG_OP_ATTENTION, m=m, shape=S32) == 0
    assert tg.tg_workspace_bytes(tg.TG_OP_GATE_SCORE, n=16384, d_model=2048, h=256) >= 16384 // 128 * 4 + 256 * 2048 * 2
    assert tg.tg_workspace_bytes(99) == 0


def test_decode_validation_and_workspace(L):
    g = ctypes.c_void_p(256)
    f = L.tg_gated_decode_attention
    # q, k, ldk, v, ldv, dtype, length, hq, hkv, head_dim, bias, gain, temp, ratio, scale, out, lse, ws, ws_bytes, stream
    assert f(None, g, 1024, g, 1024, 1, 10, 16, 8, 128, None, g, g, 1.0, 0.1, g, None, g, 1 << 20, None) == 1
    assert f(g, g, 1024, g, 1024, 1, 0, 16, 8, 128, None, g, g, 1.0, 0.1, g, None, g, 1 << 20, None) == 1   # empty cache
    assert f(g, g, 1024, g, 1024, 1, 10, 16, 6, 128, None, g, g, 1.0, 0.1, g, None, g, 1 << 20, None) == 1  # hq % hkv
    assert f(g, g, 1024, g, 1024, 1, 10, 16, 8, 96, None, g, g, 1.0, 0.1, g, None, g, 1 << 20, None) == 4   # head_dim
    assert f(g, g, 1024, g, 1024, 1, 10, 32, 2, 128, None, g, g, 1.0, 0.1, g, None, g, 1 << 20, None) == 4  # group 16
    assert f(g, g, 1000, g, 1024, 1, 10, 16, 8, 128, None, g, g, 1.0, 0.1, g, None, g, 1 << 20, None) == 2  # ldk < heads
    assert f(g, ctypes.c_void_p(258), 1024, g, 1024, 1, 10, 16, 8, 128, None, g, g, 1.0, 0.1, g, None, g, 1 << 20,
             None) == 3                                                                                        # alignment
    assert f(g, g, 1028, g, 1024, 1, 10, 16, 8, 128, None, g, g, 1.0, 0.1, g, None, g, 1 << 20, None) == 3  # row stride
    need = tg.decode_workspace_bytes(10, 16, 8, 128)
    assert need > 0
    assert f(g, g, 1024, g, 1024, 1, 10, 16, 8, 128, None, g, g, 1.0, 0.1, g, None, g, need - 1, None) == 5  # workspace
    assert f(g, g, 1024, g, 1024, 1, 10, 16, 8, 128, None, g, g, 1.0, 0.1, g, None, None, 0, None) == 5
    # the workspace holds (O, max, sum) of every chunk and query head, then the KV heads' counters
    for length in (1, 64, 2064, 8256, 131072, 262144):
        ws = tg.decode_workspace_bytes(length, 16, 8, 128)
        assert 16 * 130 * 4 * ((length + 1023) // 1024) + 8 * 4 <= ws <= 16 * 130 * 4 * 256 + 256 + 256
    assert tg.decode_workspace_bytes(2064, 16, 6, 128) == 0   # invalid head split
    assert f(g, g, 1024, g, 1024, 1, 262145, 16, 8, 128, None, g, g, 1.0, 0.1, g, None, g, 1 << 30, None) == 4


def test_decode_temperature_ratio_host_helper(L):
    # ratio = log(m_kept + t + 1) / log(max(2, n_prompt + t + 1)), in float
    assert tg.tg_decode_temperature_ratio(3, 10, 0) == pytest.approx(math.log(4) / math.log(11), rel=1e-6)
    assert tg.tg_decode_temperature_ratio(2064, 16384, 7) == pytest.approx(math.log(2072) / math.log(16392), rel=1e-6)
    assert tg.tg_decode_temperature_ratio(0, 0, 0) == 0.0
    assert tg.tg_decode_temperature_ratio(-1, 10, 0) == 0.0


def test_varlen_layer_validation(L):
    S = tg.LayerShape(1, 2048, 16, 8, 128, 6144, 1, 1e6, 1e-6)
    al = lambda b: (b + 255) // 256 * 256
    # attention space and a bias staging copy for the longest request
    assert tg.tg_layer_varlen_workspace_bytes(S, [0, 100, 300]) - tg.tg_layer_varlen_workspace_bytes(S, [0, 300]) == \
        tg.tg_workspace_bytes(tg.TG_OP_ATTENTION, m=200, shape=S) - tg.tg_workspace_bytes(tg.TG_OP_ATTENTION, m=300,
                                                                                          shape=S) \
        + al(200 * 4) - al(300 * 4)
    assert tg.tg_layer_varlen_workspace_bytes(S, [1, 100]) == 0                # must start at 0
    assert tg.tg_layer_varlen_workspace_bytes(S, [0, 100, 50]) == 0            # must not decrease
    assert tg.tg_layer_varlen_workspace_bytes(S, [0, 0]) == 0                  # no rows
    assert tg.tg_layer_varlen_workspace_bytes(S, [0, 0, 64]) > 0               # an empty request is fine
    g = ctypes.c_void_p(256)
    arr = (ctypes.c_int64 * 3)(0, 100, 50)
    assert L.tg_pruned_prefill_layer_varlen(None, ctypes.byref(S), g, g, g, g, arr, 2, g, 1 << 30, None) == 1
    W = tg.LayerWeights(*([g] * 10))
    assert L.tg_pruned_prefill_layer_varlen(ctypes.byref(W), ctypes.byref(S), g, g, g, g, arr, 2, g, 1 << 30,
                                            None) == 1                        # decreasing offsets
    arr0 = (ctypes.c_int64 * 2)(5, 100)
    assert L.tg_pruned_prefill_layer_varlen(ctypes.byref(W), ctypes.byref(S), g, g, g, g, arr0, 1, g, 1 << 30,
                                            None) == 1                        # first offset not 0
    ok = (ctypes.c_int64 * 2)(0, 100)
    assert L.tg_pruned_prefill_layer_varlen(ctypes.byref(W), ctypes.byref(S), g, g, g, g, ok, 1, g, 16,
                                            None) == 5                        # workspace too small


def test_attention_backward_validation_and_workspace(L):
    g = ctypes.c_void_p(256)
    f = L.tg_gated_attention_backward

    def call(m=100, hq=16, hkv=8, dh=128, ldq=2048, ldk=1024, dtype=1, ws=g, ws_bytes=1 << 30, lse=g):
        # q, ldq, k, ldk, v, ldv, o, ldo, dO, lddo, dtype, m, hq, hkv, head_dim, bias, gain, temp, ratio, scale,
        # lse, dq, dk, dv, dbias, dgain, dtemp, ws, ws_bytes, stream
        return f(g, ldq, g, ldk, g, ldk, g, ldq, g, ldq, dtype, m, hq, hkv, dh, None, g, g, None, 0.1, lse, g, g, g,
                 None, None, None, ws, ws_bytes, None)

    assert call(lse=None) == 1                 # the forward's log-sum-exp is required
    assert call(m=0) == 1
    assert call(hkv=6) == 1                    # hq % hkv
    assert call(dh=96) == 4
    assert call(dtype=7) == 1
    assert call(ldq=1000) == 2                 # leading dimension below the heads
    assert call(ws_bytes=16) == 5
    assert call(ws=None) == 5
    assert call(ws=ctypes.c_void_p(260)) == 3  # workspace alignment
    al = lambda b: (b + 255) // 256 * 256
    # per query head and row the dO . o row dot, per KV head and key the dbias partial,
    # per query head and key block of 32 the (dgain, dtemp) partials, and for the
    # tensor-core kernels per query head and row (rounded up to 128) four per-row
    # constants and one head's (dV, dK) partial, then two counters per KV head and
    # key block of 128
    for m in (1, 31, 32, 33, 2064):
        for dh in (64, 128):
            nkb = (m + 31) // 32
            m_pad = (m + 127) // 128 * 128
            assert tg.attention_backward_workspace_bytes(m, 16, 8, dh) == \
                al(16 * m * 4) + al(8 * m * 4) + al(16 * nkb * 8) + al(16 * m_pad * 16) + \
                al(16 * m_pad * 2 * dh * 4) + al(2 * 8 * (m_pad // 128) * 4)
    assert tg.tg_workspace_bytes(tg.TG_OP_ATTENTION_BWD, m=0) == 0
