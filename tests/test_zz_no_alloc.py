"""tg_gate_score_noalloc -- gate scores for callers that cannot allocate.

A serving runtime that owns all of HBM through its own pool, a plugin host
whose interface passes no workspace, or a latency-critical path that must not
take cudaMalloc's device-wide synchronisation cannot hand tg_gate_score a
workspace.  tg_gate_score_noalloc serves them from a fixed scratch array built
into the library.  These tests call it through the C ABI twice in a row (the
second call starts from what the first left in the shared array) and compare
it with the workspace entry point, within the gate-score tolerance the other
GPU tests use; they also check that sizes beyond the array are refused before
anything runs.  The file is named to be collected last.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from learned_token_pruning_b200 import synth, tokengate as tg
from oracle import tokengate_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"
SCORE_TOL = 1e-3   # |d score| <= SCORE_TOL * rms(score), as in the gate-score parity tests


def _dev(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV, dtype)


def _case(n, d, h, dtype, seed, with_norm):
    w = synth.Workload(name="noalloc", seed=seed, n=n, n_question=64, d_model=d, hq=2, hkv=1, head_dim=64,
                       gate_hidden=h, k=10, dtype=dtype, d_ff=128, plant_len=16)
    g = synth.gate_inputs(w)
    dt = synth.torch_dtype(dtype)
    rng = np.random.default_rng(seed)
    norm_w = _dev(rng.uniform(0.5, 1.5, d).astype(np.float32)) if with_norm else None
    args = (_dev(g["hidden"], dt), norm_w, 1e-6, _dev(g["w1"], dt), _dev(g["b1"]), _dev(g["w2"]), 0.125,
            _dev(g["prunable"], torch.uint8))
    return w, args


@pytest.mark.parametrize("n,d,h,dtype,with_norm", [
    (4096 + 77, 2048, 256, "bf16", False),
    (4096 + 77, 2048, 256, "bf16", True),
    (1000, 512, 128, "bf16", True),
    (512, 256, 64, "f32", False),
])
def test_noalloc_matches_workspace_entry_point_on_two_calls(n, d, h, dtype, with_norm):
    w, args = _case(n, d, h, dtype, seed=n + d, with_norm=with_norm)
    g = synth.gate_inputs(w)
    norm_w = args[1].cpu().numpy() if with_norm else None
    # a bf16 norm weight is folded into bf16 W1 on the tensor-core path: the
    # oracle takes the same folded weights (one bf16 rounding of W1 * w_n)
    w1_eff = g["w1"] * norm_w[None, :] if norm_w is not None else g["w1"]
    if norm_w is not None and dtype == "bf16":
        w1_eff = synth.round_to(w1_eff.astype(np.float32), "bf16")
    want = O.gate_scores(g["hidden"], None, 1e-6, w1_eff, g["b1"], g["w2"], 0.125, g["prunable"])
    want_rms = math.sqrt(float(np.mean(want ** 2)))
    ref_s = torch.empty(n, device=DEV)
    ref_q = torch.empty(1, device=DEV)
    ws = torch.empty(tg.tg_workspace_bytes(tg.TG_OP_GATE_SCORE, n=n, d_model=d, h=h), dtype=torch.uint8, device=DEV)
    tg.tg_gate_score(*args, ref_s, ref_q, ws)
    torch.cuda.synchronize()
    ref = ref_s.cpu().numpy()
    rms = math.sqrt(float(np.mean(ref.astype(np.float64) ** 2)))
    for _ in range(2):
        s = torch.full((n,), float("nan"), device=DEV)
        q = torch.full((1,), float("nan"), device=DEV)
        tg.tg_gate_score_noalloc(*args, s, q)
        assert tg.tg_check_device_error() == 0
        got = s.cpu().numpy()
        assert np.all(np.isfinite(got))
        assert np.max(np.abs(got - ref)) <= SCORE_TOL * rms
        assert abs(q.item() - ref_q.item()) <= 10 * SCORE_TOL * abs(ref_q.item())
        # and against the oracle directly
        assert np.max(np.abs(got - want)) <= SCORE_TOL * want_rms
        want_q = float(np.sum(want[g["prunable"] != 0] ** 2))
        assert abs(q.item() - want_q) <= 10 * SCORE_TOL * want_q


def test_noalloc_cuda_core_path_has_no_scratch_limit():
    # fp32 takes the CUDA-core path, which uses no scratch: a size whose
    # tensor-core scratch (2 * d_model * h bytes of folded W1 = 4 MiB) would
    # exceed the array is still served
    n, d, h = 300, 4096, 512
    assert 2 * d * h > tg.lib().tg_gate_score_noalloc_scratch_bytes()
    rng = np.random.default_rng(3)
    hid = rng.standard_normal((n, d)).astype(np.float32)
    w1 = (rng.standard_normal((h, d)) * 0.02).astype(np.float32)
    w2 = rng.standard_normal(h).astype(np.float32)
    mask = np.ones(n, np.uint8)
    mask[-5:] = 0
    s = torch.empty(n, device=DEV)
    q = torch.empty(1, device=DEV)
    tg.tg_gate_score_noalloc(_dev(hid), None, 1e-6, _dev(w1), None, _dev(w2), 0.0, _dev(mask, torch.uint8), s, q)
    assert tg.tg_check_device_error() == 0
    want = O.gate_scores(hid, None, 1e-6, w1, None, w2, 0.0, mask)
    got = s.cpu().numpy()
    assert np.max(np.abs(got - want)) <= 1e-4 * math.sqrt(float(np.mean(want ** 2)))


def test_noalloc_refuses_sizes_beyond_its_scratch():
    L = tg.lib()
    cap = L.tg_gate_score_noalloc_scratch_bytes()
    assert cap == (2 << 20) + (64 << 10)
    p = ctypes.c_void_p(256)  # never dereferenced: the size check comes first
    rc = L.tg_gate_score_noalloc(p, tg.TG_BF16, 1 << 20, 8192, None, 1e-6, p, None, p, 0.0, 256, p, p, p, None)
    assert rc == 4
    assert b"scratch bytes" in L.tg_last_error()
