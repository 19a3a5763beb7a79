"""Thin Python binding of libtokengate.so (the C ABI in include/tg.h).

Every function here only marshals arguments -- torch tensors become device
pointers, the current torch stream becomes the cudaStream_t -- and calls the
entry point of the same name.  All computation runs in the library's CUDA
kernels; there is no fallback of any kind: if the library is missing or a call
fails, a TokenGateError is raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtokengate.so")

TG_F32, TG_BF16 = 0, 1
TG_OP_GATE_SCORE, TG_OP_LAYER, TG_OP_ATTENTION, TG_OP_DECODE, TG_OP_ATTENTION_BWD, TG_OP_GATE_SELECT = 0, 1, 2, 3, 4, 5
TG_WS_KEPT_ZERO = 1
TG_LAYER_ATTENTION, TG_LAYER_MLP, TG_LAYER_FULL = 1, 2, 3
STATUS = {0: "TG_OK", 1: "TG_ERR_INVALID_ARG", 2: "TG_ERR_SHAPE", 3: "TG_ERR_ALIGN", 4: "TG_ERR_UNSUPPORTED",
          5: "TG_ERR_WORKSPACE", 6: "TG_ERR_CUDA", 7: "TG_ERR_DEVICE_TIMEOUT", 8: "TG_ERR_DEVICE_CHECK"}

# every symbol the header declares, with (restype, argtypes)
_P, _I32, _I64, _F, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_INT = ctypes.c_int


class TokenGateError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({detail})")
        self.status = status


class LayerWeights(ctypes.Structure):
    _fields_ = [("w_in_norm", _P), ("w_qkv", _P), ("w_q_norm", _P), ("w_k_norm", _P), ("w_o", _P),
                ("w_post_norm", _P), ("w_gate_up", _P), ("w_down", _P), ("head_gain", _P), ("head_temp", _P)]


class LayerShape(ctypes.Structure):
    _fields_ = [("dtype", _I32), ("d_model", _I32), ("hq", _I32), ("hkv", _I32), ("head_dim", _I32),
                ("d_ff", _I32), ("qk_norm", _I32), ("rope_theta", _F), ("norm_eps", _F)]


SIGNATURES = {
    "tg_version": (ctypes.c_char_p, []),
    "tg_status_string": (ctypes.c_char_p, [_INT]),
    "tg_last_error": (ctypes.c_char_p, []),
    "tg_check_device_error": (_INT, [_P, ctypes.POINTER(ctypes.c_uint32)]),
    "tg_gate_score": (_INT, [_P, _INT, _I64, _I32, _P, _F, _P, _P, _P, _F, _I32, _P, _P, _P, _P, _SZ, _P]),
    "tg_topk_select": (_INT, [_P, _P, _I64, _I64, _I64, _P, _I64, _P]),
    "tg_gather": (_INT, [_P, _INT, _I64, _I32, _P, _I64, _P, _P, _I64, _F, _P, _P, _P, _P, _P]),
    "tg_gated_attention": (_INT, [_P, _I64, _P, _I64, _P, _I64, _INT, _I64, _I32, _I32, _I32, _P, _P, _P, _P, _F,
                                  _P, _I64, _P, _P, _SZ, _P]),
    "tg_pruned_prefill_layer": (_INT, [ctypes.POINTER(LayerWeights), ctypes.POINTER(LayerShape), _P, _P, _P, _P,
                                       _I64, _P, _SZ, _P]),
    "tg_gated_attention_backward": (_INT, [_P, _I64, _P, _I64, _P, _I64, _P, _I64, _P, _I64, _INT, _I64, _I32, _I32,
                                           _I32, _P, _P, _P, _P, _F, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "tg_gated_decode_attention": (_INT, [_P, _P, _I64, _P, _I64, _INT, _I64, _I32, _I32, _I32, _P, _P, _P, _F, _F,
                                         _P, _P, _P, _SZ, _P]),
    "tg_decode_temperature_ratio": (_F, [_I64, _I64, _I64]),
    "tg_pruned_prefill_layer_varlen": (_INT, [ctypes.POINTER(LayerWeights), ctypes.POINTER(LayerShape), _P, _P, _P,
                                              _P, ctypes.POINTER(_I64), _I32, _P, _SZ, _P]),
    "tg_layer_varlen_workspace_bytes": (_SZ, [ctypes.POINTER(LayerShape), ctypes.POINTER(_I64), _I32]),
    "tg_linear": (_INT, [_P, _I64, _P, _P, _I64, _INT, _I64, _I32, _I32, _INT, _P]),
    "tg_workspace_bytes": (_SZ, [_INT, _I64, _I64, _I32, _I32, ctypes.POINTER(LayerShape)]),
    "tg_gate_score_noalloc": (_INT, [_P, _INT, _I64, _I32, _P, _F, _P, _P, _P, _F, _I32, _P, _P, _P, _P]),
    "tg_gate_score_noalloc_scratch_bytes": (_SZ, []),
    "tg_gate_score_select": (_INT, [_P, _INT, _I64, _I32, _P, _F, _P, _P, _P, _F, _I32, _P, _I64, _I64, _P, _P, _P,
                                     _I64, _P, _SZ, ctypes.c_uint32, _P]),
    "tg_debug_set_flag_wait": (_INT, [ctypes.c_uint64, ctypes.c_uint32]),
    "tg_gather_rmsnorm": (_INT, [_P, _INT, _I64, _I32, _P, _I64, _P, _P, _I64, _F, _P, _F, _P, _P, _P, _P, _P, _P]),
    "tg_layer_attention_block": (_INT, [ctypes.POINTER(LayerWeights), ctypes.POINTER(LayerShape), _P, _P, _P, _P,
                                        _I64, _P, _SZ, _P]),
    "tg_layer_mlp_block": (_INT, [ctypes.POINTER(LayerWeights), ctypes.POINTER(LayerShape), _P, _I64, _P, _SZ, _P]),
    "tg_gather_prefill_layer": (_INT, [ctypes.POINTER(LayerWeights), ctypes.POINTER(LayerShape), _INT, _P, _I64, _P,
                                       _I64, _P, _P, _I64, _F, _P, _P, _P, _P, _P, _SZ, _P]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libtokengate.so (built in-tree by learned_token_pruning_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise TokenGateError("load", 6, f"{LIB_PATH} is missing; run python -m learned_token_pruning_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise TokenGateError("marshal", 1, "tensor is not on a CUDA device")
    if not t.is_contiguous():
        raise TokenGateError("marshal", 1, "tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return TG_F32
    if t.dtype == torch.bfloat16:
        return TG_BF16
    raise TokenGateError("marshal", 1, f"unsupported dtype {t.dtype}")


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(name: str, rc: int):
    if rc != 0:
        raise TokenGateError(name, rc, lib().tg_last_error().decode())


def tg_version() -> str:
    return lib().tg_version().decode()


def tg_check_device_error(stream=None) -> int:
    """Synchronise the stream and return the (cleared) device error word; raise if it was set."""
    word = ctypes.c_uint32(0)
    rc = lib().tg_check_device_error(_stream(stream), ctypes.byref(word))
    _check("tg_check_device_error", rc)
    return word.value


def tg_debug_set_flag_wait(limit_ns: int = 0, merge_ready_target: int = 0):
    """Test hook: limit (ns) and target of the device's waits on flags set by other CTAs (0 = defaults)."""
    _check("tg_debug_set_flag_wait", lib().tg_debug_set_flag_wait(int(limit_ns), int(merge_ready_target)))


def tg_workspace_bytes(op: int, n: int = 0, m: int = 0, d_model: int = 0, h: int = 0,
                       shape: Optional[LayerShape] = None) -> int:
    return int(lib().tg_workspace_bytes(op, n, m, d_model, h, ctypes.byref(shape) if shape is not None else None))


def tg_gate_score(hidden, norm_w, norm_eps, w1, b1, w2, b2, prunable, scores, sumsq, ws, stream=None):
    n, d = hidden.shape
    h = w1.shape[0]
    rc = lib().tg_gate_score(_ptr(hidden), _dtype(hidden), n, d, _ptr(norm_w), float(norm_eps), _ptr(w1), _ptr(b1),
                             _ptr(w2), float(b2), h, _ptr(prunable), _ptr(scores), _ptr(sumsq), _ptr(ws),
                             ws.numel() * ws.element_size() if ws is not None else 0, _stream(stream))
    _check("tg_gate_score", rc)


def tg_gate_score_noalloc(hidden, norm_w, norm_eps, w1, b1, w2, b2, prunable, scores, sumsq, stream=None):
    """tg_gate_score for callers that cannot allocate: the scratch is the library's own fixed array."""
    n, d = hidden.shape
    h = w1.shape[0]
    rc = lib().tg_gate_score_noalloc(_ptr(hidden), _dtype(hidden), n, d, _ptr(norm_w), float(norm_eps), _ptr(w1),
                                     _ptr(b1), _ptr(w2), float(b2), h, _ptr(prunable), _ptr(scores), _ptr(sumsq),
                                     _stream(stream))
    _check("tg_gate_score_noalloc", rc)


def tg_gate_score_select(hidden, norm_w, norm_eps, w1, b1, w2, b2, prunable, n_prunable: int, k: int, scores, sumsq,
                         kept_idx, ws, stream=None, flags: int = 0):
    """tg_gate_score then tg_topk_select, the selector's first radix digit counted by the scoring kernel.
    flags=TG_WS_KEPT_ZERO: ws is zero-filled or as the previous such call left it (no memset is issued)."""
    n, d = hidden.shape
    h = w1.shape[0]
    rc = lib().tg_gate_score_select(_ptr(hidden), _dtype(hidden), n, d, _ptr(norm_w), float(norm_eps), _ptr(w1),
                                    _ptr(b1), _ptr(w2), float(b2), h, _ptr(prunable), int(n_prunable), int(k),
                                    _ptr(scores), _ptr(sumsq), _ptr(kept_idx), kept_idx.numel(), _ptr(ws),
                                    ws.numel() * ws.element_size(), int(flags), _stream(stream))
    _check("tg_gate_score_select", rc)


def tg_topk_select(scores, prunable, n_prunable: int, k: int, kept_idx, stream=None):
    rc = lib().tg_topk_select(_ptr(scores), _ptr(prunable), scores.numel(), int(n_prunable), int(k), _ptr(kept_idx),
                              kept_idx.numel(), _stream(stream))
    _check("tg_topk_select", rc)


def tg_gather(hidden, kept_idx, scores, sumsq, n_prunable: int, seq_eps: float, hidden_kept, pos=None, bias=None,
              ratio=None, stream=None):
    n, d = hidden.shape
    rc = lib().tg_gather(_ptr(hidden), _dtype(hidden), n, d, _ptr(kept_idx), kept_idx.numel(), _ptr(scores),
                         _ptr(sumsq), int(n_prunable), float(seq_eps), _ptr(hidden_kept), _ptr(pos), _ptr(bias),
                         _ptr(ratio), _stream(stream))
    _check("tg_gather", rc)


def tg_gather_rmsnorm(hidden, kept_idx, scores, sumsq, n_prunable: int, seq_eps: float, norm_w, norm_eps: float,
                      hidden_kept, x_norm, pos=None, bias=None, ratio=None, stream=None):
    """tg_gather plus x_norm = RMSNorm(hidden_kept) * norm_w in the same pass."""
    n, d = hidden.shape
    rc = lib().tg_gather_rmsnorm(_ptr(hidden), _dtype(hidden), n, d, _ptr(kept_idx), kept_idx.numel(), _ptr(scores),
                                 _ptr(sumsq), int(n_prunable), float(seq_eps), _ptr(norm_w), float(norm_eps),
                                 _ptr(hidden_kept), _ptr(x_norm), _ptr(pos), _ptr(bias), _ptr(ratio), _stream(stream))
    _check("tg_gather_rmsnorm", rc)


def _row_view(t: torch.Tensor):
    """(pointer, leading dimension) of a 2-D view whose rows may be strided."""
    if t.dim() != 2 or t.stride(1) != 1:
        raise TokenGateError("marshal", 1, "expected a 2-D view with unit inner stride")
    if not t.is_cuda:
        raise TokenGateError("marshal", 1, "tensor is not on a CUDA device")
    return ctypes.c_void_p(t.data_ptr()), t.stride(0)


def attention_workspace_bytes(m: int, hq: int, hkv: int, head_dim: int, dtype: torch.dtype) -> int:
    """Workspace bytes tg_gated_attention uses on the current device (0: none needed)."""
    shape = LayerShape(dtype=TG_BF16 if dtype == torch.bfloat16 else TG_F32, hq=hq, hkv=hkv, head_dim=head_dim)
    return tg_workspace_bytes(TG_OP_ATTENTION, m=m, shape=shape)


def tg_gated_attention(q, k, v, head_dim: int, bias, head_gain, head_temp, ratio, sm_scale: float, out, lse=None,
                       ws=None, stream=None):
    """q/k/v/out are 2-D row views [m, heads*head_dim] (rows may be strided); ws is a device
    byte buffer of attention_workspace_bytes(...) bytes or None (no key-range split)."""
    qp, ldq = _row_view(q)
    kp, ldk = _row_view(k)
    vp, ldv = _row_view(v)
    op, ldo = _row_view(out)
    m = q.shape[0]
    hq = q.shape[1] // head_dim
    hkv = k.shape[1] // head_dim
    rc = lib().tg_gated_attention(qp, ldq, kp, ldk, vp, ldv, _dtype(q), m, hq, hkv, head_dim, _ptr(bias),
                                  _ptr(head_gain), _ptr(head_temp), _ptr(ratio), float(sm_scale), op, ldo, _ptr(lse),
                                  _ptr(ws), ws.numel() * ws.element_size() if ws is not None else 0,
                                  _stream(stream))
    _check("tg_gated_attention", rc)


def attention_backward_workspace_bytes(m: int, hq: int, hkv: int, head_dim: int) -> int:
    shape = LayerShape(dtype=TG_BF16, d_model=0, hq=hq, hkv=hkv, head_dim=head_dim, d_ff=0, qk_norm=0,
                       rope_theta=0.0, norm_eps=0.0)
    return tg_workspace_bytes(TG_OP_ATTENTION_BWD, m=m, shape=shape)


def tg_gated_attention_backward(q, k, v, out, dout, head_dim: int, bias, head_gain, head_temp, ratio,
                                sm_scale: float, lse, dq, dk, dv, ws, dbias=None, dgain=None, dtemp=None,
                                stream=None):
    """q/k/v/out/dout 2-D row views as in tg_gated_attention; dq/dk/dv fp32 [m, heads*head_dim]."""
    qp, ldq = _row_view(q)
    kp, ldk = _row_view(k)
    vp, ldv = _row_view(v)
    op, ldo = _row_view(out)
    gp, lddo = _row_view(dout)
    m = q.shape[0]
    hq = q.shape[1] // head_dim
    hkv = k.shape[1] // head_dim
    rc = lib().tg_gated_attention_backward(qp, ldq, kp, ldk, vp, ldv, op, ldo, gp, lddo, _dtype(q), m, hq, hkv,
                                           head_dim, _ptr(bias), _ptr(head_gain), _ptr(head_temp), _ptr(ratio),
                                           float(sm_scale), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dbias),
                                           _ptr(dgain), _ptr(dtemp), _ptr(ws), ws.numel() * ws.element_size(),
                                           _stream(stream))
    _check("tg_gated_attention_backward", rc)


def decode_workspace_bytes(length: int, hq: int, hkv: int, head_dim: int) -> int:
    shape = LayerShape(dtype=TG_BF16, d_model=0, hq=hq, hkv=hkv, head_dim=head_dim, d_ff=0, qk_norm=0,
                       rope_theta=0.0, norm_eps=0.0)
    return tg_workspace_bytes(TG_OP_DECODE, m=length, shape=shape)


def tg_decode_temperature_ratio(m_kept: int, n_prompt: int, t: int) -> float:
    return float(lib().tg_decode_temperature_ratio(int(m_kept), int(n_prompt), int(t)))


def tg_gated_decode_attention(q, k, v, head_dim: int, bias, head_gain, head_temp, ratio: float, sm_scale: float, out,
                              ws, lse=None, stream=None):
    """q/out [hq, head_dim] (contiguous); k/v the cache as 2-D row views [length, hkv*head_dim]
    (rows may be strided); ws a device byte buffer of decode_workspace_bytes(...) bytes."""
    kp, ldk = _row_view(k)
    vp, ldv = _row_view(v)
    hq = q.numel() // head_dim
    hkv = k.shape[1] // head_dim
    rc = lib().tg_gated_decode_attention(_ptr(q), kp, ldk, vp, ldv, _dtype(q), k.shape[0], hq, hkv, head_dim,
                                         _ptr(bias), _ptr(head_gain), _ptr(head_temp), float(ratio), float(sm_scale),
                                         _ptr(out), _ptr(lse), _ptr(ws),
                                         ws.numel() * ws.element_size() if ws is not None else 0, _stream(stream))
    _check("tg_gated_decode_attention", rc)


TG_EPI_STORE, TG_EPI_RESIDUAL, TG_EPI_SWIGLU = 0, 1, 2


def tg_linear(x, w, y, epilogue: int = TG_EPI_STORE, stream=None):
    """y = x W^T, y += x W^T (TG_EPI_RESIDUAL) or y = SiLU(x Wg^T) * (x Wu^T) (TG_EPI_SWIGLU)."""
    xp, ldx = _row_view(x)
    yp, ldy = _row_view(y)
    n_out = w.shape[0] // 2 if epilogue == TG_EPI_SWIGLU else w.shape[0]
    rc = lib().tg_linear(xp, ldx, _ptr(w), yp, ldy, _dtype(x), x.shape[0], n_out, w.shape[1], int(epilogue),
                         _stream(stream))
    _check("tg_linear", rc)


def layer_structs(weights: dict, *, dtype: torch.dtype, d_model: int, hq: int, hkv: int, head_dim: int, d_ff: int,
                  qk_norm: bool, rope_theta: float, norm_eps: float = 1e-6):
    """ctypes structs for tg_pruned_prefill_layer from a dict of device tensors."""
    W = LayerWeights(*[_ptr(weights.get(f[0])) if weights.get(f[0]) is not None else None for f in LayerWeights._fields_])
    S = LayerShape(TG_BF16 if dtype == torch.bfloat16 else TG_F32, d_model, hq, hkv, head_dim, d_ff,
                   1 if qk_norm else 0, float(rope_theta), float(norm_eps))
    return W, S


def tg_pruned_prefill_layer(W: LayerWeights, S: LayerShape, hidden_kept, pos, bias, ratio, ws, stream=None):
    m = hidden_kept.shape[0]
    rc = lib().tg_pruned_prefill_layer(ctypes.byref(W), ctypes.byref(S), _ptr(hidden_kept), _ptr(pos), _ptr(bias),
                                       _ptr(ratio), m, _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check("tg_pruned_prefill_layer", rc)


def tg_layer_attention_block(W: LayerWeights, S: LayerShape, hidden, pos, bias, ratio, ws, stream=None):
    """hidden += Attn(RMSNorm(hidden)) Wo^T: the post-attention residual, in place."""
    rc = lib().tg_layer_attention_block(ctypes.byref(W), ctypes.byref(S), _ptr(hidden), _ptr(pos), _ptr(bias),
                                        _ptr(ratio), hidden.shape[0], _ptr(ws), ws.numel() * ws.element_size(),
                                        _stream(stream))
    _check("tg_layer_attention_block", rc)


def tg_layer_mlp_block(W: LayerWeights, S: LayerShape, hidden, ws, stream=None):
    """hidden += SwiGLU MLP of RMSNorm(hidden), in place."""
    rc = lib().tg_layer_mlp_block(ctypes.byref(W), ctypes.byref(S), _ptr(hidden), hidden.shape[0], _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream))
    _check("tg_layer_mlp_block", rc)


def tg_gather_prefill_layer(W: LayerWeights, S: LayerShape, part: int, hidden, kept_idx, scores, sumsq,
                            n_prunable: int, seq_eps: float, hidden_kept, pos, bias, ratio, ws, stream=None):
    """tg_gather into hidden_kept / pos / bias / ratio fused with the first RMSNorm of a layer part
    (TG_LAYER_FULL or TG_LAYER_MLP), which then runs on the kept rows."""
    n = hidden.shape[0]
    rc = lib().tg_gather_prefill_layer(ctypes.byref(W), ctypes.byref(S), int(part), _ptr(hidden), n, _ptr(kept_idx),
                                       kept_idx.numel(), _ptr(scores), _ptr(sumsq), int(n_prunable), float(seq_eps),
                                       _ptr(hidden_kept), _ptr(pos), _ptr(bias), _ptr(ratio), _ptr(ws),
                                       ws.numel() * ws.element_size(), _stream(stream))
    _check("tg_gather_prefill_layer", rc)


def _seg_array(seg_rows):
    arr = (_I64 * len(seg_rows))(*[int(x) for x in seg_rows])
    return arr, len(seg_rows) - 1


def tg_layer_varlen_workspace_bytes(S: LayerShape, seg_rows) -> int:
    arr, nseg = _seg_array(seg_rows)
    return int(lib().tg_layer_varlen_workspace_bytes(ctypes.byref(S), arr, nseg))


def tg_pruned_prefill_layer_varlen(W: LayerWeights, S: LayerShape, hidden_kept, pos, bias, ratio, seg_rows, ws,
                                   stream=None):
    """seg_rows: host sequence of nseg + 1 row offsets (0, m_0, m_0 + m_1, ...)."""
    arr, nseg = _seg_array(seg_rows)
    rc = lib().tg_pruned_prefill_layer_varlen(ctypes.byref(W), ctypes.byref(S), _ptr(hidden_kept), _ptr(pos),
                                              _ptr(bias), _ptr(ratio), arr, nseg, _ptr(ws),
                                              ws.numel() * ws.element_size(), _stream(stream))
    _check("tg_pruned_prefill_layer_varlen", rc)
