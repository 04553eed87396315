"""Python binding of libsage.so: SageAttention-style quantized attention on B200.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/sage.h.  PyTorch supplies device
memory and the current stream.  There is no fallback: if the library is not
built, or the GPU is not a B200, the calls raise.

Functions carry the names of the C entry points:
  sage_smooth_quant_qk, sage_smooth_quant_qk_noalloc, sage_quant_v_fp8,
  sage_smooth_quant_qkv, sage_smooth_quant_qkv_rope,
  sage_attn_fwd_quantized,
  sage_attn_fwd, sage_attn_fwd_ws, sage_attn_workspace_bytes,
  sage_attn_fwd_host, sage_smooth_quant_qkv_varlen, sage_attn_fwd_varlen_quantized,
  sage_attn_fwd_varlen, sage_get_device_error, sage_set_wait_timeout_ns,
  sage_selftest_wait_timeout, sage_status_string, sage_version,
  sage_v_hat_layout.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsage.so")

SAGE_OK = 0
SAGE_ERR_DEVICE_TIMEOUT = 6
VARIANTS = {"B": 0, "8+8": 1, "8+8-r56": 2}

_c = ctypes
_vp = _c.c_void_p
_i = _c.c_int
_f = _c.c_float

_SIGS = {
    "sage_smooth_quant_qk": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _f, _vp, _vp, _vp, _vp, _vp, _vp]),
    "sage_smooth_quant_qk_noalloc": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _f, _vp, _vp, _vp, _vp, _vp,
                                          _vp]),
    "sage_quant_v_fp8": (_i, [_vp, _i, _i, _i, _i, _f, _vp, _vp, _vp]),
    "sage_smooth_quant_qkv": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _f, _vp, _vp, _vp, _vp,
                                   _vp, _vp, _vp, _vp]),
    "sage_smooth_quant_qkv_rope": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _f, _vp,
                                        _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "sage_attn_fwd_quantized": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]),
    "sage_attn_workspace_bytes": (_c.c_size_t, [_i, _i, _i, _i, _i, _i]),
    "sage_attn_fwd": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp]),
    "sage_attn_fwd_ws": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp, _c.c_size_t, _vp]),
    "sage_attn_fwd_host": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp]),
    "sage_smooth_quant_qkv_varlen": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _f, _vp,
                                          _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "sage_attn_fwd_varlen_quantized": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                            _i, _i, _i, _i, _vp]),
    "sage_attn_fwd_varlen": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _i,
                                  _vp]),
    "sage_v_hat_layout": (_i, []),
    "sage_get_device_error": (_i, [_vp, _c.POINTER(_c.c_uint32)]),
    "sage_set_wait_timeout_ns": (None, [_c.c_uint64]),
    "sage_selftest_wait_timeout": (_i, [_c.c_uint64, _vp]),
    "sage_status_string": (_c.c_char_p, [_i]),
    "sage_version": (_c.c_char_p, []),
    "sage_last_error_detail": (_c.c_char_p, []),
}

_lib_handle = None


def load_library() -> ctypes.CDLL:
    """Load libsage.so (raises if it has not been built)."""
    global _lib_handle
    if _lib_handle is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build the CUDA library first "
                "(python -m quantized_attention_08_b200.build)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib_handle = lib
    return _lib_handle


class SageError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {sage_status_string(status)} (status {status}); "
                         f"last failing step: {sage_last_error_detail()}")


def sage_last_error_detail() -> str:
    return load_library().sage_last_error_detail().decode()


def sage_status_string(status: int) -> str:
    return load_library().sage_status_string(int(status)).decode()


def sage_version() -> str:
    return load_library().sage_version().decode()


def sage_v_hat_layout() -> int:
    return load_library().sage_v_hat_layout()


def _check(status: int, where: str):
    if status != SAGE_OK:
        raise SageError(status, where)


def _stream(stream=None) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, dtype, name: str, cuda: bool = True):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if cuda and not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _variant(v) -> int:
    return VARIANTS[v] if isinstance(v, str) else int(v)


def _nb(N: int) -> int:
    return (N + 127) // 128


def sage_smooth_quant_qk(q: torch.Tensor, k: torch.Tensor, sm_scale: Optional[float] = None,
                         out=None, stream=None):
    """Smooth K, quantize Q*sm_scale and smoothed K per 128-token block.
    Returns (q_hat int8, k_hat int8, delta_q fp32, delta_k fp32, mean_k fp32)."""
    _need(q, torch.float16, "q")
    _need(k, torch.float16, "k")
    B, H, N, d = q.shape
    Hk = k.shape[1]
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if out is None:
        dev = q.device
        out = (torch.empty_like(q, dtype=torch.int8), torch.empty_like(k, dtype=torch.int8),
               torch.empty(B, H, _nb(N), dtype=torch.float32, device=dev),
               torch.empty(B, Hk, _nb(N), dtype=torch.float32, device=dev),
               torch.empty(B, Hk, d, dtype=torch.float32, device=dev))
    qh, kh, dq, dk, mk = out
    st = load_library().sage_smooth_quant_qk(_ptr(q), _ptr(k), B, H, Hk, N, d, float(sm_scale),
                                             _ptr(qh), _ptr(kh), _ptr(dq), _ptr(dk), _ptr(mk),
                                             _stream(stream))
    _check(st, "sage_smooth_quant_qk")
    return out


def sage_smooth_quant_qk_noalloc(q: torch.Tensor, k: torch.Tensor, out,
                                 sm_scale: Optional[float] = None, stream=None):
    """sage_smooth_quant_qk with no device allocation inside the call: the
    caller passes the five output tensors `out` = (q_hat, k_hat, delta_q,
    delta_k, mean_k) and the library uses its static 4 MiB scratch (sizes
    with B*H_kv*ceil(N/256)*d > 524288 raise).  Calls that may overlap on
    one device race on that scratch; see include/sage.h."""
    _need(q, torch.float16, "q")
    _need(k, torch.float16, "k")
    B, H, N, d = q.shape
    Hk = k.shape[1]
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    qh, kh, dq, dk, mk = out
    st = load_library().sage_smooth_quant_qk_noalloc(
        _ptr(q), _ptr(k), B, H, Hk, N, d, float(sm_scale), _ptr(qh), _ptr(kh), _ptr(dq),
        _ptr(dk), _ptr(mk), _stream(stream))
    _check(st, "sage_smooth_quant_qk_noalloc")
    return out


def sage_quant_v_fp8(v: torch.Tensor, v_r: float = 448.0, out=None, stream=None):
    """E4M3 codes of V / delta_v with delta_v = colmax|V| / v_r per channel.
    Returns (v_hat uint8 [B,Hkv,N,d], delta_v fp32 [B,Hkv,d])."""
    _need(v, torch.float16, "v")
    B, Hk, N, d = v.shape
    if out is None:
        out = (torch.empty_like(v, dtype=torch.uint8),
               torch.empty(B, Hk, d, dtype=torch.float32, device=v.device))
    vh, dv = out
    st = load_library().sage_quant_v_fp8(_ptr(v), B, Hk, N, d, float(v_r), _ptr(vh), _ptr(dv),
                                         _stream(stream))
    _check(st, "sage_quant_v_fp8")
    return out


def sage_smooth_quant_qkv(q, k, v=None, sm_scale: Optional[float] = None, v_r: float = 448.0,
                          out=None, stream=None):
    """Whole pre-pass in three launches.  Returns (q_hat, k_hat, delta_q,
    delta_k, mean_k, v_hat, delta_v); the last two are None when v is None."""
    _need(q, torch.float16, "q")
    _need(k, torch.float16, "k")
    if v is not None:
        _need(v, torch.float16, "v")
    B, H, N, d = q.shape
    Hk = k.shape[1]
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if out is None:
        dev = q.device
        out = (torch.empty_like(q, dtype=torch.int8), torch.empty_like(k, dtype=torch.int8),
               torch.empty(B, H, _nb(N), dtype=torch.float32, device=dev),
               torch.empty(B, Hk, _nb(N), dtype=torch.float32, device=dev),
               torch.empty(B, Hk, d, dtype=torch.float32, device=dev),
               None if v is None else torch.empty_like(v, dtype=torch.uint8),
               None if v is None else torch.empty(B, Hk, d, dtype=torch.float32, device=dev))
    qh, kh, dq, dk, mk, vh, dv = out
    st = load_library().sage_smooth_quant_qkv(
        _ptr(q), _ptr(k), _ptr(v), B, H, Hk, N, d, float(sm_scale), float(v_r), _ptr(qh),
        _ptr(kh), _ptr(vh), _ptr(dq), _ptr(dk), _ptr(mk), _ptr(dv), _stream(stream))
    _check(st, "sage_smooth_quant_qkv")
    return out


def sage_smooth_quant_qkv_rope(q, k, cos_t, sin_t, v=None, sm_scale: Optional[float] = None,
                               v_r: float = 448.0, out=None, stream=None):
    """sage_smooth_quant_qkv with rotary embedding of Q and K fused in front
    of the quantizers; cos_t / sin_t are fp32 CUDA tensors [N, d/2].  Same
    outputs as sage_smooth_quant_qkv."""
    _need(q, torch.float16, "q")
    _need(k, torch.float16, "k")
    _need(cos_t, torch.float32, "cos_t")
    _need(sin_t, torch.float32, "sin_t")
    if v is not None:
        _need(v, torch.float16, "v")
    B, H, N, d = q.shape
    Hk = k.shape[1]
    if tuple(cos_t.shape) != (N, d // 2) or tuple(sin_t.shape) != (N, d // 2):
        raise ValueError(f"rotary tables must be [N, d/2] = [{N}, {d // 2}]")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if out is None:
        dev = q.device
        out = (torch.empty_like(q, dtype=torch.int8), torch.empty_like(k, dtype=torch.int8),
               torch.empty(B, H, _nb(N), dtype=torch.float32, device=dev),
               torch.empty(B, Hk, _nb(N), dtype=torch.float32, device=dev),
               torch.empty(B, Hk, d, dtype=torch.float32, device=dev),
               None if v is None else torch.empty_like(v, dtype=torch.uint8),
               None if v is None else torch.empty(B, Hk, d, dtype=torch.float32, device=dev))
    qh, kh, dq, dk, mk, vh, dv = out
    st = load_library().sage_smooth_quant_qkv_rope(
        _ptr(q), _ptr(k), _ptr(v), _ptr(cos_t), _ptr(sin_t), B, H, Hk, N, d, float(sm_scale),
        float(v_r), _ptr(qh), _ptr(kh), _ptr(vh), _ptr(dq), _ptr(dk), _ptr(mk), _ptr(dv),
        _stream(stream))
    _check(st, "sage_smooth_quant_qkv_rope")
    return out


def sage_attn_fwd_quantized(q_hat, k_hat, delta_q, delta_k, v_or_vhat, delta_v=None, *,
                            causal: bool = False, variant="B", o=None, stream=None):
    """Attention on pre-quantized operands; returns o fp16 [B,H,N,d]."""
    _need(q_hat, torch.int8, "q_hat")
    _need(k_hat, torch.int8, "k_hat")
    var = _variant(variant)
    B, H, N, d = q_hat.shape
    Hk = k_hat.shape[1]
    if o is None:
        o = torch.empty(B, H, N, d, dtype=torch.float16, device=q_hat.device)
    st = load_library().sage_attn_fwd_quantized(
        _ptr(q_hat), _ptr(k_hat), _ptr(delta_q), _ptr(delta_k), _ptr(v_or_vhat), _ptr(delta_v),
        _ptr(o), B, H, Hk, N, d, int(bool(causal)), var, _stream(stream))
    _check(st, "sage_attn_fwd_quantized")
    return o


def sage_attn_workspace_bytes(B: int, H: int, H_kv: int, N: int, d: int, variant="B") -> int:
    return load_library().sage_attn_workspace_bytes(B, H, H_kv, N, d, _variant(variant))


def sage_attn_fwd(q, k, v, *, causal: bool = False, sm_scale: Optional[float] = None,
                  variant="B", o=None, workspace: Optional[torch.Tensor] = None, stream=None):
    """Whole SageAttention forward (Smooth K, quantize, attention); returns o fp16."""
    _need(q, torch.float16, "q")
    _need(k, torch.float16, "k")
    _need(v, torch.float16, "v")
    B, H, N, d = q.shape
    Hk = k.shape[1]
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if o is None:
        o = torch.empty_like(q)
    lib = load_library()
    if workspace is None:
        st = lib.sage_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, Hk, N, d, int(bool(causal)),
                               float(sm_scale), _variant(variant), _stream(stream))
        _check(st, "sage_attn_fwd")
    else:
        st = lib.sage_attn_fwd_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, Hk, N, d,
                                  int(bool(causal)), float(sm_scale), _variant(variant),
                                  _ptr(workspace), workspace.numel() * workspace.element_size(),
                                  _stream(stream))
        _check(st, "sage_attn_fwd_ws")
    return o


def sage_attn_fwd_ws(q, k, v, workspace: torch.Tensor, *, causal: bool = False,
                     sm_scale: Optional[float] = None, variant="B", o=None, stream=None):
    """sage_attn_fwd with the intermediates carved from a caller workspace
    (a CUDA tensor of at least sage_attn_workspace_bytes() bytes)."""
    if workspace is None:
        raise ValueError("workspace is required")
    return sage_attn_fwd(q, k, v, causal=causal, sm_scale=sm_scale, variant=variant, o=o,
                         workspace=workspace, stream=stream)


def sage_attn_fwd_host(q_host, k_host, v_host, o_host, *, causal: bool = False,
                       sm_scale: Optional[float] = None, variant="B", stream=None):
    """End-to-end call on host (CPU, ideally pinned) fp16 tensors; o_host is written."""
    for t, n in ((q_host, "q_host"), (k_host, "k_host"), (v_host, "v_host"), (o_host, "o_host")):
        _need(t, torch.float16, n, cuda=False)
        if t.is_cuda:
            raise TypeError(f"{n} must be a host tensor")
    B, H, N, d = q_host.shape
    Hk = k_host.shape[1]
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    st = load_library().sage_attn_fwd_host(_ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(o_host),
                                           B, H, Hk, N, d, int(bool(causal)), float(sm_scale),
                                           _variant(variant), _stream(stream))
    _check(st, "sage_attn_fwd_host")
    return o_host


def _varlen_shape(q, k, cu_seqlens, max_seqlen):
    _need(cu_seqlens, torch.int32, "cu_seqlens")
    H, T, d = q.shape
    Hk = k.shape[0]
    B = cu_seqlens.numel() - 1
    return B, H, Hk, T, d, int(max_seqlen)


def sage_smooth_quant_qkv_varlen(q, k, cu_seqlens, max_seqlen: int, v=None,
                                 sm_scale: Optional[float] = None, v_r: float = 448.0, stream=None):
    """Pre-pass of a packed batch (q [H,T,d], k/v [H_kv,T,d], cu_seqlens int32
    [B+1] on the device).  Returns (q_hat, k_hat, delta_q [B,H,nbm],
    delta_k [B,H_kv,nbm], mean_k [B,H_kv,d], v_hat, delta_v)."""
    _need(q, torch.float16, "q")
    _need(k, torch.float16, "k")
    B, H, Hk, T, d, ms = _varlen_shape(q, k, cu_seqlens, max_seqlen)
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    dev = q.device
    nbm = _nb(ms)
    qh, kh = torch.empty_like(q, dtype=torch.int8), torch.empty_like(k, dtype=torch.int8)
    dq = torch.zeros(B, H, nbm, dtype=torch.float32, device=dev)
    dk = torch.zeros(B, Hk, nbm, dtype=torch.float32, device=dev)
    mk = torch.empty(B, Hk, d, dtype=torch.float32, device=dev)
    vh = None if v is None else torch.empty_like(v, dtype=torch.uint8)
    dv = None if v is None else torch.empty(B, Hk, d, dtype=torch.float32, device=dev)
    st = load_library().sage_smooth_quant_qkv_varlen(
        _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), B, ms, T, H, Hk, d, float(sm_scale),
        float(v_r), _ptr(qh), _ptr(kh), _ptr(vh), _ptr(dq), _ptr(dk), _ptr(mk), _ptr(dv),
        _stream(stream))
    _check(st, "sage_smooth_quant_qkv_varlen")
    return qh, kh, dq, dk, mk, vh, dv


def sage_attn_fwd_varlen_quantized(q_hat, k_hat, delta_q, delta_k, v_or_vhat, delta_v,
                                   cu_seqlens, max_seqlen: int, *, causal: bool = False,
                                   variant="B", o=None, stream=None):
    """Attention of a packed batch on pre-quantized operands; returns o
    fp16 [H,T,d]."""
    _need(q_hat, torch.int8, "q_hat")
    _need(k_hat, torch.int8, "k_hat")
    var = _variant(variant)
    B, H, Hk, T, d, ms = _varlen_shape(q_hat, k_hat, cu_seqlens, max_seqlen)
    if o is None:
        o = torch.empty(H, T, d, dtype=torch.float16, device=q_hat.device)
    st = load_library().sage_attn_fwd_varlen_quantized(
        _ptr(q_hat), _ptr(k_hat), _ptr(delta_q), _ptr(delta_k), _ptr(v_or_vhat), _ptr(delta_v),
        _ptr(o), _ptr(cu_seqlens), B, ms, T, H, Hk, d, int(bool(causal)), var, _stream(stream))
    _check(st, "sage_attn_fwd_varlen_quantized")
    return o


def sage_attn_fwd_varlen(q, k, v, cu_seqlens, max_seqlen: int, *, causal: bool = False,
                         sm_scale: Optional[float] = None, variant="B", o=None, stream=None):
    """Whole forward pass of a packed batch: q [H,T,d], k/v [H_kv,T,d] fp16,
    cu_seqlens int32 [B+1] on the device; returns o fp16 [H,T,d]."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.float16, n)
    B, H, Hk, T, d, ms = _varlen_shape(q, k, cu_seqlens, max_seqlen)
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if o is None:
        o = torch.empty_like(q)
    st = load_library().sage_attn_fwd_varlen(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(cu_seqlens), B, ms, T, H, Hk, d,
        int(bool(causal)), float(sm_scale), _variant(variant), _stream(stream))
    _check(st, "sage_attn_fwd_varlen")
    return o


def sage_get_device_error(stream=None):
    """(status, raw error word); synchronizes the stream and clears the word."""
    w = ctypes.c_uint32(0)
    st = load_library().sage_get_device_error(_stream(stream), ctypes.byref(w))
    return st, w.value


def sage_set_wait_timeout_ns(ns: int):
    load_library().sage_set_wait_timeout_ns(int(ns))


def sage_selftest_wait_timeout(timeout_ns: int, stream=None):
    _check(load_library().sage_selftest_wait_timeout(int(timeout_ns), _stream(stream)),
           "sage_selftest_wait_timeout")
