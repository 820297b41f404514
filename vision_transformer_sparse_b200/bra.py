"""ctypes binding of the C-ABI library `libbra.so` (declared in include/bra.h).

Argument marshalling only: shapes are read from the tensors, outputs are
allocated with torch when not given, and the call goes straight to the C entry
point of the same name on the current torch CUDA stream. Every step of the
computation runs in the library's CUDA kernels; there is no fallback. If the
library is missing this module raises at first use.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libbra.so")
_lib = None

BRA_F32, BRA_BF16 = 0, 1
STATUS = {0: "BRA_OK", 1: "BRA_ERR_NULL", 2: "BRA_ERR_SHAPE", 3: "BRA_ERR_ALIGN", 4: "BRA_ERR_DTYPE",
          5: "BRA_ERR_CUDA", 6: "BRA_ERR_INDEX", 7: "BRA_ERR_SCRATCH", 8: "BRA_ERR_TIMEOUT"}
VARIANT_AUTO, VARIANT_GENERIC, VARIANT_TMA, VARIANT_SPLIT, VARIANT_PIPE = 0, 1, 2, 3, 4
STATIC_SCRATCH_FLOATS = 4 * 1024 * 1024
# entry points declared in include/bra.h
SYMBOLS = ("bra_forward", "bra_route", "bra_attend", "bra_forward_host", "bra_forward_noalloc",
           "bra_status_string",
           "bra_version", "bra_launch_count", "bra_trace_begin", "bra_trace_end", "bra_kernel_name",
           "bra_set_kernel_variant", "bra_device_status", "bra_selftest_wait_timeout", "bra_trace_read",
           "bra_linear", "bra_qkv", "bra_attention_layer", "bra_backward", "bra_linear_act", "bra_block", "bra_backward_async")
ACT_NONE, ACT_GELU, ACT_RESIDUAL = 0, 1, 2
KERNEL_CLASSES = 11


class BraError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s (%s)" % (where, STATUS.get(status, status), status_string(status)))


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError("libbra.so is not built (%s); run "
                               "`python -m vision_transformer_sparse_b200.build`" % _LIB_PATH)
        L = ctypes.CDLL(_LIB_PATH)
        vp, i = ctypes.c_void_p, ctypes.c_int
        shape = [i] * 8  # N, H, W, C, heads, S, topk, dtype
        L.bra_forward.argtypes = [vp] * 5 + shape + [vp, vp, vp, vp]
        L.bra_route.argtypes = [vp] * 2 + shape + [vp, vp, vp]
        L.bra_attend.argtypes = [vp] * 5 + shape + [vp, vp, vp]
        L.bra_forward_host.argtypes = [vp] * 5 + shape + [vp, vp, vp, vp]
        L.bra_forward_noalloc.argtypes = [vp] * 5 + shape + [vp, vp, vp, vp]
        L.bra_linear.argtypes = [vp] * 3 + [i] * 4 + [vp, vp]
        L.bra_qkv.argtypes = [vp] * 3 + [i] * 3 + [vp] * 4
        L.bra_attention_layer.argtypes = [vp] * 7 + shape + [vp, vp, vp, vp]
        L.bra_backward.argtypes = [vp] * 6 + shape + [vp] * 6
        L.bra_backward_async.argtypes = [vp] * 6 + shape + [vp] * 6
        L.bra_linear_act.argtypes = [vp] * 4 + [i] * 5 + [vp, vp]
        L.bra_block.argtypes = [vp] * 17 + shape + [vp, vp, vp, vp]
        for f in ("bra_forward", "bra_route", "bra_attend", "bra_forward_host", "bra_forward_noalloc",
                  "bra_version", "bra_linear", "bra_qkv", "bra_attention_layer", "bra_backward",
                  "bra_linear_act", "bra_block", "bra_backward_async"):
            getattr(L, f).restype = i
        L.bra_status_string.argtypes = [i]
        L.bra_status_string.restype = ctypes.c_char_p
        L.bra_launch_count.restype = ctypes.c_longlong
        L.bra_trace_begin.restype = i
        L.bra_trace_end.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong)]
        L.bra_trace_end.restype = i
        L.bra_trace_read.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong)]
        L.bra_trace_read.restype = i
        L.bra_kernel_name.argtypes = [i]
        L.bra_kernel_name.restype = ctypes.c_char_p
        L.bra_set_kernel_variant.argtypes = [i]
        L.bra_set_kernel_variant.restype = i
        L.bra_device_status.argtypes = [vp]
        L.bra_device_status.restype = i
        L.bra_selftest_wait_timeout.argtypes = [ctypes.c_uint, vp]
        L.bra_selftest_wait_timeout.restype = i
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().bra_status_string(int(status)).decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BRA_BF16
    if t.dtype == torch.float32:
        return BRA_F32
    raise TypeError("BRA takes bfloat16 or float32 tensors, got %s" % t.dtype)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check_dev(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("BRA tensors must be contiguous CUDA tensors")


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _raise(rc: int, where: str):
    if rc != 0:
        raise BraError(rc, where)


def forward(q, k, v, lce_w, lce_b, heads: int, S: int, topk: int, out=None, r_idx=None, r_weight=None,
            stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """bra_forward: (N,H,W,C) q, k, v; lce_w (C,5,5); lce_b (C) -> out, r_idx, r_weight."""
    N, H, W, C = q.shape
    P = S * S
    out = torch.empty_like(q) if out is None else out
    r_idx = torch.empty((N, P, topk), dtype=torch.int32, device=q.device) if r_idx is None else r_idx
    r_weight = torch.empty((N, P, topk), dtype=torch.float32, device=q.device) if r_weight is None else r_weight
    _check_dev(q, k, v, lce_w, lce_b, out, r_idx, r_weight)
    rc = lib().bra_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(lce_w), _ptr(lce_b), N, H, W, C, heads, S, topk,
                           _dtype_code(q), _ptr(out), _ptr(r_idx), _ptr(r_weight), _stream(stream))
    _raise(rc, "bra_forward")
    return out, r_idx, r_weight


def linear(x, w, b, out=None, stream=None) -> torch.Tensor:
    """bra_linear: x (..., K) rows, w (Nout, K), b (Nout) -> x w^T + b, shape (..., Nout)."""
    K = x.shape[-1]
    Nout = w.shape[0]
    M = x.numel() // K if K else 0
    out = torch.empty(x.shape[:-1] + (Nout,), dtype=x.dtype, device=x.device) if out is None else out
    _check_dev(x, w, b, out)
    rc = lib().bra_linear(_ptr(x), _ptr(w), _ptr(b), M, K, Nout, _dtype_code(x), _ptr(out), _stream(stream))
    _raise(rc, "bra_linear")
    return out


def linear_act(x, w, b, act: int, res=None, out=None, stream=None) -> torch.Tensor:
    """bra_linear_act: act(x w^T + b) for act ACT_NONE / ACT_GELU, or res + (x w^T + b) for
    ACT_RESIDUAL (res of the output's shape)."""
    K = x.shape[-1]
    Nout = w.shape[0]
    M = x.numel() // K if K else 0
    out = torch.empty(x.shape[:-1] + (Nout,), dtype=x.dtype, device=x.device) if out is None else out
    _check_dev(*(t for t in (x, w, b, res, out) if t is not None))
    rc = lib().bra_linear_act(_ptr(x), _ptr(w), _ptr(b), _ptr(res) if res is not None else None, M, K, Nout, act,
                              _dtype_code(x), _ptr(out), _stream(stream))
    _raise(rc, "bra_linear_act")
    return out


BLOCK_PARAMS = ("pos_w", "pos_b", "ln1_g", "ln1_b", "w_qkv", "b_qkv", "w_o", "b_o", "lce_w", "lce_b", "ln2_g",
                "ln2_b", "mlp_w1", "mlp_b1", "mlp_w2", "mlp_b2")


def block(x, p: dict, heads: int, S: int, topk: int, out=None, r_idx=None, r_weight=None, stream=None):
    """bra_block: one BiFormer block (pos-embed, norm1, attention layer, norm2, MLP, residuals)
    on x (N,H,W,C); p maps BLOCK_PARAMS names to device tensors."""
    N, H, W, C = x.shape
    P = S * S
    out = torch.empty_like(x) if out is None else out
    r_idx = torch.empty((N, P, topk), dtype=torch.int32, device=x.device) if r_idx is None else r_idx
    r_weight = torch.empty((N, P, topk), dtype=torch.float32, device=x.device) if r_weight is None else r_weight
    _check_dev(x, *(p[k] for k in BLOCK_PARAMS), out, r_idx, r_weight)
    rc = lib().bra_block(_ptr(x), *(_ptr(p[k]) for k in BLOCK_PARAMS), N, H, W, C, heads, S, topk, _dtype_code(x),
                         _ptr(out), _ptr(r_idx), _ptr(r_weight), _stream(stream))
    _raise(rc, "bra_block")
    return out, r_idx, r_weight


def qkv(x, w_qkv, b_qkv, q=None, k=None, v=None, stream=None):
    """bra_qkv: x (..., C), w_qkv (3C, C), b_qkv (3C) -> q, k, v, each of x's shape."""
    C = x.shape[-1]
    M = x.numel() // C if C else 0
    q, k, v = (torch.empty_like(x) if t is None else t for t in (q, k, v))
    _check_dev(x, w_qkv, b_qkv, q, k, v)
    rc = lib().bra_qkv(_ptr(x), _ptr(w_qkv), _ptr(b_qkv), M, C, _dtype_code(x), _ptr(q), _ptr(k), _ptr(v),
                       _stream(stream))
    _raise(rc, "bra_qkv")
    return q, k, v


def attention_layer(x, w_qkv, b_qkv, w_o, b_o, lce_w, lce_b, heads: int, S: int, topk: int, out=None,
                    r_idx=None, r_weight=None, stream=None):
    """bra_attention_layer: out = wo(BRA(qkv(x))) for x (N,H,W,C) -> out, r_idx, r_weight."""
    N, H, W, C = x.shape
    P = S * S
    out = torch.empty_like(x) if out is None else out
    r_idx = torch.empty((N, P, topk), dtype=torch.int32, device=x.device) if r_idx is None else r_idx
    r_weight = torch.empty((N, P, topk), dtype=torch.float32, device=x.device) if r_weight is None else r_weight
    _check_dev(x, w_qkv, b_qkv, w_o, b_o, lce_w, lce_b, out, r_idx, r_weight)
    rc = lib().bra_attention_layer(_ptr(x), _ptr(w_qkv), _ptr(b_qkv), _ptr(w_o), _ptr(b_o), _ptr(lce_w),
                                   _ptr(lce_b), N, H, W, C, heads, S, topk, _dtype_code(x), _ptr(out),
                                   _ptr(r_idx), _ptr(r_weight), _stream(stream))
    _raise(rc, "bra_attention_layer")
    return out, r_idx, r_weight


def backward(q, k, v, lce_w, r_idx, dout, heads: int, S: int, stream=None, grads=None, sync: bool = True) -> dict:
    """bra_backward (sync=True) or bra_backward_async: gradients (float32) of
    sum(dout * forward output) for the routing r_idx (N, S*S, topk), routing detached ->
    {dq, dk, dv, dlce_w, dlce_b} (allocated here unless `grads` holds them)."""
    N, H, W, C = q.shape
    topk = r_idx.shape[-1]
    f32 = dict(dtype=torch.float32, device=q.device)
    g = grads if grads is not None else {
        "dq": torch.empty((N, H, W, C), **f32), "dk": torch.empty((N, H, W, C), **f32),
        "dv": torch.empty((N, H, W, C), **f32), "dlce_w": torch.empty((C, 5, 5), **f32),
        "dlce_b": torch.empty((C,), **f32)}
    _check_dev(q, k, v, lce_w, r_idx, dout, *g.values())
    fn = lib().bra_backward if sync else lib().bra_backward_async
    rc = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(lce_w), _ptr(r_idx), _ptr(dout), N, H, W, C, heads, S,
            topk, _dtype_code(q), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dlce_w"]),
            _ptr(g["dlce_b"]), _stream(stream))
    _raise(rc, "bra_backward" if sync else "bra_backward_async")
    return g


def forward_noalloc(q, k, v, lce_w, lce_b, heads: int, S: int, topk: int, out=None, r_idx=None,
                    r_weight=None, stream=None):
    """bra_forward_noalloc: bra_forward with its scratch in the library's static device
    array (no allocation inside the call). Outputs are allocated here with torch when not
    given; pass them in to keep the whole call allocation-free."""
    N, H, W, C = q.shape
    P = S * S
    out = torch.empty_like(q) if out is None else out
    r_idx = torch.empty((N, P, topk), dtype=torch.int32, device=q.device) if r_idx is None else r_idx
    r_weight = torch.empty((N, P, topk), dtype=torch.float32, device=q.device) if r_weight is None else r_weight
    _check_dev(q, k, v, lce_w, lce_b, out, r_idx, r_weight)
    rc = lib().bra_forward_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(lce_w), _ptr(lce_b), N, H, W, C, heads, S,
                                   topk, _dtype_code(q), _ptr(out), _ptr(r_idx), _ptr(r_weight),
                                   _stream(stream))
    _raise(rc, "bra_forward_noalloc")
    return out, r_idx, r_weight


def route(q, k, heads: int, S: int, topk: int, r_idx=None, r_weight=None, stream=None):
    """bra_route: region pooling, affinity and top-k -> r_idx (int32), r_weight (float32)."""
    N, H, W, C = q.shape
    P = S * S
    r_idx = torch.empty((N, P, topk), dtype=torch.int32, device=q.device) if r_idx is None else r_idx
    r_weight = torch.empty((N, P, topk), dtype=torch.float32, device=q.device) if r_weight is None else r_weight
    _check_dev(q, k, r_idx, r_weight)
    rc = lib().bra_route(_ptr(q), _ptr(k), N, H, W, C, heads, S, topk, _dtype_code(q), _ptr(r_idx),
                         _ptr(r_weight), _stream(stream))
    _raise(rc, "bra_route")
    return r_idx, r_weight


def attend(q, k, v, lce_w, lce_b, heads: int, S: int, r_idx, out=None, stream=None) -> torch.Tensor:
    """bra_attend: attention over a given routing r_idx (N,S*S,topk) int32, plus LCE(V)."""
    N, H, W, C = q.shape
    topk = r_idx.shape[-1]
    out = torch.empty_like(q) if out is None else out
    _check_dev(q, k, v, lce_w, lce_b, r_idx, out)
    rc = lib().bra_attend(_ptr(q), _ptr(k), _ptr(v), _ptr(lce_w), _ptr(lce_b), N, H, W, C, heads, S, topk,
                          _dtype_code(q), _ptr(r_idx), _ptr(out), _stream(stream))
    _raise(rc, "bra_attend")
    return out


def forward_host(q, k, v, lce_w, lce_b, heads: int, S: int, topk: int, out=None, r_idx=None,
                 r_weight=None, stream=None):
    """bra_forward_host: host (CPU, ideally pinned) tensors in and out; the library copies."""
    N, H, W, C = q.shape
    P = S * S
    for t in (q, k, v, lce_w, lce_b):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("bra_forward_host takes contiguous host tensors")
    out = torch.empty_like(q) if out is None else out
    r_idx = torch.empty((N, P, topk), dtype=torch.int32) if r_idx is None else r_idx
    r_weight = torch.empty((N, P, topk), dtype=torch.float32) if r_weight is None else r_weight
    rc = lib().bra_forward_host(_ptr(q), _ptr(k), _ptr(v), _ptr(lce_w), _ptr(lce_b), N, H, W, C, heads, S,
                                topk, _dtype_code(q), _ptr(out), _ptr(r_idx), _ptr(r_weight), _stream(stream))
    _raise(rc, "bra_forward_host")
    return out, r_idx, r_weight


def launch_count() -> int:
    """Kernels the library has launched since it was loaded."""
    return int(lib().bra_launch_count())


def trace_begin() -> None:
    _raise(lib().bra_trace_begin(), "bra_trace_begin")


def trace_read() -> dict:
    """{kernel name: (milliseconds, pairs)} summed over the recorded pairs, trace kept."""
    ms = (ctypes.c_double * KERNEL_CLASSES)()
    n = (ctypes.c_longlong * KERNEL_CLASSES)()
    _raise(lib().bra_trace_read(ms, n), "bra_trace_read")
    return {lib().bra_kernel_name(i).decode(): (ms[i], n[i]) for i in range(KERNEL_CLASSES)}


def trace_end() -> dict:
    """{kernel name: (milliseconds, launches)} over the traced launches."""
    ms = (ctypes.c_double * KERNEL_CLASSES)()
    n = (ctypes.c_longlong * KERNEL_CLASSES)()
    _raise(lib().bra_trace_end(ms, n), "bra_trace_end")
    return {lib().bra_kernel_name(i).decode(): (ms[i], n[i]) for i in range(KERNEL_CLASSES)}


def set_kernel_variant(variant: int) -> int:
    """bra_set_kernel_variant: VARIANT_AUTO or VARIANT_GENERIC; returns the previous one."""
    prev = lib().bra_set_kernel_variant(int(variant))
    if prev < 0:
        raise ValueError("unknown kernel variant %r" % variant)
    return prev


def device_status(stream=None) -> int:
    """bra_device_status: 0; 8 (BRA_ERR_TIMEOUT) if a kernel's bounded wait ran out; 6 (BRA_ERR_INDEX) if
    a bra_backward_async call met an out-of-range routing entry. Clears the flags."""
    return int(lib().bra_device_status(_stream(stream)))


def selftest_wait_timeout(polls: int, stream=None) -> None:
    _raise(lib().bra_selftest_wait_timeout(int(polls), _stream(stream)), "bra_selftest_wait_timeout")


def raw_call(name: str, *args) -> int:
    """Call an entry point with raw ctypes arguments (argument-check tests)."""
    return getattr(lib(), name)(*args)
