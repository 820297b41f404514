"""Float64 CPU oracle for the BRA forward pass — TEST INFRASTRUCTURE ONLY.

Only `tests/`, `__graft_entry__.smoke()` and the benchmark's CPU-baseline leg may
import this package. The CUDA library never calls it, and it imports nothing from
the CUDA package.

The forward's arithmetic lives in `bra_oracle.c` (plain C, float64, OpenMP over
regions), compiled with gcc into `liboracle_bra.so` next to it; this module marshals
numpy arrays through ctypes and adds the attention layer's projections (numpy, float64,
below). The backward pass with the routing detached is `oracle/backward.py` (numpy,
float64).

Every function follows the official BRA code as walked through on
"BiFormer ... 前向传播过程" (niftyadmin), section "BRA模块", eqs. 4-7, and
Algorithm 1 as described on bernice.tw ("Bi-Level Routing Attention"). Parity
pins: see tests/test_oracle_pins.py. No page prints a numeric worked example, so
no pin compares against printed values; every function is pinned by closed forms,
library routines on special cases, brute force and invariants instead.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bra_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_bra.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE float64: no fast-math, no reassociation)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fno-fast-math", "-ffp-contract=off", "-shared", "-fPIC",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        i = ctypes.c_int
        lib.oracle_route.argtypes = [dp, dp, i, i, i, i, i, i, i, ip, dp, dp]
        lib.oracle_attend.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, i, i, i, ip, dp]
        lib.oracle_forward.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, i, i, i, dp, ip, dp]
        lib.oracle_lce.argtypes = [dp, dp, dp, i, i, i, i, dp]
        lib.oracle_region_mean.argtypes = [dp, i, i, i, i, i, dp]
        lib.oracle_check_shape.argtypes = [i] * 7
        lib.oracle_set_threads.argtypes = [i]
        for name in ("oracle_route", "oracle_attend", "oracle_forward", "oracle_check_shape",
                     "oracle_threads"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
    return _lib


def _d(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float64)


def _p(x: np.ndarray, t=ctypes.c_double):
    return x.ctypes.data_as(ctypes.POINTER(t))


def threads() -> int:
    return _load().oracle_threads()


def set_threads(t: int) -> None:
    _load().oracle_set_threads(int(t))


def region_mean(x, S: int) -> np.ndarray:
    """Mean of each region's tokens, all channels: (N,H,W,C) -> (N,S*S,C)."""
    x = _d(x)
    N, H, W, C = x.shape
    out = np.empty((N, S * S, C), np.float64)
    _load().oracle_region_mean(_p(x), N, H, W, C, S, _p(out))
    return out


def route(q, k, heads: int, S: int, topk: int, with_logits: bool = False):
    """Region affinity, top-k region indices (descending) and their softmax weights."""
    q, k = _d(q), _d(k)
    N, H, W, C = q.shape
    P = S * S
    r_idx = np.empty((N, P, topk), np.int32)
    r_w = np.empty((N, P, topk), np.float64)
    logits = np.empty((N, P, P), np.float64) if with_logits else None
    rc = _load().oracle_route(_p(q), _p(k), N, H, W, C, heads, S, topk, _p(r_idx, ctypes.c_int32),
                              _p(r_w), _p(logits) if with_logits else None)
    if rc:
        raise ValueError("oracle_route: bad shape")
    return (r_idx, r_w, logits) if with_logits else (r_idx, r_w)


def lce(v, lce_w, lce_b) -> np.ndarray:
    """Depthwise 5x5 cross-correlation of v (zero pad 2) plus bias."""
    v, w, b = _d(v), _d(lce_w), _d(lce_b)
    N, H, W, C = v.shape
    out = np.empty_like(v)
    _load().oracle_lce(_p(v), _p(w), _p(b), N, H, W, C, _p(out))
    return out


def attend(q, k, v, lce_w, lce_b, heads: int, S: int, r_idx) -> np.ndarray:
    """Token-to-token attention over the given routing, plus LCE(V)."""
    q, k, v, w, b = _d(q), _d(k), _d(v), _d(lce_w), _d(lce_b)
    r_idx = np.ascontiguousarray(r_idx, dtype=np.int32)
    N, H, W, C = q.shape
    topk = r_idx.shape[-1]
    out = np.empty_like(q)
    rc = _load().oracle_attend(_p(q), _p(k), _p(v), _p(w), _p(b), N, H, W, C, heads, S, topk,
                               _p(r_idx, ctypes.c_int32), _p(out))
    if rc:
        raise ValueError("oracle_attend: bad shape or region index (rc=%d)" % rc)
    return out


def forward(q, k, v, lce_w, lce_b, heads: int, S: int, topk: int
            ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """The whole BRA forward: returns (out, r_idx, r_weight)."""
    q, k, v, w, b = _d(q), _d(k), _d(v), _d(lce_w), _d(lce_b)
    N, H, W, C = q.shape
    P = S * S
    out = np.empty_like(q)
    r_idx = np.empty((N, P, topk), np.int32)
    r_w = np.empty((N, P, topk), np.float64)
    rc = _load().oracle_forward(_p(q), _p(k), _p(v), _p(w), _p(b), N, H, W, C, heads, S, topk,
                                _p(out), _p(r_idx, ctypes.c_int32), _p(r_w))
    if rc:
        raise ValueError("oracle_forward: bad shape (rc=%d)" % rc)
    return out, r_idx, r_w


def check_shape(N, H, W, C, heads, S, topk) -> bool:
    return _load().oracle_check_shape(N, H, W, C, heads, S, topk) == 0


# ----------------------------------------------------------------------------- attention layer
# The two steps either side of the path: the qkv projection before it (nn.Linear C -> 3C
# with bias; q, k and v are consecutive C-wide chunks of its output, in that order) and
# the output projection `wo` after it (nn.Linear C -> C with bias). Sources: "BiFormer ...
# 前向传播过程" (niftyadmin), section "BRA模块" (the qkv projection split into q and kv, and
# the closing linear layer after out + lepe) and section "网络结构" (the module printout:
# qkv Linear(64 -> 192, bias=True), wo Linear(64 -> 64, bias=True)); Algorithm 1 as
# described on bernice.tw chunks linear_qkv(x) into query, key, value the same way.
# Between the steps every tensor is stored in the layer's dtype (a bf16 model keeps its
# activations in bf16): q, k, v and the attention output are rounded to that dtype before
# the next step reads them, as the CUDA path stores them.

def round_to(x, dtype: str) -> np.ndarray:
    """Round float64 values to the storage dtype, nearest with ties to even; float64 out.

    "f32": IEEE single (numpy's conversion). "bf16": bfloat16 straight from the float64
    value (one rounding): the 52-bit fraction is rounded to 7 bits. Valid for zero and for
    finite magnitudes in bfloat16's normal range, which the function checks.
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    if dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    if dtype != "bf16":
        raise ValueError("dtype must be 'f32' or 'bf16'")
    a = np.abs(x)
    if not np.all(np.isfinite(x)) or np.any((a != 0) & ((a < 2.0 ** -126) | (a >= 3.3e38))):
        raise ValueError("round_to bf16: value outside bfloat16's normal range")
    u = x.view(np.uint64)
    drop = np.uint64(45)
    lsb = (u >> drop) & np.uint64(1)
    r = (u + (np.uint64(1) << np.uint64(44)) - np.uint64(1) + lsb) & ~((np.uint64(1) << drop) - np.uint64(1))
    return r.view(np.float64)


def linear(x, w, b) -> np.ndarray:
    """nn.Linear in float64: y = x w^T + b, x (..., K), w (Nout, K), b (Nout)."""
    x, w, b = _d(x), _d(w), _d(b)
    return x @ w.T + b


def layer_forward(x, w_qkv, b_qkv, w_o, b_o, lce_w, lce_b, heads: int, S: int, topk: int, dtype: str,
                  intermediates: bool = False, r_idx_given=None):
    """The attention layer around the path: out = wo(BRA(qkv(x))).

    x (N,H,W,C); w_qkv (3C, C), b_qkv (3C); w_o (C, C), b_o (C); lce_w (C,5,5), lce_b (C).
    Returns (out, r_idx, r_weight), plus {"q","k","v","o"} (the stored intermediates)
    when `intermediates` is set. `out` is the float64 value before the final rounding.
    With `r_idx_given`, the attention runs over that routing instead of its own (r_idx and
    r_weight are still the layer's own routing), so that a result routed differently on a
    near tie can be checked element by element.
    """
    x = _d(x)
    N, H, W, C = x.shape
    qkv = linear(x.reshape(-1, C), w_qkv, b_qkv)
    q, k, v = (round_to(qkv[:, i * C:(i + 1) * C], dtype).reshape(N, H, W, C) for i in range(3))
    o, r_idx, r_w = forward(q, k, v, lce_w, lce_b, heads, S, topk)
    if r_idx_given is not None:
        o = attend(q, k, v, lce_w, lce_b, heads, S, r_idx_given)
    o = round_to(o, dtype)
    out = linear(o.reshape(-1, C), w_o, b_o).reshape(N, H, W, C)
    if intermediates:
        return out, r_idx, r_w, {"q": q, "k": k, "v": v, "o": o}
    return out, r_idx, r_w
