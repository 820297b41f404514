"""Float64 CPU oracle of the BiFormer block around the attention layer — TEST
INFRASTRUCTURE ONLY (only `tests/` may import it).

The block, as the walk-through ("BiFormer ... 前向传播过程", niftyadmin) prints and runs it:
section "2、BiFormer Block" gives the first two lines of its forward,
    x = x + pos_embed(x)
    x = x + drop_path(attn(norm1(x)))
and the module printout of section "网络结构" gives the parts: pos_embed =
Conv2d(C, C, 3, padding 1, groups C) (bias on: no `bias=False` is printed), norm1 / norm2 =
LayerNorm(C, eps 1e-6, affine), attn = the attention layer (qkv projection, BRA, output
projection), mlp = Linear(C, 3C) -> Identity -> GELU -> Linear(3C, C), drop_path =
Identity. The walk-through says nothing about the MLP line ("没什么好说的"); the reading
taken is the same pre-norm residual form as the attention line,
    x = x + drop_path(mlp(norm2(x))).
GELU is PyTorch's default (the exact erf form). Between the steps every stored tensor is
rounded to the block's dtype, as a bf16 model stores its activations: x after each
residual add, the LayerNorm outputs, the MLP hidden layer after the GELU, and the
attention layer's own intermediates (oracle.layer_forward).
Pins: tests/test_oracle_block_pins.py.
"""
from __future__ import annotations

import math
from typing import Dict

import numpy as np

import oracle


def dwconv3(x, w, b) -> np.ndarray:
    """Depthwise 3x3 cross-correlation, zero pad 1, plus bias: x (N,H,W,C), w (C,3,3)."""
    x = np.asarray(x, dtype=np.float64)
    N, H, W, C = x.shape
    xp = np.zeros((N, H + 2, W + 2, C))
    xp[:, 1:H + 1, 1:W + 1] = x
    out = np.broadcast_to(np.asarray(b, np.float64), x.shape).copy()
    for a in range(3):
        for c in range(3):
            out += xp[:, a:a + H, c:c + W] * np.asarray(w, np.float64)[:, a, c]
    return out


def layer_norm(x, gamma, beta, eps: float = 1e-6) -> np.ndarray:
    """LayerNorm over the last axis: (x - mean) / sqrt(var + eps) * gamma + beta, with the
    biased variance (mean of squared deviations)."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * np.asarray(gamma, np.float64) + np.asarray(beta, np.float64)


def gelu(x) -> np.ndarray:
    """x * Phi(x) with the standard normal CDF Phi(x) = (1 + erf(x / sqrt 2)) / 2."""
    x = np.asarray(x, dtype=np.float64)
    erf = np.vectorize(math.erf)
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def block_forward(x, p: Dict[str, np.ndarray], heads: int, S: int, topk: int, dtype: str, r_idx_given=None,
                  intermediates: bool = False):
    """One BiFormer block. p holds pos_w (C,3,3), pos_b (C), ln1_g, ln1_b, ln2_g, ln2_b (C),
    w_qkv (3C,C), b_qkv (3C), w_o (C,C), b_o (C), lce_w (C,5,5), lce_b (C),
    mlp_w1 (3C,C), mlp_b1 (3C), mlp_w2 (C,3C), mlp_b2 (C).
    Returns (out, r_idx, r_weight); out is the float64 value before its final rounding.
    `r_idx_given`: the attention runs over that routing (see oracle.layer_forward).
    `intermediates`: also return {"h": norm1's stored output (the attention layer's input),
    "x2": the stored residual x1 + attn, "m": the stored MLP output} (the output is x2 + m)."""
    r = lambda a: oracle.round_to(a, dtype)
    x = np.asarray(x, dtype=np.float64)
    N, H, W, C = x.shape
    x = r(x + dwconv3(x, p["pos_w"], p["pos_b"]))
    h = r(layer_norm(x, p["ln1_g"], p["ln1_b"]))
    h1 = h
    a, r_idx, r_w = oracle.layer_forward(h, p["w_qkv"], p["b_qkv"], p["w_o"], p["b_o"], p["lce_w"], p["lce_b"],
                                         heads, S, topk, dtype, r_idx_given=r_idx_given)
    x = r(x + r(a))
    h = r(layer_norm(x, p["ln2_g"], p["ln2_b"]))
    m = r(gelu(oracle.linear(h.reshape(-1, C), p["mlp_w1"], p["mlp_b1"])))
    m = oracle.linear(m, p["mlp_w2"], p["mlp_b2"]).reshape(N, H, W, C)
    if intermediates:
        return x + r(m), r_idx, r_w, {"h": h1, "x2": x, "m": r(m)}
    return x + r(m), r_idx, r_w
