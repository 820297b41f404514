"""Float64 CPU oracle of the BRA backward pass — TEST INFRASTRUCTURE ONLY.

Only `tests/` may import this module (like the rest of `oracle/`). It imports nothing from
the CUDA package.

What it computes: the gradients of a scalar loss L with respect to q, k, v and the LCE
parameters, given dL/dout, for the forward of `oracle.attend` (token-to-token attention
over a FIXED routing, plus LCE(V)). The routing carries no gradient: the walk-through's
router ("BiFormer ... 前向传播过程", niftyadmin, section "BRA模块", the `TopkRouting`
forward) detaches the region-level query and key when `diff_routing` is off (its
default), the top-k index is a discrete choice, and r_weight does not scale K or V (the
gather's soft-routing option is off). So the path is:

  per image n, query region p, head m (d channels), with Q the region's w^2 tokens and
  K, V the topk * w^2 gathered tokens of its routed regions (r_idx order, then token
  order inside a region):
    s = scale * Q K^T,  a = softmax over the gathered keys,  o = a V        (forward)
    dV += a^T dO,  da = dO V^T,  ds = a * (da - rowsum(a * da)),
    dQ = scale * ds K,  dK += scale * ds^T Q                                (backward)
  gathered rows are scatter-added back to their pixels (a pixel gathered by several
  query regions, or twice by one, accumulates every contribution);
  LCE: out[y, x, c] += b[c] + sum_{a,b} w[c, a, b] V[y + a - 2, x + b - 2, c] (zero pad), so
    dV[y', x', c] += sum_{a,b} w[c, a, b] dout[y' - a + 2, x' - b + 2, c],
    dw[c, a, b] = sum_{n,y,x} dout[n, y, x, c] Vpad[n, y + a, x + b, c],  db[c] = sum dout.

Plain numpy in float64, one (image, region, head) at a time; no blocking, no fusion.
Pins: tests/test_oracle_backward_pins.py (finite differences of the forward oracle, torch
autograd on a region-masked dense attention, closed forms of the LCE gradients).
"""
from __future__ import annotations

from typing import Dict

import numpy as np


def region_pixels(H: int, W: int, S: int) -> np.ndarray:
    """(S*S, w^2) flat pixel index y * W + x of every region's tokens: region p = j*S + i
    covers rows j*hr .. j*hr + hr - 1 and columns i*wr .. i*wr + wr - 1, tokens row-major."""
    hr, wr = H // S, W // S
    pix = np.empty((S * S, hr * wr), dtype=np.int64)
    for j in range(S):
        for i in range(S):
            ys = j * hr + np.arange(hr)
            xs = i * wr + np.arange(wr)
            pix[j * S + i] = (ys[:, None] * W + xs[None, :]).reshape(-1)
    return pix


def lce_backward(v, lce_w, dout):
    """Gradients of out += LCE(v) = b + depthwise 5x5 cross-correlation (zero pad 2):
    returns (dv, dw, db)."""
    v, w, dout = (np.asarray(a, dtype=np.float64) for a in (v, lce_w, dout))
    N, H, W, C = v.shape
    vp = np.zeros((N, H + 4, W + 4, C))
    vp[:, 2:H + 2, 2:W + 2] = v
    gp = np.zeros((N, H + 4, W + 4, C))
    dw = np.empty((C, 5, 5))
    for a in range(5):
        for b in range(5):
            # out[y, x] uses v[y + a - 2, x + b - 2] = vp[y + a, x + b] with weight w[:, a, b]
            dw[:, a, b] = np.einsum("nyxc,nyxc->c", dout, vp[:, a:a + H, b:b + W])
            gp[:, a:a + H, b:b + W] += dout * w[:, a, b]
    dv = gp[:, 2:H + 2, 2:W + 2]
    db = dout.sum(axis=(0, 1, 2))
    return dv, dw, db


def backward(q, k, v, lce_w, lce_b, heads: int, S: int, r_idx, dout) -> Dict[str, np.ndarray]:
    """Gradients {dq, dk, dv, dlce_w, dlce_b} of sum(dout * attend(q, k, v, ..., r_idx)).

    lce_b takes no part in the arithmetic (its gradient is the sum of dout); it is an
    argument so that the call mirrors the forward's."""
    q, k, v, dout = (np.asarray(a, dtype=np.float64) for a in (q, k, v, dout))
    r_idx = np.asarray(r_idx)
    N, H, W, C = q.shape
    P = S * S
    d = C // heads
    scale = d ** -0.5
    pix = region_pixels(H, W, S)
    qf, kf, vf, gf = (a.reshape(N, H * W, C) for a in (q, k, v, dout))
    dq = np.zeros_like(qf)
    dk = np.zeros_like(kf)
    dv = np.zeros_like(vf)
    for n in range(N):
        for p in range(P):
            rows = pix[p]                                # this region's query pixels
            keys = pix[r_idx[n, p]].reshape(-1)          # gathered key pixels, r_idx order
            for m in range(heads):
                ch = slice(m * d, (m + 1) * d)
                Q, K, V, dO = qf[n, rows, ch], kf[n, keys, ch], vf[n, keys, ch], gf[n, rows, ch]
                s = scale * Q @ K.T
                s -= s.max(axis=1, keepdims=True)
                a = np.exp(s)
                a /= a.sum(axis=1, keepdims=True)
                da = dO @ V.T
                ds = a * (da - (a * da).sum(axis=1, keepdims=True))
                dq[n, rows, ch] += scale * ds @ K
                np.add.at(dk[n], (keys[:, None], np.arange(m * d, (m + 1) * d)[None, :]), scale * ds.T @ Q)
                np.add.at(dv[n], (keys[:, None], np.arange(m * d, (m + 1) * d)[None, :]), a.T @ dO)
    dv_lce, dw, db = lce_backward(v, lce_w, dout)
    return {"dq": dq.reshape(N, H, W, C), "dk": dk.reshape(N, H, W, C),
            "dv": dv.reshape(N, H, W, C) + dv_lce, "dlce_w": dw, "dlce_b": db}
