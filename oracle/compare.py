"""Parity checks of a BRA result against the float64 oracle — TEST INFRASTRUCTURE ONLY.

Works on numpy arrays; knows nothing of how the result under test was produced.

Rules (fixed for this operation):
  * r_idx: per row, the SET of routed regions must equal the oracle's wherever the
    oracle's k-th and (k+1)-th largest affinities differ by more than 1e-3. Rows
    under that gap ("near ties") are counted separately; there the result's set must
    still be a valid top-k of the oracle's affinities within 1e-3.
  * r_weight: on every row (near ties included) compared index by index within 1e-5
    with the softmax over the oracle's logits of the regions the result selected
    (which is the oracle's own r_weight wherever the selections agree).
  * out: float32 inputs -> max |out - ref| <= 1e-4; bfloat16 inputs ->
    |out - ref| <= 2e-2 + 1e-2 |ref| element-wise. The reference output is the
    oracle's attention over the routing under test, so that a near-tie row is still
    checked element by element.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

import oracle

GAP = 1e-3
TOL_F32_ABS = 1e-4
TOL_BF16_ABS, TOL_BF16_REL = 2e-2, 1e-2
TOL_WEIGHT = 1e-5


@dataclasses.dataclass
class Report:
    rows: int = 0
    near_tie_rows: int = 0
    idx_mismatch_rows: int = 0
    weight_max_err: float = 0.0
    out_max_abs_err: float = 0.0
    out_worst_ratio: float = 0.0   # max over elements of err / allowed
    ok: bool = True
    notes: str = ""

    def fail(self, msg: str):
        self.ok = False
        self.notes += msg + "; "


def check_routing(logits: np.ndarray, ref_idx: np.ndarray, ref_w: np.ndarray, idx: np.ndarray,
                  w: np.ndarray, rep: Report, tol_weight: float = TOL_WEIGHT) -> None:
    N, P, topk = ref_idx.shape
    srt = -np.sort(-logits, axis=-1)
    for n in range(N):
        for p in range(P):
            rep.rows += 1
            got = idx[n, p]
            if np.any(got < 0) or np.any(got >= P) or len(set(got.tolist())) != topk:
                rep.fail("row (%d,%d): invalid index set %s" % (n, p, got))
                continue
            near = topk < P and srt[n, p, topk - 1] - srt[n, p, topk] <= GAP
            if near:
                rep.near_tie_rows += 1
                kth = srt[n, p, topk - 1]
                if np.any(logits[n, p, got] < kth - GAP):
                    rep.fail("row (%d,%d): near-tie set is not a valid top-k" % (n, p))
                    continue
            elif set(got.tolist()) != set(ref_idx[n, p].tolist()):
                rep.idx_mismatch_rows += 1
                rep.fail("row (%d,%d): r_idx %s != oracle %s" % (n, p, got, ref_idx[n, p]))
                continue
            # descending order where neighbours are separated by more than the gap
            lg = logits[n, p, got]
            if np.any(np.diff(lg) > GAP):
                rep.fail("row (%d,%d): r_idx not in descending affinity order" % (n, p))
            # r_weight is the softmax over the logits of the selected regions, so it is
            # fixed by the selection on every row, near ties included: compare it with the
            # float64 softmax over the oracle's logits at the indices under test (equal to
            # the oracle's own r_weight wherever the sets agree)
            if near or not np.array_equal(got, ref_idx[n, p]):
                e = np.exp(lg - lg.max())
                want = e / e.sum()
            else:
                want = ref_w[n, p]
            err = float(np.max(np.abs(w[n, p].astype(np.float64) - want)))
            if not np.isfinite(err):
                rep.fail("row (%d,%d): r_weight not finite" % (n, p))
                continue
            rep.weight_max_err = max(rep.weight_max_err, err)
    if rep.weight_max_err > tol_weight:
        rep.fail("r_weight err %.3g > %.1g" % (rep.weight_max_err, tol_weight))


def check_output(out: np.ndarray, ref: np.ndarray, dtype: str, rep: Report, scale: Optional[np.ndarray] = None
                 ) -> None:
    """`scale`: the magnitude the relative bf16 term is taken of (default |ref|); a result
    that is a sum of separately rounded terms passes the sum of the terms' magnitudes."""
    out = out.astype(np.float64)
    err = np.abs(out - ref)
    rep.out_max_abs_err = float(err.max()) if err.size else 0.0
    if dtype == "f32":
        allowed = np.full_like(ref, TOL_F32_ABS)
    else:
        allowed = TOL_BF16_ABS + TOL_BF16_REL * (np.abs(ref) if scale is None else scale)
    ratio = err / allowed
    rep.out_worst_ratio = float(ratio.max()) if ratio.size else 0.0
    if not np.all(np.isfinite(out)):
        rep.fail("non-finite output")
    if rep.out_worst_ratio > 1.0:
        where = np.unravel_index(np.argmax(ratio), ratio.shape)
        rep.fail("out err %.3g at %s (ref %.4g, got %.4g)" % (err[where], where, ref[where], out[where]))


def check_forward(inp: dict, heads: int, S: int, topk: int, dtype: str, out: np.ndarray, r_idx: np.ndarray,
                  r_weight: np.ndarray, ref: Optional[tuple] = None) -> Report:
    """Full parity check of one bra_forward result; `inp` holds the exact input values."""
    rep = Report()
    ref_idx, ref_w, logits = ref if ref is not None else oracle.route(inp["q"], inp["k"], heads, S, topk,
                                                                      with_logits=True)
    check_routing(logits, ref_idx, ref_w, r_idx, r_weight, rep)
    if rep.ok:
        ref_out = oracle.attend(inp["q"], inp["k"], inp["v"], inp["lce_w"], inp["lce_b"], heads, S, r_idx)
        check_output(out, ref_out, dtype, rep)
    return rep


# ----------------------------------------------------------------------------- attention layer
# The layer's q, k, v are computed on both sides from the same x and weights, but a
# float32-accumulated projection and the float64 one can round an element to neighbouring
# bfloat16 values (when the exact value lies within the float32 accumulation error of a
# rounding boundary: a fraction of a percent of the elements). Such one-ulp differences
# (2^-7 relative) move region means and affinities by ~1e-4, so for bfloat16 the layer's
# r_weight is compared within TOL_LAYER_WEIGHT instead of TOL_WEIGHT; a routing row whose
# k-th / (k+1)-th gap is under GAP is a near tie exactly as above. The output tolerance is
# the forward's: the projections add one float32-accumulated GEMM and one rounding of the
# attention output, both far below it.
TOL_LAYER_WEIGHT = 2e-3


def check_layer(inp: dict, heads: int, S: int, topk: int, dtype: str, out: np.ndarray, r_idx: np.ndarray,
                r_weight: np.ndarray) -> Report:
    """Parity check of one attention-layer result (x, w_qkv, b_qkv, w_o, b_o, lce_w, lce_b in `inp`)."""
    rep = Report()
    _, _, _, mid = oracle.layer_forward(inp["x"], inp["w_qkv"], inp["b_qkv"], inp["w_o"], inp["b_o"], inp["lce_w"],
                                        inp["lce_b"], heads, S, topk, dtype, intermediates=True)
    ref_idx, ref_w, logits = oracle.route(mid["q"], mid["k"], heads, S, topk, with_logits=True)
    check_routing(logits, ref_idx, ref_w, r_idx, r_weight, rep,
                  tol_weight=TOL_LAYER_WEIGHT if dtype == "bf16" else TOL_WEIGHT)
    if rep.ok:
        o = oracle.round_to(oracle.attend(mid["q"], mid["k"], mid["v"], inp["lce_w"], inp["lce_b"], heads, S, r_idx),
                            dtype)
        N, H, W, C = o.shape
        ref_out = oracle.linear(o.reshape(-1, C), inp["w_o"], inp["b_o"]).reshape(N, H, W, C)
        check_output(out, ref_out, dtype, rep)
    return rep
