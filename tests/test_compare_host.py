"""The parity checker itself (no GPU): it must reject the mistakes it exists to catch.

r_weight is the softmax over the affinities of the selected regions (the router of the
niftyadmin walk-through, section "BRA模块": top-k of the region logits, then softmax),
so it is fixed by the selection on every row, near ties included.
"""
import numpy as np

from oracle import compare


def _case():
    # one image, 4 regions, topk 2. Row 0 has a near tie between regions 1 and 2 for the
    # second place (gap 4e-4 <= 1e-3); rows 1-3 are well separated.
    logits = np.array([[[2.0, 1.0, 1.0004, -1.0],
                        [0.1, 0.9, -0.5, 0.3],
                        [-1.0, -2.0, 0.5, 0.0],
                        [0.0, 0.2, 0.4, 0.6]]])
    order = np.argsort(-logits, axis=-1, kind="stable")[..., :2]
    ref_idx = order.astype(np.int32)
    lg = np.take_along_axis(logits, order, axis=-1)
    e = np.exp(lg - lg.max(-1, keepdims=True))
    ref_w = e / e.sum(-1, keepdims=True)
    return logits, ref_idx, ref_w


def _run(logits, ref_idx, ref_w, idx, w):
    rep = compare.Report()
    compare.check_routing(logits, ref_idx, ref_w, idx, w.astype(np.float32), rep)
    return rep


def test_exact_result_passes_and_counts_the_near_tie():
    logits, ref_idx, ref_w = _case()
    rep = _run(logits, ref_idx, ref_w, ref_idx.copy(), ref_w)
    assert rep.ok, rep.notes
    assert rep.near_tie_rows == 1 and rep.rows == 4


def test_other_side_of_a_near_tie_passes_with_its_own_softmax():
    logits, ref_idx, ref_w = _case()
    idx = ref_idx.copy()
    idx[0, 0] = [0, 1]  # region 1 instead of 2: within the gap
    w = ref_w.copy()
    lg = logits[0, 0, [0, 1]]
    w[0, 0] = np.exp(lg - lg.max()) / np.exp(lg - lg.max()).sum()
    assert _run(logits, ref_idx, ref_w, idx, w).ok


def test_wrong_weight_on_a_near_tie_row_fails():
    logits, ref_idx, ref_w = _case()
    w = ref_w.copy()
    w[0, 0] = [0.5, 0.5]  # a wrong softmax exactly on the near-tie row
    assert not _run(logits, ref_idx, ref_w, ref_idx.copy(), w).ok
    w[0, 0] = [np.nan, 0.5]
    assert not _run(logits, ref_idx, ref_w, ref_idx.copy(), w).ok


def test_wrong_set_off_near_ties_and_invalid_rows_fail():
    logits, ref_idx, ref_w = _case()
    idx = ref_idx.copy()
    idx[0, 1] = [1, 2]  # the oracle's set is {1, 3}; no near tie in that row
    assert not _run(logits, ref_idx, ref_w, idx, ref_w).ok
    idx = ref_idx.copy()
    idx[0, 2] = [2, 2]  # a repeated region is not a top-k
    assert not _run(logits, ref_idx, ref_w, idx, ref_w).ok
    idx = ref_idx.copy()
    idx[0, 3] = [2, 3]  # right set, ascending order
    assert not _run(logits, ref_idx, ref_w, idx, ref_w[:, :, ::-1]).ok


def test_output_tolerance_form():
    ref = np.array([0.0, 1.0, -3.0])
    rep = compare.Report()
    compare.check_output(ref + np.array([0.019, 0.029, -0.049]), ref, "bf16", rep)
    assert rep.ok, rep.notes
    rep = compare.Report()
    compare.check_output(ref + np.array([0.0, 0.031, 0.0]), ref, "bf16", rep)
    assert not rep.ok
    rep = compare.Report()
    compare.check_output(ref + np.array([0.0, 1.1e-4, 0.0]), ref, "f32", rep)
    assert not rep.ok
