"""Pins for the float64 oracle, independent of the oracle itself (CPU only).

No page prints a numeric worked example of BRA, so every pin is a closed form,
a library routine on a special case, a brute-force restatement in another
formulation, an invariant, or the shape comments printed by the niftyadmin
walk-through ("BRA模块" section). Each pin is chosen so that a plausible slip in
the oracle (a swapped region row/column, a transposed token index inside a
region, a dropped scale, a wrong softmax axis, per-head routing, a flipped LCE
kernel, a missing bias, a lost zero pad) fails at least one test.
"""
import os

import numpy as np
import pytest
import scipy.signal
import scipy.special

import oracle
from vision_transformer_sparse_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand(shape, seed):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape)


def inputs(N, H, W, C, seed, bias=0.0, S=1):
    q, k, v = (rand((N, H, W, C), seed + i) for i in range(3))
    if bias:
        hr, wr = H // S, W // S
        for t, x in enumerate((q, k, v)):
            off = rand((N, S, 1, S, 1, C), seed + 10 + t) * bias
            x[...] = (x.reshape(N, S, hr, S, wr, C) + off).reshape(N, H, W, C)
    w = rand((C, 5, 5), seed + 3) * 0.2
    b = rand((C,), seed + 4) * 0.1
    return q, k, v, w, b


# ---------------------------------------------------------------- independent restatements

def region_of(H, W, S):
    """Region index of every pixel, from image coordinates: row block * S + column block."""
    ys, xs = np.meshgrid(np.arange(H), np.arange(W), indexing="ij")
    return (ys // (H // S)) * S + (xs // (W // S))


def lce_scipy(v, w, b):
    """Depthwise zero-padded 5x5 cross-correlation via scipy, plus bias."""
    N, H, W, C = v.shape
    out = np.empty_like(v)
    for n in range(N):
        for c in range(C):
            out[n, :, :, c] = scipy.signal.correlate2d(v[n, :, :, c], w[c], mode="same",
                                                       boundary="fill", fillvalue=0.0) + b[c]
    return out


def masked_dense_attention(q, k, v, heads, S, r_idx):
    """Dense multi-head attention over ALL pixels, with keys outside the query's routed
    regions masked out. Regions come from pixel coordinates, not from a gather."""
    N, H, W, C = q.shape
    d = C // heads
    reg = region_of(H, W, S).reshape(-1)
    out = np.empty_like(q)
    for n in range(N):
        allowed = np.zeros((S * S, S * S), bool)
        for p in range(S * S):
            allowed[p, r_idx[n, p]] = True
        mask = allowed[reg][:, reg]                       # (HW query, HW key)
        Q = q[n].reshape(H * W, heads, d) * d ** -0.5
        K = k[n].reshape(H * W, heads, d)
        V = v[n].reshape(H * W, heads, d)
        s = np.einsum("thd,uhd->htu", Q, K)
        s = np.where(mask[None], s, -np.inf)
        a = scipy.special.softmax(s, axis=-1)
        out[n] = np.einsum("htu,uhd->thd", a, V).reshape(H, W, C)
    return out


# ---------------------------------------------------------------- pins

def test_golden_stage1_shapes():
    """The walk-through's stage-1 shape comments at 224x224 (N=1, 56x56x64, S=7, 2 heads, topk 1)."""
    shapes = {}
    with open(os.path.join(GOLDEN, "stage1_224_shapes.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                name, shp = line.split()
                shapes[name] = tuple(int(s) for s in shp.split(","))
    N, H, W, C = shapes["x"]
    S = int(round(shapes["regions"][1] ** 0.5))
    heads, d = shapes["q_pix_heads"][1], shapes["q_pix_heads"][3]
    topk = shapes["r_idx"][2]
    wl = synth.WORKLOADS["stage1_tiny_224"]
    assert (wl.N, wl.H, wl.W, wl.C, wl.S, wl.heads, wl.topk) == (N, H, W, C, S, heads, topk)
    assert shapes["regions"][2:4] == (H // S, W // S)
    q, k, v, w, b = inputs(N, H, W, C, 7)
    assert oracle.region_mean(q, S).shape == shapes["q_win"]
    r_idx, r_w, logits = oracle.route(q, k, heads, S, topk, with_logits=True)
    assert logits.shape == shapes["attn_logit"]
    assert r_idx.shape == shapes["r_idx"] and r_w.shape == shapes["r_weight"]
    # keys per query = topk * tokens per region = last dim of attn_weight
    assert topk * (H // S) * (W // S) == shapes["attn_weight"][3] == shapes["kv_pix_sel"][3]
    assert shapes["kv_pix_sel"][4] == 2 * C and d * heads == C
    out = oracle.attend(q, k, v, w, b, heads, S, r_idx)
    assert out.shape == shapes["out"]


@pytest.mark.parametrize("N,H,W,C,S", [(2, 12, 8, 6, 4), (1, 9, 15, 4, 3), (1, 6, 6, 3, 1)])
def test_region_mean_is_block_mean(N, H, W, C, S):
    """Region p = row-block*S + column-block, mean over hr x wr tokens (library reshape-mean)."""
    x = rand((N, H, W, C), 11)
    ref = x.reshape(N, S, H // S, S, W // S, C).mean(axis=(2, 4)).reshape(N, S * S, C)
    np.testing.assert_allclose(oracle.region_mean(x, S), ref, rtol=0, atol=1e-14)


@pytest.mark.parametrize("S", [2, 3, 4])
@pytest.mark.parametrize("heads", [1, 2])
def test_route_matches_sort_all_topk(S, heads):
    """Logits = (scale*q_r) k_r^T over ALL channels; top-k = full sort (value desc, index asc)."""
    N, H, W, C = 2, 2 * S, 3 * S, 8
    q, k, _, _, _ = inputs(N, H, W, C, 100 + S)
    d = C // heads
    qr = q.reshape(N, S, H // S, S, W // S, C).mean(axis=(2, 4)).reshape(N, S * S, C)
    kr = k.reshape(N, S, H // S, S, W // S, C).mean(axis=(2, 4)).reshape(N, S * S, C)
    logits_ref = (qr * d ** -0.5) @ kr.transpose(0, 2, 1)
    for topk in range(1, S * S + 1):
        r_idx, r_w, logits = oracle.route(q, k, heads, S, topk, with_logits=True)
        np.testing.assert_allclose(logits, logits_ref, rtol=0, atol=1e-13)
        for n in range(N):
            for p in range(S * S):
                order = np.lexsort((np.arange(S * S), -logits_ref[n, p]))[:topk]
                assert list(r_idx[n, p]) == list(order)
                sel = logits_ref[n, p, order]
                np.testing.assert_allclose(r_w[n, p], scipy.special.softmax(sel), rtol=1e-13, atol=0)


def test_route_ties_go_to_lower_index():
    """Two regions with identical key content tie exactly; the lower index comes first."""
    S, C = 3, 4
    q = rand((1, 6, 6, C), 5)
    k = rand((1, 6, 6, C), 6)
    k[:, 4:6, 2:4] = k[:, 0:2, 0:2]   # region 7 (row 2, col 1) := region 0 (row 0, col 0)
    r_idx, _, logits = oracle.route(q, k, 1, S, S * S, with_logits=True)
    assert np.all(logits[0, :, 0] == logits[0, :, 7])
    for p in range(S * S):
        row = list(r_idx[0, p])
        assert row.index(0) + 1 == row.index(7)


def test_route_scale_invariance_and_weight_dependence():
    """I_r is invariant to a positive scale of q; r_weight is not (it is a softmax of logits)."""
    q, k, _, _, _ = inputs(2, 8, 8, 8, 21)
    a, wa = oracle.route(q, k, 2, 4, 5)
    b, wb = oracle.route(2.5 * q, k, 2, 4, 5)
    assert np.array_equal(a, b)
    assert not np.allclose(wa, wb)
    np.testing.assert_allclose(wa.sum(-1), 1.0, atol=1e-14)
    assert np.all(np.diff(wa, axis=-1) <= 0)


@pytest.mark.parametrize("N,H,W,C,heads,S", [(1, 8, 8, 8, 2, 4), (2, 6, 9, 6, 3, 3), (1, 4, 4, 4, 1, 2)])
def test_dense_limit_equals_mhsa_plus_lce(N, H, W, C, heads, S):
    """At topk = S^2 BRA is dense multi-head attention plus LCE (the stage-4
    AttentionLePE of the BiFormer-T printout): brute force, library softmax and scipy conv."""
    q, k, v, w, b = inputs(N, H, W, C, 31)
    out, r_idx, _ = oracle.forward(q, k, v, w, b, heads, S, S * S)
    d = C // heads
    ref = np.empty_like(q)
    for n in range(N):
        Q = q[n].reshape(-1, heads, d) * d ** -0.5
        K = k[n].reshape(-1, heads, d)
        V = v[n].reshape(-1, heads, d)
        a = scipy.special.softmax(np.einsum("thd,uhd->htu", Q, K), axis=-1)
        ref[n] = np.einsum("htu,uhd->thd", a, V).reshape(H, W, C)
    ref += lce_scipy(v, w, b)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("N,H,W,C,heads,S,topk", [
    (1, 8, 12, 8, 2, 4, 1), (2, 9, 6, 6, 2, 3, 2), (1, 12, 12, 4, 1, 4, 5), (1, 10, 10, 4, 2, 5, 3)])
def test_routed_equals_masked_dense(N, H, W, C, heads, S, topk):
    """Gathered attention == dense attention with keys outside the routed regions masked,
    regions taken from pixel coordinates. Pins the gather's token mapping."""
    q, k, v, w, b = inputs(N, H, W, C, 41, bias=0.7, S=S)
    out, r_idx, _ = oracle.forward(q, k, v, w, b, heads, S, topk)
    ref = masked_dense_attention(q, k, v, heads, S, r_idx) + lce_scipy(v, w, b)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_routed_region_order_invariance():
    """The softmax runs over the union of routed keys, so the order of I_r's entries
    does not change the output."""
    q, k, v, w, b = inputs(2, 12, 12, 8, 51, bias=0.5, S=4)
    r_idx, _ = oracle.route(q, k, 2, 4, 5)
    base = oracle.attend(q, k, v, w, b, 2, 4, r_idx)
    rng = np.random.Generator(np.random.PCG64(3))
    perm = np.array([[rng.permutation(row) for row in img] for img in r_idx], np.int32)
    assert not np.array_equal(perm, r_idx)
    np.testing.assert_allclose(oracle.attend(q, k, v, w, b, 2, 4, perm), base, rtol=0, atol=1e-13)


def test_lce_impulse_response_and_padding():
    """A V impulse reproduces the 5x5 weights (cross-correlation, kernel read reversed
    around the impulse); borders are zero padded (scipy fill); the bias is added once."""
    C, H, W = 3, 9, 11
    w = rand((C, 5, 5), 61)
    b = rand((C,), 62)
    v = np.zeros((1, H, W, C))
    y0, x0 = 4, 5
    v[0, y0, x0, 1] = 1.0
    lepe = oracle.lce(v, w, b)
    for a in range(5):
        for bb in range(5):
            assert lepe[0, y0 + 2 - a, x0 + 2 - bb, 1] == pytest.approx(w[1, a, bb] + b[1], abs=1e-15)
    np.testing.assert_allclose(lepe[0, :, :, 0], b[0], atol=1e-15)
    vr = rand((2, H, W, C), 63)
    np.testing.assert_allclose(oracle.lce(vr, w, b), lce_scipy(vr, w, b), rtol=0, atol=1e-13)


def test_constant_values_pass_through_attention():
    """With V constant per channel, attention returns that constant whatever the routing."""
    N, H, W, C, S = 1, 8, 8, 6, 4
    q, k, _, w, b = inputs(N, H, W, C, 71)
    cval = rand((C,), 72)
    v = np.broadcast_to(cval, (N, H, W, C)).copy()
    out, _, _ = oracle.forward(q, k, v, w, b, 3, S, 3)
    np.testing.assert_allclose(out - oracle.lce(v, w, b), np.broadcast_to(cval, out.shape), atol=1e-14)


def test_single_token_regions_route_to_best_pixel():
    """With one token per region (S = H = W) and topk = 1, the output is v of the
    pixel maximising q.k (all channels), plus LCE."""
    N, H, C = 2, 5, 4
    q, k, v, w, b = inputs(N, H, H, C, 81)
    out, r_idx, r_w = oracle.forward(q, k, v, w, b, 2, H, 1)
    lepe = lce_scipy(v, w, b)
    for n in range(N):
        Qf, Kf, Vf = q[n].reshape(-1, C), k[n].reshape(-1, C), v[n].reshape(-1, C)
        best = np.argmax(Qf @ Kf.T, axis=1)
        assert np.array_equal(r_idx[n, :, 0], best)
        np.testing.assert_allclose(out[n].reshape(-1, C), Vf[best] + lepe[n].reshape(-1, C), atol=1e-14)
    assert np.all(r_w == 1.0)


def test_shape_rules():
    """C divisible by heads, 1 <= topk <= S^2; H and W need not be multiples of S (the
    padded grid, pinned in test_oracle_padding_pins.py)."""
    assert oracle.check_shape(1, 56, 56, 64, 2, 7, 1)
    assert oracle.check_shape(1, 57, 56, 64, 2, 7, 1)
    assert oracle.check_shape(1, 56, 55, 64, 2, 7, 1)
    assert not oracle.check_shape(1, 56, 56, 64, 3, 7, 1)
    assert not oracle.check_shape(1, 56, 56, 64, 2, 7, 0)
    assert not oracle.check_shape(1, 56, 56, 64, 2, 7, 50)
    with pytest.raises(ValueError):
        oracle.attend(*inputs(1, 4, 4, 2, 1), 1, 2, np.full((1, 4, 1), 4, np.int32))


def test_synthetic_generator_is_seeded_and_bf16_exact():
    wl = synth.WORKLOADS["seg_stage2_512"].with_(N=1)
    a = synth.make_inputs(wl)
    b = synth.make_inputs(wl)
    for key in a:
        assert np.array_equal(a[key], b[key])
    assert np.array_equal(synth.round_bf16(a["q"]), a["q"])
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.0 ** -130, 3.3e38], np.float32)
    r = synth.round_bf16(x)
    assert r[0] == 1.0 and r[1] == 1.0 and r[2] == 1.0 + 2 ** -6 and r[3] != 0
