"""Pins for the oracle's attention layer (CPU only): the qkv projection before the path
and the output projection after it, out = wo(BRA(qkv(x))).

The pages print the two projections as nn.Linear modules with bias (qkv C -> 3C, split
into q, k, v in that order; wo C -> C), so every pin below is a closed form, a special
case that reduces to the already-pinned BRA oracle or to textbook dense attention, an
invariant, or a brute-force restatement. A slip such as swapped k / v chunks, a
transposed weight, a dropped bias, a missing rounding step or a bias applied to the
wrong chunk fails at least one of them.
"""
import numpy as np
import pytest
import scipy.special

import oracle
from vision_transformer_sparse_b200 import synth
from test_oracle_pins import lce_scipy


def rand(shape, seed, scale=1.0):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape) * scale


def layer_inputs(N, H, W, C, seed, dtype="f32"):
    r = (lambda a: synth.round_bf16(a.astype(np.float32)).astype(np.float64)) if dtype == "bf16" else (
        lambda a: a.astype(np.float32).astype(np.float64))
    return dict(
        x=r(rand((N, H, W, C), seed)),
        w_qkv=r(rand((3 * C, C), seed + 1, C ** -0.5)),
        b_qkv=r(rand((3 * C,), seed + 2, 0.05)),
        w_o=r(rand((C, C), seed + 3, C ** -0.5)),
        b_o=r(rand((C,), seed + 4, 0.05)),
        lce_w=r(rand((C, 5, 5), seed + 5, 0.1)),
        lce_b=r(rand((C,), seed + 6, 0.05)),
    )


def run(d, heads, S, topk, dtype, **kw):
    return oracle.layer_forward(d["x"], d["w_qkv"], d["b_qkv"], d["w_o"], d["b_o"], d["lce_w"], d["lce_b"],
                                heads, S, topk, dtype, **kw)


def routing_gap(q, k, heads, S, topk):
    """Smallest gap between the k-th and (k+1)-th logit over all rows (inf at topk = S^2)."""
    _, _, logits = oracle.route(q, k, heads, S, topk, with_logits=True)
    if topk == S * S:
        return np.inf
    srt = -np.sort(-logits, axis=-1)
    return float(np.min(srt[..., topk - 1] - srt[..., topk]))


# ---------------------------------------------------------------- rounding

def test_round_bf16_ties_and_closed_forms():
    """Round-to-nearest-even at exact halfway points between bfloat16 neighbours."""
    x = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 1 + 2 ** -8 + 2 ** -40, 1 - 2 ** -10,
                  3.0, 0.0, 2.0 ** -126, 255.5, 256.5, 257.0])
    want = np.array([1.0, 1 + 2 ** -6, -1.0, 1 + 2 ** -7, 1.0, 3.0, 0.0, 2.0 ** -126, 256.0, 256.0, 256.0])
    np.testing.assert_array_equal(oracle.round_to(x, "bf16"), want)


def test_round_bf16_matches_float32_path_and_error_bound():
    """On float32 values the direct rounding equals an independent float32 -> bfloat16
    rounding (no double rounding is possible there), and every result is within half a
    unit in the last place: |r - x| <= 2^-8 |x|, with at most 8 significant bits."""
    x = (rand((4096,), 7) * np.exp(rand((4096,), 8) * 4)).astype(np.float32)
    r = oracle.round_to(x.astype(np.float64), "bf16")
    np.testing.assert_array_equal(r, synth.round_bf16(x).astype(np.float64))
    y = rand((4096,), 9) * 10
    ry = oracle.round_to(y, "bf16")
    assert np.all(np.abs(ry - y) <= 2.0 ** -8 * np.abs(y))
    m, _ = np.frexp(ry)
    assert np.all(m * 2 ** 8 == np.round(m * 2 ** 8))


def test_round_f32_is_ieee_single():
    y = rand((1000,), 10)
    np.testing.assert_array_equal(oracle.round_to(y, "f32"), y.astype(np.float32).astype(np.float64))


def test_round_rejects_out_of_range():
    with pytest.raises(ValueError):
        oracle.round_to(np.array([1e-40]), "bf16")
    with pytest.raises(ValueError):
        oracle.round_to(np.array([np.inf]), "bf16")


# ---------------------------------------------------------------- linear

def test_linear_brute_force():
    """y[m, n] = b[n] + sum_k x[m, k] w[n, k], written out with Python loops."""
    x, w, b = rand((3, 5), 11), rand((4, 5), 12), rand((4,), 13)
    y = oracle.linear(x, w, b)
    for m in range(3):
        for n in range(4):
            acc = b[n]
            for kk in range(5):
                acc += x[m, kk] * w[n, kk]
            assert abs(y[m, n] - acc) <= 1e-12 * (1 + abs(acc))


# ---------------------------------------------------------------- the layer

SHAPE = dict(N=2, H=8, W=8, C=16)  # 2 heads of 8 channels, S = 2: 16 tokens per region


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_identity_weights_reduce_to_bra(dtype):
    """qkv weight [I; I; I], output weight I, zero biases: the layer is BRA(x, x, x)
    followed by one rounding of its output to the dtype."""
    C = SHAPE["C"]
    d = layer_inputs(**SHAPE, seed=20, dtype=dtype)
    eye = np.eye(C)
    d.update(w_qkv=np.vstack([eye, eye, eye]), b_qkv=np.zeros(3 * C), w_o=eye, b_o=np.zeros(C))
    out, r_idx, r_w = run(d, 2, 2, 2, dtype)
    ref, ref_idx, ref_w = oracle.forward(d["x"], d["x"], d["x"], d["lce_w"], d["lce_b"], 2, 2, 2)
    np.testing.assert_array_equal(r_idx, ref_idx)
    np.testing.assert_array_equal(r_w, ref_w)
    half_ulp = 2.0 ** -8 if dtype == "bf16" else 2.0 ** -24
    assert np.all(np.abs(out - ref) <= half_ulp * np.abs(ref))


def test_chunk_order_is_q_k_v():
    """qkv weight [I; 2I; 3I]: q = x, k = 2x, v = 3x (exact in float32 for these x), so the
    layer equals BRA(x, 2x, 3x); swapping the k and v chunks would give BRA(x, 3x, 2x)."""
    C = SHAPE["C"]
    d = layer_inputs(**SHAPE, seed=21, dtype="bf16")
    eye = np.eye(C)
    d.update(w_qkv=np.vstack([eye, 2 * eye, 3 * eye]), b_qkv=np.zeros(3 * C), w_o=eye, b_o=np.zeros(C))
    out, r_idx, _ = run(d, 2, 2, 1, "f32")
    x = d["x"]
    ref, ref_idx, _ = oracle.forward(x, 2 * x, 3 * x, d["lce_w"], d["lce_b"], 2, 2, 1)
    np.testing.assert_array_equal(r_idx, ref_idx)
    assert np.max(np.abs(out - ref)) <= 2.0 ** -24 * np.max(np.abs(ref)) * 4
    swapped, _, _ = oracle.forward(x, 3 * x, 2 * x, d["lce_w"], d["lce_b"], 2, 2, 1)
    assert np.max(np.abs(out - swapped)) > 0.1


def test_zero_output_weight_gives_output_bias():
    C = SHAPE["C"]
    d = layer_inputs(**SHAPE, seed=22)
    d["w_o"] = np.zeros((C, C))
    out, _, _ = run(d, 2, 2, 2, "f32")
    np.testing.assert_array_equal(out, np.broadcast_to(d["b_o"], out.shape))


def test_output_weight_is_applied_as_x_w_transpose():
    """A permutation matrix as output weight moves channel j of the attention output to
    channel n where w_o[n, j] = 1 (nn.Linear: y = x w^T), and nothing else changes."""
    C = SHAPE["C"]
    d = layer_inputs(**SHAPE, seed=23)
    perm = np.random.Generator(np.random.PCG64(5)).permutation(C)
    d["w_o"] = np.eye(C)[perm]
    d["b_o"] = np.zeros(C)
    out, _, _, mid = run(d, 2, 2, 2, "f32", intermediates=True)
    np.testing.assert_array_equal(out, mid["o"][..., perm])


def test_common_key_bias_leaves_routing_and_output_unchanged():
    """Adding the same vector to every key adds q.beta to every score of a query (and
    q_r.beta to every affinity of a row): softmax, top-k and r_weight are unchanged. In
    float32 storage the shifted keys round differently, hence the small tolerance."""
    C = SHAPE["C"]
    d = layer_inputs(**SHAPE, seed=24)
    out0, idx0, w0, mid = run(d, 2, 2, 2, "f32", intermediates=True)
    assert routing_gap(mid["q"], mid["k"], 2, 2, 2) > 1e-3
    d["b_qkv"] = d["b_qkv"].copy()
    d["b_qkv"][C:2 * C] += rand((C,), 25, 0.7)
    out1, idx1, w1 = run(d, 2, 2, 2, "f32")
    np.testing.assert_array_equal(idx0, idx1)
    assert np.max(np.abs(w0 - w1)) < 1e-5
    assert np.max(np.abs(out0 - out1)) < 1e-5


def test_value_bias_shifts_output_by_projected_bias():
    """With the LCE switched off (zero weight and bias), adding gamma to every value adds
    gamma to every attention output (the weights of a query sum to one), so the layer
    output moves by w_o gamma."""
    C = SHAPE["C"]
    d = layer_inputs(**SHAPE, seed=26)
    d["lce_w"] = np.zeros((C, 5, 5))
    d["lce_b"] = np.zeros(C)
    out0, _, _ = run(d, 2, 2, 2, "f32")
    gamma = rand((C,), 27, 0.5)
    d["b_qkv"] = d["b_qkv"].copy()
    d["b_qkv"][2 * C:] += gamma
    out1, _, _ = run(d, 2, 2, 2, "f32")
    np.testing.assert_allclose(out1 - out0, np.broadcast_to(d["w_o"] @ gamma, out0.shape), atol=2e-5)


def test_dense_special_case_is_textbook_attention_layer():
    """topk = S^2: every query sees every token, so the layer is textbook multi-head
    self-attention with the LCE added, between two linear maps; here written with einsum
    and scipy (float32 storage between the steps, as in the oracle)."""
    N, H, W, C, heads, S = 1, 8, 8, 16, 2, 2
    d = layer_inputs(N, H, W, C, seed=28)
    out, _, _ = run(d, heads, S, S * S, "f32")
    f32 = lambda a: a.astype(np.float32).astype(np.float64)
    qkv = np.einsum("nhwc,jc->nhwj", d["x"], d["w_qkv"]) + d["b_qkv"]
    q, k, v = f32(qkv[..., :C]), f32(qkv[..., C:2 * C]), f32(qkv[..., 2 * C:])
    dh = C // heads
    Q = q.reshape(H * W, heads, dh) * dh ** -0.5
    K = k.reshape(H * W, heads, dh)
    V = v.reshape(H * W, heads, dh)
    a = scipy.special.softmax(np.einsum("thd,uhd->htu", Q, K), axis=-1)
    att = np.einsum("htu,uhd->thd", a, V).reshape(1, H, W, C)
    o = f32(att + lce_scipy(v, d["lce_w"], d["lce_b"]))
    ref = np.einsum("nhwc,jc->nhwj", o, d["w_o"]) + d["b_o"]
    assert np.max(np.abs(out - ref)) < 1e-5


def test_workload_layer_inputs_shapes_and_scale():
    w = synth.WORKLOADS["cls_stage2_224"].with_(N=1)
    d = synth.make_layer_inputs(w)
    C = w.C
    assert d["x"].shape == (1, 28, 28, C) and d["w_qkv"].shape == (3 * C, C) and d["b_qkv"].shape == (3 * C,)
    assert d["w_o"].shape == (C, C) and d["b_o"].shape == (C,)
    for a in d.values():
        np.testing.assert_array_equal(a, synth.round_bf16(a))
    _, _, _, mid = oracle.layer_forward(d["x"], d["w_qkv"], d["b_qkv"], d["w_o"], d["b_o"], d["lce_w"],
                                        d["lce_b"], w.heads, w.S, w.topk, w.dtype, intermediates=True)
    assert 0.8 < mid["q"].std() < 1.25 and 0.8 < mid["v"].std() < 1.25
    for name in ("q", "k", "v", "o"):  # stored in the layer's dtype between the steps
        a = mid[name].astype(np.float32)
        np.testing.assert_array_equal(a, synth.round_bf16(a))
        assert np.array_equal(a.astype(np.float64), mid[name])


def test_layer_checker_accepts_the_oracle_and_rejects_a_kv_swap():
    """The GPU tests' layer check passes the oracle's own (rounded) result and fails a
    result computed with the k and v chunks of the projection swapped."""
    from oracle import compare
    w = synth.Workload("checker", 50, 1, 14, 14, 64, 2, 7, 4, "bf16", lce_b_std=0.01)
    inp = synth.make_layer_inputs(w)
    args = (w.heads, w.S, w.topk, w.dtype)
    keys = ("x", "w_qkv", "b_qkv", "w_o", "b_o", "lce_w", "lce_b")
    out, r_idx, r_w = oracle.layer_forward(*(inp[k] for k in keys), *args)
    rep = compare.check_layer(inp, *args[:3], w.dtype, oracle.round_to(out, "bf16"), r_idx, r_w.astype(np.float32))
    assert rep.ok, rep.notes
    C = w.C
    bad = dict(inp)
    bad["w_qkv"] = np.vstack([inp["w_qkv"][:C], inp["w_qkv"][2 * C:], inp["w_qkv"][C:2 * C]])
    bad["b_qkv"] = np.concatenate([inp["b_qkv"][:C], inp["b_qkv"][2 * C:], inp["b_qkv"][C:2 * C]])
    out2, idx2, w2 = oracle.layer_forward(*(bad[k] for k in keys), *args)
    rep2 = compare.check_layer(inp, *args[:3], w.dtype, oracle.round_to(out2, "bf16"), idx2, w2.astype(np.float32))
    assert not rep2.ok
