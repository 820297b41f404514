"""Pins for the oracle's padded grid (H or W not a multiple of S), CPU only.

The bernice.tw notes (section "消融實驗") say only that padding the feature map costs
compute, which is why S is chosen per task (7, 16, 8). The reading taken: q, k, v are
zero-padded at the bottom and right to Hp = S*ceil(H/S), Wp = S*ceil(W/S); region means
are taken over the whole padded region; padded tokens take part as keys (k = v = 0,
score 0); only the H x W real outputs are kept. The pins:
  * the oracle on the raw input equals the oracle's divisible-shape path on an input
    padded by hand with numpy, cropped (a different branch of the oracle, itself pinned
    by test_oracle_pins.py);
  * region means equal numpy's pad-reshape-mean;
  * at topk = S^2 the result is the closed form of dense attention over the real keys
    plus Hp*Wp - H*W extra keys of score 0 and value 0, plus scipy's LCE;
  * on a divisible shape nothing changes.
A divisor that counts only the real tokens, padded keys left out of the softmax, or a
cropping offset each fail at least two of these.
"""
import numpy as np
import pytest
import scipy.special

import oracle
from test_oracle_pins import inputs, lce_scipy

CASES = [  # N, H, W, C, heads, S, topk
    (1, 30, 30, 16, 2, 7, 3),     # a whole region row and column of padding (30 -> 35)
    (2, 13, 10, 8, 1, 4, 2),      # non-square, different pads (13 -> 16, 10 -> 12)
    (1, 16, 21, 8, 2, 4, 4),      # padding on the right only
    (1, 9, 9, 4, 1, 2, 1),        # one padded row and column of a 5 x 5 region
]


def pad(x, Hp, Wp):
    N, H, W, C = x.shape
    return np.pad(x, ((0, 0), (0, Hp - H), (0, Wp - W), (0, 0)))


def padded_size(H, W, S):
    return S * -(-H // S), S * -(-W // S)


@pytest.mark.parametrize("N,H,W,C,heads,S,topk", CASES)
def test_raw_input_equals_hand_padded_input_cropped(N, H, W, C, heads, S, topk):
    q, k, v, w, b = inputs(N, H, W, C, seed=300 + H + W)
    Hp, Wp = padded_size(H, W, S)
    out, r_idx, r_w = oracle.forward(q, k, v, w, b, heads, S, topk)
    out_p, r_idx_p, r_w_p = oracle.forward(pad(q, Hp, Wp), pad(k, Hp, Wp), pad(v, Hp, Wp), w, b, heads, S, topk)
    assert np.array_equal(r_idx, r_idx_p)
    np.testing.assert_allclose(r_w, r_w_p, rtol=0, atol=1e-14)
    np.testing.assert_allclose(out, out_p[:, :H, :W], rtol=0, atol=1e-13)


@pytest.mark.parametrize("N,H,W,C,heads,S,topk", CASES)
def test_region_means_over_the_padded_region(N, H, W, C, heads, S, topk):
    q = inputs(N, H, W, C, seed=400 + H)[0]
    Hp, Wp = padded_size(H, W, S)
    hr, wr = Hp // S, Wp // S
    want = pad(q, Hp, Wp).reshape(N, S, hr, S, wr, C).mean(axis=(2, 4)).reshape(N, S * S, C)
    np.testing.assert_allclose(oracle.region_mean(q, S), want, rtol=0, atol=1e-14)


@pytest.mark.parametrize("N,H,W,C,heads,S,topk", CASES)
def test_dense_limit_is_attention_with_zero_keys(N, H, W, C, heads, S, topk):
    q, k, v, w, b = inputs(N, H, W, C, seed=500 + H + W)
    Hp, Wp = padded_size(H, W, S)
    n_pad = Hp * Wp - H * W
    d = C // heads
    out, _, _ = oracle.forward(q, k, v, w, b, heads, S, S * S)
    lepe = lce_scipy(v, w, b)
    for n in range(N):
        Q = q[n].reshape(-1, heads, d) * d ** -0.5
        K = k[n].reshape(-1, heads, d)
        V = v[n].reshape(-1, heads, d)
        s = np.einsum("thd,uhd->htu", Q, K)                      # real keys
        s = np.concatenate([s, np.zeros(s.shape[:2] + (n_pad,))], axis=-1)  # + padded keys
        a = scipy.special.softmax(s, axis=-1)[..., :H * W]       # padded values are 0
        o = np.einsum("htu,uhd->thd", a, V).reshape(H, W, C)
        np.testing.assert_allclose(out[n], o + lepe[n], rtol=0, atol=1e-12)


def test_divisible_shape_is_unchanged():
    """On a divisible shape the padded grid is the plain one: the hand-padded input is the
    input itself, and the result equals the unpadded closed form pinned elsewhere."""
    q, k, v, w, b = inputs(1, 12, 12, 8, seed=77)
    out, r_idx, r_w = oracle.forward(q, k, v, w, b, 2, 4, 16)
    out2, _, _ = oracle.forward(pad(q, 12, 12), pad(k, 12, 12), pad(v, 12, 12), w, b, 2, 4, 16)
    assert np.array_equal(out, out2)
    d = 4
    Q = q[0].reshape(-1, 2, d) * d ** -0.5
    a = scipy.special.softmax(np.einsum("thd,uhd->htu", Q, k[0].reshape(-1, 2, d)), axis=-1)
    o = np.einsum("htu,uhd->thd", a, v[0].reshape(-1, 2, d)).reshape(12, 12, 8)
    np.testing.assert_allclose(out[0], o + lce_scipy(v, w, b)[0], rtol=0, atol=1e-12)
