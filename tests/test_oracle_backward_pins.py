"""Pins for the backward oracle (oracle/backward.py), CPU only.

The backward of the path (routing detached, as the walk-through's router does when
`diff_routing` is off) is pinned against things it shares no code with:
  * central finite differences of the pinned forward oracle (`oracle.attend` over the
    same fixed routing), element by element, including a routing row with a repeated
    region (its keys count twice);
  * PyTorch autograd in float64 on a dense multi-head attention whose keys outside the
    query's routed regions are masked out (regions taken from pixel coordinates), plus a
    grouped Conv2d for the LCE: a textbook formulation with no gather;
  * closed forms of the LCE gradients (bias = sum of dout; weight = cross-correlation of
    the zero-padded V with dout) and linearity in dout.
A slip such as a missing softmax-Jacobian term, a transposed score, keys not
scatter-added back, a lost scale factor or a flipped LCE kernel fails at least one.
"""
import numpy as np
import pytest
import scipy.signal
import torch

import oracle
from oracle import backward as ob


def rand(shape, seed, scale=1.0):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape) * scale


def case(N, H, W, C, seed):
    q, k, v = (rand((N, H, W, C), seed + i) for i in range(3))
    w = rand((C, 5, 5), seed + 3, 0.2)
    b = rand((C,), seed + 4, 0.1)
    g = rand((N, H, W, C), seed + 5)
    return q, k, v, w, b, g


def loss(q, k, v, w, b, heads, S, r_idx, g):
    return float(np.sum(g * oracle.attend(q, k, v, w, b, heads, S, r_idx)))


@pytest.mark.parametrize("dup", [False, True])
def test_finite_differences_every_element(dup):
    """Central differences (h = 1e-5, float64) of sum(dout * attend) against every element of
    the analytic gradients; with `dup`, one routing row selects the same region twice."""
    N, H, W, C, heads, S = 1, 4, 4, 4, 2, 2
    q, k, v, w, b, g = case(N, H, W, C, 30)
    r_idx, _ = oracle.route(q, k, heads, S, 2)
    if dup:
        r_idx = r_idx.copy()
        r_idx[0, 1] = [3, 3]
    grads = ob.backward(q, k, v, w, b, heads, S, r_idx, g)
    h = 1e-5
    args = {"q": q, "k": k, "v": v, "w": w, "b": b}
    names = {"q": "dq", "k": "dk", "v": "dv", "w": "dlce_w", "b": "dlce_b"}
    for key, arr in args.items():
        num = np.empty_like(arr)
        flat = arr.reshape(-1)
        for i in range(flat.size):
            old = flat[i]
            flat[i] = old + h
            lp = loss(**args, heads=heads, S=S, r_idx=r_idx, g=g)
            flat[i] = old - h
            lm = loss(**args, heads=heads, S=S, r_idx=r_idx, g=g)
            flat[i] = old
            num.reshape(-1)[i] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(grads[names[key]], num, rtol=1e-6, atol=1e-7, err_msg=key)


def masked_dense_reference(q, k, v, w, b, heads, S, r_idx, g):
    """Autograd gradients of a dense, region-masked attention plus a grouped Conv2d."""
    N, H, W, C = q.shape
    d = C // heads
    hr, wr = H // S, W // S
    ys, xs = np.meshgrid(np.arange(H), np.arange(W), indexing="ij")
    reg = ((ys // hr) * S + xs // wr).reshape(-1)
    T = [torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v, w, b)]
    tq, tk, tv, tw, tb = T
    outs = []
    for n in range(N):
        allowed = np.zeros((S * S, S * S), bool)
        for p in range(S * S):
            allowed[p, r_idx[n, p]] = True
        mask = torch.tensor(allowed[reg][:, reg])
        Q = tq[n].reshape(H * W, heads, d) * d ** -0.5
        K = tk[n].reshape(H * W, heads, d)
        V = tv[n].reshape(H * W, heads, d)
        s = torch.einsum("thd,uhd->htu", Q, K).masked_fill(~mask[None], float("-inf"))
        att = torch.einsum("htu,uhd->thd", torch.softmax(s, dim=-1), V).reshape(H, W, C)
        lce = torch.nn.functional.conv2d(tv[n].permute(2, 0, 1)[None], tw[:, None], tb, padding=2, groups=C)
        outs.append(att + lce[0].permute(1, 2, 0))
    L = (torch.stack(outs) * torch.tensor(g)).sum()
    L.backward()
    return {"dq": tq.grad.numpy(), "dk": tk.grad.numpy(), "dv": tv.grad.numpy(), "dlce_w": tw.grad.numpy(),
            "dlce_b": tb.grad.numpy()}


@pytest.mark.parametrize("shape", [(2, 8, 8, 16, 2, 2, 2), (1, 12, 12, 32, 2, 3, 4), (1, 8, 8, 8, 1, 4, 16)])
def test_matches_autograd_of_masked_dense_attention(shape):
    N, H, W, C, heads, S, topk = shape
    q, k, v, w, b, g = case(N, H, W, C, 40 + C)
    r_idx, _ = oracle.route(q, k, heads, S, topk)
    got = ob.backward(q, k, v, w, b, heads, S, r_idx, g)
    ref = masked_dense_reference(q, k, v, w, b, heads, S, r_idx, g)
    for name in ref:
        np.testing.assert_allclose(got[name], ref[name], rtol=1e-9, atol=1e-10, err_msg=name)


def test_lce_gradient_closed_forms():
    """db = sum of dout over images and pixels; dw[c] = cross-correlation of the
    zero-padded V with dout (scipy), i.e. sum over pixels of dout * shifted V."""
    N, H, W, C = 2, 6, 7, 3
    _, _, v, w, b, g = case(N, H, W, C, 50)
    dv, dw, db = ob.lce_backward(v, w, g)
    np.testing.assert_allclose(db, g.sum(axis=(0, 1, 2)), rtol=1e-12)
    for c in range(C):
        ref = sum(scipy.signal.correlate2d(np.pad(v[n, :, :, c], 2), g[n, :, :, c], mode="valid") for n in range(N))
        np.testing.assert_allclose(dw[c], ref, rtol=1e-10, atol=1e-12)
        # dv = dout correlated with the kernel flipped in both axes ("full" convolution, cropped)
        for n in range(N):
            ref_dv = scipy.signal.convolve2d(g[n, :, :, c], w[c], mode="same")
            np.testing.assert_allclose(dv[n, :, :, c], ref_dv, rtol=1e-10, atol=1e-12)


def test_linear_in_dout():
    N, H, W, C, heads, S = 1, 8, 8, 8, 2, 2
    q, k, v, w, b, g = case(N, H, W, C, 60)
    g2 = rand(g.shape, 61)
    r_idx, _ = oracle.route(q, k, heads, S, 2)
    a = ob.backward(q, k, v, w, b, heads, S, r_idx, g)
    c = ob.backward(q, k, v, w, b, heads, S, r_idx, g2)
    s = ob.backward(q, k, v, w, b, heads, S, r_idx, g + 3 * g2)
    for name in a:
        np.testing.assert_allclose(s[name], a[name] + 3 * c[name], rtol=1e-10, atol=1e-10)


def test_region_pixels_cover_the_image_once():
    for H, W, S in ((8, 8, 2), (12, 6, 3), (4, 4, 4)):
        pix = ob.region_pixels(H, W, S)
        assert sorted(pix.reshape(-1).tolist()) == list(range(H * W))
        # region p = j*S + i holds rows j*hr.., columns i*wr..; tokens row-major
        hr, wr = H // S, W // S
        assert pix[1, 0] == wr and pix[S, 0] == hr * W
        if wr > 1:
            assert pix[0, 1] == 1
