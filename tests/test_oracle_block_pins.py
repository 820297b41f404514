"""Pins for the BiFormer block oracle (oracle/block.py), CPU only: each part against the
PyTorch module the walk-through prints (Conv2d groups=C, LayerNorm eps 1e-6, GELU,
Linear), closed forms, and the whole block against a composition of those modules with
the pinned attention-layer oracle."""
import numpy as np
import pytest
import scipy.signal
import torch

import oracle
from oracle import block as ob


def rand(shape, seed, scale=1.0):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape) * scale


def params(C, seed):
    g = C ** -0.5
    return {
        "pos_w": rand((C, 3, 3), seed, 0.2), "pos_b": rand((C,), seed + 1, 0.05),
        "ln1_g": 1 + rand((C,), seed + 2, 0.1), "ln1_b": rand((C,), seed + 3, 0.05),
        "ln2_g": 1 + rand((C,), seed + 4, 0.1), "ln2_b": rand((C,), seed + 5, 0.05),
        "w_qkv": rand((3 * C, C), seed + 6, g), "b_qkv": rand((3 * C,), seed + 7, 0.02),
        "w_o": rand((C, C), seed + 8, g), "b_o": rand((C,), seed + 9, 0.02),
        "lce_w": rand((C, 5, 5), seed + 10, 0.05), "lce_b": rand((C,), seed + 11, 0.01),
        "mlp_w1": rand((3 * C, C), seed + 12, g), "mlp_b1": rand((3 * C,), seed + 13, 0.02),
        "mlp_w2": rand((C, 3 * C), seed + 14, (3 * C) ** -0.5), "mlp_b2": rand((C,), seed + 15, 0.02),
    }


def t(a):
    return torch.tensor(np.asarray(a), dtype=torch.float64)


def test_dwconv3_is_the_grouped_conv2d():
    x, w, b = rand((2, 5, 6, 4), 1), rand((4, 3, 3), 2), rand((4,), 3)
    ref = torch.nn.functional.conv2d(t(x).permute(0, 3, 1, 2), t(w)[:, None], t(b), padding=1, groups=4)
    np.testing.assert_allclose(ob.dwconv3(x, w, b), ref.permute(0, 2, 3, 1).numpy(), rtol=1e-12, atol=1e-12)
    # and a single channel against scipy's cross-correlation
    ref0 = scipy.signal.correlate2d(x[0, :, :, 0], w[0], mode="same") + b[0]
    np.testing.assert_allclose(ob.dwconv3(x, w, b)[0, :, :, 0], ref0, rtol=1e-12, atol=1e-12)


def test_layer_norm_matches_torch_and_constant_rows_give_beta():
    x, g, b = rand((3, 7, 16), 4), rand((16,), 5), rand((16,), 6)
    ref = torch.nn.functional.layer_norm(t(x), (16,), t(g), t(b), eps=1e-6)
    np.testing.assert_allclose(ob.layer_norm(x, g, b), ref.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(ob.layer_norm(np.full((2, 16), 3.5), g, b), np.broadcast_to(b, (2, 16)), atol=1e-12)


def test_gelu_is_the_exact_erf_form():
    x = rand((1000,), 7, 3)
    np.testing.assert_allclose(ob.gelu(x), torch.nn.functional.gelu(t(x)).numpy(), rtol=1e-12, atol=1e-14)
    assert ob.gelu(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(ob.gelu(np.array([10.0, -10.0])), [10.0, 0.0], atol=1e-12)


def test_zero_branches_leave_the_positional_residual():
    """Output projection and second MLP layer set to zero: both residual branches add
    nothing, so the block is x + pos_embed(x) (float32 storage)."""
    N, H, W, C = 1, 8, 8, 16
    p = params(C, 20)
    p.update(w_o=np.zeros((C, C)), b_o=np.zeros(C), mlp_w2=np.zeros((C, 3 * C)), mlp_b2=np.zeros(C))
    x = rand((N, H, W, C), 21)
    out, _, _ = ob.block_forward(x, p, 2, 2, 2, "f32")
    ref = oracle.round_to(x + ob.dwconv3(x, p["pos_w"], p["pos_b"]), "f32")
    np.testing.assert_allclose(out, ref, rtol=0, atol=0)


def torch_block(x, p, heads, S, topk):
    """The block from torch modules (float64, float32 rounding at the same stored points),
    with the attention layer from the pinned layer oracle."""
    C = x.shape[-1]
    f32 = lambda a: a.float().double()
    conv = torch.nn.Conv2d(C, C, 3, padding=1, groups=C).double()
    ln1, ln2 = torch.nn.LayerNorm(C, eps=1e-6).double(), torch.nn.LayerNorm(C, eps=1e-6).double()
    mlp = torch.nn.Sequential(torch.nn.Linear(C, 3 * C), torch.nn.Identity(), torch.nn.GELU(),
                              torch.nn.Linear(3 * C, C)).double()
    with torch.no_grad():
        conv.weight.copy_(t(p["pos_w"])[:, None])
        conv.bias.copy_(t(p["pos_b"]))
        for ln, g, b in ((ln1, "ln1_g", "ln1_b"), (ln2, "ln2_g", "ln2_b")):
            ln.weight.copy_(t(p[g]))
            ln.bias.copy_(t(p[b]))
        mlp[0].weight.copy_(t(p["mlp_w1"]))
        mlp[0].bias.copy_(t(p["mlp_b1"]))
        mlp[3].weight.copy_(t(p["mlp_w2"]))
        mlp[3].bias.copy_(t(p["mlp_b2"]))
        X = t(x)
        X = f32(X + conv(X.permute(0, 3, 1, 2)).permute(0, 2, 3, 1))
        h = f32(ln1(X))
        a, _, _ = oracle.layer_forward(h.numpy(), p["w_qkv"], p["b_qkv"], p["w_o"], p["b_o"], p["lce_w"],
                                       p["lce_b"], heads, S, topk, "f32")
        X = f32(X + f32(t(a)))
        h = f32(ln2(X))
        hid = f32(mlp[2](mlp[1](mlp[0](h))))
        return (X + f32(mlp[3](hid))).numpy()


@pytest.mark.parametrize("shape", [(1, 8, 8, 16, 2, 2, 2), (2, 12, 12, 32, 2, 3, 4)])
def test_block_matches_torch_modules(shape):
    N, H, W, C, heads, S, topk = shape
    p = params(C, 30 + C)
    x = rand((N, H, W, C), 31 + C)
    out, _, _ = ob.block_forward(x, p, heads, S, topk, "f32")
    np.testing.assert_allclose(out, torch_block(x, p, heads, S, topk), rtol=1e-6, atol=1e-6)
