"""Parity of the attention layer around BRA (qkv projection, BRA, output projection) and of
the projections alone with the float64 oracle, through the C ABI on a B200.

Tolerances: a projection result rounded to bfloat16 is within half an ulp of its
float32-accumulated value (2^-8 relative) plus the accumulation error, bounded here by
1e-4 times sum |x||w| + |b| (float32: 1e-5 times the same sum). The layer is checked by
oracle.compare.check_layer (routing set-exact off near ties, output within the forward's
tolerance); its r_weight is also checked within the forward's 1e-5 against the oracle's
routing of the q and k the GPU stored (read back through bra_qkv)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import compare
from vision_transformer_sparse_b200 import bra, synth

pytestmark = pytest.mark.gpu

TORCH = {"bf16": torch.bfloat16, "f32": torch.float32}


def rand(shape, seed, scale=1.0):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape) * scale


def store(a, dtype):
    a = np.asarray(a, dtype=np.float32)
    return synth.round_bf16(a) if dtype == "bf16" else a


def dev(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to("cuda").to(TORCH[dtype])


def host(t):
    return t.float().cpu().numpy().astype(np.float64)


def allowed(x, w, b, ref, dtype):
    scale = np.abs(x.astype(np.float64)) @ np.abs(w.astype(np.float64)).T + np.abs(b.astype(np.float64))
    if dtype == "bf16":
        return 2.0 ** -8 * np.abs(ref) + 1e-4 * scale
    return 2.0 ** -24 * np.abs(ref) + 1e-5 * scale


# (M, K, Nout): one row; a ragged 128-row tile; the qkv shapes of C = 128 and 256;
# a width that takes 32-column tiles; many tiles per CTA; the stage-2 batch's qkv.
LINEAR = [(1, 32, 32), (127, 64, 64), (300, 128, 384), (1000, 256, 768), (129, 96, 96), (5000, 128, 128),
          (50176, 128, 384)]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("M,K,Nout", LINEAR)
def test_linear_matches_oracle(M, K, Nout, dtype):
    seed = 1000 + M + K + Nout
    x = store(rand((M, K), seed), dtype)
    w = store(rand((Nout, K), seed + 1, K ** -0.5), dtype)
    b = store(rand((Nout,), seed + 2, 0.1), dtype)
    y = torch.full((M, Nout), float("nan"), dtype=TORCH[dtype], device="cuda")
    bra.linear(dev(x, dtype), dev(w, dtype), dev(b, dtype), out=y)
    torch.cuda.synchronize()
    got = host(y)
    ref = oracle.linear(x, w, b)
    assert np.all(np.isfinite(got))
    err = np.abs(got - ref)
    lim = allowed(x, w, b, ref, dtype)
    assert np.all(err <= lim), "max err %.3g, worst ratio %.3g" % (err.max(), (err / lim).max())
    assert bra.device_status() == 0


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("M,C", [(196, 64), (1000, 128), (333, 256)])
def test_qkv_writes_the_three_chunks(M, C, dtype):
    x = store(rand((M, C), 7 + C), dtype)
    w = store(rand((3 * C, C), 8 + C, C ** -0.5), dtype)
    b = store(rand((3 * C,), 9 + C, 0.1), dtype)
    q, k, v = bra.qkv(dev(x, dtype), dev(w, dtype), dev(b, dtype))
    torch.cuda.synchronize()
    ref = oracle.linear(x, w, b)
    lim = allowed(x, w, b, ref, dtype)
    for i, t in enumerate((q, k, v)):
        sl = slice(i * C, (i + 1) * C)
        assert np.all(np.abs(host(t) - ref[:, sl]) <= lim[:, sl]), "chunk %d" % i


def run_layer(inp, heads, S, topk, dtype):
    N, H, W, C = inp["x"].shape
    d = {k: dev(v, dtype) for k, v in inp.items()}
    out = torch.full((N, H, W, C), float("nan"), dtype=TORCH[dtype], device="cuda")
    r_idx = torch.full((N, S * S, topk), -1, dtype=torch.int32, device="cuda")
    r_w = torch.full((N, S * S, topk), float("nan"), dtype=torch.float32, device="cuda")
    bra.attention_layer(d["x"], d["w_qkv"], d["b_qkv"], d["w_o"], d["b_o"], d["lce_w"], d["lce_b"], heads, S, topk,
                        out=out, r_idx=r_idx, r_weight=r_w)
    torch.cuda.synchronize()
    assert bra.device_status() == 0
    return host(out), r_idx.cpu().numpy(), r_w.cpu().numpy()


# (N, H, W, C, heads, S, topk, dtype): ragged row tiles (196 tokens), the fused
# small-image path (cluster and routed forms), 256-token regions (tcgen05 attention),
# the pipeline kernel's shape, 32 channels, and float32.
LAYER = [
    (1, 14, 14, 64, 2, 7, 4, "bf16"),
    (2, 28, 28, 128, 4, 7, 4, "bf16"),
    (2, 14, 14, 256, 8, 7, 16, "bf16"),
    (1, 32, 32, 64, 2, 2, 1, "bf16"),
    (2, 64, 64, 128, 4, 8, 4, "bf16"),
    (1, 16, 16, 32, 1, 4, 2, "bf16"),
    (1, 56, 56, 64, 2, 7, 1, "f32"),
    (2, 14, 14, 64, 2, 7, 3, "f32"),
]


def check_routing_of_stored_qk(inp, heads, S, topk, dtype, r_idx, r_w):
    """The layer's routing is the routing of the q and k it stored: the oracle's float64
    routing of the GPU's own q and k (from bra_qkv, the same projection kernel) must give
    the layer's r_idx (set-exact off near ties) and r_weight within the forward's 1e-5."""
    q, k, _ = bra.qkv(dev(inp["x"], dtype), dev(inp["w_qkv"], dtype), dev(inp["b_qkv"], dtype))
    torch.cuda.synchronize()
    qh, kh = host(q), host(k)
    ref_idx, ref_w, logits = oracle.route(qh, kh, heads, S, topk, with_logits=True)
    rep = compare.Report()
    compare.check_routing(logits, ref_idx, ref_w, r_idx, r_w, rep, tol_weight=compare.TOL_WEIGHT)
    assert rep.ok, rep.notes[:2000]


@pytest.mark.parametrize("N,H,W,C,heads,S,topk,dtype", LAYER)
def test_layer_matches_oracle(N, H, W, C, heads, S, topk, dtype):
    w = synth.Workload("layer_case", 40 + C + topk, N, H, W, C, heads, S, topk, dtype, lce_b_std=0.01)
    inp = synth.make_layer_inputs(w)
    out, r_idx, r_w = run_layer(inp, heads, S, topk, dtype)
    rep = compare.check_layer(inp, heads, S, topk, dtype, out, r_idx, r_w)
    assert rep.ok, rep.notes
    check_routing_of_stored_qk(inp, heads, S, topk, dtype, r_idx, r_w)


@pytest.mark.parametrize("name", ["cls_stage2_224", "det_stage1_1024", "stage1_tiny_224"])
def test_layer_full_workload(name):
    """The benchmark workloads' full sizes, every element checked."""
    w = synth.WORKLOADS[name]
    inp = synth.make_layer_inputs(w)
    out, r_idx, r_w = run_layer(inp, w.heads, w.S, w.topk, w.dtype)
    rep = compare.check_layer(inp, w.heads, w.S, w.topk, w.dtype, out, r_idx, r_w)
    assert rep.ok, rep.notes
    check_routing_of_stored_qk(inp, w.heads, w.S, w.topk, w.dtype, r_idx, r_w)
