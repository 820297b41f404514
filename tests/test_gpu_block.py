"""The BiFormer block (bra_block) and its MLP layers (bra_linear_act) on a B200, against
the float64 block oracle (oracle/block.py, pinned in tests/test_oracle_block_pins.py).

The block as the niftyadmin walk-through prints it (section "2、BiFormer Block" and the
module printout of "网络结构"): x + pos_embed(x), the pre-norm attention layer, the
pre-norm MLP (Linear C -> 3C, GELU, Linear 3C -> C), every stored intermediate rounded to
the dtype on both sides. Routing: set-exact off near ties against the oracle's routing of
its own norm1 output, r_weight within the layer tolerance (a float32-accumulated LayerNorm
or projection can round a stored element to the neighbouring bf16 value). Output: against
the oracle block run over the GPU's routing, so that near-tie rows are checked too, within
the forward's tolerance taken of the magnitudes of the two stored terms the output adds:
for bf16 |out - ref| <= 2e-2 + 1e-2 (|x2| + |m| + |ref|), where out = x2 + m with x2 and m
each rounded to bf16 on both sides. The two sides may round x2 or m to neighbouring bf16
values (one ulp is 2^-8 relative to the term), and where the terms cancel (x2 = 2.0,
m = -1.8) such a difference is large relative to |ref|; the forward's |ref|-relative form
does not describe a sum of rounded terms. float32: the forward's 1e-4.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import block as ob
from oracle import compare
from vision_transformer_sparse_b200 import bra, synth

pytestmark = pytest.mark.gpu

TORCH = {"bf16": torch.bfloat16, "f32": torch.float32}


def dev(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda().to(TORCH[dtype])


def rand(shape, seed, scale=1.0):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape) * scale


def store(a, dtype):
    a = np.asarray(a, dtype=np.float32)
    return synth.round_bf16(a) if dtype == "bf16" else a


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("M,K,Nout", [(1, 64, 192), (300, 128, 384), (1000, 256, 768), (777, 192, 64),
                                      (5000, 384, 128)])
def test_mlp_epilogues(M, K, Nout, dtype):
    """GELU and residual epilogues of the projection GEMM against float64: the bf16 result
    is within one rounding (2^-8 relative per rounding) of the exact value plus the float32
    accumulation error (1e-4 of sum |x||w| + |b|, float32 1e-5)."""
    x = store(rand((M, K), M + K), dtype)
    w = store(rand((Nout, K), M + K + 1, K ** -0.5), dtype)
    b = store(rand((Nout,), M + K + 2, 0.1), dtype)
    res = store(rand((M, Nout), M + K + 3), dtype)
    t = oracle.linear(x, w, b)
    scale = np.abs(x.astype(np.float64)) @ np.abs(w.astype(np.float64)).T + np.abs(b.astype(np.float64))
    acc = (1e-4 if dtype == "bf16" else 1e-5) * scale
    ulp = 2.0 ** -8 if dtype == "bf16" else 2.0 ** -23
    for act in (bra.ACT_GELU, bra.ACT_RESIDUAL):
        y = torch.full((M, Nout), float("nan"), dtype=TORCH[dtype], device="cuda")
        bra.linear_act(dev(x, dtype), dev(w, dtype), dev(b, dtype), act,
                       res=dev(res, dtype) if act == bra.ACT_RESIDUAL else None, out=y)
        torch.cuda.synchronize()
        got = y.float().cpu().numpy().astype(np.float64)
        if act == bra.ACT_GELU:
            ref = ob.gelu(t)
            lim = ulp * np.abs(ref) + 1.2 * acc + 1e-30
        else:
            ref = res.astype(np.float64) + t
            lim = ulp * (np.abs(t) + np.abs(ref)) + acc + 1e-30
        err = np.abs(got - ref)
        assert np.all(np.isfinite(got))
        assert np.all(err <= lim), "act %d: max err %.3g, worst ratio %.3g" % (act, err.max(), (err / lim).max())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_gelu_erf_within_its_bound(dtype):
    """The epilogue's GELU takes erf from Abramowitz and Stegun's formula 7.1.26, whose
    absolute error is at most 1.5e-7 in exact arithmetic. Evaluated in float32 as
    1 - P(t) e with t and e from the MUFU (relative errors about 2^-22) and P a
    five-term Horner sum (a few float32 roundings of a value below 1), P e carries at
    most ~4.5e-7 of absolute error, which 1 - P e keeps where erf is small. So the
    kernel's erf is within 6e-7 of the exact one and GELU(x) = x (1 + erf(x / sqrt 2)) / 2
    within 3e-7 |x| (plus two float32 roundings and one of the stored dtype). Checked on
    65,536 values over [-10, 10] and a few special points, through an identity weight so
    that the GEMM adds nothing."""
    M, K = 1024, 64
    x = np.linspace(-10.0, 10.0, M * K).reshape(M, K)
    x[0, :8] = [0.0, -0.0, 1e-30, -1e-30, 1e-6, -1e-6, 38.0, -38.0]
    x = store(x, dtype)
    w = np.eye(K)
    b = np.zeros(K)
    y = torch.full((M, K), float("nan"), dtype=TORCH[dtype], device="cuda")
    bra.linear_act(dev(x, dtype), dev(w, dtype), dev(b, dtype), bra.ACT_GELU, out=y)
    torch.cuda.synchronize()
    got = y.float().cpu().numpy().astype(np.float64)
    ref = ob.gelu(x.astype(np.float64))
    ulp = 2.0 ** -8 if dtype == "bf16" else 2.0 ** -23
    lim = 3e-7 * np.abs(x) + (ulp + 2.0 ** -22) * np.abs(ref) + 1e-38
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got))
    assert np.all(err <= lim), "max err %.3g, worst ratio %.3g at x = %.6g" % (
        err.max(), (err / lim).max(), x.flat[np.argmax(err / lim)])


def run_block(w, inp):
    dt = TORCH[w.dtype]
    d = {k: dev(v, w.dtype) for k, v in inp.items()}
    out = torch.full((w.N, w.H, w.W, w.C), float("nan"), dtype=dt, device="cuda")
    r_idx = torch.full((w.N, w.regions, w.topk), -1, dtype=torch.int32, device="cuda")
    r_w = torch.full((w.N, w.regions, w.topk), float("nan"), dtype=torch.float32, device="cuda")
    bra.block(d["x"], d, w.heads, w.S, w.topk, out=out, r_idx=r_idx, r_weight=r_w)
    torch.cuda.synchronize()
    assert bra.device_status() == 0
    return out.float().cpu().numpy(), r_idx.cpu().numpy(), r_w.cpu().numpy()


def check_block(w, inp, out, r_idx, r_w):
    p = {k: v for k, v in inp.items() if k != "x"}
    ref, _, _, mid = ob.block_forward(inp["x"], p, w.heads, w.S, w.topk, w.dtype, r_idx_given=r_idx,
                                      intermediates=True)
    # the layer's routing from the oracle's own norm1 output
    _, _, _, lmid = oracle.layer_forward(mid["h"], p["w_qkv"], p["b_qkv"], p["w_o"], p["b_o"], p["lce_w"],
                                         p["lce_b"], w.heads, w.S, w.topk, w.dtype, intermediates=True)
    ref_idx, ref_w, logits = oracle.route(lmid["q"], lmid["k"], w.heads, w.S, w.topk, with_logits=True)
    rep = compare.Report()
    compare.check_routing(logits, ref_idx, ref_w, r_idx, r_w, rep,
                          tol_weight=compare.TOL_LAYER_WEIGHT if w.dtype == "bf16" else compare.TOL_WEIGHT)
    assert rep.ok, rep.notes[:2000]
    compare.check_output(out, ref, w.dtype, rep, scale=np.abs(mid["x2"]) + np.abs(mid["m"]) + np.abs(ref))
    print("%s: near ties %d, out max err %.3e (worst/allowed %.3f)" % (
        w.name, rep.near_tie_rows, rep.out_max_abs_err, rep.out_worst_ratio))
    assert rep.ok, rep.notes[:2000]


BLOCKS = [
    # N, H, W, C, heads, S, topk, dtype
    (2, 28, 28, 128, 4, 7, 4, "bf16"),    # classification stage 2 (fused cluster form)
    (2, 14, 14, 256, 8, 7, 16, "bf16"),   # stage 3, topk 16 (routed fused form), C = 256
    (1, 32, 32, 64, 2, 2, 1, "bf16"),     # 256-token regions (tcgen05 attention)
    (1, 64, 64, 128, 4, 8, 4, "bf16"),    # 64-token regions (pipeline attention)
    (1, 30, 30, 64, 2, 7, 3, "bf16"),     # the padded grid (30 -> 35)
    (1, 16, 16, 32, 1, 4, 2, "bf16"),     # C = 32: half the lanes of a warp hold channels
    (1, 14, 14, 96, 3, 7, 2, "bf16"),     # C = 96: two channel pairs on half the lanes
    (1, 14, 14, 64, 2, 7, 2, "f32"),      # float32
    (1, 20, 18, 128, 4, 5, 3, "f32"),     # float32, padded (20 -> 20, 18 -> 20)
]


@pytest.mark.parametrize("shape", BLOCKS, ids=lambda s: "x".join(map(str, s)))
def test_block_matches_oracle(shape):
    N, H, W, C, heads, S, topk, dtype = shape
    w = synth.Workload("block", 80 + sum(shape[:7]), N, H, W, C, heads, S, topk, dtype, region_bias=0.5,
                       lce_b_std=0.01)
    inp = synth.make_block_inputs(w)
    check_block(w, inp, *run_block(w, inp))


def test_block_full_classification_stage():
    """The classification stage-2 workload at its full size (64 images), every element."""
    w = synth.WORKLOADS["cls_stage2_224"]
    inp = synth.make_block_inputs(w)
    check_block(w, inp, *run_block(w, inp))
