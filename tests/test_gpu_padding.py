"""The padded grid on a B200: feature maps whose height or width is not a multiple of S.

Reading (bernice.tw BiFormer notes, section "消融實驗", which name padding's cost as the
reason S is chosen per task): q, k, v zero-padded at the bottom and right to multiples
of S, region means over whole padded regions, padded tokens taking part as keys with
k = v = 0, the H x W real outputs kept. The oracle implements the same reading and is
pinned against a hand-padded input (tests/test_oracle_padding_pins.py). Every shape below
runs under every kernel variant, through bra_forward, and the entry points that take the
padded path (bra_route, bra_attend, bra_forward_host, bra_attention_layer) are checked
on one shape each. Outputs start as NaN so that a pixel the crop misses cannot pass.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import compare
from test_gpu_parity import any_variant, assert_parity, to_dev  # noqa: F401  (fixture)
from vision_transformer_sparse_b200 import bra, synth

pytestmark = pytest.mark.gpu

PADDED = [
    # N, H, W, C, heads, S, topk, dtype
    (1, 30, 30, 64, 2, 7, 3, "bf16"),     # 30 -> 35: a whole region row and column of padding
    (2, 13, 10, 64, 2, 4, 2, "bf16"),     # 13 -> 16, 10 -> 12: different pads per axis
    (1, 60, 60, 128, 4, 8, 4, "bf16"),    # 60 -> 64: 64-token regions (pipeline kernel)
    (1, 30, 31, 64, 2, 2, 1, "bf16"),     # 30 -> 32, 31 -> 32: 256-token regions (tcgen05)
    (1, 26, 27, 256, 8, 7, 16, "bf16"),   # 26 -> 28: topk 16 (routed fused form)
    (2, 12, 14, 64, 2, 7, 49, "bf16"),    # 12 -> 14: dense limit, padded keys in every row
    (1, 50, 54, 64, 2, 7, 1, "f32"),      # f32, 50 -> 56
    (1, 16, 21, 64, 2, 4, 4, "f32"),      # f32, padding on the right only
]


def workload(shape):
    N, H, W, C, heads, S, topk, dtype = shape
    return synth.Workload("padded", 60 + sum(shape[:7]), N, H, W, C, heads, S, topk, dtype,
                          region_bias=0.5, lce_b_std=0.05, lce_w_std=0.1)


@pytest.mark.parametrize("shape", PADDED, ids=lambda s: "x".join(map(str, s)))
def test_padded_shapes(shape, any_variant):  # noqa: F811
    w = workload(shape)
    assert_parity(w, synth.make_inputs(w))
    assert bra.device_status() == 0


def test_padded_route_and_attend_entry_points():
    w = workload((2, 30, 30, 64, 2, 7, 3, "bf16"))
    inp = synth.make_inputs(w)
    d = to_dev(inp, w.dtype)
    r_idx, r_w = bra.route(d["q"], d["k"], w.heads, w.S, w.topk)
    _, f_idx, f_w = bra.forward(d["q"], d["k"], d["v"], d["lce_w"], d["lce_b"], w.heads, w.S, w.topk)
    assert torch.equal(r_idx, f_idx) and torch.equal(r_w, f_w)
    ref_idx, ref_w, logits = oracle.route(inp["q"], inp["k"], w.heads, w.S, w.topk, with_logits=True)
    rep = compare.Report()
    compare.check_routing(logits, ref_idx, ref_w, r_idx.cpu().numpy(), r_w.cpu().numpy(), rep)
    assert rep.ok, rep.notes
    # attention over a caller's routing: reversed rows, a repeated region
    given = ref_idx[:, :, ::-1].copy()
    given[:, 0, 1] = given[:, 0, 0]
    out = torch.full_like(d["q"], float("nan"))
    bra.attend(d["q"], d["k"], d["v"], d["lce_w"], d["lce_b"], w.heads, w.S,
               torch.from_numpy(given).cuda(), out=out)
    torch.cuda.synchronize()
    ref = oracle.attend(inp["q"], inp["k"], inp["v"], inp["lce_w"], inp["lce_b"], w.heads, w.S, given)
    rep = compare.Report()
    compare.check_output(out.float().cpu().numpy(), ref, w.dtype, rep)
    assert rep.ok, rep.notes


def test_padded_host_entry_point():
    w = workload((3, 13, 10, 64, 2, 4, 2, "bf16"))
    inp = synth.make_inputs(w)
    h = {k: torch.from_numpy(v).to(torch.bfloat16).pin_memory() for k, v in inp.items()}
    out = torch.full((w.N, w.H, w.W, w.C), float("nan"), dtype=torch.bfloat16).pin_memory()
    r_idx = torch.full((w.N, w.regions, w.topk), -1, dtype=torch.int32).pin_memory()
    r_w = torch.full((w.N, w.regions, w.topk), float("nan"), dtype=torch.float32).pin_memory()
    bra.forward_host(h["q"], h["k"], h["v"], h["lce_w"], h["lce_b"], w.heads, w.S, w.topk, out=out, r_idx=r_idx,
                     r_weight=r_w)
    rep = compare.check_forward(inp, w.heads, w.S, w.topk, w.dtype, out.float().numpy(), r_idx.numpy(), r_w.numpy())
    assert rep.ok, rep.notes


@pytest.mark.parametrize("shape", [(2, 30, 30, 64, 2, 7, 3, "bf16"), (1, 50, 54, 64, 2, 7, 1, "f32")],
                         ids=lambda s: "x".join(map(str, s)))
def test_padded_attention_layer(shape):
    w = workload(shape)
    inp = synth.make_layer_inputs(w)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    d = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda().to(dt) for k, v in inp.items()}
    out = torch.full((w.N, w.H, w.W, w.C), float("nan"), dtype=dt, device="cuda")
    r_idx = torch.full((w.N, w.regions, w.topk), -1, dtype=torch.int32, device="cuda")
    r_w = torch.full((w.N, w.regions, w.topk), float("nan"), dtype=torch.float32, device="cuda")
    bra.attention_layer(d["x"], d["w_qkv"], d["b_qkv"], d["w_o"], d["b_o"], d["lce_w"], d["lce_b"], w.heads, w.S,
                        w.topk, out=out, r_idx=r_idx, r_weight=r_w)
    torch.cuda.synchronize()
    rep = compare.check_layer(inp, w.heads, w.S, w.topk, w.dtype, out.float().cpu().numpy(), r_idx.cpu().numpy(),
                              r_w.cpu().numpy())
    assert rep.ok, rep.notes
