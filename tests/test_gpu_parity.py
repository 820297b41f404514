"""Parity of the CUDA path (through the C ABI) with the float64 oracle, on a B200.

Every BiFormer stage workload runs at its full size — the size the benchmark
launches — and is compared element by element. Edge cases: empty batch, one-token
regions, the dense limit topk = S^2, ragged key chunks, non-square regions, d = 64,
duplicated and out-of-range region indices, host-buffer entry point, determinism.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import compare
from vision_transformer_sparse_b200 import bra, synth

pytestmark = pytest.mark.gpu

TDT = {"f32": torch.float32, "bf16": torch.bfloat16}


def to_dev(inp, dtype):
    return {k: torch.from_numpy(v).to("cuda").to(TDT[dtype]).contiguous() for k, v in inp.items()}


def run_forward(w: synth.Workload, inp):
    d = to_dev(inp, w.dtype)
    # outputs start as NaN / -1, so that an element the kernels leave unwritten fails
    # instead of passing on whatever an earlier test left in that memory
    out = torch.full_like(d["q"], float("nan"))
    r_idx = torch.full((w.N, w.regions, w.topk), -1, dtype=torch.int32, device="cuda")
    r_w = torch.full((w.N, w.regions, w.topk), float("nan"), dtype=torch.float32, device="cuda")
    bra.forward(d["q"], d["k"], d["v"], d["lce_w"], d["lce_b"], w.heads, w.S, w.topk, out=out, r_idx=r_idx,
                r_weight=r_w)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), r_idx.cpu().numpy(), r_w.cpu().numpy()


def assert_parity(w: synth.Workload, inp, res=None):
    out, r_idx, r_w = run_forward(w, inp) if res is None else res
    rep = compare.check_forward(inp, w.heads, w.S, w.topk, w.dtype, out, r_idx, r_w)
    print("%s: rows %d near-tie %d weight err %.2e out max err %.3e (worst/allowed %.3f)" % (
        w.name, rep.rows, rep.near_tie_rows, rep.weight_max_err, rep.out_max_abs_err, rep.out_worst_ratio))
    assert rep.ok, rep.notes[:2000]
    return rep


@pytest.fixture(scope="module", autouse=True)
def _lib(bra_lib):
    assert torch.cuda.is_available()
    return bra_lib


VARIANTS = {"auto": 0, "generic": 1, "tma": 2, "split": 3, "pipe": 4}


@pytest.fixture(params=["auto", "split", "pipe", "generic"])
def variant(request):
    """Run a test under the automatic kernel choice (the fused one-kernel forward for
    small images, else region means + routing + the tcgen05 attention kernel for
    128/256-token regions or the persistent mma.sync pipeline), the three-kernel path
    forced, the mma.sync pipeline forced, and the generic cp.async attention kernel
    forced."""
    prev = bra.set_kernel_variant(VARIANTS[request.param])
    yield request.param
    bra.set_kernel_variant(prev)


@pytest.fixture(params=["auto", "split", "pipe", "generic", "tma"])
def any_variant(request):
    """Every kernel variant, including the one-unit-per-CTA TMA attention kernel."""
    prev = bra.set_kernel_variant(VARIANTS[request.param])
    yield request.param
    bra.set_kernel_variant(prev)


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_stage_workloads_full_size(name, variant):
    w = synth.WORKLOADS[name]
    assert_parity(w, synth.make_inputs(w))
    assert bra.device_status() == 0


SMALL = [
    # N, H, W, C, heads, S, topk, dtype
    (2, 16, 16, 64, 2, 4, 3, "bf16"),     # 16-token regions, 48 keys (ragged chunk)
    (1, 24, 24, 128, 4, 3, 5, "bf16"),    # 64-token regions, 320 keys (5 chunks)
    (3, 12, 8, 64, 2, 4, 2, "bf16"),      # non-square regions 3x2, 12 keys
    (2, 9, 9, 64, 1, 3, 9, "bf16"),       # d = 64, 3x3 regions, dense limit, 81 keys
    (1, 8, 8, 64, 2, 8, 5, "bf16"),       # one-token regions
    (1, 30, 20, 128, 2, 5, 7, "bf16"),    # d = 64, 6x4 regions (24 queries), 168 keys
    (2, 32, 32, 64, 2, 2, 4, "bf16"),     # 256-token regions, dense limit, 1024 keys
    (1, 14, 14, 64, 2, 7, 49, "f32"),     # f32 dense limit
    (2, 12, 18, 128, 2, 3, 4, "f32"),     # f32, d = 64, non-square
    (1, 16, 16, 64, 2, 16, 3, "f32"),     # f32 one-token regions, S = 16
    (1, 60, 60, 96, 3, 5, 2, "bf16"),     # 3 heads, 12x12 regions split over 6 CTAs
    (1, 12, 12, 64, 2, 6, 5, "bf16"),     # 2x2 regions, 20 keys (ragged chunk), fused path
    (2, 8, 8, 256, 8, 2, 2, "bf16"),      # 8 heads: a cluster of 8 CTAs per image
    (3, 20, 20, 64, 2, 5, 7, "bf16"),     # 4x4 regions, 112 keys (two chunks), borders
    (1, 32, 32, 64, 2, 2, 1, "bf16"),     # 256-token regions, 256 keys: tcgen05 kernel
    (2, 16, 32, 64, 2, 2, 2, "bf16"),     # 8x16 regions, topk 2 -> 256 keys: tcgen05
    (1, 16, 32, 128, 4, 2, 1, "bf16"),    # 8x16 regions, 128 keys, 4 heads: tcgen05
    (3, 48, 48, 96, 3, 3, 1, "bf16"),     # 16x16 regions, 3 heads, 3 images: tcgen05
    (1, 32, 32, 64, 2, 16, 20, "bf16"),   # 256 regions (column-per-lane routing), topk 20 (sort)
    (6, 16, 16, 64, 2, 16, 2, "bf16"),    # 256 regions, 6 images (8 routing rows per CTA)
    (2, 12, 12, 64, 2, 6, 12, "bf16"),    # 2x2 regions, topk 12: per-image routing, routed fused kernel
    (1, 20, 20, 64, 2, 5, 20, "bf16"),    # 4x4 regions, 25 of them, topk 20: the same, one column warp
    (1, 32, 32, 64, 2, 4, 4, "bf16"),     # 8x8 regions, topk 4 -> 256 keys: half-filled tcgen05 tile (split)
    (2, 16, 16, 64, 2, 2, 2, "bf16"),     # 8x8 regions, topk 2 -> 128 keys: the same, one score half
    (1, 28, 28, 192, 6, 7, 4, "bf16"),    # 6 heads (C = 192): a cluster of 6 CTAs per image
    (2, 32, 32, 160, 5, 4, 2, "bf16"),    # 5 heads (C = 160), 8x8 regions: split path
    (2, 8, 8, 64, 2, 1, 1, "bf16"),       # S = 1: one region, every query over its whole image
    (1, 16, 16, 64, 2, 16, 256, "bf16"),  # S = 16, topk = 256: one-token regions, dense limit
    (1, 16, 16, 64, 2, 16, 256, "f32"),   # the same in float32
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "x".join(map(str, s)))
def test_small_shapes(shape, any_variant):
    N, H, W, C, heads, S, topk, dtype = shape
    w = synth.Workload("small", 40 + sum(shape[:7]), N, H, W, C, heads, S, topk, dtype,
                       region_bias=0.5, lce_b_std=0.05, lce_w_std=0.1)
    assert_parity(w, synth.make_inputs(w))


def test_empty_batch():
    w = synth.WORKLOADS["cls_stage2_224"].with_(N=0)
    d = to_dev(synth.make_inputs(w), w.dtype)
    out, r_idx, r_w = bra.forward(d["q"], d["k"], d["v"], d["lce_w"], d["lce_b"], w.heads, w.S, w.topk)
    assert out.shape[0] == 0 and r_idx.shape == (0, 49, 4)


def test_route_entry_point_matches_forward():
    w = synth.WORKLOADS["seg_stage2_512"]
    inp = synth.make_inputs(w)
    d = to_dev(inp, w.dtype)
    r_idx, r_w = bra.route(d["q"], d["k"], w.heads, w.S, w.topk)
    _, f_idx, f_w = bra.forward(d["q"], d["k"], d["v"], d["lce_w"], d["lce_b"], w.heads, w.S, w.topk)
    assert torch.equal(r_idx, f_idx) and torch.equal(r_w, f_w)
    ref_idx, ref_w, logits = oracle.route(inp["q"], inp["k"], w.heads, w.S, w.topk, with_logits=True)
    rep = compare.Report()
    compare.check_routing(logits, ref_idx, ref_w, r_idx.cpu().numpy(), r_w.cpu().numpy(), rep)
    assert rep.ok, rep.notes


def test_attend_given_routing_with_duplicates_and_any_order(any_variant):
    w = synth.WORKLOADS["cls_stage2_224"].with_(N=4)
    inp = synth.make_inputs(w)
    d = to_dev(inp, w.dtype)
    rng = np.random.Generator(np.random.PCG64(5))
    r_idx = rng.integers(0, w.regions, size=(w.N, w.regions, w.topk)).astype(np.int32)
    r_idx[:, :, 1] = r_idx[:, :, 0]  # duplicates count twice
    out = bra.attend(d["q"], d["k"], d["v"], d["lce_w"], d["lce_b"], w.heads, w.S,
                     torch.from_numpy(r_idx).cuda())
    ref = oracle.attend(inp["q"], inp["k"], inp["v"], inp["lce_w"], inp["lce_b"], w.heads, w.S, r_idx)
    rep = compare.Report()
    compare.check_output(out.float().cpu().numpy(), ref, w.dtype, rep)
    assert rep.ok, rep.notes


def test_bounded_wait_reports_timeout_and_recovers():
    """A wait that can never complete gives up after its poll limit, raises the device
    flag (reported once by bra_device_status) and leaves the context usable."""
    assert bra.device_status() == 0
    bra.selftest_wait_timeout(64)
    assert bra.device_status() == 8
    assert bra.device_status() == 0
    w = synth.WORKLOADS["cls_stage2_224"].with_(N=2)
    assert_parity(w, synth.make_inputs(w))


def test_attend_rejects_out_of_range_region_index(any_variant):
    """The kernel checks every index it reads; a bad one is reported, never dereferenced."""
    w = synth.WORKLOADS["cls_stage2_224"].with_(N=1)
    d = to_dev(synth.make_inputs(w), w.dtype)
    r_idx = torch.zeros((1, w.regions, w.topk), dtype=torch.int32, device="cuda")
    r_idx[0, 3, 2] = w.regions       # one past the end
    r_idx[0, 5, 0] = -1
    with pytest.raises(bra.BraError) as e:
        bra.attend(d["q"], d["k"], d["v"], d["lce_w"], d["lce_b"], w.heads, w.S, r_idx)
    assert e.value.status == 6
    # the context is still usable
    r_idx.clamp_(0, w.regions - 1)
    bra.attend(d["q"], d["k"], d["v"], d["lce_w"], d["lce_b"], w.heads, w.S, r_idx)
    torch.cuda.synchronize()


@pytest.mark.parametrize("shape", [(2, 32, 32, 64, 2, 2, 1), (2, 16, 32, 64, 2, 2, 2), (2, 32, 32, 64, 2, 4, 4)],
                         ids=["w256k1", "w128k2", "w64k4"])
def test_tcgen05_attend_duplicates_and_bad_index(shape):
    """64/128/256-token regions (the tcgen05 kernel; 64-token regions take it when it is
    asked for): duplicated routed regions count twice; an out-of-range index is reported
    (status 6) and its keys are masked."""
    N, H, W, C, heads, S, topk = shape
    prev = bra.set_kernel_variant(VARIANTS["split"])
    try:
        _tcgen05_attend_duplicates_and_bad_index(shape)
    finally:
        bra.set_kernel_variant(prev)


def _tcgen05_attend_duplicates_and_bad_index(shape):
    N, H, W, C, heads, S, topk = shape
    w = synth.Workload("small", 77, N, H, W, C, heads, S, topk, "bf16", region_bias=0.5, lce_b_std=0.05,
                       lce_w_std=0.1)
    inp = synth.make_inputs(w)
    d = to_dev(inp, w.dtype)
    rng = np.random.Generator(np.random.PCG64(9))
    r_idx = rng.integers(0, w.regions, size=(w.N, w.regions, w.topk)).astype(np.int32)
    if topk > 1:
        r_idx[:, 1:, 1] = r_idx[:, 1:, 0]
    out = bra.attend(d["q"], d["k"], d["v"], d["lce_w"], d["lce_b"], w.heads, w.S, torch.from_numpy(r_idx).cuda())
    ref = oracle.attend(inp["q"], inp["k"], inp["v"], inp["lce_w"], inp["lce_b"], w.heads, w.S, r_idx)
    rep = compare.Report()
    compare.check_output(out.float().cpu().numpy(), ref, w.dtype, rep)
    assert rep.ok, rep.notes
    bad = torch.from_numpy(r_idx).cuda()
    bad[0, 1, 0] = w.regions
    with pytest.raises(bra.BraError) as e:
        bra.attend(d["q"], d["k"], d["v"], d["lce_w"], d["lce_b"], w.heads, w.S, bad)
    assert e.value.status == 6
    assert bra.device_status() == 0


def test_tcgen05_row_with_dominant_far_key_is_exact():
    """256-token regions (the tcgen05 kernel): one query whose logit for a key far down
    the row exceeds every logit of the first keys by hundreds, so that probabilities
    taken relative to the first keys would overflow; the row must still match the
    oracle (the kernel recomputes such a row with its true max)."""
    w = synth.Workload("small", 91, 1, 32, 32, 64, 2, 2, 1, "bf16", region_bias=0.0, lce_b_std=0.05, lce_w_std=0.1)
    inp = synth.make_inputs(w)
    e = np.full(32, 30.0 / np.sqrt(32.0))
    inp["q"][0, 5, 19, 0:32] = e          # query token 5*16+3 of region 1 (head 0)
    inp["k"][0, 28, 24, 0:32] = e         # key 200 of region 3
    inp = {k: synth.round_bf16(v) if k in ("q", "k", "v") else v for k, v in inp.items()}
    d = to_dev(inp, w.dtype)
    r_idx = np.array([[[2], [3], [0], [1]]], dtype=np.int32)
    out = bra.attend(d["q"], d["k"], d["v"], d["lce_w"], d["lce_b"], w.heads, w.S, torch.from_numpy(r_idx).cuda())
    ref = oracle.attend(inp["q"], inp["k"], inp["v"], inp["lce_w"], inp["lce_b"], w.heads, w.S, r_idx)
    rep = compare.Report()
    got = out.float().cpu().numpy()
    compare.check_output(got, ref, w.dtype, rep)
    assert rep.ok, rep.notes
    assert np.all(np.isfinite(got))


def test_host_entry_point_matches_device_entry_point():
    w = synth.WORKLOADS["cls_stage2_224"].with_(N=8)
    inp = synth.make_inputs(w)
    d = to_dev(inp, w.dtype)
    out, r_idx, r_w = bra.forward(d["q"], d["k"], d["v"], d["lce_w"], d["lce_b"], w.heads, w.S, w.topk)
    h = {k: v.cpu().pin_memory() for k, v in d.items()}
    h_out, h_idx, h_w = bra.forward_host(h["q"], h["k"], h["v"], h["lce_w"], h["lce_b"], w.heads, w.S, w.topk)
    assert torch.equal(h_out, out.cpu()) and torch.equal(h_idx, r_idx.cpu()) and torch.equal(h_w, r_w.cpu())


def test_deterministic_and_stream_ordered():
    w = synth.WORKLOADS["det_stage1_1024"]
    d = to_dev(synth.make_inputs(w), w.dtype)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        a = bra.forward(d["q"], d["k"], d["v"], d["lce_w"], d["lce_b"], w.heads, w.S, w.topk)
        b = bra.forward(d["q"], d["k"], d["v"], d["lce_w"], d["lce_b"], w.heads, w.S, w.topk)
    s.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
