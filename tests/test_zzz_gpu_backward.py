"""Parity of bra_backward (routing detached) with the float64 backward oracle, on a B200.

The cases of tests/test_backward_host.py, which runs the SIMT kernels' per-item code on the
host with every access bounds-checked (the file name keeps these tests after the rest of
the GPU suite), plus shapes for the tensor-core path that bf16 maps with 32 channels per
head take (regions of 4, 25, 32, 64 and 256 tokens, the dense limit with a ragged last key
chunk, repeated and out-of-range regions). Tolerance: float32 arithmetic against float64,
normwise per tensor: max |gpu - ref| <= 1e-4 * max(1, max |ref|). The tensor-core path
multiplies the probabilities and dS as bf16 high + low parts, so it meets the same bound,
and it is deterministic: two calls give the same bits."""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as ob
from vision_transformer_sparse_b200 import bra, synth
from test_backward_host import CASES, inputs

pytestmark = pytest.mark.gpu

TORCH = {"bf16": torch.bfloat16, "f32": torch.float32}


def dev(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to("cuda").to(TORCH[dtype])


def run_gpu(q, k, v, dout, w, r_idx, heads, S, dtype):
    g = bra.backward(dev(q, dtype), dev(k, dtype), dev(v, dtype), dev(w, dtype),
                     torch.from_numpy(np.ascontiguousarray(r_idx, np.int32)).cuda(), dev(dout, dtype), heads, S)
    torch.cuda.synchronize()
    return {name: t.cpu().numpy() for name, t in g.items()}


def check(got, ref):
    for name in ref:
        assert np.all(np.isfinite(got[name])), name
        err = np.max(np.abs(got[name].astype(np.float64) - ref[name]))
        assert err <= 1e-4 * max(1.0, np.max(np.abs(ref[name]))), (name, err)


@pytest.mark.parametrize("N,H,W,C,heads,S,topk,dtype", CASES)
def test_backward_matches_oracle(N, H, W, C, heads, S, topk, dtype):
    q, k, v, dout, w = inputs(N, H, W, C, 70 + C + topk, dtype)
    r_idx, _ = oracle.route(q, k, heads, S, topk)
    got = run_gpu(q, k, v, dout, w, r_idx, heads, S, dtype)
    check(got, ob.backward(q, k, v, w, np.zeros(C), heads, S, r_idx, dout))
    assert bra.device_status() == 0


def test_backward_repeated_and_invalid_regions():
    N, H, W, C, heads, S = 1, 8, 8, 64, 2, 2
    q, k, v, dout, w = inputs(N, H, W, C, 90, "f32")
    r_idx, _ = oracle.route(q, k, heads, S, 2)
    r_idx = r_idx.copy()
    r_idx[0, 1] = [3, 3]
    check(run_gpu(q, k, v, dout, w, r_idx, heads, S, "f32"), ob.backward(q, k, v, w, np.zeros(C), heads, S, r_idx, dout))
    r_bad = r_idx.copy()
    r_bad[0, 2, 1] = 7
    with pytest.raises(bra.BraError) as e:
        run_gpu(q, k, v, dout, w, r_bad, heads, S, "f32")
    assert e.value.status == 6  # BRA_ERR_INDEX


TC_CASES = [
    # N, H, W, C, heads, S, topk  (bf16, d = 32: the tensor-core path)
    (2, 14, 14, 256, 8, 7, 16),   # 2x2-token regions: one warp with 12 padded rows
    (1, 14, 14, 64, 2, 7, 49),    # dense limit: 196 keys, a ragged last 32-key chunk
    (1, 15, 15, 64, 2, 3, 3),     # 5x5-token regions: 25 queries, 75 keys
    (1, 12, 24, 64, 2, 3, 2),     # non-square 4x8-token regions
    (1, 32, 32, 128, 4, 4, 4),    # 64-token regions, 256 keys (the segmentation shape)
    (1, 32, 32, 64, 2, 2, 1),     # 256-token regions, 16 warps (the detection shape)
    (1, 14, 14, 96, 3, 7, 4),     # 48 channel pairs: five LCE slots per CTA, one idle
    (1, 20, 20, 32, 1, 5, 3),     # 16 channel pairs: four 4-pixel segments per tile row
    (1, 14, 14, 192, 6, 7, 4),    # 96 channel pairs: two LCE groups of 48
]


@pytest.mark.parametrize("N,H,W,C,heads,S,topk", TC_CASES)
def test_tensor_core_backward_matches_oracle(N, H, W, C, heads, S, topk):
    q, k, v, dout, w = inputs(N, H, W, C, 120 + C + topk + H, "bf16")
    r_idx, _ = oracle.route(q, k, heads, S, topk)
    got = run_gpu(q, k, v, dout, w, r_idx, heads, S, "bf16")
    check(got, ob.backward(q, k, v, w, np.zeros(C), heads, S, r_idx, dout))
    assert bra.device_status() == 0


def test_tensor_core_backward_repeated_and_invalid_regions():
    N, H, W, C, heads, S = 1, 16, 16, 64, 2, 4
    q, k, v, dout, w = inputs(N, H, W, C, 95, "bf16")
    r_idx, _ = oracle.route(q, k, heads, S, 3)
    r_idx = r_idx.copy()
    r_idx[0, 1] = [5, 5, 2]   # a region routed twice: its keys count twice in the softmax
    r_idx[0, 7] = [7, 0, 7]
    check(run_gpu(q, k, v, dout, w, r_idx, heads, S, "bf16"), ob.backward(q, k, v, w, np.zeros(C), heads, S, r_idx, dout))
    r_bad = r_idx.copy()
    r_bad[0, 2, 1] = 16
    with pytest.raises(bra.BraError) as e:
        run_gpu(q, k, v, dout, w, r_bad, heads, S, "bf16")
    assert e.value.status == 6  # BRA_ERR_INDEX


def test_tensor_core_backward_is_deterministic():
    """Two calls on the classification stage-2 batch give identical bits in every output
    (no atomics: each element has one writer, and every sum runs in a fixed order)."""
    w = synth.WORKLOADS["cls_stage2_224"].with_(N=8)
    q, k, v, dout, lw = inputs(w.N, w.H, w.W, w.C, 130, "bf16")
    r_idx, _ = oracle.route(q, k, w.heads, w.S, w.topk)
    a = run_gpu(q, k, v, dout, lw, r_idx, w.heads, w.S, "bf16")
    b = run_gpu(q, k, v, dout, lw, r_idx, w.heads, w.S, "bf16")
    for name in a:
        assert np.array_equal(a[name].view(np.uint32), b[name].view(np.uint32)), name


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_async_backward_equals_backward_and_reports_index_errors(dtype):
    """bra_backward_async: the same kernels without the host synchronisation; identical
    results (bits, on the deterministic bf16 path), and an out-of-range routing entry
    surfaces through bra_device_status as BRA_ERR_INDEX."""
    N, H, W, C, heads, S = 2, 16, 16, 64, 2, 4
    q, k, v, dout, w = inputs(N, H, W, C, 140, dtype)
    r_idx, _ = oracle.route(q, k, heads, S, 3)
    d = [dev(x, dtype) for x in (q, k, v, w)]
    ri = torch.from_numpy(np.ascontiguousarray(r_idx, np.int32)).cuda()
    do = dev(dout, dtype)
    a = bra.backward(d[0], d[1], d[2], d[3], ri, do, heads, S)
    b = bra.backward(d[0], d[1], d[2], d[3], ri, do, heads, S, sync=False)
    assert bra.device_status() == 0
    ref = ob.backward(q, k, v, w, np.zeros(C), heads, S, r_idx, dout)
    check({n_: t.cpu().numpy() for n_, t in b.items()}, ref)
    if dtype == "bf16":
        for n_ in a:
            assert torch.equal(a[n_].view(torch.int32), b[n_].view(torch.int32)), n_
    bad = r_idx.copy()
    bad[1, 3, 2] = -1
    bra.backward(d[0], d[1], d[2], d[3], torch.from_numpy(bad).cuda(), do, heads, S, sync=False)
    assert bra.device_status() == 6  # BRA_ERR_INDEX, then cleared
    assert bra.device_status() == 0


def test_backward_with_element_aligned_buffers():
    """bf16 with 32 channels per head but q, k, v, dout one element past a 16-byte
    boundary: the tensor-core kernels need 16-byte pieces, so the SIMT kernels run, and
    the gradients still match the oracle."""
    N, H, W, C, heads, S, topk = 1, 14, 14, 64, 2, 7, 3
    q, k, v, dout, w = inputs(N, H, W, C, 777, "bf16")
    r_idx, _ = oracle.route(q, k, heads, S, topk)

    def shifted(a):  # the same bf16 values at an address 2 bytes past a 16-byte boundary
        buf = torch.empty(a.size + 8, dtype=torch.bfloat16, device="cuda")
        t = buf[1:1 + a.size]
        t.copy_(dev(a, "bf16").reshape(-1))
        return t.view(a.shape)

    g = bra.backward(shifted(q), shifted(k), shifted(v), dev(w, "bf16"),
                     torch.from_numpy(np.ascontiguousarray(r_idx, np.int32)).cuda(), shifted(dout), heads, S)
    torch.cuda.synchronize()
    got = {name: t.cpu().numpy() for name, t in g.items()}
    check(got, ob.backward(q, k, v, w, np.zeros(C), heads, S, r_idx, dout))
    assert bra.device_status() == 0
