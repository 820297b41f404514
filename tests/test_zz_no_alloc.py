"""bra_forward_noalloc on a B200: the allocation-free entry point gives the same
results as bra_forward.

bra_forward_noalloc exists for callers that cannot allocate device memory when they
call in (a framework whose caching allocator already holds the device's memory, a
real-time loop that forbids allocation after start-up, a process whose memory pool is
disabled or capped). Its scratch is a static device array inside the library, shared
by every call, so this test makes two calls in a row — the second reuses whatever the
first left in the array — plus a call on a different shape, and compares each with
bra_forward under the parity tolerance of the other GPU tests. This file is collected
last so that a failure here does not stop the rest of a `-x` run; it passes alone in a
fresh process too, where its first call is the one that looks up the array's address.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import compare
from vision_transformer_sparse_b200 import bra, synth

pytestmark = pytest.mark.gpu


def _device_inputs(w):
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    return {k: torch.from_numpy(v).cuda().to(dt).contiguous() for k, v in synth.make_inputs(w).items()}


def _close(a: torch.Tensor, b: torch.Tensor, dtype: str):
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    if dtype == "f32":
        return np.max(np.abs(a - b)) <= compare.TOL_F32_ABS
    return np.all(np.abs(a - b) <= compare.TOL_BF16_ABS + compare.TOL_BF16_REL * np.abs(b))


def _check(w, d, noalloc):
    ref_out, ref_idx, ref_w = bra.forward(d["q"], d["k"], d["v"], d["lce_w"], d["lce_b"], w.heads, w.S, w.topk)
    out, r_idx, r_w = noalloc
    torch.cuda.synchronize()
    assert torch.equal(r_idx, ref_idx)
    assert torch.max(torch.abs(r_w - ref_w)).item() <= compare.TOL_WEIGHT
    assert _close(out, ref_out, w.dtype)


def test_noalloc_matches_forward_on_consecutive_calls(bra_lib):
    w = synth.WORKLOADS["cls_stage2_224"]
    d = _device_inputs(w)
    for _ in range(2):  # the second call starts from the first call's scratch contents
        res = bra.forward_noalloc(d["q"], d["k"], d["v"], d["lce_w"], d["lce_b"], w.heads, w.S, w.topk)
        _check(w, d, res)
    # a different shape right after, through the same array
    w2 = synth.WORKLOADS["stage1_tiny_224"]
    d2 = _device_inputs(w2)
    res = bra.forward_noalloc(d2["q"], d2["k"], d2["v"], d2["lce_w"], d2["lce_b"], w2.heads, w2.S, w2.topk)
    _check(w2, d2, res)


def test_noalloc_rejects_problems_beyond_the_static_array(bra_lib):
    w = synth.WORKLOADS["cls_stage2_224"]
    N = bra.STATIC_SCRATCH_FLOATS // (2 * w.regions * w.C) + 1   # one image too many
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check fails first
    rc = bra.raw_call("bra_forward_noalloc", *[fake] * 5, N, w.H, w.W, w.C, w.heads, w.S, w.topk, 1,
                      fake, fake, fake, None)
    assert rc == 7 and "static" in bra.status_string(rc)
