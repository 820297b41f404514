"""bra_forward_noalloc on a B200: the allocation-free entry point gives, bit for bit, the
results of bra_forward, and those results pass the parity check against the float64
oracle.

bra_forward_noalloc exists for callers that cannot allocate device memory when they
call in (a framework whose caching allocator already holds the device's memory, a
real-time loop that forbids allocation after start-up, a process whose memory pool is
disabled or capped). Its scratch is a static device array inside the library, shared
by every call, so each case makes two calls in a row — the second reuses whatever the
previous call left in the array — and the cases run one after another through the
same array with different shapes. Outputs start as NaN / -1 so that an element a call
leaves unwritten cannot pass. The cases cover the one-kernel fused forward (which
needs no scratch), the pipeline and tcgen05 attention paths (which do) and float32.
This file is collected last so that a failure here does not stop the rest of a `-x`
run; it passes alone in a fresh process too.
"""
import ctypes

import pytest
import torch

from oracle import compare
from vision_transformer_sparse_b200 import bra, synth

pytestmark = pytest.mark.gpu

CASES = [("cls_stage2_224", 8), ("seg_stage2_512", 1), ("det_stage1_1024", 1), ("stage1_tiny_224", 1)]


def _device_inputs(w, inp):
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    return {k: torch.from_numpy(v).cuda().to(dt).contiguous() for k, v in inp.items()}


def _outputs(w, like):
    return (torch.full_like(like, float("nan")),
            torch.full((w.N, w.regions, w.topk), -1, dtype=torch.int32, device="cuda"),
            torch.full((w.N, w.regions, w.topk), float("nan"), dtype=torch.float32, device="cuda"))


def test_noalloc_equals_forward_and_the_oracle_on_consecutive_calls(bra_lib):
    for name, batch in CASES:
        w = synth.WORKLOADS[name].with_(N=batch)
        inp = synth.make_inputs(w)
        d = _device_inputs(w, inp)
        ref = _outputs(w, d["q"])
        bra.forward(d["q"], d["k"], d["v"], d["lce_w"], d["lce_b"], w.heads, w.S, w.topk, out=ref[0],
                    r_idx=ref[1], r_weight=ref[2])
        for call in range(2):  # the second call starts from the first call's scratch contents
            got = _outputs(w, d["q"])
            bra.forward_noalloc(d["q"], d["k"], d["v"], d["lce_w"], d["lce_b"], w.heads, w.S, w.topk, out=got[0],
                                r_idx=got[1], r_weight=got[2])
            torch.cuda.synchronize()
            for a, b in zip(got, ref):  # the same kernels as bra_forward: identical bits
                assert torch.equal(a.view(torch.uint8) if a.is_floating_point() else a,
                                   b.view(torch.uint8) if b.is_floating_point() else b), (name, call)
            rep = compare.check_forward(inp, w.heads, w.S, w.topk, w.dtype, got[0].float().cpu().numpy(),
                                        got[1].cpu().numpy(), got[2].cpu().numpy())
            assert rep.ok, (name, call, rep.notes[:1000])


def test_noalloc_rejects_problems_beyond_the_static_array(bra_lib):
    w = synth.WORKLOADS["cls_stage2_224"]
    N = bra.STATIC_SCRATCH_FLOATS // (2 * w.regions * w.C) + 1   # one image too many
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check fails first
    rc = bra.raw_call("bra_forward_noalloc", *[fake] * 5, N, w.H, w.W, w.C, w.heads, w.S, w.topk, 1,
                      fake, fake, fake, None)
    assert rc == 7 and "static" in bra.status_string(rc)
