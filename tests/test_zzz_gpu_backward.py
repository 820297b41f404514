"""Parity of bra_backward (routing detached) with the float64 backward oracle, on a B200.

The cases of tests/test_backward_host.py, which runs the kernels' per-item code on the
host with every access bounds-checked (the file name keeps these tests after the rest of
the GPU suite). Tolerance:
float32 arithmetic with atomically accumulated dk and dv against float64, normwise per
tensor: max |gpu - ref| <= 1e-4 * max(1, max |ref|)."""
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
