"""The backward kernels' per-item code run on the host (CPU, no GPU): every memory access
bounds-checked against its buffer, results compared with the float64 backward oracle.

tests/host/bwd_host_harness.cu compiles csrc/backward.cuh for the host with
BRA_BWD_HOST_CHECK and replays the kernels' partition (the LCE dv pass, the zeroed dk,
every (image, region, head, query token) item, the 256-way partial sums of the LCE
parameter gradients). Tolerance: float32 arithmetic against float64, normwise per tensor,
max |got - ref| <= 1e-4 * max(1, max |ref|).
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle
from oracle import backward as ob
from vision_transformer_sparse_b200 import synth

HERE = os.path.dirname(os.path.abspath(__file__))
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("bwd") / "libbwdhost.so")
    cmd = [NVCC, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a", "-Xcompiler", "-fPIC",
           "-shared", "-o", out, os.path.join(HERE, "host", "bwd_host_harness.cu")]
    subprocess.check_call(cmd)
    lib = ctypes.CDLL(out)
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.bwd_host_run.argtypes = [vp] * 6 + [i] * 8 + [vp] * 6
    lib.bwd_host_run.restype = ctypes.c_longlong
    return lib


def ptr(a):
    return ctypes.c_void_p(a.ctypes.data)


def run(lib, q, k, v, dout, w, r_idx, heads, S, dtype):
    N, H, W, C = q.shape
    topk = r_idx.shape[-1]
    if dtype == "bf16":
        conv = lambda a: np.ascontiguousarray((np.asarray(a, np.float32).view(np.uint32) >> 16).astype(np.uint16))
    else:
        conv = lambda a: np.ascontiguousarray(a, dtype=np.float32)
    ins = [conv(a) for a in (q, k, v, dout, w)]
    r = np.ascontiguousarray(r_idx, dtype=np.int32)
    g = {"dq": np.full((N, H, W, C), np.nan, np.float32), "dk": np.full((N, H, W, C), np.nan, np.float32),
         "dv": np.full((N, H, W, C), np.nan, np.float32), "dlce_w": np.full((C, 5, 5), np.nan, np.float32),
         "dlce_b": np.full((C,), np.nan, np.float32)}
    bad = np.zeros(1, np.int32)
    fails = lib.bwd_host_run(*(ptr(a) for a in ins), ptr(r), N, H, W, C, heads, S, topk, int(dtype == "bf16"),
                             *(ptr(a) for a in g.values()), ptr(bad))
    return g, int(fails), int(bad[0])


def inputs(N, H, W, C, seed, dtype):
    w = synth.Workload("bwd", seed, N, H, W, C, 2, 2, 1, dtype, lce_b_std=0.01)
    d = synth.make_inputs(w)
    dout = synth.make_inputs(w, seed_base=0xB0D0 + seed)["q"]  # any seeded map, stored in the dtype
    return d["q"], d["k"], d["v"], dout, d["lce_w"]


def check(got, ref):
    for name in ref:
        err = np.max(np.abs(got[name].astype(np.float64) - ref[name]))
        assert err <= 1e-4 * max(1.0, np.max(np.abs(ref[name]))), (name, err)


# (N, H, W, C, heads, S, topk, dtype): d = 32 and 64, 1-, 4- and 16-token regions, dense
# routing (topk = S^2), float32 and bf16 storage
CASES = [
    (1, 8, 8, 64, 2, 2, 2, "f32"),
    (2, 8, 8, 128, 2, 2, 4, "f32"),
    (1, 14, 14, 64, 2, 7, 3, "f32"),
    (1, 8, 8, 64, 2, 8, 5, "f32"),
    (1, 8, 8, 64, 2, 2, 2, "bf16"),
    (1, 12, 12, 128, 4, 3, 2, "bf16"),
    (2, 28, 28, 128, 4, 7, 4, "bf16"),
]


@pytest.mark.parametrize("N,H,W,C,heads,S,topk,dtype", CASES)
def test_host_run_matches_oracle(harness, N, H, W, C, heads, S, topk, dtype):
    q, k, v, dout, w = inputs(N, H, W, C, 70 + C + topk, dtype)
    r_idx, _ = oracle.route(q, k, heads, S, topk)
    got, fails, bad = run(harness, q, k, v, dout, w, r_idx, heads, S, dtype)
    assert fails == 0 and bad == 0
    check(got, ob.backward(q, k, v, w, np.zeros(C), heads, S, r_idx, dout))


def test_host_run_repeated_and_invalid_regions(harness):
    """A routing row that repeats a region counts its keys twice (as the oracle does); an
    index outside [0, S*S) is skipped and raises the flag, with every access in bounds."""
    N, H, W, C, heads, S = 1, 8, 8, 64, 2, 2
    q, k, v, dout, w = inputs(N, H, W, C, 90, "f32")
    r_idx, _ = oracle.route(q, k, heads, S, 2)
    r_idx = r_idx.copy()
    r_idx[0, 1] = [3, 3]
    got, fails, bad = run(harness, q, k, v, dout, w, r_idx, heads, S, "f32")
    assert fails == 0 and bad == 0
    check(got, ob.backward(q, k, v, w, np.zeros(C), heads, S, r_idx, dout))
    r_bad = r_idx.copy()
    r_bad[0, 2, 1] = 7
    r_bad[0, 0, 0] = -1
    _, fails, bad = run(harness, q, k, v, dout, w, r_bad, heads, S, "f32")
    assert fails == 0 and bad == 1
