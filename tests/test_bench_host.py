"""Host-side logic of bench.py (no GPU): how a committed ncu summary is matched to the
source it was captured on, and the algorithmic figures the roofline divides by."""
import importlib.util
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "vision_transformer_sparse_b200", "csrc")


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def includes(name):
    with open(os.path.join(CSRC, name)) as f:
        return re.findall(r'^\s*#include "([^"]+)"', f.read(), flags=re.M)


def test_kernel_sources_are_the_include_closure(bench):
    for kernel, heads in bench.KERNEL_HEADERS.items():
        got = set(bench.kernel_sources(kernel))
        assert set(heads) <= got, kernel
        for name in got:  # closed under #include
            assert set(includes(name)) <= got, (kernel, name)
        # every kernel builds on the shared helpers, except the self-contained per-element
        # ones (the block's per-pixel kernels and the padded grid's copies)
        assert "common.cuh" in got or kernel in ("block_pixel_kernels", "pad_crop_kernels"), kernel


def test_fp32_kernel_does_not_depend_on_the_tensor_core_kernels(bench):
    got = set(bench.kernel_sources("attn_f32_kernel"))
    assert "attn_umma.cuh" not in got and "umma.cuh" not in got and "fused_image.cuh" not in got


def test_profile_lookup_matches_only_the_current_source(bench, tmp_path, monkeypatch):
    # a summary is used for traffic only while its hash is the kernel's current one
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    os.makedirs(tmp_path / "profiles")
    os.makedirs(tmp_path / "vision_transformer_sparse_b200")
    os.symlink(CSRC, tmp_path / "vision_transformer_sparse_b200" / "csrc")
    h = bench.kernel_source_hash("attn_umma_kernel")
    (tmp_path / "profiles" / "attn_umma_kernel_w.txt").write_text(
        "source_hash: %s\ndram_bytes_per_launch: 1234\n" % h)
    (tmp_path / "profiles" / "attn_umma_kernel_old.txt").write_text(
        "source_hash: 0000000000000000\ndram_bytes_per_launch: 99\n")
    assert bench.profiled_traffic("attn_umma_kernel", "w")[0] == 1234.0
    assert bench.profiled_traffic("attn_umma_kernel", "old")[0] is None
    assert bench.profiled_traffic("attn_umma_kernel", "missing") == (None, None)


def test_algorithmic_figures_of_the_detection_stage(bench):
    from vision_transformer_sparse_b200 import synth
    w = synth.WORKLOADS["det_stage1_1024"]
    acc = bench.algorithmic(w)
    T = w.N * w.H * w.W
    L = w.topk * (w.H // w.S) * (w.W // w.S)
    assert acc["tokens"] == T
    assert acc["flops"] == 4 * T * L * w.C
    assert acc["gathered_bytes"] == w.N * w.S * w.S * L * 2 * w.C * 2


def test_source_hash_ignores_comments_only(bench):
    """A profile stays matched across comment edits, and not across code edits."""
    src = 'int a = 1; // note\n/* block\n comment */ const char *s = "x // kept"; char q = \'/\';\n\n  int b;\n'
    assert bench.strip_comments(src) == 'int a = 1;\n const char *s = "x // kept"; char q = \'/\';\n  int b;'
    assert bench.strip_comments(src.replace("// note", "// other note")) == bench.strip_comments(src)
    assert bench.strip_comments(src.replace("int b;", "int c;")) != bench.strip_comments(src)


def test_algorithmic_figures_of_the_layer_and_the_backward(bench):
    """Bytes per launch of the projections (the mean of the qkv and output launches) and
    per call of the backward, written out from their tensors' sizes."""
    from vision_transformer_sparse_b200 import synth
    w = synth.WORKLOADS["cls_stage2_224"]
    acc = bench.algorithmic(w)
    T, C, b = w.tokens, w.C, 2
    qkv = T * C * b + 3 * C * C * b + 3 * T * C * b      # x, w_qkv read; q, k, v written
    wo = T * C * b + C * C * b + T * C * b               # o, w_o read; out written
    assert acc["linear_bytes"] == (qkv + wo) / 2
    assert acc["linear_flops"] == 2 * T * C * 3 * C + 2 * T * C * C
    bwd = (4 * T * C * b                                 # q, k, v, dout read
           + 3 * T * C * 4                               # dq, dk, dv written (float32)
           + w.N * w.regions * w.topk * 4                # r_idx
           + C * 25 * b + C * 25 * 4 + C * 4)            # lce_w read; dlce_w, dlce_b written
    assert acc["bwd_bytes"] == bwd


def test_method_roofline_picks_the_slower_term(bench):
    """The detection stage is bound by its FLOPs at the burst bf16 peak, the classification
    stage by its gathered K/V bytes at HBM bandwidth; frac = roofline time / kernel time."""
    from vision_transformer_sparse_b200 import synth
    peaks = {"hbm_gbs": 6540.8, "bf16_tflops": 1645.8, "bf16_tflops_sustained": 1369.4}
    det = bench.algorithmic(synth.WORKLOADS["det_stage1_1024"])
    r = bench.method_roofline(det, peaks, 20e-6)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] == 1645.8
    t_flop = det["flops"] / 1645.8e12
    assert abs(r["frac"] - t_flop / 20e-6) < 1e-12
    assert abs(r["roofline_us"] - t_flop * 1e6) < 1e-9
    cls = bench.algorithmic(synth.WORKLOADS["cls_stage2_224"])
    r = bench.method_roofline(cls, peaks, 50e-6)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["frac"] - cls["gathered_bytes"] / 6540.8e9 / 50e-6) < 1e-12
