"""Seeded synthetic inputs for Bi-Level Routing Attention (BRA) workloads.

This module only draws numbers and rounds them to the storage dtype; it holds
none of the attention, pooling, routing or convolution arithmetic. Both the
float64 oracle (through the tests) and the CUDA path (through the tests and the
benchmark) receive exactly the arrays produced here.

Workload shapes follow the BiFormer stage shapes of the pages:
  * stage-1 shape comments for a 224x224 image (niftyadmin walk-through,
    section "BRA模块": x (1,56,56,64), 49 regions of 8x8 tokens, 2 heads of 32,
    topk 1);
  * per-stage top-k 1, 4, 16, S^2 and S = 7 / 16 / 8 for classification /
    detection / segmentation (bernice.tw, "Biformer" and "消融實驗" sections);
  * one detection map whose size is not a multiple of S (a 1000x1000 input: 250x250
    at stage 1, S = 16), for the padded grid.

Value recipe (stated once, used everywhere):
  * q, k, v ~ N(0, 1) i.i.d.;
  * for the detection and segmentation workloads, a per-(image, region,
    channel) offset ~ N(0, 0.5^2) is added to each of q, k, v separately, so
    that region means differ and routing is non-uniform;
  * LCE depthwise 5x5 weight ~ N(0, 0.02^2); LCE bias ~ N(0, 0.01^2) for the
    classification stage-2/3 workloads, 0 otherwise;
  * values are drawn in float64, cast to float32, then rounded to bfloat16
    (round-to-nearest-even) when the workload dtype is bf16.
Seeds: workload c, tensor slot i -> seed 0xB1F0 + 16*c + i, with slots
q=0, k=1, v=2, lce_w=3, lce_b=4, q/k/v region offsets = 5/6/7.

Attention-layer inputs (make_layer_inputs: the qkv projection before the path and
the output projection after it) draw the layer input x instead of q, k, v:
  * x ~ N(0, 1), plus the same kind of per-(image, region, channel) offset for the
    detection and segmentation workloads;
  * qkv weight (3C, C) and output weight (C, C) ~ N(0, 1/C), so that q, k, v and the
    layer output have unit scale; both biases ~ N(0, 0.02^2);
  * LCE weight and bias as above; slots x=8, x offset=9, qkv weight/bias=10/11,
    output weight/bias=12/13.

BiFormer-block inputs (make_block_inputs) add the block's own parameters to the layer's:
  * pos-embed depthwise 3x3 weight ~ N(0, 0.2^2), bias ~ N(0, 0.05^2);
  * LayerNorm gains 1 + N(0, 0.1^2), shifts ~ N(0, 0.05^2);
  * MLP weights (3C, C) ~ N(0, 1/C) and (C, 3C) ~ N(0, 1/(3C)), biases ~ N(0, 0.02^2);
  * slots 14-23.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

SLOT = {"q": 0, "k": 1, "v": 2, "lce_w": 3, "lce_b": 4, "q_off": 5, "k_off": 6, "v_off": 7,
        "x": 8, "x_off": 9, "w_qkv": 10, "b_qkv": 11, "w_o": 12, "b_o": 13,
        "pos_w": 14, "pos_b": 15, "ln1_g": 16, "ln1_b": 17, "ln2_g": 18, "ln2_b": 19,
        "mlp_w1": 20, "mlp_b1": 21, "mlp_w2": 22, "mlp_b2": 23}


@dataclasses.dataclass(frozen=True)
class Workload:
    """One BRA forward problem: feature maps (N,H,W,C), `heads` heads, S x S regions."""

    name: str
    index: int          # seed namespace
    N: int
    H: int
    W: int
    C: int
    heads: int
    S: int
    topk: int
    dtype: str          # "f32" or "bf16"
    region_bias: float = 0.0   # std of the per-(image, region, channel) offset
    lce_b_std: float = 0.0
    lce_w_std: float = 0.02

    @property
    def d(self) -> int:
        return self.C // self.heads

    @property
    def regions(self) -> int:
        return self.S * self.S

    @property
    def hr(self) -> int:
        """Region height: ceil(H / S) (the padded grid when S does not divide H)."""
        return -(-self.H // self.S)

    @property
    def wr(self) -> int:
        return -(-self.W // self.S)

    @property
    def w2(self) -> int:
        return self.hr * self.wr

    @property
    def tokens(self) -> int:
        return self.N * self.H * self.W

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The BiFormer stage shapes used as parity cases and as the benchmark workload.
WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("stage1_tiny_224", 1, 1, 56, 56, 64, 2, 7, 1, "f32"),
        Workload("cls_stage2_224", 2, 64, 28, 28, 128, 4, 7, 4, "bf16", lce_b_std=0.01),
        Workload("cls_stage3_224", 3, 128, 14, 14, 256, 8, 7, 16, "bf16", lce_b_std=0.01),
        Workload("cls_stage3_224_dense", 6, 128, 14, 14, 256, 8, 7, 49, "bf16", lce_b_std=0.01),
        Workload("det_stage1_1024", 4, 2, 256, 256, 64, 2, 16, 1, "bf16", region_bias=0.5),
        Workload("seg_stage2_512", 5, 8, 64, 64, 128, 4, 8, 4, "bf16", region_bias=0.5),
        # a detection input whose stage-1 map (1000 / 4 = 250) is not a multiple of S = 16:
        # the padded grid (250 -> 256)
        Workload("det_stage1_1000", 7, 2, 250, 250, 64, 2, 16, 1, "bf16", region_bias=0.5),
    ]
}

# the benchmark default: the largest single-GPU workload (most tokens and attention FLOPs)
BENCH_WORKLOAD = "det_stage1_1024"


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)).astype(np.uint32)
    return r.view(np.float32)


def _rng(w: Workload, slot: str, seed_base: Optional[int]) -> np.random.Generator:
    base = 0xB1F0 + 16 * w.index if seed_base is None else seed_base
    return np.random.Generator(np.random.PCG64(base + SLOT[slot]))


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    x32 = x.astype(np.float32)
    return round_bf16(x32) if dtype == "bf16" else x32


def _region_field(off: np.ndarray, w: Workload) -> np.ndarray:
    """Spread per-region offsets (N,S,1,S,1,C) over the pixels of their regions, on the
    (padded) grid of ceil(H/S) x ceil(W/S) regions, cropped to H x W."""
    N, C = off.shape[0], off.shape[-1]
    full = np.broadcast_to(off, (N, w.S, w.hr, w.S, w.wr, C)).reshape(N, w.S * w.hr, w.S * w.wr, C)
    return full[:, :w.H, :w.W]


def make_inputs(w: Workload, seed_base: Optional[int] = None, batch: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Return q, k, v (N,H,W,C), lce_w (C,5,5), lce_b (C) as float32 arrays.

    When the workload dtype is bf16 every value is exactly representable in
    bfloat16. `batch` overrides N (the first `batch` images of a longer draw are
    NOT the same as a shorter draw; each call is its own sample).
    """
    N = w.N if batch is None else batch
    shape = (N, w.H, w.W, w.C)
    out = {}
    for name in ("q", "k", "v"):
        x = _rng(w, name, seed_base).standard_normal(shape)
        if w.region_bias > 0:
            off = _rng(w, name + "_off", seed_base).standard_normal((N, w.S, 1, w.S, 1, w.C)) * w.region_bias
            x = x + _region_field(off, w)
        out[name] = _store(x, w.dtype)
    out["lce_w"] = _store(_rng(w, "lce_w", seed_base).standard_normal((w.C, 5, 5)) * w.lce_w_std, w.dtype)
    if w.lce_b_std > 0:
        b = _rng(w, "lce_b", seed_base).standard_normal((w.C,)) * w.lce_b_std
    else:
        b = np.zeros((w.C,))
    out["lce_b"] = _store(b, w.dtype)
    return out


def make_layer_inputs(w: Workload, seed_base: Optional[int] = None, batch: Optional[int] = None
                      ) -> Dict[str, np.ndarray]:
    """Return x (N,H,W,C), w_qkv (3C,C), b_qkv (3C), w_o (C,C), b_o (C), lce_w, lce_b.

    float32 arrays whose values are exactly representable in the workload dtype.
    """
    N = w.N if batch is None else batch
    shape = (N, w.H, w.W, w.C)
    x = _rng(w, "x", seed_base).standard_normal(shape)
    if w.region_bias > 0:
        off = _rng(w, "x_off", seed_base).standard_normal((N, w.S, 1, w.S, 1, w.C)) * w.region_bias
        x = x + _region_field(off, w)
    g = 1.0 / np.sqrt(w.C)
    out = {
        "x": _store(x, w.dtype),
        "w_qkv": _store(_rng(w, "w_qkv", seed_base).standard_normal((3 * w.C, w.C)) * g, w.dtype),
        "b_qkv": _store(_rng(w, "b_qkv", seed_base).standard_normal((3 * w.C,)) * 0.02, w.dtype),
        "w_o": _store(_rng(w, "w_o", seed_base).standard_normal((w.C, w.C)) * g, w.dtype),
        "b_o": _store(_rng(w, "b_o", seed_base).standard_normal((w.C,)) * 0.02, w.dtype),
    }
    base = make_inputs(w, seed_base, batch)
    out["lce_w"] = base["lce_w"]
    out["lce_b"] = base["lce_b"]
    return out


def make_block_inputs(w: Workload, seed_base: Optional[int] = None, batch: Optional[int] = None
                      ) -> Dict[str, np.ndarray]:
    """make_layer_inputs plus pos_w (C,3,3), pos_b, ln1_g, ln1_b, ln2_g, ln2_b (C),
    mlp_w1 (3C,C), mlp_b1 (3C), mlp_w2 (C,3C), mlp_b2 (C): float32 arrays exactly
    representable in the workload dtype."""
    out = make_layer_inputs(w, seed_base, batch)
    C = w.C
    draw = lambda slot, shape, scale, shift=0.0: _store(
        shift + _rng(w, slot, seed_base).standard_normal(shape) * scale, w.dtype)
    out.update({
        "pos_w": draw("pos_w", (C, 3, 3), 0.2), "pos_b": draw("pos_b", (C,), 0.05),
        "ln1_g": draw("ln1_g", (C,), 0.1, 1.0), "ln1_b": draw("ln1_b", (C,), 0.05),
        "ln2_g": draw("ln2_g", (C,), 0.1, 1.0), "ln2_b": draw("ln2_b", (C,), 0.05),
        "mlp_w1": draw("mlp_w1", (3 * C, C), C ** -0.5), "mlp_b1": draw("mlp_b1", (3 * C,), 0.02),
        "mlp_w2": draw("mlp_w2", (C, 3 * C), (3 * C) ** -0.5), "mlp_b2": draw("mlp_b2", (C,), 0.02),
    })
    return out
