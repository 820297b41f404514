"""Benchmark of the B200 BRA forward (Bi-Level Routing Attention, BiFormer).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one whole BRA forward (region means, routing, routed attention + LCE)
over one batch of the workload, through the C ABI (`bra_forward`). Prints ONE JSON
line on rank 0.

Timing: W untimed warm-up steps, then exactly K steps bracketed by a barrier and a
device synchronise, timed with CUDA events on the launching stream; the max over
ranks is taken. Each step reads a different input set from a rotation whose total
size is at least three times the L2 cache, so inputs come from HBM, not L2. The
steps are replayed as CUDA graphs (one per input set) to take host launch cost out.
A second, traced pass over the same K steps times each kernel with CUDA events on
its own stream (bra_trace_*), for the roofline of the dominant kernel.

Multi-GPU (torchrun): images are independent, so every rank runs its own batch of
the workload with no collective on the data path ("scaling": "weak"); `value` is
the tokens of all ranks over the slowest rank's time.

--impl reference times the float64 CPU oracle on this host's cores (the only
reference this method has): each step is a bounded sample of the same workload.

--block times the whole BiFormer block (bra_block: pos-embed, LayerNorms, the attention
layer, the MLP) with the block's seeded inputs, under its own metric name.

--layer times the attention layer around BRA instead (bra_attention_layer: the qkv
projection, the BRA forward, the output projection) on the same workload shape, with
the layer's seeded inputs (x and the two projections' weights); its line carries its
own metric name.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from vision_transformer_sparse_b200 import synth  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "BRA fwd tokens/s and TFLOP/s at 1 B200; % of bf16 tensor/HBM roofline"
METRIC_LAYER = "BRA attention layer fwd (qkv projection + BRA + output projection) tokens/s at 1 B200"
METRIC_BLOCK = "BiFormer block fwd (pos-embed, LayerNorms, BRA attention layer, MLP) tokens/s at 1 B200"
METRIC_BWD = "BRA backward (routing detached) tokens/s at 1 B200"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--workload", default=synth.BENCH_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch each step directly")
    ap.add_argument("--layer", action="store_true",
                    help="time the whole attention layer (bra_attention_layer) instead of the BRA forward")
    ap.add_argument("--block", action="store_true",
                    help="time the whole BiFormer block (bra_block) instead of the BRA forward")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (bra_backward, routing detached) instead of the forward")
    ap.add_argument("--variant", default="auto", choices=["auto", "generic", "tma", "split", "pipe"],
                    help="attention kernel (auto: persistent TMA pipeline where the shape allows)")
    ap.add_argument("--source-hash", metavar="KERNEL",
                    help="print the source hash of a traced kernel class (for a profiles/ summary) and exit")
    return ap.parse_args()


# ----------------------------------------------------------------------------- accounting

def algorithmic(w: synth.Workload):
    """Per-forward algorithmic figures of the workload (one batch of N images)."""
    b = 2 if w.dtype == "bf16" else 4
    T = w.tokens
    L = w.topk * w.w2                               # keys per query
    flops = 4.0 * T * L * w.C                       # QK^T and PV, 2 flops per MAC
    gathered = float(w.N * w.regions * w.topk * w.w2 * 2 * w.C * b)  # K+V tiles per query region
    route_bytes = w.N * w.regions * w.topk * 8      # r_idx + r_weight
    # bytes the attention kernel must move at least once: q, k, v read, out written,
    # the routing read, the LCE parameters
    attn_unique = 4.0 * T * w.C * b + w.N * w.regions * w.topk * 4 + w.C * 26 * b
    pool_bytes = 2.0 * T * w.C * b + 2 * w.N * w.regions * w.C * 4
    # the one-kernel forward: q, k, v read once, out written once, r_idx and r_weight,
    # the LCE parameters
    fused_bytes = 4.0 * T * w.C * b + route_bytes + w.C * 26 * b
    # the projections (attention layer): qkv reads x and its weight and writes q, k, v;
    # wo reads the attention output and its weight and writes out. Per launch, averaged
    # over the two launches of a layer forward.
    lin_bytes = (4.0 * T * w.C * b + 3 * w.C * w.C * b + 2.0 * T * w.C * b + w.C * w.C * b) / 2
    lin_flops = 8.0 * T * w.C * w.C
    # the backward: q, k, v and dout read, dq, dk, dv written in float32, the routing and
    # the LCE weight read, its float32 gradients written (per call, all its kernels)
    bwd_bytes = 4.0 * T * w.C * b + 3.0 * T * w.C * 4 + w.N * w.regions * w.topk * 4 + w.C * 25 * (b + 4) + w.C * 4
    # the block's per-pixel kernels: pos_ln reads x and writes x1 and norm1's output; add_ln
    # reads x1 and the attention output and writes x2 and norm2's output (mean per launch)
    block_bytes = (3.0 * T * w.C * b + 4.0 * T * w.C * b) / 2
    return {"tokens": T, "flops": flops, "gathered_bytes": gathered, "attn_bytes": attn_unique,
            "block_bytes": block_bytes,
            "pool_bytes": pool_bytes, "route_bytes": route_bytes, "fused_bytes": fused_bytes,
            "linear_bytes": lin_bytes, "linear_flops": lin_flops, "bwd_bytes": bwd_bytes, "elem_bytes": b}


def method_roofline(acc, peaks, kernel_s):
    """The roofline of the method's own accounting for one forward: the slower of the
    attention FLOPs at the dense bf16 tensor peak (the burst figure: the kernel runs in
    sub-second graph replays, not a seconds-long loop) and the gathered K/V bytes at HBM
    bandwidth; `achieved` is that bound's quantity over the kernel's time `kernel_s`."""
    t_flop = acc["flops"] / (peaks["bf16_tflops"] * 1e12)
    t_gath = acc["gathered_bytes"] / (peaks["hbm_gbs"] * 1e9)
    common = {"algorithmic_flops_per_launch": acc["flops"], "gathered_bytes_per_launch": acc["gathered_bytes"],
              "definition": "max(attention FLOP / bf16 peak, gathered K/V bytes / HBM)"}
    if t_flop > t_gath:
        ach = acc["flops"] / kernel_s / 1e12
        return dict(common, bound="tensor", achieved=ach, peak=peaks["bf16_tflops"], unit="TFLOP/s",
                    frac=ach / peaks["bf16_tflops"], roofline_us=t_flop * 1e6)
    ach = acc["gathered_bytes"] / kernel_s / 1e9
    return dict(common, bound="hbm", achieved=ach, peak=peaks["hbm_gbs"], unit="GB/s", frac=ach / peaks["hbm_gbs"],
                roofline_us=t_gath * 1e6)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": float(pk["hbm_gbs"]), "bf16_tflops": float(pk["bf16_tflops"]),
                "bf16_tflops_sustained": float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"]))}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# The header that defines each traced kernel class; a class's source is that header and
# every header it includes from csrc/, so a committed profile stays valid until one of
# those files changes.
KERNEL_HEADERS = {
    "attn_umma_kernel": ["attn_umma.cuh"],
    "bra_image_kernel": ["fused_image.cuh"],
    "attn_bf16_kernel": ["attn_pipe.cuh", "attn_tma.cuh", "attn.cuh"],
    "attn_f32_kernel": ["attn.cuh"],
    "region_mean_kernel": ["route.cuh"],
    "route_kernel": ["route.cuh"],
    "linear_umma_kernel": ["linear.cuh"],
    "linear_f32_kernel": ["linear.cuh"],
    "bwd_kernels": ["backward.cuh", "backward_tc.cuh"],
    "block_pixel_kernels": ["block.cuh"],
    "pad_crop_kernels": ["pad.cuh"],
}


def kernel_sources(kernel: str):
    """Sorted csrc/ headers that make up `kernel` (its #include closure)."""
    csrc = os.path.join(ROOT, "vision_transformer_sparse_b200", "csrc")
    todo, seen = list(KERNEL_HEADERS.get(kernel, [])), set()
    if not todo:
        todo = [n for n in os.listdir(csrc) if n.endswith(".cuh")]
    while todo:
        name = todo.pop()
        if name in seen or not os.path.exists(os.path.join(csrc, name)):
            continue
        seen.add(name)
        with open(os.path.join(csrc, name)) as f:
            for line in f:
                line = line.strip()
                if line.startswith("#include \"") and line.endswith("\""):
                    todo.append(line[len("#include \""):-1])
    return sorted(seen)


def strip_comments(src: str) -> str:
    """C/C++ source without its comments, trailing blanks and empty lines (string and
    character literals kept as they are), so that a comment edit leaves the hash alone."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            while i < n and src[i] != "\n":
                i += 1
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (line.rstrip() for line in "".join(out).split("\n"))
    return "\n".join(line for line in lines if line)


def kernel_source_hash(kernel: str) -> str:
    """Hash of the kernel's header closure with comments and blank lines removed."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "vision_transformer_sparse_b200", "csrc")
    for name in kernel_sources(kernel):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from a committed ncu summary
    (profiles/<kernel>_<workload>.txt), if it was taken on the current kernel source
    (else None)."""
    path = os.path.join(ROOT, "profiles", "%s_%s.txt" % (kernel, workload))
    if not os.path.exists(path):
        return None, None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.split(":", 1)[0].strip() in ("source_hash", "dram_bytes_per_launch",
                                                                   "units_scale"):
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("source_hash") != kernel_source_hash(kernel) or "dram_bytes_per_launch" not in vals:
        return None, path
    return float(vals["dram_bytes_per_launch"]), path


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML in a background thread."""

    REASONS = {"gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
               "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
               "display_clock_setting": 0x100}

    def __init__(self, index: int, period_s: float = 0.005):
        self.samples = []
        self.ok = False
        self.period = period_s
        self._stop = threading.Event()
        self._mark = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report without clocks
            self.err = str(e)

    def _read(self):
        nv = self.nv
        sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        return sm, r

    def _run(self):
        while not self._stop.is_set():
            try:
                sm, r = self._read()
                self.samples.append((time.perf_counter(), sm, r, self._mark))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def mark(self, tag):
        self._mark = tag

    def sample_now(self):
        """One sample from the calling thread (used while the timed work drains)."""
        if self.ok:
            try:
                sm, r = self._read()
                self.samples.append((time.perf_counter(), sm, r, self._mark))
            except Exception:
                pass

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, tag="timed"):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        sel = [s for s in self.samples if s[3] == tag]
        note = "samples during the timed region"
        if not sel:
            sel = self.samples[-5:]
            note = "timed region shorter than the sampling period; nearest samples"
        mhz = [s[1] for s in sel]
        bits = 0
        for s in sel:
            bits |= s[2]
        reasons = [k for k, v in self.REASONS.items() if bits & v and k != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(sel), "note": note}


# ----------------------------------------------------------------------------- reference arm

def oracle_step(w: synth.Workload, sample: synth.Workload, layer: bool, backward: bool = False, block: bool = False):
    """One call of the oracle on `sample` (the BRA forward, the whole layer, the block, or the
    backward for the forward's routing)."""
    import oracle
    if block:
        from oracle import block as ob
        inp = {k: v.astype(np.float64) for k, v in synth.make_block_inputs(sample).items()}
        prm = {k: v for k, v in inp.items() if k != "x"}
        return lambda: ob.block_forward(inp["x"], prm, w.heads, w.S, w.topk, w.dtype)
    if backward:
        from oracle import backward as ob
        inp = {k: v.astype(np.float64) for k, v in synth.make_inputs(sample).items()}
        dout = synth.make_inputs(sample, seed_base=0xB0D0 + sample.index)["q"].astype(np.float64)
        r_idx, _ = oracle.route(inp["q"], inp["k"], w.heads, w.S, w.topk)
        return lambda: ob.backward(inp["q"], inp["k"], inp["v"], inp["lce_w"], inp["lce_b"], w.heads, w.S, r_idx, dout)
    if layer:
        inp = {k: v.astype(np.float64) for k, v in synth.make_layer_inputs(sample).items()}
        keys = ("x", "w_qkv", "b_qkv", "w_o", "b_o", "lce_w", "lce_b")
        return lambda: oracle.layer_forward(*(inp[k] for k in keys), w.heads, w.S, w.topk, w.dtype)
    inp = {k: v.astype(np.float64) for k, v in synth.make_inputs(sample).items()}
    return lambda: oracle.forward(inp["q"], inp["k"], inp["v"], inp["lce_w"], inp["lce_b"], w.heads, w.S, w.topk)


def bench_reference(args, w: synth.Workload, rank: int):
    """The float64 CPU oracle on this host's cores; each step one image of the workload."""
    import oracle
    if rank != 0:
        return None
    sample = w.with_(N=1)
    step = oracle_step(w, sample, args.layer, args.backward, args.block)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = sample.tokens * args.steps / dt
    cores = oracle.threads()
    line = {
        "impl": "reference", "metric": METRIC_BWD if args.backward else (
            METRIC_BLOCK if args.block else (METRIC_LAYER if args.layer else METRIC)),
        "value": value, "unit": "tokens/s", "n_gpus": 0,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1), BiFormer stage shape)",
        "config": {"workload": w.name, "N_per_gpu": w.N, "images_per_step": sample.N, "H": w.H, "W": w.W,
                   "C": w.C, "heads": w.heads, "S": w.S, "topk": w.topk, "input_dtype": w.dtype,
                   "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": "1 image (%d tokens) of the workload per step; ms_per_step is per image"
                                   % sample.tokens},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


def cpu_baseline(w: synth.Workload, budget_s: float = 12.0, layer: bool = False, backward: bool = False,
                 block: bool = False):
    """The oracle as it stands on a bounded sample: whole images (at most 8), repeated
    until about `budget_s` seconds of host time are used (at least once)."""
    import oracle
    sample = w.with_(N=max(1, min(w.N, 8)))
    step = oracle_step(w, sample, layer, backward, block)
    reps, t0 = 0, time.perf_counter()
    while True:
        step()
        reps += 1
        dt = time.perf_counter() - t0
        if dt > budget_s:
            break
    return {"value": sample.tokens * reps / dt, "unit": "tokens/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": "%d x %s of %d images (%d tokens), %.1f s" % (reps, "backward" if backward else
                                                                   ("block" if block else
                                                                    ("layer" if layer else "forward")),
                                                                   sample.N, sample.tokens, dt)}


# ----------------------------------------------------------------------------- our arm

def main():
    args = parse()
    if args.source_hash:
        print("%s %s (%s)" % (args.source_hash, kernel_source_hash(args.source_hash),
                              " ".join(kernel_sources(args.source_hash))))
        return
    w = synth.WORKLOADS[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if world > 1:
            # rank 0 alone runs and prints; the others exit without work
            if rank != 0:
                return
        line = bench_reference(args, w, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist

    from vision_transformer_sparse_b200 import bra

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    bra.set_kernel_variant({"auto": bra.VARIANT_AUTO, "generic": bra.VARIANT_GENERIC,
                            "tma": bra.VARIANT_TMA, "split": bra.VARIANT_SPLIT,
                            "pipe": bra.VARIANT_PIPE}[args.variant])
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    acc = algorithmic(w)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    # inputs: this rank's own batch (weak scaling); seeded per rank
    seed = None if rank == 0 else 0xB1F0 + 16 * w.index + 1000 * rank
    block = args.block
    layer, backward = args.layer or block, args.backward
    inp = (synth.make_block_inputs(w, seed_base=seed) if block else
           synth.make_layer_inputs(w, seed_base=seed) if layer else synth.make_inputs(w, seed_base=seed))
    if backward:  # dL/dout: another seeded map of the same shape, stored in the dtype
        inp["dout"] = synth.make_inputs(w, seed_base=0xB0D0 + w.index + 1000 * rank)["q"]
    base = {k: torch.from_numpy(v).to(dev).to(tdt).contiguous() for k, v in inp.items()}
    lead = "x" if layer else "q"  # the (N,H,W,C) input whose shape the output takes
    if backward:  # the forward's routing, computed once on the device
        _, r0, _ = bra.forward(base["q"], base["k"], base["v"], base["lce_w"], base["lce_b"], w.heads, w.S, w.topk)
        base["r_idx"] = r0
        torch.cuda.synchronize(dev)
    # bytes of one input set plus its output (the layer's q, k, v and attention output
    # are the library's scratch, produced and consumed inside the step)
    set_bytes = (2 if layer else 4) * w.tokens * w.C * acc["elem_bytes"]
    if backward:
        set_bytes = 5 * w.tokens * w.C * acc["elem_bytes"] + 3 * w.tokens * w.C * 4
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    n_sets = max(2, math.ceil(3 * l2 / set_bytes))
    sets = []
    for _ in range(n_sets):
        s = {k: v.clone() for k, v in base.items()}
        s["out"] = torch.empty_like(base[lead])
        if not backward:  # the backward reads the forward's routing (copied with the set)
            s["r_idx"] = torch.empty((w.N, w.regions, w.topk), dtype=torch.int32, device=dev)
        s["r_w"] = torch.empty((w.N, w.regions, w.topk), dtype=torch.float32, device=dev)
        if backward:  # the gradients of each set, written in place by every step
            f32 = dict(dtype=torch.float32, device=dev)
            s["grads"] = {"dq": torch.empty((w.N, w.H, w.W, w.C), **f32), "dk": torch.empty((w.N, w.H, w.W, w.C), **f32),
                          "dv": torch.empty((w.N, w.H, w.W, w.C), **f32), "dlce_w": torch.empty((w.C, 5, 5), **f32),
                          "dlce_b": torch.empty((w.C,), **f32)}
        sets.append(s)

    stream = torch.cuda.Stream(device=dev)

    def fwd(s, sync=False):
        if backward:  # timed and traced: the asynchronous entry point (graph-capturable)
            bra.backward(s["q"], s["k"], s["v"], s["lce_w"], s["r_idx"], s["dout"], w.heads, w.S, stream=stream,
                         grads=s["grads"], sync=sync)
        elif block:
            bra.block(s["x"], s, w.heads, w.S, w.topk, out=s["out"], r_idx=s["r_idx"], r_weight=s["r_w"],
                      stream=stream)
        elif layer:
            bra.attention_layer(s["x"], s["w_qkv"], s["b_qkv"], s["w_o"], s["b_o"], s["lce_w"], s["lce_b"],
                                w.heads, w.S, w.topk, out=s["out"], r_idx=s["r_idx"], r_weight=s["r_w"],
                                stream=stream)
        else:
            bra.forward(s["q"], s["k"], s["v"], s["lce_w"], s["lce_b"], w.heads, w.S, w.topk,
                        out=s["out"], r_idx=s["r_idx"], r_weight=s["r_w"], stream=stream)

    # one CUDA graph per input set
    graphs = []
    kernels_per_step = None
    with torch.cuda.stream(stream):
        fwd(sets[0])  # first call outside capture: lazy module load, pool init
    stream.synchronize()
    if not args.no_graph:
        for s in sets:
            g = torch.cuda.CUDAGraph()
            c0 = bra.launch_count()
            with torch.cuda.graph(g, stream=stream):
                fwd(s)
            kernels_per_step = bra.launch_count() - c0
            graphs.append(g)

    def run_step(i):
        if graphs:
            graphs[i % n_sets].replay()
        else:
            fwd(sets[i % n_sets])

    clocks = ClockSampler(local)
    clocks.start()
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            run_step(i)
    stream.synchronize()

    # ---- timed region
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    c_launch0 = bra.launch_count()
    clocks.mark("timed")
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for i in range(args.steps):
            run_step(i)
        ev1.record(stream)
    # the host enqueues far faster than the device runs: sample the clocks until the
    # timed work has drained, so that even a short timed region has samples inside it
    while not ev1.query():
        clocks.sample_now()
    torch.cuda.synchronize(dev)
    clocks.mark(None)
    if world > 1:
        dist.barrier()
    ms = ev0.elapsed_time(ev1)
    direct_launches = bra.launch_count() - c_launch0
    gpu_launches = direct_launches if not graphs else kernels_per_step * args.steps
    if world > 1:
        t = torch.tensor([ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())

    # ---- traced pass: per-kernel device time. Each input set's forward is captured
    # again with an event pair around every kernel (event-record nodes), the graphs are
    # replayed for at least K steps, and the pairs are read after every round.
    torch.cuda.synchronize(dev)
    bra.trace_begin()
    trace = {}
    traced = []
    with torch.cuda.stream(stream):
        for s_ in sets:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                fwd(s_)
            traced.append(g)
    rounds = max(1, math.ceil(args.steps / n_sets))
    for _ in range(rounds):
        with torch.cuda.stream(stream):
            for g in traced:
                g.replay()
        torch.cuda.synchronize(dev)
        for k_, (t_ms, t_n) in bra.trace_read().items():
            a_ = trace.setdefault(k_, [0.0, 0])
            a_[0] += t_ms
            a_[1] += t_n
    del traced
    traced_steps = rounds * n_sets
    bra.trace_end()
    clocks.stop()

    # ---- end to end through the public API from pinned host memory: the host-buffer
    # entry point for the forward; for the layer, copies on the stream around the
    # device call
    host = {k: v.cpu().pin_memory() for k, v in base.items()}
    h_out = torch.empty_like(host[lead]).pin_memory()
    h_idx = torch.empty((w.N, w.regions, w.topk), dtype=torch.int32).pin_memory()
    h_w = torch.empty((w.N, w.regions, w.topk), dtype=torch.float32).pin_memory()
    d_in = sets[0]
    if backward:
        host = {k: v.cpu().pin_memory() for k, v in base.items()}
        h_grads = {k: torch.empty(v.shape, dtype=torch.float32).pin_memory() for k, v in sets[0]["grads"].items()}

    def e2e_step():
        if backward:
            with torch.cuda.stream(stream):
                for k_, v_ in host.items():
                    d_in[k_].copy_(v_, non_blocking=True)
                fwd(d_in, sync=True)  # the synchronising public entry point
                for k_, t_ in d_in["grads"].items():
                    h_grads[k_].copy_(t_, non_blocking=True)
            stream.synchronize()
        elif layer:
            with torch.cuda.stream(stream):
                for k_, v_ in host.items():
                    d_in[k_].copy_(v_, non_blocking=True)
                fwd(d_in)
                h_out.copy_(d_in["out"], non_blocking=True)
                h_idx.copy_(d_in["r_idx"], non_blocking=True)
                h_w.copy_(d_in["r_w"], non_blocking=True)
            stream.synchronize()
        else:
            bra.forward_host(host["q"], host["k"], host["v"], host["lce_w"], host["lce_b"], w.heads, w.S, w.topk,
                             out=h_out, r_idx=h_idx, r_weight=h_w, stream=stream)

    for _ in range(3):
        e2e_step()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    if world > 1:
        t = torch.tensor([e2e_ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = h_out.numel() * h_out.element_size() + h_idx.numel() * 4 + h_w.numel() * 4
    if backward:
        d2h = sum(t.numel() * 4 for t in h_grads.values())

    if rank != 0:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return

    ms_step = ms / args.steps
    tokens_all = acc["tokens"] * world
    value = tokens_all * args.steps / (ms / 1e3)
    tflops = acc["flops"] * world * args.steps / (ms / 1e3) / 1e12

    peaks, peak_kind = load_peaks()
    # the dominant kernel (largest share of device time) and its algorithmic bytes
    attn_name = max((v[0], k) for k, v in trace.items() if v[1])[1]
    t_ms, t_n = trace[attn_name]
    traced_s = t_ms / max(t_n, 1) / 1e3
    launches_per_step = t_n / max(traced_steps, 1)
    # the traced time carries the cost of its event pair; no launch can take longer than
    # its share of the timed step, so the kernel time used below is the smaller of the two
    attn_s = min(traced_s, ms_step / 1e3 / max(launches_per_step, 1e-9))
    alg_bytes = {"bra_image_kernel": acc["fused_bytes"], "region_mean_kernel": acc["pool_bytes"],
                 "route_kernel": acc["route_bytes"], "linear_umma_kernel": acc["linear_bytes"],
                 "linear_f32_kernel": acc["linear_bytes"],
                 "block_pixel_kernels": acc["block_bytes"]}.get(attn_name, acc["attn_bytes"])
    if backward:  # the backward's kernels form one traced class: time per call
        traced_s = t_ms / max(traced_steps, 1) / 1e3
        attn_s = min(traced_s, ms_step / 1e3)
        alg_bytes = acc["bwd_bytes"]
    step_traced_ms = sum(v[0] for v in trace.values()) / traced_steps
    share = {k: round(v[0] / max(1e-12, sum(x[0] for x in trace.values())), 4) for k, v in trace.items() if v[1]}
    traffic, _ = profiled_traffic(attn_name, w.name)
    unique = {"bound": "hbm", "kernel": attn_name, "achieved": alg_bytes / attn_s / 1e9, "peak": peaks["hbm_gbs"],
              "unit": "GB/s", "frac": alg_bytes / attn_s / 1e9 / peaks["hbm_gbs"], "traffic": traffic,
              "algorithmic_bytes_per_launch": alg_bytes, "avg_launch_us": attn_s * 1e6,
              "traced_launch_us": traced_s * 1e6, "peak_source": peak_kind,
              "definition": "bytes the kernel must move at least once (q, k, v read, out written, routing, "
                            "LCE parameters) / HBM"}
    if backward or layer:
        roofline = unique
    else:
        roofline = method_roofline(acc, peaks, attn_s)
        roofline.update({"kernel": attn_name, "traffic": traffic, "avg_launch_us": attn_s * 1e6,
                         "traced_launch_us": traced_s * 1e6, "step_frac": roofline["roofline_us"] / (ms_step * 1e3),
                         "peak_source": peak_kind + (" (burst bf16)" if roofline["bound"] == "tensor" else "")})
    line = {
        "metric": METRIC_BWD if backward else (METRIC_BLOCK if block else (METRIC_LAYER if layer else METRIC)),
        "value": value,
        "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded N(0,1), BiFormer stage shape; no dataset)",
        "config": {"workload": w.name, "N_per_gpu": w.N, "H": w.H, "W": w.W, "C": w.C, "heads": w.heads,
                   "S": w.S, "topk": w.topk, "global_batch": w.N * world,
                   "l2": "inputs larger than L2: %d rotating input sets, %.0f MB each, %.0f MB total vs L2 %.0f MB"
                         % (n_sets, set_bytes / 1e6, n_sets * set_bytes / 1e6, l2 / 1e6),
                   "launch": "CUDA graph per step" if graphs else "direct launches",
                   "attention_kernel": args.variant,
                   "step": "bra_backward_async (routing detached, the forward's r_idx)" if backward else
                           ("bra_block (pos-embed, norm1, attention layer, norm2, MLP)" if block else
                            "bra_attention_layer (qkv projection, BRA, output projection)" if layer
                            else "bra_forward"),
                   "parallelism": "dp%d (independent images, no collective)" % world},
        "tflops": tflops,
        "gpu_launches": gpu_launches,
        "roofline": roofline,
        "roofline_unique": unique,
        "kernels": {k: {"ms_total": round(v[0], 4), "launches": v[1], "us_per_launch": round(v[0] * 1e3 / v[1], 3),
                        "share": share.get(k)} for k, v in trace.items() if v[1]},
        "traced_step_ms": step_traced_ms,
        "clocks": clocks.summary(),
        "e2e": {"value": tokens_all * args.e2e_steps / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
                "entry": "bra_backward (synchronising) with stream copies (pinned host buffers)" if backward else
                         ("bra_block with stream copies (pinned host buffers)" if block else
                          "bra_attention_layer with stream copies (pinned host buffers)" if layer
                          else "bra_forward_host (pinned host buffers)")},
    }
    if backward:  # the forward's FLOP accounting does not describe this step
        line.pop("tflops")
    if backward or layer:
        line.pop("roofline_unique")
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, layer=layer, backward=backward, block=block)
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
