"""Multi-process (gloo, world size 2, CPU) checks of the batch-sharded path.

BRA never crosses images: region means, routing, the routed attention and the LCE
all stay inside one image (and the projections of the attention layer act per token). So N images split over ranks, each rank running its own
share with no exchange, must give exactly the full-batch result, and the benchmark
only needs a max-over-ranks reduction of its timings. The ranks here run the oracle
(there is no GPU in this test); the property checked is the partition itself.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from vision_transformer_sparse_b200 import synth

W = synth.WORKLOADS["seg_stage2_512"].with_(N=4, H=16, W=16)   # 4 images of 16x16, S=8


def shard(n_items: int, world: int, rank: int):
    """Contiguous, near-equal split of n_items over ranks."""
    base, extra = divmod(n_items, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


LAYER_KEYS = ("x", "w_qkv", "b_qkv", "w_o", "b_o", "lce_w", "lce_b")


def _run(inp, a, b, layer):
    """The forward (or the whole layer) of images a .. b-1."""
    if layer:
        args = [inp[k] for k in LAYER_KEYS]
        args[0] = args[0][a:b]
        return oracle.layer_forward(*args, W.heads, W.S, W.topk, W.dtype)
    return oracle.forward(*(inp[k][a:b] for k in ("q", "k", "v")), inp["lce_w"], inp["lce_b"], W.heads, W.S,
                          W.topk)


def _rank_main(rank, world, port, result_path, layer=False):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = synth.make_layer_inputs(W) if layer else synth.make_inputs(W)
        a, b = shard(W.N, world, rank)
        out, r_idx, r_w = _run(inp, a, b, layer)
        parts = [None] * world
        dist.all_gather_object(parts, (a, b, out, r_idx, r_w))
        t = torch.tensor([1.0 + rank], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        if rank == 0:
            full_out, full_idx, full_w = _run(inp, 0, W.N, layer)
            cat_out = np.concatenate([p[2] for p in parts])
            cat_idx = np.concatenate([p[3] for p in parts])
            cat_w = np.concatenate([p[4] for p in parts])
            ok = (np.array_equal(cat_idx, full_idx) and np.array_equal(cat_w, full_w)
                  and np.array_equal(cat_out, full_out) and t.item() == float(world)
                  and [p[:2] for p in parts] == [shard(W.N, world, r) for r in range(world)])
            with open(result_path, "w") as f:
                f.write("ok" if ok else "mismatch")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_shard_covers_batch():
    for n in range(0, 9):
        for world in (1, 2, 3, 4):
            spans = [shard(n, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            assert max(b - a for a, b in spans) - min(b - a for a, b in spans) <= 1


@pytest.mark.timeout(300)
def test_two_rank_batch_split_equals_full_batch(tmp_path):
    result = str(tmp_path / "result.txt")
    mp.spawn(_rank_main, args=(2, _free_port(), result), nprocs=2, join=True)
    assert open(result).read() == "ok"


@pytest.mark.timeout(300)
def test_two_rank_layer_split_equals_full_batch(tmp_path):
    """The same partition for the attention layer (qkv projection, BRA, output projection)."""
    result = str(tmp_path / "result.txt")
    mp.spawn(_rank_main, args=(2, _free_port(), result, True), nprocs=2, join=True)
    with open(result) as f:
        assert f.read() == "ok"


def _rank_backward(rank, world, port, result_path):
    """Data-parallel backward: each rank takes its images; the per-image gradients (dq, dk,
    dv) are concatenated, the LCE parameter gradients (sums over the batch) all-reduced."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import backward as ob
        inp = synth.make_inputs(W)
        dout = synth.make_inputs(W, seed_base=0xB0D0)["q"]
        r_idx, _ = oracle.route(inp["q"], inp["k"], W.heads, W.S, W.topk)
        a, b = shard(W.N, world, rank)
        g = ob.backward(*(inp[k][a:b] for k in ("q", "k", "v")), inp["lce_w"], inp["lce_b"], W.heads, W.S,
                        r_idx[a:b], dout[a:b])
        for name in ("dlce_w", "dlce_b"):
            t = torch.from_numpy(g[name].copy())
            dist.all_reduce(t, op=dist.ReduceOp.SUM)
            g[name] = t.numpy()
        parts = [None] * world
        dist.all_gather_object(parts, {k: g[k] for k in ("dq", "dk", "dv")})
        if rank == 0:
            full = ob.backward(inp["q"], inp["k"], inp["v"], inp["lce_w"], inp["lce_b"], W.heads, W.S, r_idx, dout)
            ok = all(np.allclose(np.concatenate([p[k] for p in parts]), full[k], rtol=1e-12, atol=1e-12)
                     for k in ("dq", "dk", "dv"))
            ok = ok and all(np.allclose(g[k], full[k], rtol=1e-12, atol=1e-12) for k in ("dlce_w", "dlce_b"))
            with open(result_path, "w") as f:
                f.write("ok" if ok else "mismatch")
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_rank_backward_shards_and_all_reduces_parameter_gradients(tmp_path):
    result = str(tmp_path / "result.txt")
    mp.spawn(_rank_backward, args=(2, _free_port(), result), nprocs=2, join=True)
    with open(result) as f:
        assert f.read() == "ok"
