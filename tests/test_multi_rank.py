"""The multi-rank path on CPU: two gloo ranks share the heads of one layer.

Each rank attends its own shard of GQA groups (computed here with the fp64
oracle standing in for the per-rank kernels), the shards are gathered with the
padded all-gather the benchmark uses, and the result must equal the
single-process layer; the timing reduction returns the maximum over ranks.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from dynamic_sparse_attention_est_b200 import shard, synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, result_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle

    w = synth.WORKLOADS["mixed-gqa-1m"]
    pats = synth.mixed_head_patterns(w, seed=3, hq=8)
    x = synth.generate(synth.Workload("mr", "vs", 8, 4, 256, "vertical", n_heavy=4), seed=5)
    parts = shard.partition_heads(pats, 4, world)
    mine = parts[rank]
    orc = oracle.get()
    out, _ = orc.dense_attention(x["q"], x["k"], x["v"], 0.088, head_ids=mine)
    full = shard.gather_heads(torch.from_numpy(out), parts, 8)  # padded all-gather, head order restored
    t = shard.max_over_ranks(1.0 + rank)
    if rank == 0:
        ref, _ = orc.dense_attention(x["q"], x["k"], x["v"], 0.088)
        np.save(result_path, np.array([np.abs(full.numpy() - ref).max(), t,
                                       len(set(parts[0]) & set(parts[1])), sum(len(p) for p in parts)]))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_assemble_the_layer(tmp_path):
    res = str(tmp_path / "res.npy")
    mp.start_processes(_worker, args=(2, _free_port(), res), nprocs=2, join=True, start_method="spawn")
    err, tmax, overlap, total = np.load(res)
    assert err == 0.0
    assert tmax == 2.0
    assert overlap == 0 and total == 8


@pytest.mark.parametrize("n", [32768, 1 << 20])
def test_partition_is_balanced_and_keeps_groups_whole(n):
    w = synth.WORKLOADS["mixed-gqa-1m"]
    pats = synth.mixed_head_patterns(w, seed=0)
    cost = {p: shard.pattern_cost(p, n) for p in set(pats)}
    for world in (1, 2, 4, 8):
        parts = shard.partition_heads(pats, 8, world, n)
        flat = sorted(h for p in parts for h in p)
        assert flat == list(range(32))
        for p in parts:
            assert all(((h // 4) * 4 + i) in p for h in p for i in range(4))  # whole groups
        loads = shard.shard_summary(parts, pats, n)
        heaviest_group = max(sum(cost[pats[g * 4 + i]] for i in range(4)) for g in range(8))
        assert max(loads.values()) - min(loads.values()) <= heaviest_group + 1e-9


def test_pattern_costs_follow_the_tile_plan():
    """Closed forms against hand counts of the kernel's tile plan."""
    # dense causal at 256 tokens: query tiles 0 and 1 compute 1 and 2 tiles
    assert shard.head_tiles("dense", 256) == 3
    # A-shape whose window covers everything is dense
    assert shard.head_tiles("ashape", 4096, window=4096) == shard.head_tiles("dense", 4096)
    # Tri-shape with every row in the dense tail is dense; with none it is A-shape
    assert shard.head_tiles("trishape", 8192, n_last=8192) == shard.head_tiles("dense", 8192)
    assert shard.head_tiles("trishape", 8192, n_last=0) == shard.head_tiles("ashape", 8192)
    # A-shape at 128K, counted tile by tile: 2 sink halves, then the window's halves
    # from the one holding key r0 - 4095 up to the diagonal half (or every causal
    # half while the window still reaches the sinks)
    n, tiles = 131072, 0
    for t in range(n // 128):
        r0, hi = 128 * t, 2 * t + 1
        w_lo = max(0, r0 - 4095) // 64
        halves = (2 + hi - w_lo + 1) if w_lo > 2 else hi + 1
        tiles += (halves + 1) // 2  # a tile is two halves
    assert shard.head_tiles("ashape", n) == tiles
    # Block-Sparse with every block selected is dense
    assert shard.head_tiles("block", 4096, topk=64) == shard.head_tiles("dense", 4096)
    # Vertical-Slash: at 32K the slash ranges cover the causal tiles; at 1M about half
    assert shard.pattern_cost("vs", 32768) > 0.99
    assert 0.4 < shard.pattern_cost("vs", 1 << 20) < 0.7
    assert shard.pattern_cost("block", 1 << 20) < shard.pattern_cost("block", 32768)


def test_rank_seeds_differ():
    assert len({shard.rank_seed(0, r) for r in range(8)}) == 8


def _gather_worker(rank, world, port, result_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    # 4 GQA groups of 2 q-heads over 3 ranks: shards of unequal size
    pats = ["vs", "vs", "block", "block", "ashape", "ashape", "dense", "dense"]
    parts = shard.partition_heads(pats, 4, world)
    local = torch.stack([torch.full((3, 5), float(h)) for h in parts[rank]]) if parts[rank] else torch.zeros(0, 3, 5)
    full = shard.gather_heads(local, parts, 8)
    if rank == 0:
        np.save(result_path, np.array([full[h].eq(float(h)).all().item() for h in range(8)] +
                                      [len(p) for p in parts]))
    dist.barrier()
    dist.destroy_process_group()


def test_gather_heads_unequal_shards(tmp_path):
    """Three ranks with shards of different sizes: the padded all-gather puts every head back in place."""
    res = str(tmp_path / "gather.npy")
    mp.start_processes(_gather_worker, args=(3, _free_port(), res), nprocs=3, join=True, start_method="spawn")
    r = np.load(res)
    assert r[:8].all()
    sizes = r[8:].tolist()
    assert sum(sizes) == 8 and max(sizes) != min(sizes), sizes  # the padding was exercised
