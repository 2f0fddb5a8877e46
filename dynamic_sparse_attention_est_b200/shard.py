"""Host-side pieces of running the path on several GPUs.

The path has no exchange step: every head (and every layer) is independent
(news article "单卡A100实现百万token推理…", section 方法介绍: patterns and indices
are per head).  So multi-GPU runs either replicate layers (one layer per rank,
weak scaling) or shard the heads of one layer (whole GQA groups per rank, then
one all-gather that assembles the output on every rank); the other collective
is the max-over-ranks reduction of the measured time.
"""
from __future__ import annotations

from typing import Dict, List, Sequence

import torch

# Relative cost of one q-head by pattern: the share of the causal key tiles its
# mask makes the kernel compute, measured on the 1M-token synthetic layer
# (Vertical-Slash ~0.5, Block-Sparse 100/16384 blocks, A-shape 4224/1M keys).
PATTERN_COST = {"dense": 1.0, "vs": 0.5, "block": 0.0125, "ashape": 0.005, "trishape": 0.006}


def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws its own layer."""
    return seed + 1009 * rank


def partition_heads(head_patterns: Sequence[str], hkv: int, world: int) -> List[List[int]]:
    """Longest-processing-time assignment of whole GQA groups to ranks.

    A group (one kv-head and its q-heads) stays on one rank so that its K and V
    are read by one GPU only.  Returns, per rank, the ascending q-head ids.
    """
    hq = len(head_patterns)
    grp = hq // hkv
    costs = []
    for g in range(hkv):
        heads = list(range(g * grp, (g + 1) * grp))
        costs.append((sum(PATTERN_COST[head_patterns[h]] for h in heads), g, heads))
    costs.sort(key=lambda c: (-c[0], c[1]))
    load = [0.0] * world
    out: List[List[int]] = [[] for _ in range(world)]
    for cost, _, heads in costs:
        r = min(range(world), key=lambda i: (load[i], i))
        load[r] += cost
        out[r].extend(heads)
    return [sorted(x) for x in out]


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of `value` over the ranks of the default process group."""
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_summary(parts: List[List[int]], head_patterns: Sequence[str]) -> Dict[int, float]:
    return {r: sum(PATTERN_COST[head_patterns[h]] for h in p) for r, p in enumerate(parts)}


def gather_heads(local: torch.Tensor, parts: List[List[int]], hq: int) -> torch.Tensor:
    """Assembles the per-rank head outputs of one layer on every rank.

    ``local`` holds this rank's heads, in the order of ``parts[rank]``, along
    dim 0.  Every rank pads its shard to the largest shard, one all-gather
    (NCCL on GPUs, gloo on CPU) exchanges them, and the rows are put back in
    head order: the result has ``hq`` heads along dim 0.
    """
    import torch.distributed as dist

    world = dist.get_world_size()
    m = max(len(p) for p in parts)
    pad = torch.zeros((m,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    pad[:local.shape[0]] = local
    bufs = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(bufs, pad)
    out = torch.empty((hq,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    for r, p in enumerate(parts):
        if p:
            out[torch.tensor(p, device=local.device)] = bufs[r][:len(p)]
    return out
