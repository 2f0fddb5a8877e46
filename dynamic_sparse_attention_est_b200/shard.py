"""Host-side pieces of running the path on several GPUs.

The path has no exchange step: every head (and every layer) is independent
(news article "单卡A100实现百万token推理…", section 方法介绍: patterns and indices
are per head).  So multi-GPU runs either replicate layers (one layer per rank,
weak scaling) or shard the heads of one layer; the only collective is the
max-over-ranks reduction of the measured time.
"""
from __future__ import annotations

from typing import Dict, List, Sequence

import torch

# Relative cost of one q-head by pattern: the share of the causal key tiles its
# mask makes the kernel compute, measured on the 1M-token synthetic layer
# (Vertical-Slash ~0.5, Block-Sparse 100/16384 blocks, A-shape 4224/1M keys).
PATTERN_COST = {"dense": 1.0, "vs": 0.5, "block": 0.0125, "ashape": 0.005}


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
