"""Host-side pieces of running the path on several GPUs.

The path has no exchange step: every head (and every layer) is independent
(news article "单卡A100实现百万token推理…", section 方法介绍: patterns and indices
are per head).  So multi-GPU runs either replicate layers (one layer per rank,
weak scaling) or shard the heads of one layer (whole GQA groups per rank, then
one all-gather that assembles the output on every rank); the other collective
is the max-over-ranks reduction of the measured time.
"""
from __future__ import annotations

import functools
import math
from typing import Dict, List, Sequence

import numpy as np
import torch

# Relative cost of one q-head by pattern: the 128x128 tiles the attention
# kernel computes for it at n tokens, from the kernel's own tile plan (dense,
# A-shape, Tri-shape exactly; Block-Sparse and Vertical-Slash from their
# budgets under a model of the index sets, see `head_tiles`), as a share of the
# dense causal head.  A Vertical-Slash head at 32K tokens costs a dense head
# (its 6,096 slash ranges cover every causal tile); at 1M about half of one.
DEFAULT_PARAMS = dict(n_vertical=1000, n_slash=6096, topk=100, n_sink=128, window=4096, n_last=64)


@functools.lru_cache(maxsize=256)
def head_tiles(pattern: str, n: int, n_vertical: int = 1000, n_slash: int = 6096, topk: int = 100,
               n_sink: int = 128, window: int = 4096, n_last: int = 64) -> float:
    """Predicted 128x128 tiles (two 64-key halves each) computed for one q-head.

    Per 128-row query tile t (rows r0 = 128 t ...):
      dense          the causal halves, min(2t + 2, n / 64);
      ashape         the sink halves plus the window halves (or the causal ones
                     where they meet), as the kernel's tile plan walks them;
      trishape       the same, with tiles holding the last n_last rows dense;
      block          the union of the two query blocks' lists of min(topk, b + 1)
                     blocks, their overlap taken as that of independent draws
                     from the causal prefix;
      vs             slash offsets spread evenly over [0, n): each reaches a
                     128-key range, so a key is covered with probability
                     1 - exp(-128 n_slash / n); the verticals fill the uncovered
                     rest, 64 per half.
    """
    nb64 = n // 64
    t = np.arange((n + 127) // 128, dtype=np.float64)
    r0 = 128.0 * t
    hi = np.minimum(2.0 * t + 1, nb64 - 1)
    causal = hi + 1
    if pattern == "dense":
        halves = causal
    elif pattern in ("ashape", "trishape"):
        sink_h = min(-(-n_sink // 64), nb64)
        w_lo = np.floor(np.maximum(0.0, r0 - window + 1) / 64)
        split = w_lo > sink_h
        if pattern == "trishape":
            split &= np.minimum(r0 + 127, n - 1) < n - n_last
        halves = np.where(split, sink_h + (hi - w_lo + 1), causal)
    elif pattern == "block":
        b0, b1 = 2.0 * t, 2.0 * t + 1
        k0 = np.minimum(topk, b0 + 1)
        k1 = np.where(b1 < nb64, np.minimum(topk, b1 + 1), 0.0)
        halves = np.minimum(causal, k0 + k1 - k0 * k1 / (b1 + 1))
    elif pattern == "vs":
        keys = np.minimum(r0 + 128, n)
        cov = 1.0 - math.exp(-128.0 * min(n_slash, n) / n)
        halves = np.minimum(causal, keys * cov / 64 + np.minimum(n_vertical, keys) * (1 - cov) / 64 + 1)
    else:
        raise ValueError(pattern)
    return float(np.ceil(halves / 2).sum())


def pattern_cost(pattern: str, n: int, **params) -> float:
    """Cost of one q-head of `pattern` at n tokens, relative to a dense causal head."""
    p = {**DEFAULT_PARAMS, **params}
    return head_tiles(pattern, n, **p) / head_tiles("dense", n)


def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws its own layer."""
    return seed + 1009 * rank


def partition_heads(head_patterns: Sequence[str], hkv: int, world: int, n: int = 1 << 20,
                    **params) -> List[List[int]]:
    """Longest-processing-time assignment of whole GQA groups to ranks.

    A group (one kv-head and its q-heads) stays on one rank so that its K and V
    are read by one GPU only; each head weighs `pattern_cost` at n tokens with
    the layer's pattern parameters.  Returns, per rank, the ascending q-head ids.
    """
    hq = len(head_patterns)
    grp = hq // hkv
    costs = []
    for g in range(hkv):
        heads = list(range(g * grp, (g + 1) * grp))
        costs.append((sum(pattern_cost(head_patterns[h], n, **params) for h in heads), g, heads))
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


def shard_summary(parts: List[List[int]], head_patterns: Sequence[str], n: int = 1 << 20,
                  **params) -> Dict[int, float]:
    return {r: sum(pattern_cost(head_patterns[h], n, **params) for h in p) for r, p in enumerate(parts)}


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
