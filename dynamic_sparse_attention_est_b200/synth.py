"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no arithmetic of the method itself (no estimation, no masks,
no attention): it only draws Q, K, V of the shapes and structure of the
workloads, so that the CUDA path and the fp64 oracle can be fed the same bf16
tensors.  Every draw comes from a ``torch.Generator`` seeded by the caller.

Recipe (shared by all workloads):
  * Q, K, V ~ N(0, 1) in fp32, shape [heads, n, 128];
  * rotary position embedding on Q and K, rotate-half convention,
    inv_freq_i = theta ** (-2 i / d) with theta = 500000;
  * a planted structure, added after the rotation so that it survives it;
  * rounded to bf16.

Planted structures:
  * ``vertical``: for each kv-head g a unit vector u_g; key 0 plus ``n_heavy``
    random other keys get +4 u_g, every query of the q-heads of group g gets
    +1.5 u_g (heavy "vertical" keys every query attends to).
  * ``clustered``: for each kv-head g, 64 clusters of 8 consecutive 64-token key
    blocks (512 hot blocks); each cluster has a unit direction w_c, its key
    tokens get +4 w_c, and for each q-head of the group 16 random later query
    blocks get +1.5 w_c on all their tokens.
  * ``plain``: nothing planted.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import torch

D_HEAD = 128
ROPE_THETA = 500000.0


@dataclass(frozen=True)
class Workload:
    name: str
    pattern: str          # "vs", "block", "ashape", "trishape", "dense" or "mixed"
    hq: int
    hkv: int
    n: int
    structure: str        # "vertical", "clustered" or "plain"
    n_heavy: int = 0      # extra heavy keys besides key 0 ("vertical")
    heavy_frac: float = 0.0
    last_q: int = 64
    n_vertical: int = 1000
    n_slash: int = 6096
    block: int = 64
    topk: int = 100
    n_sink: int = 128
    window: int = 4096
    mix: Dict[str, float] = field(default_factory=dict)

    def heavy_count(self) -> int:
        if self.n_heavy:
            return self.n_heavy
        return int(round(self.heavy_frac * self.n))


WORKLOADS: Dict[str, Workload] = {
    "vs-1h-4k": Workload("vs-1h-4k", "vs", 1, 1, 4096, "vertical", n_heavy=16,
                          last_q=64, n_vertical=256, n_slash=512),
    "vs-gqa-32k": Workload("vs-gqa-32k", "vs", 32, 8, 32768, "vertical", heavy_frac=0.005,
                            last_q=64, n_vertical=1000, n_slash=6096),
    "block-gqa-128k": Workload("block-gqa-128k", "block", 32, 8, 131072, "clustered",
                                block=64, topk=100),
    "ashape-gqa-128k": Workload("ashape-gqa-128k", "ashape", 32, 8, 131072, "plain",
                                 n_sink=128, window=4096),
    "trishape-gqa-128k": Workload("trishape-gqa-128k", "trishape", 32, 8, 131072, "plain",
                                   n_sink=128, window=4096, last_q=64),
    # one Vertical-Slash head at 256K tokens with the layer's budgets: a profiling-size case
    # for the sparse-slash pass (a few hundred MB on the device)
    "vs-1h-256k": Workload("vs-1h-256k", "vs", 1, 1, 262144, "vertical", heavy_frac=0.005,
                            last_q=64, n_vertical=1000, n_slash=6096),
    # one Vertical-Slash head at 1M tokens with the layer's budgets: a profiling-size case
    "vs-1h-1m": Workload("vs-1h-1m", "vs", 1, 1, 1048576, "vertical", heavy_frac=0.005,
                          last_q=64, n_vertical=1000, n_slash=6096),
    "mixed-gqa-1m": Workload("mixed-gqa-1m", "mixed", 32, 8, 1048576, "vertical",
                              heavy_frac=0.005, last_q=64, n_vertical=1000, n_slash=6096,
                              block=64, topk=100, n_sink=128, window=4096,
                              mix={"vs": 0.6, "block": 0.3, "ashape": 0.1}),
}


def _rope_tables(n: int, d: int, device) -> tuple:
    half = d // 2
    inv = ROPE_THETA ** (-torch.arange(0, half, dtype=torch.float64, device=device) * 2.0 / d)
    pos = torch.arange(n, dtype=torch.float64, device=device)
    ang = pos[:, None] * inv[None, :]
    return torch.cos(ang).float(), torch.sin(ang).float()


def _rotate(x: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor) -> torch.Tensor:
    half = x.shape[-1] // 2
    x1, x2 = x[..., :half], x[..., half:]
    return torch.cat([x1 * cos - x2 * sin, x2 * cos + x1 * sin], dim=-1)


def _unit(g: torch.Generator, d: int, device) -> torch.Tensor:
    u = torch.randn(d, generator=g, device=device)
    return u / u.norm()


def generate(w: Workload, seed: int = 0, device="cpu", n: Optional[int] = None,
             hq: Optional[int] = None, hkv: Optional[int] = None) -> dict:
    """Draws Q, K, V (bf16, [heads, n, 128]) for workload ``w``.

    ``n``/``hq``/``hkv`` override the workload's sizes (smaller test cases keep
    its structure).  Heads are drawn one at a time so that the fp32 temporaries
    stay small at 1M tokens.  Returns a dict with q, k, v and what was planted.
    """
    n = n or w.n
    hq = hq or w.hq
    hkv = hkv or w.hkv
    assert hq % hkv == 0
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    cos, sin = _rope_tables(n, D_HEAD, device)
    q = torch.empty(hq, n, D_HEAD, dtype=torch.bfloat16, device=device)
    k = torch.empty(hkv, n, D_HEAD, dtype=torch.bfloat16, device=device)
    v = torch.empty(hkv, n, D_HEAD, dtype=torch.bfloat16, device=device)
    grp = hq // hkv
    planted: dict = {"heavy": [], "clusters": []}
    for gh in range(hkv):
        kk = _rotate(torch.randn(n, D_HEAD, generator=g, device=device), cos, sin)
        v[gh] = torch.randn(n, D_HEAD, generator=g, device=device).to(torch.bfloat16)
        q_add = [None] * grp
        if w.structure == "vertical":
            u = _unit(g, D_HEAD, device)
            extra = min(w.heavy_count(), n - 1)
            pos = torch.randperm(n - 1, generator=g, device=device)[:extra] + 1
            heavy = torch.cat([torch.zeros(1, dtype=torch.long, device=device), pos])
            kk[heavy] += 4.0 * u
            planted["heavy"].append(heavy.sort().values.cpu())
            for j in range(grp):
                q_add[j] = ("all", 1.5 * u)
        elif w.structure == "clustered":
            nb = n // 64
            n_clusters = min(64, max(1, nb // 16))
            span = 8 if nb >= 16 else 1
            slots = max(1, nb // span)
            starts = torch.randperm(slots, generator=g, device=device)[:n_clusters] * span
            dirs = [_unit(g, D_HEAD, device) for _ in range(n_clusters)]
            links: List[list] = [[] for _ in range(grp)]
            for c in range(n_clusters):
                b0 = int(starts[c])
                kk[b0 * 64:(b0 + span) * 64] += 4.0 * dirs[c]
                for j in range(grp):
                    later = nb - (b0 + span)
                    if later <= 0:
                        continue
                    tgt = torch.randint(b0 + span, nb, (16,), generator=g, device=device)
                    links[j].append((c, tgt.cpu()))
            planted["clusters"].append((starts.cpu(), links))
            for j in range(grp):
                q_add[j] = ("blocks", links[j], dirs)
        k[gh] = kk.to(torch.bfloat16)
        del kk
        for j in range(grp):
            h = gh * grp + j
            qq = _rotate(torch.randn(n, D_HEAD, generator=g, device=device), cos, sin)
            if q_add[j] is not None:
                if q_add[j][0] == "all":
                    qq += q_add[j][1]
                else:
                    _, lk, dirs = q_add[j]
                    for c, tgt in lk:
                        for b in tgt.tolist():
                            qq[b * 64:(b + 1) * 64] += 1.5 * dirs[c]
            q[h] = qq.to(torch.bfloat16)
            del qq
    return {"q": q, "k": k, "v": v, "planted": planted, "n": n, "hq": hq, "hkv": hkv}


def mixed_head_patterns(w: Workload, seed: int = 0, hq: Optional[int] = None) -> List[str]:
    """Head -> pattern assignment of a mixed layer, drawn from the seed.

    The shares in ``w.mix`` are rounded to whole heads (largest remainder), and
    a seeded permutation places them over the q-heads.
    """
    hq = hq or w.hq
    names = list(w.mix.keys())
    raw = [w.mix[nm] * hq for nm in names]
    counts = [int(math.floor(x)) for x in raw]
    rem = hq - sum(counts)
    order = sorted(range(len(names)), key=lambda i: (-(raw[i] - counts[i]), i))
    for i in order[:rem]:
        counts[i] += 1
    labels: List[str] = []
    for nm, c in zip(names, counts):
        labels += [nm] * c
    g = torch.Generator()
    g.manual_seed(seed + 7919)
    perm = torch.randperm(hq, generator=g).tolist()
    return [labels[p] for p in perm]
