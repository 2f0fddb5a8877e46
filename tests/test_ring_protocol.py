"""The chunk ring of the Vertical-Slash CUDA-core pass, as a model checked on the CPU.

`vs_diag_kernel` stages each sparse slash group's key range in 128-key chunks
of K and V through a three-stage ring: one producer warp loads chunk c into
stage c % 3 once the eight consumer warps have all released chunk c - 3; each
consumer warp, per slash offset, needs the chunks that hold its 16 rows' keys
(at most two) and first releases every chunk below them -- seeing and releasing
one by one the chunks it skips -- so it never waits while holding a chunk it
no longer needs.  This model replays those rules under random interleavings of
the producer and the warps, on the groups and windows the kernel derives from
sparse index sets (the grouping of offsets at most 128 apart and the routing
m < ratio * H of the kernel's planner), and checks that
- no interleaving deadlocks,
- a warp reads only chunks it has seen full and not released,
- no stage is refilled while a warp may still read it,
- every chunk is released by every warp.
The GPU tests check the kernel's results; this checks the protocol they rely on.
"""
import random

import numpy as np
import pytest

NST, NW, CH, ROWS = 3, 8, 128, 16  # stages, consumer warps, keys per chunk, rows per warp


def _groups(si, n, ratio):
    """Sorted distinct offsets and the groups routed to the CUDA cores:
    (first offset, last offset, first index, last index)."""
    soff = np.unique(si[(si >= 0) & (si < n)])
    groups, start = [], 0
    for e in range(1, len(soff) + 1):
        if e == len(soff) or soff[e] - soff[e - 1] > 128:
            groups.append((int(soff[start]), int(soff[e - 1]), start, e - 1))
            start = e
    diag = []
    for (x, y, f, l) in groups:
        m, halves = l - f + 1, (y - x + 128 + 63) // 64
        if ratio > 0 and m < ratio * halves:
            diag.append((x, y, f, l))
    return [int(v) for v in soff], diag


def _chunks(x, y, r0, rmax):
    a, b = max(0, r0 - y), rmax - x
    return a, (b - a + CH) // CH


def _warp_program(heads, n, nq, w, items):
    """('need', lo, hi) and ('read', lo, hi) steps of warp w, in global chunk numbers."""
    c_base = 0
    for it in items:
        t, hp = nq - 1 - it // len(heads), it % len(heads)
        soff, dg = heads[hp]
        r0, rmax = 128 * t, min(128 * t + 127, n - 1)
        last_r, rw = rmax - r0, ROWS * w
        for (x, y, f, l) in dg:
            if x > rmax:
                break
            a, nc = _chunks(x, y, r0, rmax)
            for j in range(l - f, -1, -1):  # largest offset first: the windows move forward
                u0 = r0 - soff[f + j] - a
                ulo, uhi = max(0, u0 + rw), min(u0 + rw + ROWS - 1, u0 + last_r)
                if ulo > uhi:
                    continue
                lo, hi = c_base + ulo // CH, c_base + uhi // CH
                assert hi - lo <= 1
                yield ("need", lo, hi)
                yield ("read", lo, hi)
            yield ("need", c_base + nc, c_base + nc - 1)  # the group's remaining chunks
            c_base += nc


def _producer_total(heads, n, nq, items):
    c = 0
    for it in items:
        t, hp = nq - 1 - it // len(heads), it % len(heads)
        _, dg = heads[hp]
        r0, rmax = 128 * t, min(128 * t + 127, n - 1)
        for (x, y, f, l) in dg:
            if x > rmax:
                break
            c += _chunks(x, y, r0, rmax)[1]
    return c


def _simulate(heads, n, items, seed, release_first=True):
    """release_first=False models the rule's absence: a warp sees the chunks up to
    its window's end before it releases the ones below it."""
    rng = random.Random(seed)
    nq = (n + 127) // 128
    total = _producer_total(heads, n, nq, items)
    loaded, released, holder = [False] * total, [0] * total, {}
    pc = 0
    warps = [{"prog": _warp_program(heads, n, nq, w, items), "got": 0, "rel": 0, "step": None, "done": False}
             for w in range(NW)]
    while True:
        runnable = []
        if pc < total and (pc < NST or released[pc - NST] == NW):
            runnable.append("P")
        for i, W in enumerate(warps):
            if W["done"]:
                continue
            if W["step"] is None:
                W["step"] = next(W["prog"], None)
                if W["step"] is None:
                    W["done"] = True
                    continue
            kind, lo, hi = W["step"]
            if not release_first and kind == "need" and W["got"] <= hi:
                if W["got"] < total and loaded[W["got"]]:
                    runnable.append(i)
            elif kind == "read" or (W["rel"] < lo and W["rel"] < W["got"]):
                runnable.append(i)
            elif W["got"] < lo or W["got"] <= hi:
                if W["got"] < total and loaded[W["got"]]:
                    runnable.append(i)
            else:
                runnable.append(i)  # need satisfied
        if not runnable:
            assert all(W["done"] for W in warps) and pc == total, "deadlock"
            break
        a = rng.choice(runnable)
        if a == "P":
            loaded[pc] = True
            holder[pc % NST] = pc
            pc += 1
            continue
        W = warps[a]
        kind, lo, hi = W["step"]
        if not release_first and kind == "need" and W["got"] <= hi:
            W["got"] += 1
        elif kind == "read":
            for c in range(lo, hi + 1):
                assert W["rel"] <= c < W["got"], "read outside the seen, unreleased window"
                assert holder[c % NST] == c, "stage refilled while still read"
            W["step"] = None
        elif W["rel"] < lo and W["rel"] < W["got"]:
            released[W["rel"]] += 1
            W["rel"] += 1
        elif W["got"] < lo:  # a chunk this warp skips: seen, then released
            W["got"] += 1
            released[W["rel"]] += 1
            W["rel"] += 1
        elif W["got"] <= hi:
            W["got"] += 1
        else:
            W["step"] = None
    assert all(r == NW for r in released), "every chunk released by every warp"


def _sparse_indices(rng, n, nh, n_far):
    """Slash offsets mostly far apart (lone offsets), some in pairs and triples
    within 128 of each other, offset 0 and one past n."""
    si = []
    for _ in range(nh):
        base = np.sort(rng.choice(np.arange(1, n), n_far, replace=False))
        extra = [b + rng.integers(1, 100) for b in base[::3]] + [b + rng.integers(1, 60) for b in base[::5]]
        si.append(np.unique(np.concatenate([[0], base, extra, [n + 5]])).astype(np.int64))
    return si


@pytest.mark.parametrize("n,nh,n_far,ratio", [(4160, 2, 24, 1.0), (4160, 2, 24, 1000.0), (8192, 3, 60, 2.0),
                                              (1088, 1, 6, 1000.0)])
def test_chunk_ring_never_deadlocks_nor_reads_stale_stages(n, nh, n_far, ratio):
    rng = np.random.default_rng(n + nh)
    heads = [_groups(si, n, ratio) for si in _sparse_indices(rng, n, nh, n_far)]
    assert any(dg for _, dg in heads)
    n_items = nh * ((n + 127) // 128)
    for grid in (1, 3):
        for cta in range(grid):
            items = list(range(cta, n_items, grid))  # the persistent CTA's stride over the work items
            for seed in range(2):
                _simulate(heads, n, items, seed)


def test_model_catches_waiting_while_holding_a_stale_chunk():
    """Without release-before-wait the same inputs deadlock: a warp holding a
    chunk below its window waits for a stage that chunk keeps occupied."""
    rng = np.random.default_rng(4160 + 2)
    heads = [_groups(si, 4160, 1000.0) for si in _sparse_indices(rng, 4160, 2, 24)]
    items = list(range(2 * ((4160 + 127) // 128)))
    with pytest.raises(AssertionError, match="deadlock"):
        for seed in range(20):
            _simulate(heads, 4160, items, seed, release_first=False)
