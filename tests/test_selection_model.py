"""The Block-Sparse row selection's algorithm, on the CPU.

`block_topk_warp_kernel` picks the best k of a score row in two stages: a
histogram of 256 bins linear in value between the row's minimum and maximum
finds the bin holding the k-th best (everything above it is taken), then the
scores of that bin are settled exactly -- up to 32 by rank (score descending,
index ascending), more by a radix select over their order-preserving keys that
starts below the bits they all share.  This is a plain model of those steps
(fp32 arithmetic where the kernel uses it), checked against a brute-force
top-k on rows with distinct scores, heavy ties, all-equal rows, long common
key prefixes and signed zeros.  The GPU kernel itself is checked against the
oracle by the -m gpu parity tests.
"""
import numpy as np


def _key(x):
    """Order-preserving unsigned key of an fp32 value (negatives reversed)."""
    u = int(np.float32(x).view(np.uint32))
    return (~u) & 0xFFFFFFFF if u & 0x80000000 else u | 0x80000000


def _select(row, take):
    x = [np.float32(v) + np.float32(0.0) for v in row]  # -0 read as +0
    xmin, xmax = min(x), max(x)
    with np.errstate(all="ignore"):
        scale = np.float32(256.0) / np.float32(xmax - xmin)
    if not scale < np.float32(3.0e38):
        scale = np.float32(0.0)

    def bin_of(v):
        return min(255, int(np.float32(np.float32(v - xmin) * scale)))

    hist = [0] * 256
    for v in x:
        hist[bin_of(v)] += 1
    cum = 0
    for b in range(255, -1, -1):
        if cum + hist[b] >= take:
            bstar, in_bin = b, hist[b]
            break
        cum += hist[b]
    rem = take - cum
    taken = {j for j, v in enumerate(x) if bin_of(v) > bstar}
    cands = [j for j, v in enumerate(x) if bin_of(v) == bstar]
    if rem == in_bin:
        taken |= set(cands)
    elif in_bin <= 32:
        for j in cands:
            rank = sum(1 for c in cands if x[c] > x[j] or (x[c] == x[j] and c < j))
            if rank < rem:
                taken.add(j)
    else:
        keys = {j: _key(x[j]) for j in cands}
        kmin, kmax = min(keys.values()), max(keys.values())
        diff = kmin ^ kmax
        top = diff.bit_length() - 1 if diff else -1
        pmask = 0xFFFFFFFF if top < 0 else (0 if top == 31 else (~((2 << top) - 1)) & 0xFFFFFFFF)
        prefix, rem2 = kmax & pmask, rem
        while top >= 0:
            w = min(8, top + 1)
            shift, dm = top + 1 - w, (1 << w) - 1
            h = [0] * 256
            for k in keys.values():
                if k & pmask == prefix:
                    h[(k >> shift) & dm] += 1
            c2 = 0
            for dg in range(255, -1, -1):
                if c2 + h[dg] >= rem2:
                    ib = h[dg]
                    break
                c2 += h[dg]
            prefix |= dg << shift
            pmask |= dm << shift
            rem2 -= c2
            top -= w
            if ib == rem2:
                break
        eq_seen = 0
        for j in cands:
            u = keys[j] & pmask
            if u > prefix:
                taken.add(j)
            elif u == prefix:
                if eq_seen < rem2:
                    taken.add(j)
                eq_seen += 1
    return sorted(taken)


def test_two_stage_selection_matches_brute_force():
    rng = np.random.default_rng(11)
    for trial in range(600):
        i = int(rng.integers(2, 300))
        take = int(rng.integers(1, i))
        kind = trial % 5
        if kind == 0:
            row = rng.standard_normal(i)                       # distinct
        elif kind == 1:
            row = rng.integers(-3, 3, i).astype(float)         # heavy ties, > 32 in a bin
        elif kind == 2:
            row = np.full(i, 0.5)                              # one value
        elif kind == 3:
            row = rng.random(i) * 1e-3 + 1.0                   # long shared key prefix
        else:
            row = np.where(rng.random(i) < 0.5, 0.0, -0.0) + (rng.random(i) < 0.1) * rng.standard_normal(i)
        row = row.astype(np.float32)
        order = sorted(range(i), key=lambda j: (-float(row[j]), j))  # -0 == +0 as floats
        assert _select(list(row), take) == sorted(order[:take]), (trial, kind, i, take)
