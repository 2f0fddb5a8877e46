"""Checks that pin the fp64 oracle to something other than itself.

Every pin recomputes its expectation from the definitions with independent
numpy code (a dense logit matrix, ``np.trace`` for diagonals, explicit boolean
masks, block means of the raw logits) or from a closed form, never by calling
the oracle a second way.  Each takes an ``oracle.Oracle`` so that the mutation
test can run the same pins against builds with a planted mistake.

Sources the definitions follow:
  [NEWS] news article "单卡A100实现百万token推理，速度快10倍，这是微软官方的大模型推理加速",
         section 方法介绍 (Vertical-Slash from the last queries, Block-Sparse by mean pooling)
         and Figure 4 (verticals and slashes inside the kernel).
  [TALK] AICon 2025 talk transcript "以 KV 缓存为中心的高效长文本方法", second
         observation (A-shape, vertical, slash and block patterns).
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np
import torch

from dynamic_sparse_attention_est_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _inputs(n, hq=2, hkv=1, seed=0, structure="vertical", n_heavy=4):
    w = synth.Workload("pin", "vs", hq, hkv, n, structure, n_heavy=n_heavy)
    x = synth.generate(w, seed=seed)
    f = lambda t: t.float().numpy().astype(np.float64)
    return f(x["q"]), f(x["k"]), f(x["v"]), x


def _softmax_rows(z):
    m = np.max(z, axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(z - m)
    s = e.sum(axis=-1, keepdims=True)
    return np.divide(e, s, out=np.zeros_like(e), where=s > 0), s, m


def _masked_attention(q, k, v, scale, mask):
    """Textbook softmax(scale*QK^T masked) V for one head; mask [n, n] bool."""
    z = scale * (q @ k.T)
    z = np.where(mask, z, -np.inf)
    p, s, m = _softmax_rows(z)
    lse = np.where(s[:, 0] > 0, m[:, 0] + np.log(np.where(s[:, 0] > 0, s[:, 0], 1.0)), -np.inf)
    return p @ v, lse, p


def _topk_ref(scores, kk):
    """Indices of the kk best by (score desc, index asc), ascending."""
    idx = np.arange(len(scores))
    order = np.lexsort((idx, -scores))
    return np.sort(order[:min(kk, len(scores))])


# --------------------------------------------------------------------------- VS estimate
def pin_vs_estimate_bruteforce(orc):
    """Column/diagonal sums of the last-L softmax rows, from a dense logit matrix."""
    for n, L, nv, ns in [(200, 64, 30, 40), (256, 64, 50, 70), (96, 128, 10, 12)]:
        q, k, _, _ = _inputs(n)
        scale = 1.0 / math.sqrt(128)
        vi, si, vert, slash = orc.vs_estimate(q.astype(np.float32), k.astype(np.float32), L, nv,
                                              ns, scale, return_scores=True)
        Lr = min(L, n)
        for hp in range(q.shape[0]):
            rows = np.arange(n - Lr, n)
            z = scale * (q[hp, rows] @ k[0].T)
            z = np.where(np.arange(n)[None, :] <= rows[:, None], z, -np.inf)
            a, _, _ = _softmax_rows(z)
            v_ref = a.sum(axis=0)
            # slash[o] = sum_i A[i, i-o]; row r is query n-Lr+r, so k - r = n - Lr - o
            s_ref = np.array([np.trace(a, offset=n - Lr - o) for o in range(n)])
            assert np.allclose(vert[hp], v_ref, rtol=1e-12, atol=1e-15), "vertical sums"
            assert np.isinf(slash[hp, 0]) and slash[hp, 0] > 0, "offset 0 forced"
            assert np.allclose(slash[hp, 1:], s_ref[1:], rtol=1e-12, atol=1e-15), "slash sums"
            s_forced = s_ref.copy()
            s_forced[0] = np.inf
            assert np.array_equal(vi[hp][:min(nv, n)], _topk_ref(v_ref, nv)), "vertical top-k"
            assert np.array_equal(si[hp][:min(ns, n)], _topk_ref(s_forced, ns)), "slash top-k"


def pin_vs_estimate_uniform_closed_form(orc):
    """Q = 0 makes every softmax row uniform: A_ik = 1/(i+1), so the sums are harmonic."""
    n, L = 160, 64
    q = np.zeros((1, n, 128), np.float32)
    k = np.random.default_rng(3).standard_normal((1, n, 128)).astype(np.float32)
    _, _, vert, slash = orc.vs_estimate(q, k, L, 8, 8, 0.1, return_scores=True)
    for kk in range(n):
        ref = math.fsum(1.0 / (i + 1) for i in range(max(kk, n - L), n))
        assert abs(vert[0, kk] - ref) <= 1e-12 * ref, f"vert[{kk}]"
    for o in range(1, n):
        ref = math.fsum(1.0 / (i + 1) for i in range(max(o, n - L), n))
        assert abs(slash[0, o] - ref) <= 1e-12 * max(ref, 1e-300), f"slash[{o}]"


def pin_vs_estimate_golden(orc):
    """Hand-worked 4-token example (tests/golden/vs_estimate_tiny.json)."""
    with open(os.path.join(GOLDEN, "vs_estimate_tiny.json")) as f:
        g = json.load(f)
    q = np.array(g["q"], np.float32)[None]
    k = np.array(g["k"], np.float32)[None]
    vi, si, vert, slash = orc.vs_estimate(q, k, g["last_q"], g["n_vertical"], g["n_slash"],
                                          g["scale"], return_scores=True)
    ev = [float(Fraction(x)) for x in g["expected_vertical"]]
    es = [float(Fraction(x)) for x in g["expected_slash_from_1"]]
    assert np.allclose(vert[0], ev, rtol=g["rtol"]), "golden vertical sums"
    assert np.allclose(slash[0, 1:], es, rtol=g["rtol"]), "golden slash sums"
    assert vi[0].tolist() == g["expected_v_idx"], "golden v_idx"
    assert si[0].tolist() == g["expected_s_idx"], "golden s_idx"


# --------------------------------------------------------------------------- BS estimate
def pin_block_estimate_commutes(orc):
    """Pooled score = block mean of the raw logits (pooling commutes with the product)."""
    n, block = 512, 64
    q, k, _, _ = _inputs(n, hq=2, hkv=1, structure="plain")
    _, _, pq, pk, sc = orc.block_estimate(q.astype(np.float32), k.astype(np.float32), block, 3,
                                          return_scores=True)
    nb = n // block
    for hp in range(2):
        z = q[hp] @ k[0].T
        ref = z.reshape(nb, block, nb, block).mean(axis=(1, 3))
        low = np.tril(np.ones((nb, nb), bool))
        assert np.allclose(sc[hp][low], ref[low], rtol=1e-12, atol=1e-13), "commutativity"
        assert np.all(np.isneginf(sc[hp][~low])), "future blocks excluded"
        assert np.allclose(pq[hp], q[hp].reshape(nb, block, 128).mean(axis=1), rtol=1e-13)


def pin_block_estimate_topk_bruteforce(orc):
    """Diagonal block forced, best topk-1 earlier blocks by (score desc, index asc)."""
    n, block = 1024, 64
    for topk in (1, 3, 5, 16, 40):
        q, k, _, _ = _inputs(n, hq=2, hkv=1, structure="plain", seed=topk)
        bi, bc = orc.block_estimate(q.astype(np.float32), k.astype(np.float32), block, topk)
        nb = n // block
        for hp in range(2):
            qp = q[hp].reshape(nb, block, 128).mean(axis=1)
            kp = k[0].reshape(nb, block, 128).mean(axis=1)
            s = qp @ kp.T
            for i in range(nb):
                rest = _topk_ref(s[i, :i], topk - 1) if (topk > 1 and i > 0) else np.array([], int)
                ref = np.sort(np.concatenate([rest, [i]]))
                assert bc[hp, i] == len(ref), "block count"
                assert np.array_equal(bi[hp, i, :bc[hp, i]], ref), f"row {i}"
                assert np.all(bi[hp, i, bc[hp, i]:] == -1), "padding"


# --------------------------------------------------------------------------- attention
def _vs_mask(n, vi, si):
    i = np.arange(n)[:, None]
    kk = np.arange(n)[None, :]
    vs = set(int(x) for x in vi if x >= 0)
    ss = set(int(x) for x in si if x >= 0)
    inv = np.array([c in vs for c in range(n)])[None, :]
    ons = np.isin(i - kk, list(ss)) if ss else np.zeros((n, n), bool)
    return (kk <= i) & (inv | ons)


def _block_mask(n, block, bi, bc):
    i = np.arange(n)[:, None]
    kk = np.arange(n)[None, :]
    nb = n // block
    sel = np.zeros((nb, nb), bool)
    for b in range(nb):
        for j in bi[b, :bc[b]]:
            if j >= 0:
                sel[b, j] = True
    return (kk <= i) & sel[i // block, kk // block]


def _ashape_mask(n, sink, window):
    i = np.arange(n)[:, None]
    kk = np.arange(n)[None, :]
    return (kk <= i) & ((kk < sink) | (i - kk < window))


def pin_attention_masks_bruteforce(orc):
    """Each pattern against dense-mask softmax attention built from its definition."""
    n = 256
    scale = 1.0 / math.sqrt(128)
    q, k, v, _ = _inputs(n, hq=2, hkv=1, seed=5)
    f32 = lambda a: a.astype(np.float32)
    rng = np.random.default_rng(11)
    # Vertical-Slash with random index sets (-1 padded)
    vi = np.full((2, 20), -1, np.int32)
    si = np.full((2, 24), -1, np.int32)
    for hp in range(2):
        a = np.sort(rng.choice(n, 17, replace=False))
        b = np.sort(np.concatenate([[0], rng.choice(np.arange(1, n), 20, replace=False)]))
        vi[hp, :17], si[hp, :21] = a, b
    out, lse = orc.vs_attention(f32(q), f32(k), f32(v), scale, vi, si)
    for hp in range(2):
        ref, rl, _ = _masked_attention(q[hp], k[0], v[0], scale, _vs_mask(n, vi[hp], si[hp]))
        assert np.allclose(out[hp], ref, rtol=1e-11, atol=1e-12), "VS attention"
        assert np.allclose(lse[hp], rl, rtol=1e-12), "VS lse"
    # Block-Sparse with a forced diagonal and random earlier blocks
    block, topk = 32, 3
    nb = n // block
    bi = np.full((2, nb, topk), -1, np.int32)
    bc = np.zeros((2, nb), np.int32)
    for hp in range(2):
        for b in range(nb):
            extra = rng.choice(b, min(b, topk - 1), replace=False) if b else np.array([], int)
            row = np.sort(np.concatenate([extra, [b]]))
            bi[hp, b, :len(row)] = row
            bc[hp, b] = len(row)
    out, lse = orc.block_attention(f32(q), f32(k), f32(v), scale, block, bi, bc)
    for hp in range(2):
        ref, rl, _ = _masked_attention(q[hp], k[0], v[0], scale, _block_mask(n, block, bi[hp], bc[hp]))
        assert np.allclose(out[hp], ref, rtol=1e-11, atol=1e-12), "BS attention"
        assert np.allclose(lse[hp], rl, rtol=1e-12), "BS lse"
    # A-shape
    for sink, window in [(16, 40), (0, 1), (64, 300), (5, 7)]:
        out, lse = orc.ashape_attention(f32(q), f32(k), f32(v), scale, sink, window)
        for hp in range(2):
            ref, rl, _ = _masked_attention(q[hp], k[0], v[0], scale, _ashape_mask(n, sink, window))
            assert np.allclose(out[hp], ref, rtol=1e-11, atol=1e-12), f"A-shape {sink}/{window}"
            assert np.allclose(lse[hp], rl, rtol=1e-12), "A-shape lse"


def _trishape_mask(n, sink, window, n_last):
    i = np.arange(n)[:, None]
    return _ashape_mask(n, sink, window) | ((np.arange(n)[None, :] <= i) & (i >= n - n_last))


def pin_trishape_bruteforce(orc):
    """Tri-shape: A-shape lines plus dense last rows, vs its dense-mask definition;
    n_last = 0 is A-shape, n_last = n is dense."""
    n = 256
    scale = 1.0 / math.sqrt(128)
    q, k, v, _ = _inputs(n, hq=2, hkv=1, seed=13)
    f32 = lambda a: a.astype(np.float32)
    for sink, window, n_last in [(16, 40, 64), (0, 1, 100), (5, 7, 1), (64, 300, 30)]:
        out, lse = orc.trishape_attention(f32(q), f32(k), f32(v), scale, sink, window, n_last)
        for hp in range(2):
            ref, rl, _ = _masked_attention(q[hp], k[0], v[0], scale, _trishape_mask(n, sink, window, n_last))
            assert np.allclose(out[hp], ref, rtol=1e-11, atol=1e-12), f"Tri-shape {sink}/{window}/{n_last}"
            assert np.allclose(lse[hp], rl, rtol=1e-12), "Tri-shape lse"
    a, _ = orc.ashape_attention(f32(q), f32(k), f32(v), scale, 16, 40)
    t, _ = orc.trishape_attention(f32(q), f32(k), f32(v), scale, 16, 40, 0)
    assert np.array_equal(a, t), "n_last = 0 is A-shape"
    dns, _ = orc.dense_attention(f32(q), f32(k), f32(v), scale)
    t, _ = orc.trishape_attention(f32(q), f32(k), f32(v), scale, 16, 40, n)
    assert np.allclose(t, dns, rtol=1e-12, atol=1e-13), "n_last = n is dense"


def pin_vs_tiles_forms(orc):
    """Vertical-Slash with whole slash tiles ([NEWS] Figure 4: slashes computed as
    dense blocks), against forms that follow from its definition:
      * offset 0 alone: row i attends its tile's causal prefix, keys r0 .. i;
      * one offset o >= tile: every row of the tile starting at r0 attends exactly
        the tile_rows keys r0 - o .. r0 + tile_rows - 1 - o (none for the first
        tiles, which then give o = 0 and lse = -inf);
      * tile_rows = 1 is the token-exact pattern;
      * the token-exact key set is a subset: lse can only grow;
      * every offset selected is dense attention."""
    n, T = 320, 128
    scale = 1.0 / math.sqrt(128)
    q, k, v, _ = _inputs(n, hq=2, hkv=1, seed=23)
    f32 = lambda a: a.astype(np.float32)
    i = np.arange(n)[:, None]
    kk = np.arange(n)[None, :]
    r0 = (i // T) * T
    none_v = np.full((2, 1), -1, np.int32)
    out, lse = orc.vs_tiles_attention(f32(q), f32(k), f32(v), scale, none_v, np.zeros((2, 1), np.int32), T)
    for hp in range(2):
        ref, rl, _ = _masked_attention(q[hp], k[0], v[0], scale, (kk >= r0) & (kk <= i))
        assert np.allclose(out[hp], ref, rtol=1e-11, atol=1e-12), "offset 0: tile prefix"
        assert np.allclose(lse[hp], rl, rtol=1e-12), "offset 0: lse"
    o = 200
    out, lse = orc.vs_tiles_attention(f32(q), f32(k), f32(v), scale, none_v, np.full((2, 1), o, np.int32), T)
    for hp in range(2):
        mask = (kk >= r0 - o) & (kk < r0 - o + T) & (kk >= 0)
        ref, rl, _ = _masked_attention(q[hp], k[0], v[0], scale, mask)
        assert np.allclose(out[hp], ref, rtol=1e-11, atol=1e-12), "one far offset: a fixed key range per tile"
        assert np.array_equal(np.isfinite(lse[hp]), np.isfinite(rl)), "empty rows"
        fin = np.isfinite(rl)
        assert np.allclose(lse[hp][fin], rl[fin], rtol=1e-12), "one far offset: lse"
        counts = mask.sum(axis=1)
        assert set(np.unique(counts[i[:, 0] >= 2 * T]).tolist()) == {T}, "tile_rows keys per row"
    rng = np.random.default_rng(29)
    vi = np.sort(rng.choice(n, (2, 12), replace=False), axis=1).astype(np.int32)
    si = np.concatenate([np.zeros((2, 1), np.int32),
                         np.sort(rng.choice(np.arange(1, n), (2, 15), replace=False), axis=1)], axis=1).astype(np.int32)
    exact, el = orc.vs_attention(f32(q), f32(k), f32(v), scale, vi, si)
    one, ol = orc.vs_tiles_attention(f32(q), f32(k), f32(v), scale, vi, si, 1)
    assert np.allclose(one, exact, rtol=1e-12, atol=1e-13) and np.allclose(ol, el, rtol=1e-12), \
        "tile_rows = 1 is token-exact"
    _, tl = orc.vs_tiles_attention(f32(q), f32(k), f32(v), scale, vi, si, T)
    assert np.all(tl >= el - 1e-12), "whole tiles attend a superset"
    assert np.any(tl > el + 1e-6), "and strictly more somewhere"
    dense, _ = orc.dense_attention(f32(q), f32(k), f32(v), scale)
    all_o = np.tile(np.arange(n, dtype=np.int32), (2, 1))
    out, _ = orc.vs_tiles_attention(f32(q), f32(k), f32(v), scale, none_v, all_o, T)
    assert np.allclose(out, dense, rtol=1e-12, atol=1e-13), "every offset: dense"


def pin_vs_topp_forms(orc):
    """Top-p budgets ([TALK], work that followed MInference: a top-p of the attention
    weights instead of a fixed top-k), against what the definition fixes:
      * Q = 0 makes every row's softmax uniform, so vert[k] and slash[o] have closed
        forms (sums of 1/(i+1)); the selected counts and sets follow from them, ties
        to the lower index;
      * the set is the top-k set of its own size (a prefix of the same order);
      * it reaches p of the mass and is the shortest prefix that does;
      * the caps bound the counts."""
    n, L = 256, 64
    rng = np.random.default_rng(3)
    q = np.zeros((1, n, 128), np.float32)
    k = rng.standard_normal((1, n, 128)).astype(np.float32)
    rows = np.arange(n - L, n)
    inv = 1.0 / (rows + 1.0)
    vert = np.array([inv[rows >= kk].sum() for kk in range(n)])       # column kk: rows i >= kk
    slash = np.array([inv[rows >= o].sum() for o in range(n)])       # offset o: rows i >= o
    pv, ps = 0.5, 0.3
    vi, si, vc, sc = orc.vs_estimate_topp(q, k, L, 200, 150, pv, ps, 0.1)
    order = np.lexsort((np.arange(n), -vert))
    cv = int(np.searchsorted(np.cumsum(vert[order]), pv * vert.sum(), side="left")) + 1
    assert vc[0] == cv and np.array_equal(vi[0, :cv], np.sort(order[:cv])) and np.all(vi[0, cv:] == -1), \
        "uniform rows: vertical count and set"
    rest = np.arange(1, n)
    order = rest[np.lexsort((rest, -slash[1:]))]
    need = ps * slash.sum() - slash[0]
    cs = int(np.searchsorted(np.cumsum(slash[order]), need, side="left")) + 1
    assert sc[0] == cs + 1, "uniform rows: slash count (offset 0 forced, its mass counted)"
    assert np.array_equal(si[0, :cs + 1], np.sort(np.concatenate([[0], order[:cs]]))), "uniform rows: slash set"
    # planted inputs: prefix of the top-k order, minimal mass cover, caps
    qq, kk_, _, _ = _inputs(512, hq=2, hkv=1, seed=41)
    f32 = lambda a: a.astype(np.float32)
    vi, si, vc, sc, vs, ss = orc.vs_estimate_topp(f32(qq), f32(kk_), 64, 512, 512, 0.9, 0.8, 1 / math.sqrt(128),
                                                  return_scores=True)
    for hp in range(2):
        a, b = orc.vs_estimate(f32(qq), f32(kk_), 64, int(vc[hp]), int(sc[hp]), 1 / math.sqrt(128), head_ids=[hp])
        assert np.array_equal(vi[hp, :vc[hp]], a[0]) and np.array_equal(si[hp, :sc[hp]], b[0]), "prefix of top-k"
        sel = vs[hp, vi[hp, :vc[hp]]]
        assert sel.sum() >= 0.9 * vs[hp].sum() and sel.sum() - sel.min() < 0.9 * vs[hp].sum(), "shortest vertical cover"
        sel = ss[hp, si[hp, :sc[hp]]]
        others = np.sort(ss[hp, si[hp, 1:sc[hp]]])
        assert sel.sum() >= 0.8 * ss[hp].sum(), "slash cover"
        assert len(others) == 0 or sel.sum() - others[0] < 0.8 * ss[hp].sum(), "shortest slash cover"
    vi, si, vc, sc = orc.vs_estimate_topp(f32(qq), f32(kk_), 64, 5, 3, 0.99, 0.99, 1 / math.sqrt(128))
    assert np.all(vc == 5) and np.all(sc == 3) and np.all(vi >= 0) and np.all(si[:, 0] == 0), "caps"


def pin_full_budget_is_dense(orc):
    """Budgets that cover every key reduce each pattern to dense causal attention."""
    n = 320
    scale = 0.07
    q, k, v, _ = _inputs(n, hq=4, hkv=2, seed=9)
    f32 = lambda a: a.astype(np.float32)
    dense, dl = orc.dense_attention(f32(q), f32(k), f32(v), scale)
    for hp in range(4):
        i = np.arange(n)[:, None]
        ref, rl, p = _masked_attention(q[hp], k[hp // 2], v[hp // 2], scale, np.arange(n)[None, :] <= i)
        assert np.allclose(dense[hp], ref, rtol=1e-11, atol=1e-12), "dense vs textbook"
        assert np.allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12), "softmax rows sum to 1"
        assert np.allclose(dl[hp], rl, rtol=1e-12), "dense lse"
    vi, si = orc.vs_estimate(f32(q), f32(k), 64, n, 1, scale)        # every key vertical
    out, _ = orc.vs_attention(f32(q), f32(k), f32(v), scale, vi, si)
    assert np.allclose(out, dense, rtol=1e-12, atol=1e-13), "VS, all verticals"
    vi, si = orc.vs_estimate(f32(q), f32(k), 64, 1, n + 5, scale)    # every offset slash
    out, _ = orc.vs_attention(f32(q), f32(k), f32(v), scale, vi, si)
    assert np.allclose(out, dense, rtol=1e-12, atol=1e-13), "VS, all slashes"
    bi, bc = orc.block_estimate(f32(q), f32(k), 64, n // 64)
    out, _ = orc.block_attention(f32(q), f32(k), f32(v), scale, 64, bi, bc)
    assert np.allclose(out, dense, rtol=1e-12, atol=1e-13), "BS, all blocks"
    out, _ = orc.ashape_attention(f32(q), f32(k), f32(v), scale, 0, n)
    assert np.allclose(out, dense, rtol=1e-12, atol=1e-13), "A-shape, window = n"


def pin_attention_closed_forms(orc):
    """Q = 0 gives the mean of V over the key set; lse = log(#keys)."""
    n = 192
    rng = np.random.default_rng(2)
    q = np.zeros((1, n, 128), np.float32)
    k = rng.standard_normal((1, n, 128)).astype(np.float32)
    v = rng.standard_normal((1, n, 128)).astype(np.float32)
    out, lse = orc.ashape_attention(q, k, v, 0.1, 3, 10)
    for i in range(n):
        keys = [kk for kk in range(i + 1) if kk < 3 or i - kk < 10]
        ref = v[0, keys].astype(np.float64).mean(axis=0)
        assert np.allclose(out[0, i], ref, rtol=1e-12, atol=1e-13), f"mean of V, row {i}"
        assert abs(lse[0, i] - math.log(len(keys))) < 1e-12, "lse = log count"


def pin_planted_recovery(orc):
    """On the 4K single-head planted input, key 0 and >= 70% of heavy keys are verticals.

    The plant (+4u on heavy keys, +1.5u on queries, scale 1/sqrt(128)) shifts a
    heavy key's logit by about +0.5 against unit noise, so a few heavy keys land
    below the 256-key budget; random choice would recover 256/4096 = 6%.
    """
    w = synth.WORKLOADS["vs-1h-4k"]
    x = synth.generate(w, seed=0)
    vi, si = orc.vs_estimate(x["q"], x["k"], w.last_q, w.n_vertical, w.n_slash,
                             1.0 / math.sqrt(128))
    heavy = set(x["planted"]["heavy"][0].tolist())
    got = set(vi[0].tolist())
    assert 0 in got, "key 0 recovered"
    assert len(heavy & got) >= 0.7 * len(heavy), "planted verticals recovered"
    assert 0 in set(si[0].tolist()), "main diagonal present"


ALL_PINS = [
    pin_vs_estimate_bruteforce,
    pin_vs_estimate_uniform_closed_form,
    pin_vs_estimate_golden,
    pin_block_estimate_commutes,
    pin_block_estimate_topk_bruteforce,
    pin_attention_masks_bruteforce,
    pin_full_budget_is_dense,
    pin_trishape_bruteforce,
    pin_vs_tiles_forms,
    pin_vs_topp_forms,
    pin_attention_closed_forms,
    pin_planted_recovery,
]
