"""Parity at the benchmark's full sizes, in the launch configuration bench.py times.

The whole layer runs on the GPU (every head); the oracle then checks sampled
heads: their index sets against the oracle's scores (tie band), and sampled
output rows (the first and last rows, and rows spread over the sequence)
against the fp64 attention with the same indices.
"""
import math

import numpy as np
import pytest
import torch

from dynamic_sparse_attention_est_b200 import minf, synth
from parity import bs_score_error, check_attention, check_topk_band

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(128)


def sample_rows(n, k=160):
    rows = np.unique(np.concatenate([np.arange(64), np.linspace(0, n - 1, k).astype(np.int64), np.arange(n - 64, n)]))
    return rows.astype(np.int32)


def head_inputs(x, h, group):
    """One q-head and its kv-head as host tensors (the oracle sees hq = hkv = 1)."""
    g = h // group
    return x["q"][h:h + 1].cpu(), x["k"][g:g + 1].cpu(), x["v"][g:g + 1].cpu()


@pytest.fixture(scope="module")
def vs32k():
    w = synth.WORKLOADS["vs-gqa-32k"]
    return w, synth.generate(w, seed=0, device="cuda")


def test_vs_32k_layer(orc, vs32k):
    w, x = vs32k
    q, k, v = x["q"], x["k"], x["v"]
    gv, gs = minf.minf_vs_estimate(q, k, w.last_q, w.n_vertical, w.n_slash, SCALE)
    out, lse = minf.minf_vs_attention(q, k, v, gv, gs, SCALE)
    torch.cuda.synchronize()
    rows = sample_rows(w.n)
    grp = w.hq // w.hkv
    for h in (0, 13, 31):
        qh, kh, vh = head_inputs(x, h, grp)
        vi, si, vert, slash = orc.vs_estimate(qh, kh, w.last_q, w.n_vertical, w.n_slash, SCALE, return_scores=True)
        check_topk_band(gv[h].cpu().numpy(), vert[0], w.n_vertical, f"vertical h{h}")
        check_topk_band(gs[h].cpu().numpy(), slash[0], w.n_slash, f"slash h{h}")
        # attention on the GPU's own indices (the benchmarked configuration)
        ref, rl = orc.vs_attention(qh, kh, vh, SCALE, gv[h:h + 1].cpu().numpy(), gs[h:h + 1].cpu().numpy(), rows=rows)
        check_attention(out[h, rows], lse[h, rows], ref[0], rl[0], f"VS 32K head {h}")
        # attention with the oracle's indices fed in
        o2, l2 = minf.minf_vs_attention(q, k, v, torch.from_numpy(vi).cuda(), torch.from_numpy(si).cuda(), SCALE,
                                        head_ids=[h])
        ref2, rl2 = orc.vs_attention(qh, kh, vh, SCALE, vi, si, rows=rows)
        check_attention(o2[0, rows], l2[0, rows], ref2[0], rl2[0], f"VS 32K head {h}, oracle indices")


def test_vs_32k_layer_whole_tiles(orc, vs32k):
    """The whole-slash-tile variant at full size on the GPU's own indices, sampled rows."""
    w, x = vs32k
    q, k, v = x["q"], x["k"], x["v"]
    gv, gs = minf.minf_vs_estimate(q, k, w.last_q, w.n_vertical, w.n_slash, SCALE)
    out, lse = minf.minf_vs_attention_tiles(q, k, v, gv, gs, SCALE)
    torch.cuda.synchronize()
    rows = sample_rows(w.n)
    grp = w.hq // w.hkv
    for h in (2, 29):
        qh, kh, vh = head_inputs(x, h, grp)
        ref, rl = orc.vs_tiles_attention(qh, kh, vh, SCALE, gv[h:h + 1].cpu().numpy(), gs[h:h + 1].cpu().numpy(),
                                         128, rows=rows)
        check_attention(out[h, rows], lse[h, rows], ref[0], rl[0], f"VS tiles 32K head {h}")


def test_dense_32k_layer(orc, vs32k):
    w, x = vs32k
    out, lse = minf.minf_dense_attention(x["q"], x["k"], x["v"], SCALE)
    torch.cuda.synchronize()
    rows = sample_rows(w.n, 96)
    for h in (5, 30):
        qh, kh, vh = head_inputs(x, h, w.hq // w.hkv)
        ref, rl = orc.dense_attention(qh, kh, vh, SCALE, rows=rows)
        check_attention(out[h, rows], lse[h, rows], ref[0], rl[0], f"dense 32K head {h}")


def test_block_128k_layer(orc):
    w = synth.WORKLOADS["block-gqa-128k"]
    x = synth.generate(w, seed=0, device="cuda")
    q, k, v = x["q"], x["k"], x["v"]
    bi, bc = minf.minf_block_estimate(q, k, w.topk)
    out, lse = minf.minf_block_attention(q, k, v, bi, bc, SCALE)
    torch.cuda.synchronize()
    rows = sample_rows(w.n, 128)
    grp = w.hq // w.hkv
    nb = w.n // 64
    for h in (0, 17):
        qh, kh, vh = head_inputs(x, h, grp)
        obi, obc, _, _, sc = orc.block_estimate(qh, kh, 64, w.topk, return_scores=True)
        gbi, gbc = bi[h].cpu().numpy(), bc[h].cpu().numpy()
        eb = bs_score_error(qh, kh)[0]
        for i in list(range(0, nb, 37)) + [nb - 1]:
            assert gbc[i] == min(w.topk, i + 1) and gbi[i, gbc[i] - 1] == i
            check_topk_band(gbi[i, :gbc[i] - 1], sc[0, i, :i], w.topk - 1, f"block row {h}/{i}", abs_band=eb[i])
        ref, rl = orc.block_attention(qh, kh, vh, SCALE, 64, gbi[None], gbc[None], rows=rows)
        check_attention(out[h, rows], lse[h, rows], ref[0], rl[0], f"block 128K head {h}")
        o2, l2 = minf.minf_block_attention(q, k, v, torch.from_numpy(obi).cuda(), torch.from_numpy(obc).cuda(),
                                           SCALE, head_ids=[h])
        ref2, rl2 = orc.block_attention(qh, kh, vh, SCALE, 64, obi, obc, rows=rows)
        check_attention(o2[0, rows], l2[0, rows], ref2[0], rl2[0], f"block 128K head {h}, oracle indices")


def test_ashape_128k_layer(orc):
    w = synth.WORKLOADS["ashape-gqa-128k"]
    x = synth.generate(w, seed=0, device="cuda")
    out, lse = minf.minf_ashape_attention(x["q"], x["k"], x["v"], w.n_sink, w.window, SCALE)
    torch.cuda.synchronize()
    rows = sample_rows(w.n, 128)
    for h in (0, 31):
        qh, kh, vh = head_inputs(x, h, w.hq // w.hkv)
        ref, rl = orc.ashape_attention(qh, kh, vh, SCALE, w.n_sink, w.window, rows=rows)
        check_attention(out[h, rows], lse[h, rows], ref[0], rl[0], f"A-shape 128K head {h}")


def test_mixed_1m_layer(orc):
    w = synth.WORKLOADS["mixed-gqa-1m"]
    x = synth.generate(w, seed=0, device="cuda")
    q, k, v = x["q"], x["k"], x["v"]
    pats = synth.mixed_head_patterns(w, seed=0)
    out, lse = minf.minf_mixed_layer(q, k, v, pats, w.last_q, w.n_vertical, w.n_slash, w.topk, w.n_sink, w.window,
                                     SCALE)
    torch.cuda.synchronize()
    rows = sample_rows(w.n, 48)
    grp = w.hq // w.hkv
    for p in ("vs", "block", "ashape"):
        h = pats.index(p)
        qh, kh, vh = head_inputs(x, h, grp)
        if p == "vs":
            gv, gs = minf.minf_vs_estimate(q, k, w.last_q, w.n_vertical, w.n_slash, SCALE, head_ids=[h])
            vi, si, vert, slash = orc.vs_estimate(qh, kh, w.last_q, w.n_vertical, w.n_slash, SCALE,
                                                  return_scores=True)
            check_topk_band(gv[0].cpu().numpy(), vert[0], w.n_vertical, f"1M vertical h{h}")
            check_topk_band(gs[0].cpu().numpy(), slash[0], w.n_slash, f"1M slash h{h}")
            ref, rl = orc.vs_attention(qh, kh, vh, SCALE, gv.cpu().numpy(), gs.cpu().numpy(), rows=rows)
        elif p == "block":
            gbi, gbc = minf.minf_block_estimate(q, k, w.topk, head_ids=[h])
            ref, rl = orc.block_attention(qh, kh, vh, SCALE, 64, gbi.cpu().numpy(), gbc.cpu().numpy(), rows=rows)
        else:
            ref, rl = orc.ashape_attention(qh, kh, vh, SCALE, w.n_sink, w.window, rows=rows)
        check_attention(out[h, rows], lse[h, rows], ref[0], rl[0], f"mixed 1M head {h} ({p})")


def test_trishape_128k_layer(orc):
    """Tri-shape at the bench's size (n_last = last_q = 64 dense tail rows)."""
    w = synth.WORKLOADS["trishape-gqa-128k"]
    x = synth.generate(w, seed=0, device="cuda")
    out, lse = minf.minf_trishape_attention(x["q"], x["k"], x["v"], w.n_sink, w.window, w.last_q, SCALE)
    torch.cuda.synchronize()
    rows = sample_rows(w.n, 96)  # includes the last 64 rows, the dense tail
    for h in (5, 26):
        qh, kh, vh = head_inputs(x, h, w.hq // w.hkv)
        ref, rl = orc.trishape_attention(qh, kh, vh, SCALE, w.n_sink, w.window, w.last_q, rows=rows)
        check_attention(out[h, rows], lse[h, rows], ref[0], rl[0], f"Tri-shape 128K head {h}")


def test_vs_32k_layer_topp(orc, vs32k):
    """Top-p budgets (p = 0.95, the fixed budgets as caps) on the 32K layer: sampled
    heads' sets are the shortest covers of the oracle's mass, and the attention on
    them matches the oracle's."""
    from parity import check_topp

    w, x = vs32k
    q, k, v = x["q"], x["k"], x["v"]
    p = 0.95
    gv, gs, gvc, gsc = minf.minf_vs_estimate_topp(q, k, w.last_q, w.n_vertical, w.n_slash, p, p, SCALE)
    out, lse = minf.minf_vs_attention(q, k, v, gv, gs, SCALE)
    torch.cuda.synchronize()
    rows = sample_rows(w.n, 96)
    grp = w.hq // w.hkv
    for h in (3, 30):
        qh, kh, vh = head_inputs(x, h, grp)
        _, _, _, _, vert, slash = orc.vs_estimate_topp(qh, kh, w.last_q, w.n_vertical, w.n_slash, p, p, SCALE,
                                                       return_scores=True)
        check_topp(gv[h].cpu().numpy(), int(gvc[h]), vert[0], p, w.n_vertical, False, f"32K top-p vertical h{h}")
        check_topp(gs[h].cpu().numpy(), int(gsc[h]), slash[0], p, w.n_slash, True, f"32K top-p slash h{h}")
        ref, rl = orc.vs_attention(qh, kh, vh, SCALE, gv[h:h + 1].cpu().numpy(), gs[h:h + 1].cpu().numpy(),
                                   rows=rows)
        check_attention(out[h, rows], lse[h, rows], ref[0], rl[0], f"VS 32K top-p head {h}")
