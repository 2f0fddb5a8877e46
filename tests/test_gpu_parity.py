"""CUDA path (through the C ABI) against the fp64 oracle on the same seeded inputs.

Sizes here are small enough for the oracle to finish in seconds, yet span
several 128-row tiles and ragged tails (n % 128 == 64).
"""
import math

import numpy as np
import pytest
import torch

from dynamic_sparse_attention_est_b200 import minf, synth
from parity import (BS_TC_ACC_COEF, bs_score_bound, bs_score_error, check_attention, check_topk_band, check_topp,
                    pooled_fp32_model, tc_pooled_scores_model, to_np)

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(128)


def inputs(n, hq, hkv, structure="vertical", seed=0, n_heavy=8):
    w = synth.Workload("test", "vs", hq, hkv, n, structure, n_heavy=n_heavy)
    x = synth.generate(w, seed=seed)
    return x["q"], x["k"], x["v"]


def cuda(*ts):
    return [t.cuda() for t in ts]


@pytest.mark.parametrize("n,hq,hkv", [(128, 1, 1), (320, 1, 1), (1024, 4, 2), (1088, 2, 2)])
def test_dense(orc, n, hq, hkv):
    q, k, v = inputs(n, hq, hkv, seed=n)
    ref, rl = orc.dense_attention(q, k, v, SCALE)
    out, lse = minf.minf_dense_attention(*cuda(q, k, v), scale=SCALE)
    check_attention(out, lse, ref, rl, f"dense n={n}")


def test_dense_head_subset(orc):
    q, k, v = inputs(576, 4, 2, seed=3)
    ids = [3, 0]
    ref, rl = orc.dense_attention(q, k, v, SCALE, head_ids=ids)
    out, lse = minf.minf_dense_attention(*cuda(q, k, v), scale=SCALE, head_ids=ids)
    check_attention(out, lse, ref, rl, "dense subset")


@pytest.mark.parametrize("sink,window", [(128, 256), (100, 300), (0, 1), (64, 5000), (7, 64)])
def test_ashape(orc, sink, window):
    n = 1344
    q, k, v = inputs(n, 2, 1, structure="plain", seed=sink + window)
    ref, rl = orc.ashape_attention(q, k, v, SCALE, sink, window)
    out, lse = minf.minf_ashape_attention(*cuda(q, k, v), n_sink=sink, window=window, scale=SCALE)
    check_attention(out, lse, ref, rl, f"A-shape {sink}/{window}")


@pytest.mark.parametrize("topk", [1, 4, 16])
def test_block_attention_oracle_indices(orc, topk):
    n = 1216
    q, k, v = inputs(n, 4, 2, structure="plain", seed=topk)
    bi, bc = orc.block_estimate(q, k, 64, topk)
    ref, rl = orc.block_attention(q, k, v, SCALE, 64, bi, bc)
    out, lse = minf.minf_block_attention(*cuda(q, k, v), torch.from_numpy(bi).cuda(), torch.from_numpy(bc).cuda(),
                                         scale=SCALE)
    check_attention(out, lse, ref, rl, f"block topk={topk}")


@pytest.mark.parametrize("n,hq,hkv,topk", [(2048, 4, 2, 8),
                                           (64 * 263, 2, 1, 100),    # several 128-block score tiles, nb % 4 != 0
                                           (64 * 2100, 1, 1, 100)])  # rows longer than the warp-per-row limit
def test_block_estimate_band(orc, n, hq, hkv, topk):
    w = synth.Workload("t", "block", hq, hkv, n, "clustered")
    x = synth.generate(w, seed=1)
    q, k = x["q"], x["k"]
    bi, bc, _, _, sc = orc.block_estimate(q, k, 64, topk, return_scores=True)
    gi, gc = minf.minf_block_estimate(*cuda(q, k), topk=topk)
    gi, gc = gi.cpu().numpy(), gc.cpu().numpy()
    nb = n // 64
    eb = bs_score_error(q, k)
    for hp in range(hq):
        for i in range(nb):
            row = gi[hp, i, :gc[hp, i]]
            assert gc[hp, i] == min(topk, i + 1)
            assert row[-1] == i, "diagonal block forced"
            check_topk_band(row[:-1], sc[hp, i, :i], topk - 1, f"block row {hp}/{i}", abs_band=eb[hp, i])
            assert np.all(gi[hp, i, gc[hp, i]:] == -1)


@pytest.mark.parametrize("n_proto", [1, 3, 40])
def test_block_estimate_exact_ties_go_to_lower_index(orc, n_proto):
    """Key blocks copied from a few prototypes give pooled scores with exact ties
    (bit-identical on both sides: identical operands, identical arithmetic), and
    query blocks of zeros give rows of zeros.  The selection must then match the
    oracle exactly, ties to the lower block index: with one prototype every row
    is one tie (the whole row in one bin); with 3, each score value is shared by
    about a third of the row (more than 32 candidates in the threshold bin: the
    radix path); with 40, about 1/40 (the ranked path)."""
    n, hq, hkv, topk = 64 * 300, 2, 1, 40
    rng = np.random.default_rng(n_proto)
    proto = rng.standard_normal((n_proto, 64, 128)).astype(np.float32)
    pick = rng.integers(0, n_proto, n // 64)
    k = torch.from_numpy(proto[pick].reshape(1, n, 128)).to(torch.bfloat16)
    q = torch.from_numpy(rng.standard_normal((hq, n, 128)).astype(np.float32)).to(torch.bfloat16)
    q[1, :64 * 20] = 0  # the first 20 query blocks of head 1: all-zero score rows
    bi, bc = orc.block_estimate(q, k, 64, topk)
    gi, gc = minf.minf_block_estimate(*cuda(q, k), topk=topk)
    assert np.array_equal(gc.cpu().numpy(), bc)
    assert np.array_equal(gi.cpu().numpy(), bi)


@pytest.mark.parametrize("n,hq,hkv,ids", [(64 * 300, 4, 2, [3, 0, 2]),   # three row tiles, the last ragged
                                           (64 * 263, 2, 1, None),        # nb % 4 != 0: scalar stores
                                           (64 * 5, 2, 2, None)])         # one tile, fewer rows than a TMA box
def test_block_scores_tensor_core_error(orc, n, hq, hkv, ids):
    """The tensor-core pooled scores, entry by entry for j <= i:
    - against the exact (fp64) scores, within the worst-case bound of the split-bf16
      arithmetic (which lies inside the fp32 dot-product bound of the index band);
    - against a CPU model of the same arithmetic (identical fp32 pooling and bf16
      parts, truncating fp32 accumulation per K = 16 step), within twice the bound
      of the accumulation alone: a missing or misplaced part product fails this."""
    w = synth.Workload("t", "block", hq, hkv, n, "clustered")
    x = synth.generate(w, seed=4)
    q, k = x["q"], x["k"]
    heads = list(range(hq)) if ids is None else ids
    _, _, _, _, sc = orc.block_estimate(q, k, 64, 1, head_ids=heads, return_scores=True)
    gs = minf.minf_block_scores(*cuda(q, k), head_ids=ids).cpu().numpy().astype(np.float64)
    nb = n // 64
    tril = np.tril(np.ones((nb, nb), bool))
    bound = bs_score_bound(q, k)[heads]
    model = tc_pooled_scores_model(q, k)[heads]
    qp, kp = np.abs(pooled_fp32_model(q).astype(np.float64)), np.abs(pooled_fp32_model(k).astype(np.float64))
    g = hq // hkv
    s_abs = np.stack([qp[h] @ kp[h // g].T for h in heads])
    for hp in range(len(heads)):
        err = np.abs(gs[hp] - sc[hp])[tril]
        assert np.all(np.isfinite(gs[hp][tril]))
        assert np.all(err <= bound[hp][tril]), f"head {heads[hp]}: max err/bound {np.max(err / bound[hp][tril]):.3g}"
        dm = np.abs(gs[hp] - model[hp])[tril]
        lim = 2 * BS_TC_ACC_COEF * s_abs[hp][tril]
        assert np.all(dm <= lim), f"head {heads[hp]}: max |gpu - model| / limit {np.max(dm / lim):.3g}"


def _rand_vs_indices(rng, n, nh, nv, ns):
    vi = np.full((nh, nv), -1, np.int32)
    si = np.full((nh, ns), -1, np.int32)
    for hp in range(nh):
        a = rng.choice(n, nv - 3, replace=False)
        vi[hp, :nv - 3] = a[rng.permutation(len(a))]           # unsorted
        vi[hp, nv - 3] = a[0]                                    # a duplicate
        b = rng.choice(n, ns - 2, replace=False)
        si[hp, :ns - 2] = b
    return vi, si


@pytest.mark.parametrize("n,hq,hkv,nv,ns", [(1024, 4, 2, 40, 60), (1344, 2, 1, 100, 30), (4096, 1, 1, 256, 512)])
def test_vs_attention_oracle_indices(orc, n, hq, hkv, nv, ns):
    q, k, v = inputs(n, hq, hkv, seed=nv)
    vi, si = orc.vs_estimate(q, k, 64, nv, ns, SCALE)
    ref, rl = orc.vs_attention(q, k, v, SCALE, vi, si)
    out, lse = minf.minf_vs_attention(*cuda(q, k, v), torch.from_numpy(vi).cuda(), torch.from_numpy(si).cuda(),
                                      scale=SCALE)
    check_attention(out, lse, ref, rl, f"VS n={n}")


def test_vs_attention_unsorted_duplicate_indices(orc):
    n, hq, hkv = 1088, 2, 1
    q, k, v = inputs(n, hq, hkv, seed=77)
    vi, si = _rand_vs_indices(np.random.default_rng(5), n, hq, 50, 70)
    ref, rl = orc.vs_attention(q, k, v, SCALE, vi, si)
    out, lse = minf.minf_vs_attention(*cuda(q, k, v), torch.from_numpy(vi).cuda(), torch.from_numpy(si).cuda(),
                                      scale=SCALE)
    check_attention(out, lse, ref, rl, "VS random sets")


@pytest.mark.parametrize("n,hq,hkv,last_q,nv,ns", [(4096, 1, 1, 64, 256, 512), (2048, 4, 2, 64, 100, 300),
                                                   (1088, 3, 1, 17, 30, 40),
                                                   (65600, 2, 1, 64, 1000, 2000)])  # rows split over blocks
def test_vs_estimate_band(orc, n, hq, hkv, last_q, nv, ns):
    q, k, _ = inputs(n, hq, hkv, seed=n + hq)
    vi, si, vert, slash = orc.vs_estimate(q, k, last_q, nv, ns, SCALE, return_scores=True)
    gv, gs = minf.minf_vs_estimate(*cuda(q, k), last_q=last_q, n_vertical=nv, n_slash=ns, scale=SCALE)
    gv, gs = gv.cpu().numpy(), gs.cpu().numpy()
    for hp in range(hq):
        check_topk_band(gv[hp], vert[hp], nv, f"vertical h{hp}")
        check_topk_band(gs[hp], slash[hp], ns, f"slash h{hp}")
        assert 0 in set(gs[hp].tolist()), "offset 0 forced"


def test_vs_end_to_end_4k(orc):
    """4K single head, planted verticals: GPU estimate, then GPU attention on the GPU's indices vs the
    oracle attention on the same indices."""
    w = synth.WORKLOADS["vs-1h-4k"]
    x = synth.generate(w, seed=0)
    q, k, v = x["q"], x["k"], x["v"]
    gv, gs = minf.minf_vs_estimate(*cuda(q, k), last_q=64, n_vertical=256, n_slash=512, scale=SCALE)
    out, lse = minf.minf_vs_attention(*cuda(q, k, v), gv, gs, scale=SCALE)
    ref, rl = orc.vs_attention(q, k, v, SCALE, gv.cpu().numpy(), gs.cpu().numpy())
    check_attention(out, lse, ref, rl, "VS 4k end to end")


def test_mixed_layer(orc):
    n, hq, hkv = 1280, 8, 2
    q, k, v = inputs(n, hq, hkv, seed=11)
    pats = ["vs", "block", "ashape", "dense", "vs", "vs", "block", "ashape"]
    nv, ns, topk, sink, window = 40, 80, 6, 64, 256
    out, lse = minf.minf_mixed_layer(*cuda(q, k, v), pats, last_q=64, n_vertical=nv, n_slash=ns, topk=topk,
                                     n_sink=sink, window=window, scale=SCALE)
    for h, p in enumerate(pats):
        ids = [h]
        if p == "vs":
            vi, si = orc.vs_estimate(q, k, 64, nv, ns, SCALE, head_ids=ids)
            ref, rl = orc.vs_attention(q, k, v, SCALE, vi, si, head_ids=ids)
        elif p == "block":
            bi, bc = orc.block_estimate(q, k, 64, topk, head_ids=ids)
            ref, rl = orc.block_attention(q, k, v, SCALE, 64, bi, bc, head_ids=ids)
        elif p == "ashape":
            ref, rl = orc.ashape_attention(q, k, v, SCALE, sink, window, head_ids=ids)
        else:
            ref, rl = orc.dense_attention(q, k, v, SCALE, head_ids=ids)
        check_attention(out[h:h + 1], lse[h:h + 1], ref, rl, f"mixed head {h} ({p})")


def test_stats_count_dense_tiles():
    n, hq, hkv = 1088, 2, 1
    q, k, v = cuda(*inputs(n, hq, hkv, seed=2))
    ws = minf.workspace(256, q.device)
    minf.minf_dense_attention(q, k, v, scale=SCALE, ws=ws)
    tiles, pairs = minf.minf_stats(ws)
    nt = (n + 127) // 128
    halves = sum(min(2 * t + 2, n // 64) for t in range(nt))
    assert tiles == hq * sum((min(2 * t + 2, n // 64) + 1) // 2 for t in range(nt))
    assert pairs == hq * n * (n + 1) // 2
    assert halves > 0
    assert minf.minf_status(ws) == minf.MINF_OK


def test_bounded_wait_reports_timeout():
    ws = minf.workspace(256, torch.device("cuda"))
    minf.minf_check_wait_timeout(ws, 2_000_000)  # 2 ms
    assert minf.minf_status(ws) == minf.MINF_ERR_TIMEOUT
    assert minf.minf_status(ws) == minf.MINF_OK  # reading resets it
    # the context is still usable
    q, k, v = cuda(*inputs(128, 1, 1, seed=0))
    out, _ = minf.minf_dense_attention(q, k, v)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()


# ----------------------------------------------------------------------------- edge cases
@pytest.mark.parametrize("n", [64, 192])
def test_single_and_ragged_blocks_every_pattern(orc, n):
    q, k, v = inputs(n, 2, 1, seed=n + 1)
    qc, kc, vc = cuda(q, k, v)
    ref, rl = orc.dense_attention(q, k, v, SCALE)
    out, lse = minf.minf_dense_attention(qc, kc, vc, scale=SCALE)
    check_attention(out, lse, ref, rl, f"dense n={n}")
    ref, rl = orc.ashape_attention(q, k, v, SCALE, 16, 40)
    out, lse = minf.minf_ashape_attention(qc, kc, vc, 16, 40, scale=SCALE)
    check_attention(out, lse, ref, rl, f"A-shape n={n}")
    bi, bc = orc.block_estimate(q, k, 64, 2)
    gbi, gbc = minf.minf_block_estimate(qc, kc, topk=2)
    assert np.array_equal(gbi.cpu().numpy(), bi) and np.array_equal(gbc.cpu().numpy(), bc)
    ref, rl = orc.block_attention(q, k, v, SCALE, 64, bi, bc)
    out, lse = minf.minf_block_attention(qc, kc, vc, gbi, gbc, scale=SCALE)
    check_attention(out, lse, ref, rl, f"block n={n}")
    vi, si, vert, slash = orc.vs_estimate(q, k, 64, 8, 16, SCALE, return_scores=True)
    gv, gs = minf.minf_vs_estimate(qc, kc, 64, 8, 16, scale=SCALE)
    for hp in range(2):
        check_topk_band(gv[hp].cpu().numpy(), vert[hp], 8, f"vertical n={n}")
        check_topk_band(gs[hp].cpu().numpy(), slash[hp], 16, f"slash n={n}")
    ref, rl = orc.vs_attention(q, k, v, SCALE, vi, si)
    out, lse = minf.minf_vs_attention(qc, kc, vc, torch.from_numpy(vi).cuda(), torch.from_numpy(si).cuda(),
                                      scale=SCALE)
    check_attention(out, lse, ref, rl, f"VS n={n}")


def test_budgets_above_n_pad_and_cover_everything(orc):
    n = 256
    q, k, v = inputs(n, 2, 1, seed=21)
    qc, kc, vc = cuda(q, k, v)
    gv, gs = minf.minf_vs_estimate(qc, kc, 64, 300, 400, scale=SCALE)
    gv, gs = gv.cpu().numpy(), gs.cpu().numpy()
    assert np.array_equal(gv[:, :n], np.tile(np.arange(n), (2, 1))) and np.all(gv[:, n:] == -1)
    assert np.array_equal(gs[:, :n], np.tile(np.arange(n), (2, 1))) and np.all(gs[:, n:] == -1)
    out, lse = minf.minf_vs_attention(qc, kc, vc, torch.from_numpy(gv).cuda(), torch.from_numpy(gs).cuda(),
                                      scale=SCALE)
    ref, rl = orc.dense_attention(q, k, v, SCALE)
    check_attention(out, lse, ref, rl, "VS full budgets = dense")
    bi, bc = minf.minf_block_estimate(qc, kc, topk=9)  # topk above the 4 blocks
    out, lse = minf.minf_block_attention(qc, kc, vc, bi, bc, scale=SCALE)
    check_attention(out, lse, ref, rl, "BS full budgets = dense")


def test_empty_key_sets_give_zero_and_minus_inf(orc):
    n = 320
    q, k, v = inputs(n, 2, 1, seed=4)
    qc, kc, vc = cuda(q, k, v)
    nb = n // 64
    bi = torch.full((2, nb, 3), -1, dtype=torch.int32)
    bc = torch.zeros(2, nb, dtype=torch.int32)
    bi[0, 2, 0] = 1  # one query block of head 0 sees key block 1; everything else is empty
    bc[0, 2] = 1
    ref, rl = orc.block_attention(q, k, v, SCALE, 64, bi.numpy(), bc.numpy())
    out, lse = minf.minf_block_attention(qc, kc, vc, bi.cuda(), bc.cuda(), scale=SCALE)
    check_attention(out, lse, ref, rl, "block with empty rows")
    assert torch.all(out[1] == 0) and torch.all(torch.isneginf(lse[1]))
    vi = torch.full((2, 4), -1, dtype=torch.int32)
    si = torch.full((2, 4), -1, dtype=torch.int32)
    si[0, 0] = 0  # head 0: the main diagonal only (each query attends to itself)
    ref, rl = orc.vs_attention(q, k, v, SCALE, vi.numpy(), si.numpy())
    out, lse = minf.minf_vs_attention(qc, kc, vc, vi.cuda(), si.cuda(), scale=SCALE)
    check_attention(out, lse, ref, rl, "VS diagonal only / empty")
    assert torch.equal(out[0], vc[0])  # softmax over one key returns that value row exactly
    assert torch.all(out[1] == 0) and torch.all(torch.isneginf(lse[1]))


def test_many_heads_and_unsorted_head_subset(orc):
    n, hq, hkv = 384, 16, 4
    q, k, v = inputs(n, hq, hkv, seed=8)
    ids = [15, 2, 7, 8, 3]
    qc, kc, vc = cuda(q, k, v)
    ref, rl = orc.ashape_attention(q, k, v, SCALE, 64, 100, head_ids=ids)
    out, lse = minf.minf_ashape_attention(qc, kc, vc, 64, 100, scale=SCALE, head_ids=ids)
    check_attention(out, lse, ref, rl, "A-shape head subset")
    vi, si, vert, slash = orc.vs_estimate(q, k, 48, 20, 30, SCALE, head_ids=ids, return_scores=True)
    gv, gs = minf.minf_vs_estimate(qc, kc, 48, 20, 30, scale=SCALE, head_ids=ids)
    for p in range(len(ids)):
        check_topk_band(gv[p].cpu().numpy(), vert[p], 20, f"vertical subset {p}")
        check_topk_band(gs[p].cpu().numpy(), slash[p], 30, f"slash subset {p}")
    ref, rl = orc.vs_attention(q, k, v, SCALE, vi, si, head_ids=ids)
    out, lse = minf.minf_vs_attention(qc, kc, vc, torch.from_numpy(vi).cuda(), torch.from_numpy(si).cuda(),
                                      scale=SCALE, head_ids=ids)
    check_attention(out, lse, ref, rl, "VS head subset")


@pytest.mark.parametrize("sink,window,n_last", [(128, 256, 64), (100, 300, 200), (0, 1, 1), (64, 64, 0), (7, 64, 5000)])
def test_trishape(orc, sink, window, n_last):
    n = 1344
    q, k, v = inputs(n, 2, 1, structure="plain", seed=sink + window + n_last)
    ref, rl = orc.trishape_attention(q, k, v, SCALE, sink, window, n_last)
    out, lse = minf.minf_trishape_attention(*cuda(q, k, v), n_sink=sink, window=window, n_last=n_last, scale=SCALE)
    check_attention(out, lse, ref, rl, f"Tri-shape {sink}/{window}/{n_last}")


def test_mixed_layer_with_trishape(orc):
    n, hq, hkv = 704, 4, 2
    q, k, v = inputs(n, hq, hkv, seed=12)
    pats = ["trishape", "vs", "trishape", "block"]
    out, lse = minf.minf_mixed_layer(*cuda(q, k, v), pats, last_q=48, n_vertical=16, n_slash=32, topk=3,
                                     n_sink=32, window=96, scale=SCALE)
    for h in (0, 2):
        ref, rl = orc.trishape_attention(q, k, v, SCALE, 32, 96, 48, head_ids=[h])
        check_attention(out[h:h + 1], lse[h:h + 1], ref, rl, f"mixed Tri-shape head {h}")


@pytest.mark.parametrize("n", [49216, 65600])
def test_long_rows_budgets_above_n(n):
    """Rows longer than one block's shared memory: budgets at or above n take every index, -1 padded."""
    q, k, _ = inputs(n, 1, 1, seed=3)
    gv, gs = minf.minf_vs_estimate(*cuda(q, k), last_q=64, n_vertical=n + 5, n_slash=n, scale=SCALE)
    gv, gs = gv.cpu().numpy()[0], gs.cpu().numpy()[0]
    assert np.array_equal(gv[:n], np.arange(n)) and np.all(gv[n:] == -1)
    assert np.array_equal(gs, np.arange(n))


@pytest.mark.parametrize("n,nv", [(4096, 1000), (65600, 20000)])
def test_vertical_exact_ties_go_to_lower_index(orc, n, nv):
    """q = 0 gives every query row a uniform causal softmax, so every key column that all
    the last rows see has the same vertical score, summed in the same order: an exact tie
    that the selection breaks towards the lower index (as the oracle does)."""
    last_q = 64
    q, k, _ = inputs(n, 1, 1, seed=9)
    q = torch.zeros_like(q)
    vi, _, vert, _ = orc.vs_estimate(q, k, last_q, nv, 16, SCALE, return_scores=True)
    assert np.array_equal(vi[0], np.arange(nv))
    gv, _ = minf.minf_vs_estimate(*cuda(q, k), last_q=last_q, n_vertical=nv, n_slash=16, scale=SCALE)
    assert np.array_equal(gv.cpu().numpy()[0], np.arange(nv))


def test_vs_attention_many_slash_groups(orc):
    """More than a thousand separate slash groups (offsets 130 apart) with merged extras,
    over 140K keys: the group list spans several extraction sweeps; sampled rows."""
    n = 140096
    q, k, v = inputs(n, 1, 1, seed=17)
    offs = sorted(set([j * 130 for j in range(1078)] + [j * 130 + 60 for j in range(0, 1078, 7)]))
    si = np.array([offs], np.int32)
    rng = np.random.default_rng(4)
    vi = np.sort(rng.choice(n, 64, replace=False)).astype(np.int32)[None, :]
    rows = np.unique(np.concatenate([rng.integers(0, n, 200), np.arange(n - 64, n), [0, 127, 128, 140000]]))
    ref, rl = orc.vs_attention(q, k, v, SCALE, vi, si, rows=rows)
    out, lse = minf.minf_vs_attention(*cuda(q, k, v), torch.from_numpy(vi).cuda(), torch.from_numpy(si).cuda(),
                                      scale=SCALE)
    check_attention(out[:, rows], lse[:, rows], ref, rl, "VS many groups")


# ----------------------------------------------------------------------------- whole slash tiles
@pytest.mark.parametrize("n,hq,hkv,nv,ns", [(1024, 4, 2, 40, 60), (1344, 2, 1, 100, 30), (4096, 1, 1, 256, 512),
                                            (192, 2, 1, 8, 16), (64, 1, 1, 4, 8)])
def test_vs_tiles_oracle_indices(orc, n, hq, hkv, nv, ns):
    """Whole-slash-tile Vertical-Slash against the oracle's variant on the oracle's index sets."""
    q, k, v = inputs(n, hq, hkv, seed=nv + 3)
    vi, si = orc.vs_estimate(q, k, 64, nv, ns, SCALE)
    ref, rl = orc.vs_tiles_attention(q, k, v, SCALE, vi, si, 128)
    out, lse = minf.minf_vs_attention_tiles(*cuda(q, k, v), torch.from_numpy(vi).cuda(),
                                            torch.from_numpy(si).cuda(), scale=SCALE)
    check_attention(out, lse, ref, rl, f"VS tiles n={n}")


def test_vs_tiles_unsorted_duplicates_and_far_offsets(orc):
    """Unsorted rows with duplicates, -1 padding, offsets past n and a lone far offset."""
    n, hq, hkv = 1088, 2, 1
    q, k, v = inputs(n, hq, hkv, seed=78)
    vi, si = _rand_vs_indices(np.random.default_rng(6), n, hq, 50, 70)
    si[0, -1] = n + 100       # out of range: ignored
    si[1, :] = -1
    si[1, 0] = 300            # head 1: one far offset and the verticals
    ref, rl = orc.vs_tiles_attention(q, k, v, SCALE, vi, si, 128)
    out, lse = minf.minf_vs_attention_tiles(*cuda(q, k, v), torch.from_numpy(vi).cuda(),
                                            torch.from_numpy(si).cuda(), scale=SCALE)
    check_attention(out, lse, ref, rl, "VS tiles random sets")


def test_vs_tiles_superset_of_exact():
    """On the same indices the whole-tile key set contains the token-exact one: lse never drops."""
    n = 2048
    q, k, v = cuda(*inputs(n, 2, 1, seed=31))
    gv, gs = minf.minf_vs_estimate(q, k, 64, 100, 300, scale=SCALE)
    _, le = minf.minf_vs_attention(q, k, v, gv, gs, scale=SCALE)
    _, lt = minf.minf_vs_attention_tiles(q, k, v, gv, gs, scale=SCALE)
    assert torch.all(lt >= le - 1e-2)
    assert torch.any(lt > le + 1e-2)


def test_vs_tiles_many_slash_groups(orc):
    """Over a thousand separate slash groups at 140K keys, sampled rows."""
    n = 140096
    q, k, v = inputs(n, 1, 1, seed=18)
    offs = sorted(set([j * 130 for j in range(1078)] + [j * 130 + 60 for j in range(0, 1078, 7)]))
    si = np.array([offs], np.int32)
    rng = np.random.default_rng(5)
    vi = np.sort(rng.choice(n, 64, replace=False)).astype(np.int32)[None, :]
    rows = np.unique(np.concatenate([rng.integers(0, n, 200), np.arange(n - 64, n), [0, 127, 128, 140000]]))
    ref, rl = orc.vs_tiles_attention(q, k, v, SCALE, vi, si, 128, rows=rows)
    out, lse = minf.minf_vs_attention_tiles(*cuda(q, k, v), torch.from_numpy(vi).cuda(),
                                            torch.from_numpy(si).cuda(), scale=SCALE)
    check_attention(out[:, rows], lse[:, rows], ref, rl, "VS tiles many groups")


# ----------------------------------------------------------------------------- top-p budgets
@pytest.mark.parametrize("n,hq,hkv,pv,ps,cv,cs", [(1024, 4, 2, 0.9, 0.9, 1024, 1024), (4096, 1, 1, 0.5, 0.95, 4096, 4096),
                                                  (2048, 2, 1, 0.99, 0.99, 40, 30),
                                                  (65600, 1, 1, 0.8, 0.7, 65600, 65600)])
def test_vs_estimate_topp(orc, n, hq, hkv, pv, ps, cv, cs):
    q, k, _ = inputs(n, hq, hkv, seed=n + 7)
    vi, si, vc, sc, vert, slash = orc.vs_estimate_topp(q, k, 64, cv, cs, pv, ps, SCALE, return_scores=True)
    gv, gs, gvc, gsc = minf.minf_vs_estimate_topp(*cuda(q, k), 64, cv, cs, pv, ps, scale=SCALE)
    gv, gs, gvc, gsc = gv.cpu().numpy(), gs.cpu().numpy(), gvc.cpu().numpy(), gsc.cpu().numpy()
    for hp in range(hq):
        check_topp(gv[hp], gvc[hp], vert[hp], pv, cv, False, f"top-p vertical h{hp}")
        check_topp(gs[hp], gsc[hp], slash[hp], ps, cs, True, f"top-p slash h{hp}")
        assert abs(int(gvc[hp]) - int(vc[hp])) <= max(2, vc[hp] // 200), "vertical count near the oracle's"
        assert abs(int(gsc[hp]) - int(sc[hp])) <= max(2, sc[hp] // 200), "slash count near the oracle's"


def test_vs_topp_exact_ties_uniform_rows(orc):
    """Q = 0: every key column the last rows all see ties exactly (each column is summed
    over the same rows in the same order), so the vertical top-p set is the oracle's:
    the lowest indices among the ties, and the same count.  The diagonal sums are
    assembled from per-tile partials in an order that depends on the offset, so the
    slashes are checked within the band."""
    n = 4096
    q, k, _ = inputs(n, 1, 1, seed=12)
    q = torch.zeros_like(q)
    vi, si, vc, sc, vert, slash = orc.vs_estimate_topp(q, k, 64, 3000, 3000, 0.5, 0.3, SCALE, return_scores=True)
    gv, gs, gvc, gsc = minf.minf_vs_estimate_topp(*cuda(q, k), 64, 3000, 3000, 0.5, 0.3, scale=SCALE)
    assert int(gvc[0]) == int(vc[0]) and np.array_equal(gv[0].cpu().numpy(), vi[0])
    check_topp(gs[0].cpu().numpy(), gsc[0].item(), slash[0], 0.3, 3000, True, "uniform rows, slashes")


def test_vs_topp_then_attention(orc):
    """Top-p indices feed the attention unchanged (-1 padding ignored)."""
    n = 2048
    q, k, v = inputs(n, 2, 1, seed=19)
    vi, si, _, _ = orc.vs_estimate_topp(q, k, 64, 512, 512, 0.9, 0.9, SCALE)
    ref, rl = orc.vs_attention(q, k, v, SCALE, vi, si)
    out, lse = minf.minf_vs_attention(*cuda(q, k, v), torch.from_numpy(vi).cuda(), torch.from_numpy(si).cuda(),
                                      scale=SCALE)
    check_attention(out, lse, ref, rl, "VS attention on top-p indices")


def test_new_variants_on_an_unsorted_head_subset(orc):
    """Whole slash tiles, top-p budgets and Block-Sparse on a listed, unsorted head subset
    of a GQA layer with a ragged tail (n % 128 == 64)."""
    n, hq, hkv = 448, 16, 4
    q, k, v = inputs(n, hq, hkv, seed=28)
    ids = [14, 1, 6, 9, 4]
    qc, kc, vc = cuda(q, k, v)
    vi, si = orc.vs_estimate(q, k, 40, 24, 36, SCALE, head_ids=ids)
    ref, rl = orc.vs_tiles_attention(q, k, v, SCALE, vi, si, 128, head_ids=ids)
    out, lse = minf.minf_vs_attention_tiles(qc, kc, vc, torch.from_numpy(vi).cuda(), torch.from_numpy(si).cuda(),
                                            scale=SCALE, head_ids=ids)
    check_attention(out, lse, ref, rl, "VS whole tiles, head subset")
    tv, ts, tvc, tsc, vert, slash = orc.vs_estimate_topp(q, k, 40, 200, 200, 0.8, 0.6, SCALE, head_ids=ids,
                                                         return_scores=True)
    gv, gs, gvc, gsc = minf.minf_vs_estimate_topp(qc, kc, 40, 200, 200, 0.8, 0.6, scale=SCALE, head_ids=ids)
    for p in range(len(ids)):
        check_topp(gv[p].cpu().numpy(), gvc[p].item(), vert[p], 0.8, 200, False, f"top-p vertical subset {p}")
        check_topp(gs[p].cpu().numpy(), gsc[p].item(), slash[p], 0.6, 200, True, f"top-p slash subset {p}")
    bi, bc = orc.block_estimate(q, k, 64, 3, head_ids=ids)
    gbi, gbc = minf.minf_block_estimate(qc, kc, topk=3, head_ids=ids)
    ref, rl = orc.block_attention(q, k, v, SCALE, 64, bi, bc, head_ids=ids)
    out, lse = minf.minf_block_attention(qc, kc, vc, torch.from_numpy(bi).cuda(), torch.from_numpy(bc).cuda(),
                                         scale=SCALE, head_ids=ids)
    check_attention(out, lse, ref, rl, "Block-Sparse head subset (kv-head-major launch)")


def test_topp_p_one_and_tiny_p(orc):
    """p = 1 with caps above n keeps (nearly) every key; a tiny p keeps one vertical and
    offset 0 plus at most one more offset."""
    n = 320
    q, k, _ = inputs(n, 2, 1, seed=33)
    qc, kc = cuda(q, k)
    vi, si, vc, sc, vert, slash = orc.vs_estimate_topp(q, k, 64, n + 8, n + 8, 1.0, 1.0, SCALE, return_scores=True)
    gv, gs, gvc, gsc = minf.minf_vs_estimate_topp(qc, kc, 64, n + 8, n + 8, 1.0, 1.0, scale=SCALE)
    for p in range(2):
        assert int(gvc[p]) >= n - 8 and int(gsc[p]) >= n - 8, "p = 1 keeps almost every key"
        check_topp(gv[p].cpu().numpy(), gvc[p].item(), vert[p], 1.0, n + 8, False, "p = 1 vertical")
    gv, gs, gvc, gsc = minf.minf_vs_estimate_topp(qc, kc, 64, 50, 50, 1e-6, 1e-6, scale=SCALE)
    assert torch.all(gvc == 1) and torch.all(gsc <= 2) and torch.all(gs[:, 0] == 0)


def test_repeat_runs_bit_identical():
    """Estimates and attention are deterministic: no atomics decide a value (the
    diagonal partials are added in a fixed order, each work item is one CTA), so
    two runs on the same inputs, with other launches between them, agree bit for bit."""
    n, hq, hkv = 4160, 4, 2
    q, k, v = cuda(*inputs(n, hq, hkv, seed=7))
    xb = synth.generate(synth.Workload("t", "block", hq, hkv, n, "clustered"), seed=7)
    qb, kb, vb = cuda(xb["q"], xb["k"], xb["v"])

    def once():
        gv, gs = minf.minf_vs_estimate(q, k, last_q=64, n_vertical=200, n_slash=400, scale=SCALE)
        o, l = minf.minf_vs_attention(q, k, v, gv, gs, scale=SCALE)
        bi, bc = minf.minf_block_estimate(qb, kb, topk=20)
        ob, lb = minf.minf_block_attention(qb, kb, vb, bi, bc, scale=SCALE)
        torch.cuda.synchronize()
        return [t.cpu() for t in (gv, gs, o, l, bi, bc, ob, lb)]

    first = once()
    minf.minf_dense_attention(qb, kb, vb, scale=SCALE)  # unrelated work between the two runs
    second = once()
    names = ["v_idx", "s_idx", "vs out", "vs lse", "blk_idx", "blk_cnt", "bs out", "bs lse"]
    for name, a, b in zip(names, first, second):
        assert torch.equal(a.view(torch.uint8) if a.dtype == torch.bfloat16 else a,
                           b.view(torch.uint8) if b.dtype == torch.bfloat16 else b), f"{name} differs between runs"


# ----------------------------------------------------------------------------- sparse slash groups
def _sparse_vs_indices(rng, n, nh, nv, n_far):
    """Verticals anywhere; slash offsets mostly far apart (lone offsets), some in
    pairs and triples within 128 of each other, offset 0 and one past n."""
    vi = np.full((nh, nv), -1, np.int32)
    si = np.full((nh, 3 * n_far + 2), -1, np.int32)
    for hp in range(nh):
        vi[hp] = rng.choice(n, nv, replace=False)
        base = np.sort(rng.choice(np.arange(1, n), n_far, replace=False))
        extra = [b + rng.integers(1, 100) for b in base[::3]] + [b + rng.integers(1, 60) for b in base[::5]]
        offs = np.unique(np.concatenate([[0], base, extra, [n + 5]]))
        si[hp, :len(offs)] = rng.permutation(offs)
    return vi, si


@pytest.mark.parametrize("n,hq,hkv,nv,n_far", [(4160, 2, 1, 40, 24), (8192, 4, 2, 100, 60), (1088, 1, 1, 8, 6)])
def test_vs_sparse_slash_groups_cuda_core_path(orc, n, hq, hkv, nv, n_far):
    """Lone and small slash groups take the CUDA-core pass (the default routing), the
    rest the tile kernel; verticals that lie on those diagonals count once.  Both
    routings agree with the oracle on the same indices."""
    q, k, v = inputs(n, hq, hkv, seed=n + nv)
    vi, si = _sparse_vs_indices(np.random.default_rng(n), n, hq, nv, n_far)
    ref, rl = orc.vs_attention(q, k, v, SCALE, vi, si)
    qc, kc, vc = cuda(q, k, v)
    vt, st = torch.from_numpy(vi).cuda(), torch.from_numpy(si).cuda()
    ws = minf.workspace(minf.workspace_bytes(minf.OP_VS_ATTENTION, hq, hkv, n, hq, vi.shape[1], si.shape[1]),
                        qc.device)
    try:
        for ratio in (1.0, 0.0, 1000.0):  # default, tensor cores only, CUDA cores for every group
            minf.minf_set_vs_diag_ratio(ratio)
            out, lse = minf.minf_vs_attention(qc, kc, vc, vt, st, scale=SCALE, ws=ws)
            check_attention(out, lse, ref, rl, f"VS sparse groups n={n} ratio={ratio}")
            tiles, pairs = minf.minf_stats(ws)
            assert minf.minf_status(ws) == minf.MINF_OK
            # every in-mask pair is counted once, by one of the two paths
            assert pairs == _mask_pairs(vi, si, n), (ratio, pairs)
    finally:
        minf.minf_set_vs_diag_ratio(1.0)


def _mask_pairs(vi, si, n):
    """Number of (query, key) pairs of the Vertical-Slash mask, counted from its definition."""
    total = 0
    for hp in range(vi.shape[0]):
        vset = np.zeros(n, bool)
        vset[vi[hp][(vi[hp] >= 0) & (vi[hp] < n)]] = True
        sset = np.unique(si[hp][(si[hp] >= 0) & (si[hp] < n)])
        for i in range(n):
            keys = np.zeros(i + 1, bool)
            keys |= vset[:i + 1]
            o = sset[sset <= i]
            keys[i - o] = True
            total += int(keys.sum())
    return total


def test_vs_sparse_groups_head_subset_and_determinism(orc):
    """A listed head subset through the CUDA-core pass, twice: bit-identical results."""
    n, hq, hkv = 2112, 8, 2
    q, k, v = inputs(n, hq, hkv, seed=41)
    ids = [6, 1, 3]
    vi, si = _sparse_vs_indices(np.random.default_rng(41), n, len(ids), 30, 20)
    ref, rl = orc.vs_attention(q, k, v, SCALE, vi, si, head_ids=ids)
    qc, kc, vc = cuda(q, k, v)
    vt, st = torch.from_numpy(vi).cuda(), torch.from_numpy(si).cuda()
    o1, l1 = minf.minf_vs_attention(qc, kc, vc, vt, st, scale=SCALE, head_ids=ids)
    check_attention(o1, l1, ref, rl, "VS sparse groups, head subset")
    minf.minf_dense_attention(qc, kc, vc, scale=SCALE)  # unrelated work in between
    o2, l2 = minf.minf_vs_attention(qc, kc, vc, vt, st, scale=SCALE, head_ids=ids)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.uint8), o2.view(torch.uint8)) and torch.equal(l1, l2)


def test_vs_only_sparse_groups_no_tiles(orc):
    """Lone far offsets and no verticals: rows whose keys all come from the CUDA-core
    pass (the tile kernel has nothing for them but offset 0's diagonal tile)."""
    n = 1024
    q, k, v = inputs(n, 1, 1, seed=44)
    vi = np.full((1, 4), -1, np.int32)
    si = np.array([[300, 700, 1000, -1]], np.int32)  # no offset 0: rows below 300 see no key
    ref, rl = orc.vs_attention(q, k, v, SCALE, vi, si)
    out, lse = minf.minf_vs_attention(*cuda(q, k, v), torch.from_numpy(vi).cuda(), torch.from_numpy(si).cuda(),
                                      scale=SCALE)
    check_attention(out, lse, ref, rl, "VS lone offsets only")
    assert torch.all(out[0, :300] == 0) and torch.all(torch.isneginf(lse[0, :300]))


# ----------------------------------------------------------------------------- counters and launch timing
def test_stats_detail_and_launch_timing():
    """Per-kernel counters add up to the totals and match the dense tile count; the
    launch timing names every kernel sequence of the call, once per call."""
    n, hq, hkv = 1088, 2, 1
    q, k, v = cuda(*inputs(n, hq, hkv, seed=2))
    ws = minf.workspace(256, q.device)
    minf.minf_profile_read()  # nothing pending
    minf.minf_profile_enable(True)
    try:
        minf.minf_dense_attention(q, k, v, scale=SCALE, ws=ws)
        minf.minf_dense_attention(q, k, v, scale=SCALE, ws=ws)
    finally:
        minf.minf_profile_enable(False)
    prof = minf.minf_profile_read()
    assert set(prof) == {"attn_kernel<DENSE>"} and prof["attn_kernel<DENSE>"][0] == 2
    assert prof["attn_kernel<DENSE>"][1] > 0
    assert minf.minf_profile_read() == {}  # read clears
    det = minf.minf_stats_detail(ws)
    nt = (n + 127) // 128
    dense_tiles = hq * sum((min(2 * t + 2, n // 64) + 1) // 2 for t in range(nt))
    assert det["tiles"] == det["tiles_dense"] == dense_tiles
    assert det["tiles_vs"] == det["tiles_block"] == det["tiles_ashape"] == det["diag_pairs"] == 0
    assert det["pairs"] == hq * n * (n + 1) // 2
    # Vertical-Slash with lone offsets: the CUDA-core pass's pairs are part of the total
    vi = np.full((hq, 4), -1, np.int32)
    si = np.array([[0, 300, 700, -1], [5, 500, -1, -1]], np.int32)
    wsv = minf.workspace(minf.workspace_bytes(minf.OP_VS_ATTENTION, hq, hkv, n, hq, 4, 4), q.device)
    minf.minf_vs_attention(q, k, v, torch.from_numpy(vi).cuda(), torch.from_numpy(si).cuda(), scale=SCALE, ws=wsv)
    det = minf.minf_stats_detail(wsv)
    assert det["pairs"] == sum(n - o for o in (0, 300, 700, 5, 500))
    assert 0 < det["diag_pairs"] <= det["pairs"] and det["tiles"] == det["tiles_vs"]
