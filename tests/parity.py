"""Comparison rules of the CUDA path against the fp64 oracle.

* Attention outputs (oracle indices fed to both sides): max |gpu - oracle|
  <= 2e-2 and mean |gpu - oracle| <= 2e-3 on bf16 inputs; the log-sum-exp
  within 1e-2 absolute (fp32 accumulation, ex2.approx).
* Index sets: with t the oracle's k-th best score, every item scoring above
  t + band is in the GPU set, every item below t - band is not, and the set
  holds exactly k items.  band = 1e-3 |t| (the relative tie band) for the
  Vertical-Slash column and diagonal sums, which are positive sums of softmax
  weights.  Block-Sparse pooled scores are raw dot products that can sit at
  or near zero, where a relative band vanishes; their band adds twice the
  worst-case fp32 error of the GPU's pooled score (`bs_score_error`).
"""
from __future__ import annotations

import numpy as np
import torch

MAX_ABS = 2e-2
MEAN_ABS = 2e-3
LSE_ABS = 1e-2
REL_BAND = 1e-3
U32 = 2.0 ** -24  # unit roundoff of fp32


def _gamma(m):
    """Higham's gamma_m = m u / (1 - m u): the relative error bound of m sequential fp32 roundings."""
    return m * U32 / (1.0 - m * U32)


# Worst-case error of one GPU pooled score s^_ij against the exact dot product of
# the exact block means, in units of sum_d a_i,d * b_j,d with a, b the block means
# of |q| and |k|.  The GPU sums the 64 bf16 rows of a block in fp32, one rounding
# per add (63; the first add is exact) and scales by 1/64 (exact), so each pooled
# value is off by at most gamma_63 a (or b); it then accumulates the 128 products
# with one fp32 FMA each, off by at most gamma_128 sum |p^q||p^k|.  With
# |p| <= a and |p^| <= (1 + gamma_63) a:
#   |s^ - s| <= [gamma_128 (1 + gamma_63)^2 + 2 gamma_63 + gamma_63^2] sum_d a_d b_d.
BS_ERR_COEF = _gamma(128) * (1 + _gamma(63)) ** 2 + 2 * _gamma(63) + _gamma(63) ** 2
# That bound is the index band's floor.  The GPU's own score arithmetic stays
# inside a smaller one.  It keeps each pooled fp32 value p^ as three bf16 parts
# h + m + l with |p^ - h - m - l| <= 2^-24 |p^| (three roundings to 8 significant
# bits; each residual is exact in fp32).  Of the nine part products it forms the
# six down to 2^-16 relative size, dropping (with the residuals) at most
# (4 + 2^-6) 2^-24 |p^q||p^k| per term; bf16 products are exact in fp32.  The
# tensor core's fp32 accumulation is modelled as: one K = 16 step returns
# c + (its 16 products) within 2^-22 (|c| + sum |p|), i.e. within two fp32 ulps
# (truncation and a lost guard bit).  The five small part products, together
# at most BS_TC_SMALL of S = sum |p^q||p^k|, take the first 40 steps (each step
# with |c| + sum |p| <= 2 BS_TC_SMALL S); the eight hi.hi steps follow, each
# with |c| + sum |p| <= (BS_TC_SMALL + (1 + 2^-8)^2) S.
BS_TC_SMALL = (2 * 2.0 ** -8 + 3 * 2.0 ** -16) * (1 + 2.0 ** -8) ** 2
BS_TC_STEP = 2.0 ** -22
# the accumulation alone, per unit of S (the pooled values' sum_d |p^q||p^k|)
BS_TC_ACC_COEF = BS_TC_STEP * (40 * 2 * BS_TC_SMALL + 8 * (BS_TC_SMALL + (1 + 2.0 ** -8) ** 2))
BS_TC_ERR_COEF = ((4 + 2.0 ** -6) * U32 + BS_TC_ACC_COEF) * (1 + _gamma(63)) ** 2 \
    + 2 * _gamma(63) + _gamma(63) ** 2


def bs_score_error(q, k, block=64, coef=BS_ERR_COEF):
    """Per (q-head, query block i): twice the largest worst-case error (coef per
    unit of sum_d a b; the fp32 dot-product bound by default) of the pooled
    scores s_ij over the candidates j < i (zero for i = 0).

    With that error at most E on every candidate of a row, an item whose exact
    score exceeds the k-th best exact score t by more than 2E outranks, on the GPU,
    every item that does not score above t exactly -- at most k - 1 others -- so it
    must be selected; symmetrically below t - 2E.  q: [hq][n][128], k: [hkv][n][128]
    (bf16 tensors or arrays; GQA groups contiguous)."""
    qa = np.abs(to_np(q))
    ka = np.abs(to_np(k))
    hq, n, d = qa.shape
    hkv = ka.shape[0]
    nb = n // block
    aq = qa.reshape(hq, nb, block, d).mean(axis=2)
    ak = ka.reshape(hkv, nb, block, d).mean(axis=2)
    out = np.zeros((hq, nb))
    below = np.tril(np.ones((nb, nb), bool), -1)
    for h in range(hq):
        m = aq[h] @ ak[h // (hq // hkv)].T
        out[h] = 2.0 * coef * np.where(below, m, 0.0).max(axis=1)
    return out


def bs_score_bound(q, k, block=64, coef=BS_TC_ERR_COEF):
    """Per (q-head, i, j): coef * sum_d a_i,d b_j,d, the worst-case error of one
    pooled score (a, b the block means of |q| and |k|)."""
    qa = np.abs(to_np(q))
    ka = np.abs(to_np(k))
    hq, n, d = qa.shape
    hkv = ka.shape[0]
    nb = n // block
    aq = qa.reshape(hq, nb, block, d).mean(axis=2)
    ak = ka.reshape(hkv, nb, block, d).mean(axis=2)
    g = hq // hkv
    return coef * np.stack([aq[h] @ ak[h // g].T for h in range(hq)])


def pooled_fp32_model(x):
    """Block means as the GPU forms them: sequential fp32 sums of 64 rows, times 1/64."""
    x = x.float().numpy()
    h, n, d = x.shape
    xb = x.reshape(h, n // 64, 64, d)
    acc = np.zeros((h, n // 64, d), np.float32)
    for r in range(64):
        acc = (acc + xb[:, :, r, :]).astype(np.float32)
    return (acc * np.float32(1.0 / 64)).astype(np.float32)


def _bf16_parts(p):
    """hi, mid, lo bf16 parts of fp32 values (round to nearest even at each step)."""
    parts, r = [], torch.from_numpy(p)
    for _ in range(3):
        b = r.to(torch.bfloat16).float()
        parts.append(b.numpy().astype(np.float64))
        r = (r - b).float()  # exact in fp32
    return parts


def _trunc_f32(x):
    """fp64 -> fp32 rounded toward zero."""
    f = x.astype(np.float32)
    over = np.abs(f.astype(np.float64)) > np.abs(x)
    f[over] = np.nextafter(f[over], np.float32(0))
    return f


def tc_pooled_scores_model(q, k, products=("hl", "mm", "hm", "lh", "mh", "hh")):
    """Emulation of the tensor-core score arithmetic: split parts, the listed
    part products (Q part, K part) in order, each 128-deep product as eight
    K = 16 steps whose 16 exact products and the accumulator are summed exactly
    and truncated to fp32 (a pessimistic accumulation)."""
    qp, kp = pooled_fp32_model(q), pooled_fp32_model(k)
    qs, ks = _bf16_parts(qp), _bf16_parts(kp)
    idx = {"h": 0, "m": 1, "l": 2}
    g = q.shape[0] // k.shape[0]
    out = []
    for h in range(q.shape[0]):
        c = np.zeros((qp.shape[1], kp.shape[1]), np.float32)
        for pr in products:
            a, b = qs[idx[pr[0]]][h], ks[idx[pr[1]]][h // g]
            for s0 in range(0, 128, 16):
                c = _trunc_f32(c.astype(np.float64) + a[:, s0:s0 + 16] @ b[:, s0:s0 + 16].T)
        out.append(c.astype(np.float64))
    return np.stack(out)


def to_np(t):
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy().astype(np.float64)
    return np.asarray(t, dtype=np.float64)


MASS_TOL = 2e-5  # fp32 column / diagonal sums against the fp64 ones, as a share of the row mass


def check_attention(gpu_out, gpu_lse, ref_out, ref_lse, what=""):
    g = to_np(gpu_out)
    r = np.asarray(ref_out, np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU output"
    err = np.abs(g - r)
    assert err.max() <= MAX_ABS, f"{what}: max abs err {err.max():.3e}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean abs err {err.mean():.3e}"
    if gpu_lse is not None and ref_lse is not None:
        gl = to_np(gpu_lse)
        rl = np.asarray(ref_lse, np.float64)
        fin = np.isfinite(rl)
        assert np.array_equal(np.isfinite(gl), fin), f"{what}: lse finiteness differs"
        if fin.any():
            le = np.abs(gl[fin] - rl[fin]).max()
            assert le <= LSE_ABS, f"{what}: lse max abs err {le:.3e}"
    return float(err.max()), float(err.mean())


def check_topk_band(gpu_idx, scores, k, what="", abs_band=0.0):
    """gpu_idx: 1-D indices (-1 padded); scores: oracle fp64 scores of every candidate.
    abs_band: added to the relative band (Block-Sparse rows: `bs_score_error`)."""
    scores = np.asarray(scores, np.float64)
    kk = min(k, len(scores))
    got = [int(x) for x in np.asarray(gpu_idx).ravel() if x >= 0]
    assert len(got) == kk, f"{what}: {len(got)} indices, expected {kk}"
    assert len(set(got)) == kk, f"{what}: duplicate indices"
    assert got == sorted(got), f"{what}: not ascending"
    if kk == 0:
        return 0
    order = np.sort(scores)[::-1]
    t = order[kk - 1]
    band = REL_BAND * abs(t) + abs_band if np.isfinite(t) else 0.0
    gs = set(got)
    must = np.nonzero(scores > t + band)[0]
    never = np.nonzero(scores < t - band)[0]
    miss = [int(i) for i in must if int(i) not in gs]
    extra = [int(i) for i in never if int(i) in gs]
    assert not miss, f"{what}: missing clear winners {miss[:10]}"
    assert not extra, f"{what}: took clear losers {extra[:10]}"
    return len(got) - len(set(must.tolist()) & gs)  # picks decided inside the band


def check_topp(gpu_idx, gpu_cnt, scores, p, cap, forced0=False, what=""):
    """Top-p parity.  gpu_idx: 1-D indices (-1 padded); gpu_cnt: the GPU's count;
    scores: the oracle's fp64 scores of every candidate (for slashes the true
    mass of offset 0, which is forced when forced0).

    The GPU set must be the top-c set of the oracle's order for its own count c
    (tie band), and c must be the shortest cover of p of the mass under the
    oracle's scores, within the fp32 rounding of the scores (MASS_TOL of the total).
    """
    scores = np.asarray(scores, np.float64)
    idx = np.asarray(gpu_idx).ravel()
    c = int(gpu_cnt)
    assert 1 <= c <= cap, f"{what}: count {c} outside [1, {cap}]"
    got = idx[:c]
    assert np.all(got >= 0) and np.all(idx[c:] == -1), f"{what}: count and padding disagree"
    ranked = scores.copy()
    if forced0:
        ranked[0] = np.inf
        assert 0 in set(got.tolist()), f"{what}: forced offset 0 missing"
    check_topk_band(idx, ranked, c, what)
    total = scores.sum()
    mass = scores[got].sum()
    tol = MASS_TOL * total
    if c < cap:
        assert mass >= p * total - tol, f"{what}: mass {mass:.6g} below p*total {p * total:.6g}"
    rest = np.sort(scores[got[got != 0]] if forced0 else scores[got])
    if len(rest):
        assert mass - rest[0] < p * total + tol, f"{what}: not the shortest cover"
