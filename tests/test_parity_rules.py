"""The comparison rules themselves, on the CPU: the index tie band, the
Block-Sparse fp32 error floor that widens it, and the error model of the
tensor-core pooled scores.
"""
import numpy as np
import torch

from dynamic_sparse_attention_est_b200 import synth
from parity import (BS_ERR_COEF, BS_TC_ERR_COEF, bs_score_bound, bs_score_error,
                    check_topk_band, tc_pooled_scores_model)

import pytest


def _fp32_pooled_scores(q, k):
    """fp32 emulation of an fp32 pooled-score dot product (the arithmetic the
    index band's floor is derived for): sequential fp32 sums of the 64 rows of a
    block, times 1/64, then 128 sequential fp32 FMAs (each FMA emulated as an
    exact fp64 product-sum rounded once to fp32)."""
    q = q.float().numpy()
    k = k.float().numpy()
    hq, n, d = q.shape
    nb = n // 64

    def pool(x):
        acc = np.zeros((x.shape[0], nb, d), np.float32)
        xb = x.reshape(x.shape[0], nb, 64, d)
        for r in range(64):
            acc = (acc + xb[:, :, r, :]).astype(np.float32)
        return (acc * np.float32(1.0 / 64)).astype(np.float32)

    qp, kp = pool(q), pool(k)
    g = hq // k.shape[0]
    out = np.zeros((hq, nb, nb), np.float32)
    for h in range(hq):
        a = qp[h].astype(np.float64)
        b = kp[h // g].astype(np.float64)
        acc = np.zeros((nb, nb), np.float32)
        for dd in range(d):
            acc = (np.outer(a[:, dd], b[:, dd]) + acc.astype(np.float64)).astype(np.float32)
        out[h] = acc
    return out


@pytest.mark.parametrize("structure", ["clustered", "plain"])
def test_bs_error_floor_bounds_fp32_pooled_scores(structure):
    w = synth.Workload("t", "block", 2, 1, 64 * 48, structure)
    x = synth.generate(w, seed=3)
    q, k = x["q"], x["k"]
    nb = q.shape[1] // 64
    exact = np.einsum("hid,hjd->hij", q.double().numpy().reshape(2, nb, 64, 128).mean(2),
                      k.double().numpy().reshape(1, nb, 64, 128).mean(2).repeat(2, 0))
    got = _fp32_pooled_scores(q, k).astype(np.float64)
    eb = bs_score_error(q, k)  # twice the per-row bound
    err = np.abs(got - exact)
    for h in range(2):
        for i in range(1, nb):
            assert err[h, i, :i].max() <= eb[h, i] / 2, (h, i)
    # the bound is a few e-5 of the score scale, far above the observed rounding
    assert 0 < BS_ERR_COEF < 2e-5
    assert err[:, 1:, :].max() < eb[:, 1:].max()


def test_band_is_relative_without_a_floor():
    # scores near 1e-4, as the Vertical-Slash sums are at 1M keys
    rng = np.random.default_rng(0)
    s = 1e-4 * (1 + rng.random(200))
    order = np.argsort(-s, kind="stable")
    k = 50
    top = np.sort(order[:k])
    check_topk_band(top, s, k, "exact top-k")
    t = s[order[k - 1]]
    # swap the k-th item for the best loser: allowed only if it sits within 1e-3 |t|
    loser = order[k]
    swapped = np.sort(np.append(order[:k - 1], loser))
    if s[loser] < t * (1 - 1e-3):
        with pytest.raises(AssertionError):
            check_topk_band(swapped, s, k, "swap outside the band")
    # a score 2e-7 below t (1e-3 relative of 1e-4 is 1e-7) is outside the band
    s2 = s.copy()
    s2[loser] = t - 2e-7
    swapped = np.sort(np.append(order[:k - 1], loser))
    with pytest.raises(AssertionError):
        check_topk_band(swapped, s2, k, "2e-3 relative below t")
    # 0.5e-3 relative below t is inside the band
    s2[loser] = t * (1 - 5e-4)
    check_topk_band(swapped, s2, k, "inside the band")


def test_band_floor_admits_near_zero_ties():
    s = np.array([0.5, 0.4, 1e-9, -1e-9, -0.3])
    # t = 1e-9: the relative band alone (1e-12) would reject taking item 3
    with pytest.raises(AssertionError):
        check_topk_band(np.array([0, 1, 3]), s, 3, "no floor")
    check_topk_band(np.array([0, 1, 3]), s, 3, "with floor", abs_band=1e-6)
    with pytest.raises(AssertionError):
        check_topk_band(np.array([0, 1, 4]), s, 3, "clear loser", abs_band=1e-6)


@pytest.mark.parametrize("structure", ["clustered", "plain"])
def test_tensor_core_score_model_within_its_bound(structure):
    w = synth.Workload("t", "block", 2, 1, 64 * 40, structure)
    x = synth.generate(w, seed=5)
    q, k = x["q"], x["k"]
    nb = q.shape[1] // 64
    exact = np.einsum("hid,hjd->hij", q.double().numpy().reshape(2, nb, 64, 128).mean(2),
                      k.double().numpy().reshape(1, nb, 64, 128).mean(2).repeat(2, 0))
    bound = bs_score_bound(q, k)
    assert BS_TC_ERR_COEF < BS_ERR_COEF  # inside the index band's floor
    err = np.abs(tc_pooled_scores_model(q, k) - exact)
    assert np.all(err <= bound)
    # dropping a part product the kernel forms (hi.mid) breaks the bound: the
    # model is tight enough to see a missing term
    err_drop = np.abs(tc_pooled_scores_model(q, k, ("hl", "mm", "lh", "mh", "hh")) - exact)
    assert np.any(err_drop > bound)
