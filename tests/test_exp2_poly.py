"""The FMA-pipe exponential of the softmax: its coefficients come from the
committed Remez derivation, and its error stays within the derived bound.

Method: Cody-Waite range reduction for base 2 (x = n + f, n = rint(x),
f in [-1/2, 1/2]) and a degree-3 minimax polynomial for 2^f.
"""
import os
import re
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "dynamic_sparse_attention_est_b200", "csrc")
sys.path.insert(0, CSRC)
import exp2_poly  # noqa: E402

BOUND = 1e-4  # relative; the derivation reports 7.5e-5 for fp32 Horner evaluation


def kernel_coefficients():
    src = open(os.path.join(CSRC, "attention.cu")).read()
    body = src[src.index("exp2_poly_pair(float &a"):]
    body = body[:body.index("f32x2_unpack(t, t0, t1)")]
    return [float(x) for x in re.findall(r"f32x2_splat\(([-0-9.e+]+)f\)", body)[1:]]


def test_kernel_uses_the_derived_coefficients():
    c, rel = exp2_poly.coefficients(3)
    k = kernel_coefficients()  # Horner order in the kernel: c3, c2, c1, c0
    assert len(k) == 4
    assert np.allclose(k[::-1], c.astype(np.float64), rtol=1e-7, atol=0), (k, c)
    assert rel < BOUND


def _poly_reference(x):
    """The kernel's arithmetic restated in numpy fp32 (magic-number rounding, Horner, exponent bits)."""
    c = exp2_poly.coefficients(3)[0]
    x = np.maximum(x.astype(np.float32), np.float32(-127.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic)).astype(np.float32)
    p = np.float32(c[3])
    for cj in (c[2], c[1], c[0]):
        p = (p * f + np.float32(cj)).astype(np.float32)
    scale_bits = (t.view(np.uint32).astype(np.uint64) * (1 << 23) + 0x3F800000) & 0xFFFFFFFF
    return (p * scale_bits.astype(np.uint32).view(np.float32)).astype(np.float32)


def test_numpy_restatement_within_bound():
    x = np.concatenate([np.linspace(-126, 8, 400001), np.linspace(-1, 1, 100001)]).astype(np.float32)
    y = _poly_reference(x)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < BOUND
    z = _poly_reference(np.array([-127.0, -300.0, -np.inf], np.float32))
    assert np.all(z == 0.0)


@pytest.mark.gpu
def test_device_polynomial_within_bound():
    from dynamic_sparse_attention_est_b200 import minf

    x = torch.cat([torch.linspace(-126, 8, 400001), torch.linspace(-1, 1, 100001),
                   torch.tensor([-127.0, -500.0, float("-inf")])]).cuda()
    y_poly, y_hw = minf.minf_selftest_exp2(x)
    torch.cuda.synchronize()
    xs = x[:-3].double().cpu().numpy()
    ref = np.exp2(xs)
    yp = y_poly[:-3].double().cpu().numpy()
    yh = y_hw[:-3].double().cpu().numpy()
    assert np.max(np.abs(yp - ref) / ref) < BOUND
    assert np.max(np.abs(yh - ref) / ref) < 1e-5  # the hardware approximation, for comparison
    assert torch.all(y_poly[-3:] == 0)
    # the device result equals the numpy restatement of the same arithmetic up to fp32 rounding order
    assert np.max(np.abs(yp - _poly_reference(x[:-3].cpu().numpy())) / ref) < 1e-6
