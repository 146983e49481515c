"""Error bound of the FMA-pipe exp2 used for part of the softmax exponentials.

The CUDA helper ex2_fma (sparse_flashattention_b200/csrc/sfa_device.cuh) evaluates 2^x by
rounding-to-nearest range reduction and a degree-3 polynomial.  This test reads its four
coefficients from the header and replays the same float32 operations in numpy against an
exact 2^x: the relative error must stay below 2e-4, well under the 2^-9 (about 2e-3)
rounding of the bf16 probabilities the kernels feed to the P.V product."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "sparse_flashattention_b200", "csrc",
                   "sfa_device.cuh")


def _coeffs():
    text = open(HDR).read()
    return [np.float32(float(re.search(rf"kExp2C{i} = ([0-9.e+-]+)f;", text).group(1))) for i in range(4)]


def ex2_fma_replay(x):
    c0, c1, c2, c3 = _coeffs()
    x = x.astype(np.float32)
    xc = np.maximum(x, np.float32(-126.0))
    t = (xc + np.float32(12582912.0)).astype(np.float32)
    j = (t - np.float32(12582912.0)).astype(np.float32)
    f = (xc - j).astype(np.float32)
    p = np.float32(c3)
    for c in (c2, c1, c0):
        p = (p * f + c).astype(np.float32)  # the kernel fuses these into FMAs (one rounding fewer)
    ji = t.view(np.int32) - np.int32(0x4B400000)
    r = (p.view(np.int32) + (ji << 23)).view(np.float32)
    return np.where(x < -126.0, np.float32(0.0), r)


def test_relative_error_bound():
    x = np.linspace(-126.0, 8.0, 4_000_001, dtype=np.float64)
    got = ex2_fma_replay(x).astype(np.float64)
    want = np.exp2(x.astype(np.float32).astype(np.float64))
    assert (np.abs(got - want) / want).max() < 2e-4


def test_exact_zero_below_range_and_at_minus_inf():
    x = np.array([-np.inf, -1000.0, -126.5], dtype=np.float32)
    assert (ex2_fma_replay(x) == 0.0).all()


def test_integers_near_exact():
    x = np.arange(-100, 9, dtype=np.float32)
    got = ex2_fma_replay(x).astype(np.float64)
    assert (np.abs(got / np.exp2(x.astype(np.float64)) - 1.0) < 1e-4).all()
