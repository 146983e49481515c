"""The arithmetic the index scoring kernel relies on, checked on the CPU against exact rationals
(the kernel itself is checked bit for bit against oracle.index_topk in test_gpu_index_topk.py).

1. An E4M3 code's exponent field E and mantissa field M, placed in the low bits of the fp64 exponent
   and the top of its fraction (sign in the sign bit), read as the code's value times 2^-1016: normals
   as (1 + M/8) 2^(E-1023), the format's subnormals as fp64 subnormals (M/8) 2^-1022.
2. With key values so scaled, products with the group's summed query values and their row sums are
   exact in fp64 up to G = 1024 query heads per group, whatever the order of the sum, so a power-of-two
   rescale of the result is the exact score."""
import itertools
from fractions import Fraction

import numpy as np

import oracle

SCALE = 2.0 ** 1016


def field_placed(codes):
    c = np.asarray(codes, np.uint64)
    hi = ((c & np.uint64(0x7F)) << np.uint64(17)) | ((c & np.uint64(0x80)) << np.uint64(24))
    return (hi << np.uint64(32)).view(np.float64)


def test_field_placement_is_the_scaled_value_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    want = oracle.e4m3_decode(codes)
    got = field_placed(codes)
    finite = ~np.isnan(want)
    assert finite.sum() == 254
    # exact: a power-of-two rescale of an fp64 value (normal or subnormal) that lands in range
    np.testing.assert_array_equal(got[finite] * SCALE, want[finite])
    for c, v in zip(codes[finite], got[finite]):
        assert Fraction(float(v)) * Fraction(2) ** 1016 == Fraction(float(oracle.e4m3_decode(np.uint8(c))))
    # subnormal codes (E = 0) really are fp64 subnormals, and the NaN codes read as +-480
    sub = (codes & 0x78) == 0
    assert np.all(np.abs(got[sub & (codes & 7 != 0)]) < np.finfo(np.float64).tiny)
    np.testing.assert_array_equal(got[~finite] * SCALE, [480.0, -480.0])


def _exact_row_sum(k_codes, qsum):
    return sum(Fraction(float(oracle.e4m3_decode(np.uint8(c)))) * Fraction(float(q)) for c, q in zip(k_codes, qsum))


def _scaled_fp64_sum(k_codes, qsum, order):
    acc = 0.0
    ks = field_placed(k_codes)
    for i in order:
        acc = float(np.float64(ks[i]) * np.float64(qsum[i]) + np.float64(acc))
    return acc


def test_scaled_sums_exact_at_the_group_bound():
    rng = np.random.default_rng(7)
    d, G = 128, 1024
    finite_codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    top = np.uint8(0x7E)          # 448
    tiny = np.uint8(0x01)         # 2^-9
    rows = []
    # widest span: 127 terms at 448 * (G * 448), one term at 2^-9 * 2^-9
    q_big = np.full(d, G * 448.0)
    q_big[-1] = 2.0 ** -9
    k_big = np.full(d, top)
    k_big[-1] = tiny
    rows.append((k_big, q_big))
    # mixed signs and magnitudes: query sums of G random codes of the format
    for _ in range(6):
        qcodes = rng.choice(finite_codes, size=(G, d))
        qsum = oracle.e4m3_decode(qcodes).sum(axis=0)  # exact: multiples of 2^-9 below 2^19
        rows.append((rng.choice(finite_codes, size=d), qsum))
    for k_codes, qsum in rows:
        exact = _exact_row_sum(k_codes, qsum)
        orders = [range(d), range(d - 1, -1, -1)] + [rng.permutation(d) for _ in range(3)]
        for order in orders:
            s = _scaled_fp64_sum(k_codes, qsum, order)
            assert Fraction(s) * Fraction(2) ** 1016 == exact


def test_scaled_keys_keep_order_and_ties():
    """A power-of-two rescale keeps every comparison: keys of scaled scores order and tie like the
    scores (checked on all pairs of a small set that includes ties, signs and zero)."""
    vals = [0.0, -0.0, 2.0 ** -18, -2.0 ** -18, 1.5, 1.5, -448.0 * 448, 3.0 * 2 ** -9]
    for a, b in itertools.product(vals, repeat=2):
        sa, sb = a / SCALE, b / SCALE
        assert (sa < sb) == (a < b) and (sa == sb) == (a == b)
