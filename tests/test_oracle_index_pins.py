"""Pins for the decode index producer oracle (oracle.index_topk, oracle.e4m3_round), independent of
its code: the FP8 E4M3 rounding against PyTorch's float8_e4m3fn conversion and the format's defining
values, exact scores against rational arithmetic, and top-k sets whose answer is known by
construction (ordered keys, ties, short sequences, forced recent positions, paging invariance)."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import sfa_workloads as W

torch = pytest.importorskip("torch")


def test_e4m3_rounding_matches_torch_and_saturates():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1.0, 30.0, 150.0)])
    x = x[np.abs(x) <= 448.0]
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(oracle.e4m3_round(x), want)
    # the format's defining values: largest finite 448, smallest subnormal 2^-9, spacing 2^(e-3)
    assert oracle.e4m3_round([448.0, 1e6, -1e6, 2.0 ** -9, 2.0 ** -10 + 1e-9, 1.0 + 2 ** -4]).tolist() == \
        [448.0, 448.0, -448.0, 2.0 ** -9, 2.0 ** -9, 1.0]


def _paged(rng, L, Hkv, d, page, values=None):
    npg = -(-L // page)
    perm = rng.permutation(npg + 3).astype(np.int32)[:npg]
    kc = np.zeros((npg + 3, page, Hkv, d))
    logical = rng.standard_normal((L, Hkv, d)) if values is None else values
    for j in range(L):
        kc[perm[j // page], j % page] = logical[j]
    return kc, perm[None, :], logical


def test_scores_are_exact():
    rng = np.random.default_rng(2)
    B, Hq, Hkv, d, L, page = 1, 4, 2, 16, 37, 8
    q = rng.standard_normal((B, Hq, d)) * 3
    kc, bt, logical = _paged(rng, L, Hkv, d, page)
    _, scores, _ = oracle.index_topk(q, kc, bt, np.array([L]), Hkv, 8)
    qf, kf = oracle.e4m3_round(q), oracle.e4m3_round(logical)
    for hk in range(Hkv):
        for j in range(L):
            exact = sum(Fraction(qf[0, hk * 2 + g, c]) * Fraction(kf[j, hk, c]) for g in range(2) for c in range(d))
            assert Fraction(scores[0][hk, j]) == exact


def test_ordered_keys_ties_short_and_local():
    rng = np.random.default_rng(3)
    Hkv, d, page, L = 1, 8, 4, 20
    vals = oracle.e4m3_round(np.linspace(0.1, 3.0, L))       # increasing, distinct in E4M3
    order = rng.permutation(L)
    logical = np.repeat(vals[order][:, None, None], d, axis=2)  # key j: all components vals[order[j]]
    kc, bt, _ = _paged(rng, L, Hkv, d, page, logical)
    q = np.ones((1, 2, d))
    sel, _, _ = oracle.index_topk(q, kc, bt, np.array([L]), Hkv, 5)
    want = np.sort(np.argsort(-vals[order])[:5])
    np.testing.assert_array_equal(sel[0, 0], want)
    # the last 3 positions forced, then the 2 best of the others
    sel, _, _ = oracle.index_topk(q, kc, bt, np.array([L]), Hkv, 5, n_local=3)
    best = [j for j in np.argsort(-vals[order], kind="stable") if j < L - 3][:2]
    np.testing.assert_array_equal(sel[0, 0], np.sort(np.r_[np.arange(L - 3, L), best]))
    # all keys equal: a tie everywhere goes to the lowest positions
    kc2, bt2, _ = _paged(rng, L, Hkv, d, page, np.ones((L, Hkv, d)))
    sel, _, _ = oracle.index_topk(q, kc2, bt2, np.array([L]), Hkv, 6)
    np.testing.assert_array_equal(sel[0, 0], np.arange(6))
    # fewer positions than topk: all of them, then -1
    sel, _, _ = oracle.index_topk(q, kc2, bt2, np.array([4]), Hkv, 6)
    np.testing.assert_array_equal(sel[0, 0], [0, 1, 2, 3, -1, -1])


def test_paging_invariance_on_the_decode_workload():
    c = W.make_decode(7, 3, 8, 2, 64, 16, 50, 300, 32, 4)
    sel, _, _ = oracle.index_topk(c.q, c.k_cache, c.block_table, c.cache_seqlens, c.Hkv, 32, n_local=4)
    # the same logical cache laid out with pages in a different order
    rng = np.random.default_rng(11)
    perm = rng.permutation(c.num_pages)
    inv = np.argsort(perm)
    kc2 = c.k_cache[perm]
    bt2 = np.where(c.block_table >= 0, inv[np.maximum(c.block_table, 0)], -1).astype(np.int32)
    sel2, _, _ = oracle.index_topk(c.q, kc2, bt2, c.cache_seqlens, c.Hkv, 32, n_local=4)
    np.testing.assert_array_equal(sel, sel2)
    for b in range(c.B):
        L = int(c.cache_seqlens[b])
        assert set(range(L - 4, L)) <= set(sel[b, 0].tolist())


def test_invalid_pages_are_no_candidates():
    """A position whose page id is outside the cache is never selected and is counted."""
    rng = np.random.default_rng(4)
    L, page = 24, 4
    kc, bt, _ = _paged(rng, L, 1, 8, page, np.full((L, 1, 8), 2.0))
    bt = bt.copy()
    bt[0, 1] = kc.shape[0] + 3   # positions 4..7
    q = np.ones((1, 1, 8))
    sel, _, bad = oracle.index_topk(q, kc, bt, np.array([L]), 1, 10, n_local=2)
    assert bad == 4
    # all scores tie: the lowest valid positions, then the two forced last ones
    np.testing.assert_array_equal(sel[0, 0], [0, 1, 2, 3, 8, 9, 10, 11, 22, 23])
