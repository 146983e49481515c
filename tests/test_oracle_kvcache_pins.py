"""Pins of the non-paged cache oracles (oracle.decode_kvcache, oracle.kv_append_kvcache), on the CPU.

cache_batch_idx (flash_attn_with_kvcache docstrings, flash-attention-npu page) picks the batch entry of
a non-paged (batch_cache, seqlen_cache, Hkv, d) cache for each sequence.  The Python oracles index it
directly; they are pinned against the C paged decode oracle and the paged append oracle on the same
rows repacked into randomly placed pages of another size, against closed forms, and against a
hand-worked append."""
import numpy as np
import pytest

import oracle
import sfa_workloads as W


@pytest.mark.parametrize("page,wl", [(16, -1), (100, -1), (64, 50)])
def test_decode_kvcache_equals_paged_oracle(page, wl):
    c = W.make_decode_kvcache(31 + page, 4, 7, 900, 8, 2, 64, 1, 900, 96, 8)
    c.wl = wl
    out, lse, bad = oracle.decode_kvcache(c.q, c.k_cache, c.v_cache, c.cache_seqlens, c.sel, c.cache_batch_idx,
                                          c.Hkv, c.softmax_scale, wl=wl)
    ro, rl, rbad = oracle.decode(W.kvcache_as_paged(c, page, seed=page))
    assert bad == 0 and int(rbad[0]) == 0 and int(rbad[1]) == 0
    np.testing.assert_allclose(out, ro, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=1e-12, atol=1e-12)


def test_decode_kvcache_closed_forms():
    c = W.make_decode_kvcache(5, 3, 4, 64, 4, 2, 64, 40, 64, 8, 1)
    sel = np.full_like(c.sel, -1)
    sel[:, :, 0] = 7                           # one kept position: out = v row, lse = scale * q . k
    sel[2, :, 1:4] = 7                         # duplicates count once
    idx = c.cache_batch_idx.copy()
    idx[1] = 99                                # outside the cache: nothing kept
    out, lse, bad = oracle.decode_kvcache(c.q, c.k_cache, c.v_cache, c.cache_seqlens, sel, idx, c.Hkv,
                                          c.softmax_scale)
    f = lambda a: (np.asarray(a).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for b in (0, 2):
        for h in range(c.Hq):
            hk = h // (c.Hq // c.Hkv)
            np.testing.assert_array_equal(out[b, h], f(c.v_cache[idx[b], 7, hk]))
            want = c.softmax_scale * float(f(c.q[b, h]) @ f(c.k_cache[idx[b], 7, hk]))
            assert lse[b, h] == pytest.approx(want, rel=1e-14, abs=1e-14)
    assert np.all(out[1] == 0) and np.all(np.isneginf(lse[1]))
    assert bad == 0


def test_decode_kvcache_batch_idx_moves_the_rows():
    """Swapping two cache entries and their indices leaves the result unchanged."""
    c = W.make_decode_kvcache(9, 3, 5, 300, 8, 4, 64, 50, 300, 40, 4)
    a = oracle.decode_kvcache(c.q, c.k_cache, c.v_cache, c.cache_seqlens, c.sel, c.cache_batch_idx, c.Hkv,
                              c.softmax_scale)
    i, j = int(c.cache_batch_idx[0]), int(c.cache_batch_idx[1])
    kc, vc = c.k_cache.copy(), c.v_cache.copy()
    kc[[i, j]], vc[[i, j]] = kc[[j, i]], vc[[j, i]]
    idx = c.cache_batch_idx.copy()
    idx[0], idx[1] = j, i
    b = oracle.decode_kvcache(c.q, kc, vc, c.cache_seqlens, c.sel, idx, c.Hkv, c.softmax_scale)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_kv_append_kvcache_hand_worked():
    """Cache of 3 entries x 4 rows, one kv head, d 1: sequence 0 on entry 2 at length 1, sequence 1 on
    entry 0 at length 3; two new rows each.  Sequence 1's second row (position 4) is past the cache."""
    kc = np.zeros((3, 4, 1, 1), np.uint16)
    vc = np.zeros((3, 4, 1, 1), np.uint16)
    kn = np.array([[1, 2], [3, 4]], np.uint16).reshape(2, 2, 1, 1)
    vn = kn + 10
    k2, v2, bad = oracle.kv_append_kvcache(kc, vc, np.array([2, 0], np.int32), np.array([1, 3], np.int32), kn, vn)
    want = np.zeros((3, 4), np.uint16)
    want[2, 1], want[2, 2], want[0, 3] = 1, 2, 3
    np.testing.assert_array_equal(k2[..., 0, 0], want)
    np.testing.assert_array_equal(v2[..., 0, 0], np.where(want > 0, want + 10, 0))
    assert bad == 1
    assert np.all(kc == 0)  # inputs untouched


def test_kv_append_kvcache_equals_paged_append():
    c = W.make_decode_kvcache(12, 3, 5, 200, 4, 2, 16, 10, 150, 8, 2)
    rng = np.random.default_rng(3)
    kn = rng.integers(0, 1 << 15, size=(3, 60, 2, 16)).astype(np.uint16)
    vn = rng.integers(0, 1 << 15, size=(3, 60, 2, 16)).astype(np.uint16)
    k2, v2, bad = oracle.kv_append_kvcache(c.k_cache, c.v_cache, c.cache_batch_idx, c.cache_seqlens, kn, vn)
    page = 32
    pc = W.kvcache_as_paged(c, page, seed=4)
    kp, vp, pbad = oracle.kv_append(pc.k_cache, pc.v_cache, pc.block_table, c.cache_seqlens, kn, vn)
    # positions 200.. of a sequence lie past the non-paged cache but inside its last page's padding (224
    # rows of pages): the paged append writes them, the non-paged one cannot; compare the rows both hold
    assert bad == sum(max(0, int(L) + 60 - 200) for L in c.cache_seqlens)
    for b in range(c.B):
        for pos in range(200):
            pg, r = pc.block_table[b, pos // page], pos % page
            np.testing.assert_array_equal(k2[c.cache_batch_idx[b], pos], kp[pg, r])
            np.testing.assert_array_equal(v2[c.cache_batch_idx[b], pos], vp[pg, r])
