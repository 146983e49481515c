"""Pins of the fp64 oracle against facts fixed by the pages and by the mathematics.

Each test names what it pins.  None of them compares the oracle with a retyped copy of
itself: they use printed examples (tests/golden), closed forms, invariants, and a dense
brute-force reference that knows nothing of block selection.
"""
import os

import numpy as np
import pytest

import sfa_workloads as W
from tests.dense_ref import dense_attention, dense_decode, mask_matrix

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BF16_ONE = 0x3F80


def _read_masks():
    cases, cur = [], None
    for line in open(os.path.join(GOLDEN, "causal_mask_examples.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("case"):
            kv = dict(p.split("=") for p in line.split()[1:])
            cur = (int(kv["sq"]), int(kv["sk"]), [])
            cases.append(cur)
        else:
            cur[2].append([int(c) for c in line])
    return [(sq, sk, np.array(rows, dtype=np.int64)) for sq, sk, rows in cases]


def _case(q, k, v, cu_q, cu_k, sel, Hq, Hkv, d, bs, causal=1, wl=-1, wr=-1, scale=0.0):
    return W.PrefillCase("t", np.asarray(q, np.uint16), np.asarray(k, np.uint16), np.asarray(v, np.uint16),
                         np.asarray(cu_q, np.int32), np.asarray(cu_k, np.int32), np.asarray(sel, np.int32),
                         Hq, Hkv, d, bs, sel.shape[-1], causal, wl, wr, scale)


def _all_blocks_sel(total_q, Hkv, nblk):
    return np.broadcast_to(np.arange(nblk, dtype=np.int32), (total_q, Hkv, nblk)).copy()


def _rand_bf16(rng, shape):
    return W.f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))


@pytest.mark.parametrize("sq,sk,expect", _read_masks())
def test_causal_mask_examples(oracle_lib, sq, sk, expect):
    """Printed bottom-right causal masks: one-hot values make out[i, j] = p_ij, so the kept
    set of each row is read off the attention output itself (and off the index oracle)."""
    d = 8
    rng = np.random.default_rng(0)
    q = _rand_bf16(rng, (sq, 1, d))
    k = _rand_bf16(rng, (sk, 1, d))
    v = np.zeros((sk, 1, d), np.uint16)
    for j in range(sk):
        v[j, 0, j] = BF16_ONE
    sel = _all_blocks_sel(sq, 1, sk)  # block size 1, every block selected
    c = _case(q, k, v, [0, sq], [0, sk], sel, 1, 1, d, 1, causal=1)
    out, lse, bad = oracle_lib.fwd(c)
    assert bad == 0
    got = (out[:, 0, :sk] > 0).astype(np.int64)
    np.testing.assert_array_equal(got, expect)
    sel_c, cnt, _ = oracle_lib.fwd_index(c)
    kept = np.zeros((sq, sk), np.int64)
    for i in range(sq):
        kept[i, sel_c[i, 0, :cnt[i, 0]]] = 1
    np.testing.assert_array_equal(kept, expect)
    for i in range(sq):
        if expect[i].sum() == 0:  # all-masked row: output exactly 0, lse -inf
            assert np.all(out[i] == 0.0) and lse[0, i] == -np.inf
        else:
            assert abs(out[i, 0, :sk].sum() - 1.0) < 1e-12


def test_gqa_mapping(oracle_lib):
    """6 query heads on 2 kv heads: constant V per kv head reveals which kv head each q head reads."""
    lines = [l for l in open(os.path.join(GOLDEN, "gqa_mapping.txt")) if l.strip() and not l.startswith("#")]
    Hq, Hkv = [int(x.split("=")[1]) for x in lines[0].split()]
    mapping = {int(a): int(b) for a, b in (l.split() for l in lines[1:])}
    d, n = 16, 40
    rng = np.random.default_rng(1)
    q = _rand_bf16(rng, (n, Hq, d))
    k = _rand_bf16(rng, (n, Hkv, d))
    vals = [W.f32_to_bf16_bits(np.float32(x)) for x in (3.0, -5.0)]
    v = np.zeros((n, Hkv, d), np.uint16)
    for hk in range(Hkv):
        v[:, hk, :] = vals[hk]
    c = _case(q, k, v, [0, n], [0, n], _all_blocks_sel(n, Hkv, 5), Hq, Hkv, d, 8)
    out, _, _ = oracle_lib.fwd(c)
    for h in range(Hq):
        want = 3.0 if mapping[h] == 0 else -5.0
        assert np.allclose(out[:, h, :], want, atol=1e-12), h


@pytest.mark.parametrize("causal,wl,wr,sq,sk,bs", [(1, -1, -1, 150, 150, 16), (1, 40, 0, 70, 300, 32),
                                                     (0, 20, 35, 100, 90, 8), (1, -1, -1, 90, 40, 16),
                                                     (0, -1, -1, 33, 77, 64)])
def test_dense_limit(oracle_lib, causal, wl, wr, sq, sk, bs):
    """Selection of every block == brute-force dense masked attention (which has no blocks)."""
    rng = np.random.default_rng(sq * 7 + sk)
    Hq, Hkv, d, B = 4, 2, 32, 2
    q = _rand_bf16(rng, (B * sq, Hq, d))
    k = _rand_bf16(rng, (B * sk, Hkv, d))
    v = _rand_bf16(rng, (B * sk, Hkv, d))
    nblk = (sk + bs - 1) // bs
    sel = _all_blocks_sel(B * sq, Hkv, nblk)
    sel = W._shuffle_rows(rng, sel.reshape(-1, nblk)).reshape(sel.shape)
    c = _case(q, k, v, [0, sq, 2 * sq], [0, sk, 2 * sk], sel, Hq, Hkv, d, bs, causal, wl, wr)
    out, lse, bad = oracle_lib.fwd(c)
    ro, rl = dense_attention(c)
    assert bad == 0
    np.testing.assert_allclose(out, ro, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(np.isinf(lse), np.isinf(rl))
    fin = np.isfinite(rl)
    np.testing.assert_allclose(lse[fin], rl[fin], rtol=0, atol=1e-12)


def test_window_minus1_0_is_causal(oracle_lib):
    """window (-1, 0) without causal == causal without window (tutorial section 4.3)."""
    c = W.small_config(2)
    a, la, _ = oracle_lib.fwd(c)
    c2 = W.PrefillCase(**{**c.__dict__, "causal": 0, "wl": -1, "wr": 0})
    b, lb, _ = oracle_lib.fwd(c2)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(la, lb)


def test_rows_sum_to_one(oracle_lib):
    """v == 1 everywhere: every non-empty row outputs exactly 1 (softmax sums to 1); empty rows 0."""
    c = W.small_config(2)
    c = W.PrefillCase(**{**c.__dict__, "v": np.full_like(c.v, BF16_ONE)})
    out, lse, _ = oracle_lib.fwd(c)
    fin = np.isfinite(lse.T)  # (total_q, Hq)
    assert fin.all()
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-12)


def test_closed_forms(oracle_lib):
    """One kept key j: out = v_j, lse = scale*q.k_j.  q = 0: out = mean of v over kept keys,
    lse = ln(#kept keys)."""
    rng = np.random.default_rng(5)
    d, n, bs = 16, 64, 8
    q = _rand_bf16(rng, (n, 1, d))
    k = _rand_bf16(rng, (n, 1, d))
    v = _rand_bf16(rng, (n, 1, d))
    # Window (0, 0) keeps exactly the key at j = i.
    c = _case(q, k, v, [0, n], [0, n], _all_blocks_sel(n, 1, n // bs), 1, 1, d, bs, causal=0, wl=0, wr=0)
    out, lse, _ = oracle_lib.fwd(c)
    qf, kf, vf = (W.bf16_bits_to_f32(x).astype(np.float64) for x in (q, k, v))
    np.testing.assert_array_equal(out[:, 0, :], vf[:, 0, :])
    np.testing.assert_allclose(lse[0], (qf[:, 0, :] * kf[:, 0, :]).sum(1) / np.sqrt(d), rtol=1e-14, atol=1e-14)
    # q = 0, causal NSA selection: lse = ln(number of kept keys); out = mean of kept v.
    c = W.small_config(2)
    c = W.PrefillCase(**{**c.__dict__, "q": np.zeros_like(c.q)})
    out, lse, _ = oracle_lib.fwd(c)
    kept = np.exp(lse)  # (Hq, total_q)
    seqlens = np.diff(c.cu_q)
    want = []
    for L in seqlens:
        p = np.arange(L)
        b = p // c.bs
        want.append((np.minimum(c.topk, b + 1) - 1) * c.bs + p % c.bs + 1)
    want = np.concatenate(want)
    for h in range(c.Hq):
        np.testing.assert_allclose(kept[h], want, rtol=1e-12)
    assert int(round(kept[0].sum())) == W.kept_pairs_nsa(seqlens, c.bs, c.topk)
    t, h = 700, 5
    sel_c, cnt, _ = oracle_lib.fwd_index(c)
    hk = h // (c.Hq // c.Hkv)
    blocks = sel_c[t, hk, :cnt[t, hk]]
    i = t
    keys = [j for s in blocks for j in range(s * c.bs, min(s * c.bs + c.bs, 1024)) if j <= i]
    vf = W.bf16_bits_to_f32(c.v).astype(np.float64)
    np.testing.assert_allclose(out[t, h], vf[keys, hk, :].mean(0), rtol=0, atol=1e-12)


def test_selection_is_a_set(oracle_lib):
    """Permuting a row's slots, or duplicating ids into its padding, changes nothing."""
    c = W.small_config(4)
    out, lse, _ = oracle_lib.fwd(c)
    sc, cnt, _ = oracle_lib.fwd_index(c)
    rng = np.random.default_rng(9)
    sel = W._shuffle_rows(rng, c.sel.reshape(-1, c.topk)).reshape(c.sel.shape)
    dup = sel.copy().reshape(-1, c.topk)
    for r in range(dup.shape[0]):
        valid = dup[r][dup[r] >= 0]
        pads = np.where(dup[r] < 0)[0]
        if valid.size and pads.size:
            dup[r, pads] = rng.choice(valid, size=pads.size)
    dup = dup.reshape(c.sel.shape)
    for s in (sel, dup):
        o2, l2, _ = oracle_lib.fwd(c, sel=s)
        np.testing.assert_array_equal(out, o2)
        np.testing.assert_array_equal(lse, l2)
        sc2, cnt2, _ = oracle_lib.fwd_index(c, sel=s)
        np.testing.assert_array_equal(sc, sc2)
        np.testing.assert_array_equal(cnt, cnt2)


def test_bad_ids_counted_and_ignored(oracle_lib):
    c = W.small_config(2)
    out, lse, bad0 = oracle_lib.fwd(c)
    assert bad0 == 0
    sel = c.sel.copy()
    rows = np.where((sel == -1).any(axis=2))
    t, hk = rows[0][0], rows[1][0]
    slot = np.where(sel[t, hk] == -1)[0][0]
    sel[t, hk, slot] = 10 ** 6
    o2, l2, bad = oracle_lib.fwd(c, sel=sel)
    assert bad == 1
    np.testing.assert_array_equal(out, o2)
    _, _, bad_i = oracle_lib.fwd_index(c, sel=sel)
    assert bad_i == 1


def _brute_index(c):
    """Canonical set by brute force over keys: block s is kept iff some key of s survives the mask."""
    topk = c.sel.shape[-1]
    sc = np.full((c.total_q, c.Hkv, topk), -1, np.int32)
    cnt = np.zeros((c.total_q, c.Hkv), np.int32)
    for b in range(c.batch):
        sq, sk = c.cu_q[b + 1] - c.cu_q[b], c.cu_k[b + 1] - c.cu_k[b]
        keep = mask_matrix(sq, sk, c.causal, c.wl, c.wr)
        nblk = -(-sk // c.bs)
        for i in range(sq):
            t = c.cu_q[b] + i
            for hk in range(c.Hkv):
                s = sorted({int(x) for x in c.sel[t, hk] if 0 <= x < nblk and keep[i, x * c.bs:(x + 1) * c.bs].any()})
                sc[t, hk, :len(s)] = s
                cnt[t, hk] = len(s)
    return sc, cnt


@pytest.mark.parametrize("n", [1, 3])
def test_index_canonical_bruteforce(oracle_lib, n):
    c = W.small_config(n)
    sc, cnt, bad = oracle_lib.fwd_index(c)
    bsc, bcnt = _brute_index(c)
    assert bad == 0
    np.testing.assert_array_equal(sc, bsc)
    np.testing.assert_array_equal(cnt, bcnt)


def test_dense_window_config_matches_dense(oracle_lib):
    """The dense-limit workload (window (wl, 0), every touched block) equals dense attention."""
    c = W.small_config(3)
    out, lse, _ = oracle_lib.fwd(c)
    ro, rl = dense_attention(c)
    np.testing.assert_allclose(out, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-12)


def test_decode_matches_dense_gather(oracle_lib):
    c = W.small_config(5)
    out, lse, bad = oracle_lib.decode(c)
    assert list(bad) == [0, 0]
    ro, rl = dense_decode(c)
    np.testing.assert_allclose(out, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-12)


def test_decode_paging_invariance(oracle_lib):
    """Identity block table over contiguous pages == the seeded permuted table over the permuted pool."""
    c = W.small_config(5)
    out, lse, _ = oracle_lib.decode(c)
    npg = c.max_pages
    kc = np.zeros((c.B * npg, c.page, c.Hkv, c.d), np.uint16)
    vc = np.zeros_like(kc)
    bt = np.full((c.B, npg), -1, np.int32)
    for b in range(c.B):
        for p in range(npg):
            src = c.block_table[b, p]
            if src >= 0:
                kc[b * npg + p] = c.k_cache[src]
                vc[b * npg + p] = c.v_cache[src]
                bt[b, p] = b * npg + p
    c2 = W.DecodeCase(**{**c.__dict__, "k_cache": kc, "v_cache": vc, "block_table": bt})
    o2, l2, _ = oracle_lib.decode(c2)
    np.testing.assert_array_equal(out, o2)
    np.testing.assert_array_equal(lse, l2)


def test_decode_split_combine_identity(oracle_lib):
    """Attention over a token set split in two halves, merged through the LSEs
    (lse = log(e^lse1 + e^lse2), out = sum_s e^(lse_s - lse) out_s), equals the whole:
    this pins lse as the natural-log normaliser that the split-KV combine relies on."""
    c = W.small_config(5)
    out, lse, _ = oracle_lib.decode(c)
    half = c.topk // 2
    s1 = c.sel.copy(); s1[:, :, half:] = -1
    s2 = c.sel.copy(); s2[:, :, :half] = -1
    o1, l1, _ = oracle_lib.decode(c, sel=s1)
    o2, l2, _ = oracle_lib.decode(c, sel=s2)
    m = np.maximum(l1, l2)
    l = m + np.log(np.exp(l1 - m) + np.exp(l2 - m))
    o = np.exp(l1 - l)[..., None] * o1 + np.exp(l2 - l)[..., None] * o2
    np.testing.assert_allclose(o, out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, lse, rtol=0, atol=1e-12)


def test_decode_index_and_bad_ids(oracle_lib):
    c = W.small_config(5)
    tc, cnt, bad = oracle_lib.decode_index(c)
    assert bad == 0
    for b in range(c.B):
        for hk in range(c.Hkv):
            s = sorted({int(j) for j in c.sel[b, hk] if 0 <= j < c.cache_seqlens[b]})
            assert cnt[b, hk] == len(s)
            np.testing.assert_array_equal(tc[b, hk, :len(s)], s)
            assert (tc[b, hk, len(s):] == -1).all()
    sel = c.sel.copy()
    sel[0, 0, 0] = c.cache_seqlens[0] + 5  # beyond the cache length: an error, ignored
    o2, l2, badd = oracle_lib.decode(c, sel=sel)
    assert badd[0] == 1
    bt = c.block_table.copy()
    bt[1, 0] = c.num_pages + 3  # a bad page drops the tokens on it
    o3, l3, badp = oracle_lib.decode(c, block_table=bt)
    assert badp[1] > 0


def test_workload_kept_pairs_closed_form():
    """The NSA recipe's kept-pair count (closed form) equals the figures stated with the workloads."""
    assert W.kept_pairs_nsa([256], 32, 4) == 22656
    assert W.kept_pairs_nsa([8192, 4096, 2048, 2048], 64, 16) == 14295040
    assert W.kept_pairs_nsa([65536, 32768], 64, 16) == 96583680


def test_gated_combine_worked_example_and_gates():
    """The gated mix out = sum_c g_c * o_c: a hand-computed value (0.25*4 + 0.75*8 = 7 and
    0.25*(-2) + 0.75*2 = 1), a one-hot gate returning that branch unchanged, zero gates giving 0."""
    import oracle
    o1 = np.array([[[4.0, -2.0]]])
    o2 = np.array([[[8.0, 2.0]]])
    out = oracle.gated_combine([(o1, np.array([[0.25]])), (o2, np.array([[0.75]]))])
    np.testing.assert_array_equal(out, [[[7.0, 1.0]]])
    rng = np.random.default_rng(0)
    bits = W.f32_to_bf16_bits(rng.standard_normal((3, 2, 8), dtype=np.float32))
    other = W.f32_to_bf16_bits(rng.standard_normal((3, 2, 8), dtype=np.float32))
    one, zero = np.ones((3, 2)), np.zeros((3, 2))
    np.testing.assert_array_equal(oracle.gated_combine([(bits, one), (other, zero)]),
                                  W.bf16_bits_to_f32(bits).astype(np.float64))
    assert not oracle.gated_combine([(bits, zero), (other, zero)]).any()


def test_kv_append_worked_example():
    """oracle.kv_append against the hand-worked positions in tests/golden/kv_append_example.txt."""
    import oracle
    rows = [tuple(int(x) for x in ln.split()) for ln in open(os.path.join(GOLDEN, "kv_append_example.txt"))
            if ln.strip() and not ln.startswith("#")]
    kc = np.full((6, 2, 1, 1), -1.0)
    vc = np.full((6, 2, 1, 1), -2.0)
    bt = np.array([[4, 1, 5], [0, 3, 2]], np.int32)
    lens = np.array([3, 0], np.int32)
    kn = np.array([[10.0, 11.0], [20.0, 21.0]]).reshape(2, 2, 1, 1)
    k2, v2, bad = oracle.kv_append(kc, vc, bt, lens, kn, kn + 100)
    assert bad == 0
    want_k = kc.copy()
    want_v = vc.copy()
    for pg, row, val in rows:
        want_k[pg, row] = val
        want_v[pg, row] = val + 100
    np.testing.assert_array_equal(k2, want_k)
    np.testing.assert_array_equal(v2, want_v)
    # cache_seqlens [5, 0]: position 5 of sequence 0 -> block 2 -> page 5, row 1; position 6 -> block 3,
    # past the 3-entry block table: not written, counted.
    k3, _, bad3 = oracle.kv_append(kc, vc, bt, np.array([5, 0], np.int32), kn, kn)
    assert bad3 == 1
    assert k3[5, 1, 0, 0] == 10.0 and k3[0, 0, 0, 0] == 20.0 and k3[0, 1, 0, 0] == 21.0
    assert (k3 != kc).sum() == 3
