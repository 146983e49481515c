"""Seeded synthetic inputs for top-k sparse FlashAttention (prefill and paged decode).

This module only draws inputs. It holds none of the attention arithmetic: no
masking, no softmax, no index canonicalisation. Both the fp64 CPU oracle and the
CUDA path consume exactly the arrays produced here.

Value recipe: q/k/v ~ N(0, 1) drawn in float32 by numpy's PCG64 and rounded to
bfloat16 with round-to-nearest-even; the bf16 bit patterns are kept as uint16.

Selection recipe (NSA block selection, as parameterised on the
"Relaxed-System-Lab/Flash-Sparse-Attention" project page, quick-start example:
block_size, topk, init_blocks, local_blocks): for a query at position p of a
sequence (causal, equal q/k lengths), its own block is b = p // bs; the causally
valid blocks are {0..b}.  Always selected: the first `init_blocks` blocks and the
`local_blocks` blocks ending at b ({b, b-1, ...} clipped to >= 0).  The remaining
min(topk, b+1) - |forced| slots are drawn uniformly without replacement from the
other valid blocks.  The row of `topk` slots is -1 padded and then shuffled, so
padding and order are arbitrary.  One selection per (token, kv head), shared by
the G query heads of that kv head.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np

INVALID = -1


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round finite float32 values to bfloat16 (round to nearest, ties to even); return uint16
    bits.  For finite inputs u + 0x7FFF + lsb stays below 2^32, so uint32 arithmetic is exact."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).copy()
    lsb = (u >> 16) & np.uint32(1)
    u += np.uint32(0x7FFF)
    u += lsb
    u >>= np.uint32(16)
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_e4m3_bits(x: np.ndarray) -> np.ndarray:
    """Round finite float32 values to FP8 E4M3 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa
    bits; largest finite 448, no infinities): round to nearest, ties to even, magnitudes past 448
    saturated to 448; return uint8 codes.  Input preparation for FP8 caches."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    sign = np.signbit(x).astype(np.uint8)
    a = np.minimum(np.abs(x), 448.0)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)                 # below 2^-6 the spacing stays 2^-9 (subnormals)
    q = np.exp2(e - 3.0)
    r = np.round(a / q)                     # multiples of the spacing, halves to even
    # r is in [0, 16]; 16 means the next binade (exponent e + 1, mantissa 0)
    up = r >= 16
    e = np.where(up, e + 1, e)
    r = np.where(up, 8.0, r)
    normal = r >= 8                         # 1.mmm x 2^e
    E = np.where(normal, e + 7, 0).astype(np.int64)
    M = np.where(normal, r - 8, r).astype(np.int64)  # subnormal: r = mmm (value r * 2^-9)
    return ((sign.astype(np.int64) << 7) | (E << 3) | M).astype(np.uint8)


def _normal_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    step = 1 << 24
    for s in range(0, n, step):
        e = min(n, s + step)
        out[s:e] = f32_to_bf16_bits(rng.standard_normal(e - s, dtype=np.float32))
    return out.reshape(shape)


def _normal_bf16_parallel(seed_seq: np.random.SeedSequence, shape, chunk=1 << 24, threads=None) -> np.ndarray:
    """Large N(0,1) bf16 arrays: one child stream per fixed-size chunk (result independent of thread count)."""
    import concurrent.futures as cf
    import os

    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    nchunks = (n + chunk - 1) // chunk
    kids = seed_seq.spawn(nchunks)

    def work(i):
        s = i * chunk
        e = min(n, s + chunk)
        g = np.random.Generator(np.random.PCG64(kids[i]))
        out[s:e] = f32_to_bf16_bits(g.standard_normal(e - s, dtype=np.float32))

    threads = threads or min(32, os.cpu_count() or 1)
    with cf.ThreadPoolExecutor(threads) as ex:
        list(ex.map(work, range(nchunks)))
    return out.reshape(shape)


def _shuffle_rows(rng: np.random.Generator, a: np.ndarray) -> np.ndarray:
    keys = rng.random(a.shape)
    order = np.argsort(keys, axis=1, kind="stable")
    return np.take_along_axis(a, order, axis=1)


def nsa_block_selection(rng: np.random.Generator, seqlens: Sequence[int], hkv: int, bs: int, topk: int,
                        init_blocks: int, local_blocks: int) -> np.ndarray:
    """(total, hkv, topk) int32 block ids, -1 padded, shuffled per row."""
    total = int(sum(seqlens))
    sel = np.full((total, hkv, topk), INVALID, dtype=np.int32)
    base = 0
    for L in seqlens:
        nb = (L + bs - 1) // bs
        for b in range(nb):
            t0, t1 = base + b * bs, base + min(L, (b + 1) * bs)
            rows = (t1 - t0) * hkv
            forced = sorted(set(range(min(init_blocks, b + 1))) |
                            set(x for x in range(b - local_blocks + 1, b + 1) if x >= 0))
            forced = forced[:topk]
            nsel = min(topk, b + 1)
            nrand = nsel - len(forced)
            block = np.full((rows, topk), INVALID, dtype=np.int32)
            block[:, :len(forced)] = np.asarray(forced, dtype=np.int32)
            if nrand > 0:
                cand = np.asarray([x for x in range(b + 1) if x not in set(forced)], dtype=np.int32)
                keys = rng.random((rows, cand.size))
                pick = np.argpartition(keys, nrand - 1, axis=1)[:, :nrand]
                block[:, len(forced):nsel] = cand[pick]
            block = _shuffle_rows(rng, block)
            sel[t0:t1] = block.reshape(t1 - t0, hkv, topk)
        base += L
    return sel


def window_block_selection(rng: np.random.Generator, sq: int, sk: int, batch: int, hkv: int, bs: int,
                           causal: bool, wl: int, wr: int, topk: Optional[int] = None) -> np.ndarray:
    """Every block touching a query's key window [i+sk-sq-wl, i+sk-sq+wr] (clipped to [0, sk)); shuffled.

    This lists blocks by the window arithmetic alone, so it is an input recipe, not the
    kernel's mask: the kernel still applies the mask inside each block."""
    delta = sk - sq
    lo = np.arange(sq) + delta - (wl if wl >= 0 else 10 ** 9)
    hi = np.arange(sq) + delta + (wr if wr >= 0 else 10 ** 9)
    if causal:
        hi = np.minimum(hi, np.arange(sq) + delta)
    lo = np.clip(lo, 0, sk - 1)
    hi = np.clip(hi, -1, sk - 1)
    nmax = int(((hi // bs) - (lo // bs) + 1).max()) if sq else 0
    topk = topk or max(nmax, 1)
    rows = np.full((sq, topk), INVALID, dtype=np.int32)
    for i in range(sq):
        if hi[i] < lo[i]:
            continue
        blocks = np.arange(lo[i] // bs, hi[i] // bs + 1, dtype=np.int32)[:topk]
        rows[i, :blocks.size] = blocks
    sel = np.broadcast_to(rows[None, :, None, :], (batch, sq, hkv, topk)).reshape(batch * sq, hkv, topk).copy()
    flat = sel.reshape(-1, topk)
    return _shuffle_rows(rng, flat).reshape(sel.shape).astype(np.int32)


@dataclasses.dataclass
class PrefillCase:
    name: str
    q: np.ndarray            # uint16 bf16 bits (total_q, Hq, d)
    k: np.ndarray            # uint16 (total_k, Hkv, d)
    v: np.ndarray            # uint16 (total_k, Hkv, d)
    cu_q: np.ndarray         # int32 (batch+1)
    cu_k: np.ndarray         # int32 (batch+1)
    sel: np.ndarray          # int32 (total_q, Hkv, topk)
    Hq: int
    Hkv: int
    d: int
    bs: int
    topk: int
    causal: int = 1
    wl: int = -1
    wr: int = -1
    scale: float = 0.0       # <= 0 means 1/sqrt(d)

    @property
    def batch(self):
        return int(self.cu_q.size - 1)

    @property
    def total_q(self):
        return int(self.cu_q[-1])

    @property
    def total_k(self):
        return int(self.cu_k[-1])

    @property
    def max_sq(self):
        return int(np.diff(self.cu_q).max()) if self.batch else 0

    @property
    def max_sk(self):
        return int(np.diff(self.cu_k).max()) if self.batch else 0

    @property
    def softmax_scale(self):
        return self.scale if self.scale > 0 else 1.0 / np.sqrt(self.d)


@dataclasses.dataclass
class DecodeCase:
    name: str
    q: np.ndarray            # uint16 (B, Hq, d)
    k_cache: np.ndarray      # uint16 (num_pages, page, Hkv, d)
    v_cache: np.ndarray
    block_table: np.ndarray  # int32 (B, max_pages)
    cache_seqlens: np.ndarray  # int32 (B,)
    sel: np.ndarray          # int32 (B, Hkv, topk_tok)
    Hq: int
    Hkv: int
    d: int
    page: int
    wl: int = -1
    scale: float = 0.0
    # FP8 caches: k_cache / v_cache hold E4M3 codes (uint8) and a cached value is code * descale of its
    # (sequence, kv head); None for bf16 caches.
    k_descale: Optional[np.ndarray] = None   # float32 (B, Hkv)
    v_descale: Optional[np.ndarray] = None

    @property
    def B(self):
        return int(self.q.shape[0])

    @property
    def num_pages(self):
        return int(self.k_cache.shape[0])

    @property
    def max_pages(self):
        return int(self.block_table.shape[1])

    @property
    def topk(self):
        return int(self.sel.shape[2])

    @property
    def softmax_scale(self):
        return self.scale if self.scale > 0 else 1.0 / np.sqrt(self.d)


@dataclasses.dataclass
class KVCacheCase:
    """Decode inputs over a non-paged cache addressed through cache_batch_idx."""
    name: str
    q: np.ndarray               # uint16 (B, Hq, d)
    k_cache: np.ndarray         # uint16 (batch_cache, seqlen_cache, Hkv, d)
    v_cache: np.ndarray
    cache_batch_idx: np.ndarray  # int32 (B,): the cache entry of each sequence
    cache_seqlens: np.ndarray   # int32 (B,)
    sel: np.ndarray             # int32 (B, Hkv, topk_tok)
    Hq: int
    Hkv: int
    d: int
    wl: int = -1

    @property
    def B(self):
        return int(self.q.shape[0])

    @property
    def softmax_scale(self):
        return 1.0 / np.sqrt(self.d)


def make_decode_kvcache(seed: int, B, batch_cache, seqlen_cache, Hq, Hkv, d, len_lo, len_hi, topk_tok, n_last,
                        name="decode_kvcache") -> KVCacheCase:
    """Non-paged decode inputs: cache_seqlens ~ U[len_lo, len_hi] (<= seqlen_cache), each sequence on
    a distinct cache entry drawn from [0, batch_cache), selections as make_decode draws them."""
    ss = np.random.SeedSequence(seed)
    s_len, s_idx, s_q, s_k, s_v, s_sel = ss.spawn(6)
    L = np.random.Generator(np.random.PCG64(s_len)).integers(len_lo, len_hi + 1, size=B).astype(np.int32)
    idx = np.random.Generator(np.random.PCG64(s_idx)).permutation(batch_cache)[:B].astype(np.int32)
    q = _normal_bf16(np.random.Generator(np.random.PCG64(s_q)), (B, Hq, d))
    kc = _normal_bf16(np.random.Generator(np.random.PCG64(s_k)), (batch_cache, seqlen_cache, Hkv, d))
    vc = _normal_bf16(np.random.Generator(np.random.PCG64(s_v)), (batch_cache, seqlen_cache, Hkv, d))
    g_sel = np.random.Generator(np.random.PCG64(s_sel))
    sel = np.full((B, Hkv, topk_tok), INVALID, dtype=np.int32)
    for b in range(B):
        Lb = int(L[b])
        nl = min(n_last, Lb, topk_tok)
        last = np.arange(Lb - nl, Lb, dtype=np.int32)
        nr = min(topk_tok - nl, Lb - nl)
        for h in range(Hkv):
            rest = g_sel.choice(Lb - nl, size=nr, replace=False).astype(np.int32) if nr > 0 else \
                np.zeros(0, np.int32)
            row = np.concatenate([last, rest])
            g_sel.shuffle(row)
            sel[b, h, :row.size] = row
    return KVCacheCase(name, q, kc, vc, idx, L, sel, Hq, Hkv, d)


def kvcache_as_paged(c: KVCacheCase, page: int, seed: int) -> DecodeCase:
    """The same logical rows as a paged cache: each sequence's rows cut into pages of `page` rows,
    the pages placed at random physical slots.  Returns a DecodeCase for the C oracle."""
    rng = np.random.default_rng(seed)
    seqlen_cache = c.k_cache.shape[1]
    npp = (seqlen_cache + page - 1) // page
    num_pages = c.B * npp
    perm = rng.permutation(num_pages).astype(np.int32)
    shape = (num_pages, page) + c.k_cache.shape[2:]
    kp, vp = np.zeros(shape, np.uint16), np.zeros(shape, np.uint16)
    bt = perm.reshape(c.B, npp)
    for b in range(c.B):
        for p in range(npp):
            rows = slice(p * page, min((p + 1) * page, seqlen_cache))
            n = rows.stop - rows.start
            kp[bt[b, p], :n] = c.k_cache[c.cache_batch_idx[b], rows]
            vp[bt[b, p], :n] = c.v_cache[c.cache_batch_idx[b], rows]
    return DecodeCase("repacked", c.q, kp, vp, bt, c.cache_seqlens, c.sel, c.Hq, c.Hkv, c.d, page, wl=c.wl,
                        scale=c.softmax_scale)


def _cu(lens):
    return np.concatenate([[0], np.cumsum(np.asarray(lens, dtype=np.int64))]).astype(np.int32)


def make_nsa_prefill(seed: int, seqlens, Hq, Hkv, d, bs, topk, init_blocks, local_blocks, name="nsa",
                     parallel_values=False) -> PrefillCase:
    ss = np.random.SeedSequence(seed)
    s_q, s_k, s_v, s_sel = ss.spawn(4)
    total = int(sum(seqlens))
    if parallel_values:
        q = _normal_bf16_parallel(s_q, (total, Hq, d))
        k = _normal_bf16_parallel(s_k, (total, Hkv, d))
        v = _normal_bf16_parallel(s_v, (total, Hkv, d))
    else:
        q = _normal_bf16(np.random.Generator(np.random.PCG64(s_q)), (total, Hq, d))
        k = _normal_bf16(np.random.Generator(np.random.PCG64(s_k)), (total, Hkv, d))
        v = _normal_bf16(np.random.Generator(np.random.PCG64(s_v)), (total, Hkv, d))
    sel = nsa_block_selection(np.random.Generator(np.random.PCG64(s_sel)), seqlens, Hkv, bs, topk,
                              init_blocks, local_blocks)
    cu = _cu(seqlens)
    return PrefillCase(name, q, k, v, cu, cu.copy(), sel, Hq, Hkv, d, bs, topk, causal=1)


def make_window_prefill(seed: int, batch, sq, sk, Hq, Hkv, d, bs, wl, wr, causal=1, name="window") -> PrefillCase:
    ss = np.random.SeedSequence(seed)
    s_q, s_k, s_v, s_sel = ss.spawn(4)
    q = _normal_bf16(np.random.Generator(np.random.PCG64(s_q)), (batch * sq, Hq, d))
    k = _normal_bf16(np.random.Generator(np.random.PCG64(s_k)), (batch * sk, Hkv, d))
    v = _normal_bf16(np.random.Generator(np.random.PCG64(s_v)), (batch * sk, Hkv, d))
    sel = window_block_selection(np.random.Generator(np.random.PCG64(s_sel)), sq, sk, batch, Hkv, bs,
                                 bool(causal), wl, wr)
    return PrefillCase(name, q, k, v, _cu([sq] * batch), _cu([sk] * batch), sel, Hq, Hkv, d, bs,
                       int(sel.shape[2]), causal=causal, wl=wl, wr=wr)


def make_decode(seed: int, B, Hq, Hkv, d, page, len_lo, len_hi, topk_tok, n_last, name="decode",
                parallel_values=False, max_len=None) -> DecodeCase:
    """Paged top-k decode inputs.  cache_seqlens ~ U[len_lo, len_hi] (inclusive); pages are placed
    through a seeded permutation; each (b, kv head) selects the last `n_last` positions plus
    topk_tok - n_last positions drawn without replacement from [0, L - n_last), shuffled."""
    ss = np.random.SeedSequence(seed)
    s_len, s_perm, s_q, s_k, s_v, s_sel = ss.spawn(6)
    g_len = np.random.Generator(np.random.PCG64(s_len))
    L = g_len.integers(len_lo, len_hi + 1, size=B).astype(np.int32)
    max_len = max_len or len_hi
    max_pages = (max_len + page - 1) // page
    npages_b = (L + page - 1) // page
    num_pages = int(npages_b.sum())
    perm = np.random.Generator(np.random.PCG64(s_perm)).permutation(num_pages).astype(np.int32)
    bt = np.full((B, max_pages), INVALID, dtype=np.int32)
    off = 0
    for b in range(B):
        bt[b, :npages_b[b]] = perm[off:off + npages_b[b]]
        off += npages_b[b]
    q = _normal_bf16(np.random.Generator(np.random.PCG64(s_q)), (B, Hq, d))
    shape = (num_pages, page, Hkv, d)
    if parallel_values:
        kc = _normal_bf16_parallel(s_k, shape)
        vc = _normal_bf16_parallel(s_v, shape)
    else:
        kc = _normal_bf16(np.random.Generator(np.random.PCG64(s_k)), shape)
        vc = _normal_bf16(np.random.Generator(np.random.PCG64(s_v)), shape)
    g_sel = np.random.Generator(np.random.PCG64(s_sel))
    sel = np.full((B, Hkv, topk_tok), INVALID, dtype=np.int32)
    for b in range(B):
        Lb = int(L[b])
        nl = min(n_last, Lb, topk_tok)
        last = np.arange(Lb - nl, Lb, dtype=np.int32)
        nr = min(topk_tok - nl, Lb - nl)
        for h in range(Hkv):
            rest = g_sel.choice(Lb - nl, size=nr, replace=False).astype(np.int32) if nr > 0 else \
                np.zeros(0, np.int32)
            row = np.concatenate([last, rest])
            g_sel.shuffle(row)
            sel[b, h, :row.size] = row
    return DecodeCase(name, q, kc, vc, bt, L, sel, Hq, Hkv, d, page)


# ---------------------------------------------------------------------------------------------
# The five named workloads and their oracle-sized variants.
# ---------------------------------------------------------------------------------------------

def make_decode_fp8(seed: int, B, Hq, Hkv, d, page, len_lo, len_hi, topk_tok, n_last, name="decode_fp8",
                    parallel_values=False, max_len=None) -> DecodeCase:
    """The paged decode inputs of make_decode with the caches stored as FP8 E4M3: per (sequence, kv
    head) a descale = max |value| of the sequence's cached rows / 448 (float32), and every cached
    value of that sequence stored as e4m3(value / descale)."""
    c = make_decode(seed, B, Hq, Hkv, d, page, len_lo, len_hi, topk_tok, n_last, name=name,
                    parallel_values=parallel_values, max_len=max_len)
    kq = np.zeros(c.k_cache.shape, np.uint8)
    vq = np.zeros(c.v_cache.shape, np.uint8)
    kd = np.ones((B, Hkv), np.float32)
    vd = np.ones((B, Hkv), np.float32)
    for b in range(B):
        pages = c.block_table[b][c.block_table[b] >= 0]
        for h in range(Hkv):
            for src, dst, ds in ((c.k_cache, kq, kd), (c.v_cache, vq, vd)):
                vals = bf16_bits_to_f32(src[pages, :, h, :])
                amax = float(np.abs(vals).max()) if vals.size else 0.0
                ds[b, h] = np.float32(amax / 448.0) if amax > 0 else np.float32(1.0)
                dst[pages, :, h, :] = f32_to_e4m3_bits(vals / ds[b, h])
    return dataclasses.replace(c, k_cache=kq, v_cache=vq, k_descale=kd, v_descale=vd)


def config1():
    """Tiny selected attention: 1 x 256 tokens, Hq4/Hkv1, d64, bs32, topk4 (block 0 + own block forced)."""
    return make_nsa_prefill(1, [256], 4, 1, 64, 32, 4, init_blocks=1, local_blocks=1, name="tiny_256_d64")


def config2(parallel_values=False, shrink=1):
    """Varlen NSA: lengths [8192, 4096, 2048, 2048], Hq16/Hkv4, d128, bs64, topk16, init 1, local 2.
    shrink > 1 divides the lengths (a smaller case of the same kernels, for profiler captures)."""
    return make_nsa_prefill(2, [n // shrink for n in (8192, 4096, 2048, 2048)], 16, 4, 128, 64, 16, 1, 2,
                            name="nsa_varlen_16k" if shrink == 1 else f"nsa_varlen_16k/{shrink}",
                            parallel_values=parallel_values)


def config3():
    """Dense limit: B2, sq1024, sk4096, Hq32/Hkv8, d128, causal, window (1024, 0), every touched 64-block."""
    return make_window_prefill(3, 2, 1024, 4096, 32, 8, 128, 64, 1024, 0, causal=1, name="dense_window_1k_4k")


def config4(parallel_values=False, shrink=1):
    """Long context: lengths [65536, 32768], Hq=Hkv=4, d128, bs64, topk16, init 1, local 2.
    shrink > 1 divides the lengths (a smaller case of the same kernels, for profiler captures)."""
    return make_nsa_prefill(4, [n // shrink for n in (65536, 32768)], 4, 4, 128, 64, 16, 1, 2,
                            name="nsa_long_96k" if shrink == 1 else f"nsa_long_96k/{shrink}",
                            parallel_values=parallel_values)


def config5(parallel_values=True):
    """Paged top-k decode: B32, Hq32/Hkv8, d128, L ~ U[16384, 131072], page 256, 2048 tokens (last 128 forced)."""
    return make_decode(5, 32, 32, 8, 128, 256, 16384, 131072, 2048, 128, name="paged_topk_decode_b32",
                       parallel_values=parallel_values)


def small_config(n: int):
    """Oracle-sized variants of the five workloads (several tiles, ragged tails)."""
    if n == 1:
        return config1()
    if n == 2:
        return make_nsa_prefill(12, [1024, 517, 300, 77], 16, 4, 128, 64, 16, 1, 2, name="nsa_varlen_small")
    if n == 3:
        return make_window_prefill(13, 2, 200, 700, 32, 8, 128, 64, 256, 0, causal=1, name="dense_window_small")
    if n == 4:
        return make_nsa_prefill(14, [2048, 1000], 4, 4, 128, 64, 16, 1, 2, name="nsa_long_small")
    if n == 5:
        return make_decode(15, 4, 32, 8, 128, 256, 700, 3000, 256, 32, name="decode_small")
    raise ValueError(n)


def kept_pairs_nsa(seqlens, bs, topk):
    """Closed form of kept (query, key) pairs per query head for the NSA recipe with causal mask:
    a query at p with b = p // bs keeps (min(topk, b+1) - 1) * bs + (p % bs + 1) keys."""
    tot = 0
    for L in seqlens:
        p = np.arange(L)
        b = p // bs
        tot += int(((np.minimum(topk, b + 1) - 1) * bs + (p % bs + 1)).sum())
    return tot


# ---------------------------------------------------------------------------------------------
# Device upload of a case (torch is imported only here: the generators above need numpy alone)
# ---------------------------------------------------------------------------------------------
def dev_tensor(a, dtype=None, device="cuda"):
    """A numpy array as a torch tensor on `device`; `dtype` reinterprets the bits (bf16 from uint16)."""
    import torch
    x = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        x = x.view(dtype)
    return x.to(device)


def upload_prefill(c, device="cuda"):
    import torch
    return dict(q=dev_tensor(c.q, torch.bfloat16, device), k=dev_tensor(c.k, torch.bfloat16, device),
                v=dev_tensor(c.v, torch.bfloat16, device), cu_q=dev_tensor(c.cu_q, None, device),
                cu_k=dev_tensor(c.cu_k, None, device), sel=dev_tensor(c.sel, None, device))


def upload_decode(c, device="cuda"):
    import torch
    return dict(q=dev_tensor(c.q, torch.bfloat16, device), k_cache=dev_tensor(c.k_cache, torch.bfloat16, device),
                v_cache=dev_tensor(c.v_cache, torch.bfloat16, device),
                block_table=dev_tensor(c.block_table, None, device),
                cache_seqlens=dev_tensor(c.cache_seqlens, None, device), sel=dev_tensor(c.sel, None, device))


def quantize_cache_e4m3_device(c, d):
    """FP8 E4M3 codes (uint8) and descales (B, Hkv) of an uploaded bf16 paged cache, made on the device
    with torch for workloads too large to quantize on the host: per (sequence, kv head) descale =
    max |value| / 448, codes = round-to-nearest-even E4M3 of value / descale (make_decode_fp8's recipe).
    Returns (k_codes, v_codes, k_descale, v_descale) device tensors."""
    import torch
    kq = torch.empty(d["k_cache"].shape, dtype=torch.uint8, device=d["k_cache"].device)
    vq = torch.empty_like(kq)
    kd = torch.ones((c.B, c.Hkv), dtype=torch.float32, device=kq.device)
    vd = torch.ones_like(kd)
    bt = c.block_table
    for b in range(c.B):
        pages = torch.as_tensor(bt[b][bt[b] >= 0], device=kq.device, dtype=torch.long)
        for src, dst, ds in ((d["k_cache"], kq, kd), (d["v_cache"], vq, vd)):
            vals = src.index_select(0, pages).float()           # (pages, page, Hkv, d)
            amax = vals.abs().amax(dim=(0, 1, 3))                # (Hkv,)
            sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
            ds[b] = sc
            codes = (vals / sc.view(1, 1, -1, 1)).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
            dst.index_copy_(0, pages, codes)
    return kq, vq, kd, vd
