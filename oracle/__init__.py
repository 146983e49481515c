"""Python access to the fp64 CPU oracle (oracle/sfa_oracle.c).

TEST INFRASTRUCTURE ONLY: tests/, __graft_entry__.smoke() and bench.py's CPU
baseline leg use it.  The product path (sparse_flashattention_b200) never
imports it.  It takes the numpy arrays made by sfa_workloads and returns float64
results.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sfa_oracle.c")
_LIB = os.path.join(_HERE, "libsfa_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain C, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-D_POSIX_C_SOURCE=200809L", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.sfa_oracle_fwd.restype = ctypes.c_int64
        lib.sfa_oracle_fwd.argtypes = [P, P, P, P, P, I, I, I, I, P, I, I, I, I, I, ctypes.c_double,
                                       P, ctypes.c_int64, P, P, I]
        lib.sfa_oracle_fwd_index.restype = ctypes.c_int64
        lib.sfa_oracle_fwd_index.argtypes = [P, P, I, I, P, I, I, I, I, I, P, P]
        lib.sfa_oracle_bwd.restype = ctypes.c_int64
        lib.sfa_oracle_bwd.argtypes = [P, P, P, P, P, P, I, I, I, I, P, I, I, I, I, I, ctypes.c_double,
                                       P, P, P, I]
        lib.sfa_oracle_decode.restype = None
        lib.sfa_oracle_decode.argtypes = [P, P, P, P, I, I, I, P, P, I, I, I, I, I, I, ctypes.c_double,
                                          P, P, I, P]
        lib.sfa_oracle_decode_index.restype = ctypes.c_int64
        lib.sfa_oracle_decode_index.argtypes = [P, P, I, I, I, I, P, P]
        _lib = lib
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def default_threads():
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)


def fwd(case, rows=None, nthreads=None, sel=None):
    """Prefill oracle.  rows=None: out (total_q, Hq, d), lse (Hq, total_q).
    rows = int64 flat ids t*Hq+h: out (n, d), lse (n,).  Returns (out, lse, bad_ids)."""
    lib = _load()
    q, k, v = _c(case.q, np.uint16), _c(case.k, np.uint16), _c(case.v, np.uint16)
    cu_q, cu_k = _c(case.cu_q, np.int32), _c(case.cu_k, np.int32)
    sel = _c(case.sel if sel is None else sel, np.int32)
    if rows is None:
        out = np.zeros((case.total_q, case.Hq, case.d), np.float64)
        lse = np.zeros((case.Hq, case.total_q), np.float64)
        r, n = None, 0
    else:
        r = _c(rows, np.int64)
        n = r.size
        out = np.zeros((n, case.d), np.float64)
        lse = np.zeros((n,), np.float64)
    bad = lib.sfa_oracle_fwd(_p(q), _p(k), _p(v), _p(cu_q), _p(cu_k), case.batch, case.Hq, case.Hkv, case.d,
                             _p(sel), sel.shape[-1], case.bs, case.causal, case.wl, case.wr, float(case.scale),
                             _p(r), n, _p(out), _p(lse), nthreads or default_threads())
    return out, lse, int(bad)


def bwd(case, dout, nthreads=None, sel=None):
    """Prefill backward oracle: gradients of sum(dout * out) through the selected attention.
    dout: bf16 bit patterns (uint16), (total_q, Hq, d).  Returns (dq (total_q, Hq, d),
    dk (total_k, Hkv, d), dv (total_k, Hkv, d), bad_ids), float64."""
    lib = _load()
    q, k, v = _c(case.q, np.uint16), _c(case.k, np.uint16), _c(case.v, np.uint16)
    do = _c(dout, np.uint16)
    cu_q, cu_k = _c(case.cu_q, np.int32), _c(case.cu_k, np.int32)
    sel = _c(case.sel if sel is None else sel, np.int32)
    dq = np.zeros((case.total_q, case.Hq, case.d), np.float64)
    dk = np.zeros((case.total_k, case.Hkv, case.d), np.float64)
    dv = np.zeros((case.total_k, case.Hkv, case.d), np.float64)
    bad = lib.sfa_oracle_bwd(_p(q), _p(k), _p(v), _p(do), _p(cu_q), _p(cu_k), case.batch, case.Hq, case.Hkv,
                             case.d, _p(sel), sel.shape[-1], case.bs, case.causal, case.wl, case.wr,
                             float(case.scale), _p(dq), _p(dk), _p(dv), nthreads or default_threads())
    return dq, dk, dv, int(bad)


def fwd_index(case, sel=None):
    """Canonical (sel_c, cnt, bad_ids) of every (token, kv head)."""
    lib = _load()
    sel = _c(case.sel if sel is None else sel, np.int32)
    topk = sel.shape[-1]
    sel_c = np.zeros((case.total_q, case.Hkv, topk), np.int32)
    cnt = np.zeros((case.total_q, case.Hkv), np.int32)
    bad = lib.sfa_oracle_fwd_index(_p(_c(case.cu_q, np.int32)), _p(_c(case.cu_k, np.int32)), case.batch, case.Hkv,
                                   _p(sel), topk, case.bs, case.causal, case.wl, case.wr, _p(sel_c), _p(cnt))
    return sel_c, cnt, int(bad)


def decode(case, nthreads=None, sel=None, block_table=None):
    """Decode oracle: out (B, Hq, d), lse (B, Hq), bad = [bad token ids, bad pages]."""
    lib = _load()
    sel = _c(case.sel if sel is None else sel, np.int32)
    bt = _c(case.block_table if block_table is None else block_table, np.int32)
    out = np.zeros((case.B, case.Hq, case.d), np.float64)
    lse = np.zeros((case.B, case.Hq), np.float64)
    bad = np.zeros(2, np.int64)
    lib.sfa_oracle_decode(_p(_c(case.q, np.uint16)), _p(_c(case.k_cache, np.uint16)),
                          _p(_c(case.v_cache, np.uint16)), _p(bt), bt.shape[1], case.num_pages, case.page,
                          _p(_c(case.cache_seqlens, np.int32)), _p(sel), sel.shape[-1], case.B, case.Hq,
                          case.Hkv, case.d, case.wl, float(case.scale), _p(out), _p(lse),
                          nthreads or default_threads(), _p(bad))
    return out, lse, bad


def decode_index(case, sel=None):
    lib = _load()
    sel = _c(case.sel if sel is None else sel, np.int32)
    topk = sel.shape[-1]
    tok_c = np.zeros((case.B, case.Hkv, topk), np.int32)
    cnt = np.zeros((case.B, case.Hkv), np.int32)
    bad = lib.sfa_oracle_decode_index(_p(_c(case.cache_seqlens, np.int32)), _p(sel), topk, case.B, case.Hkv,
                                      case.wl, _p(tok_c), _p(cnt))
    return tok_c, cnt, int(bad)


def gated_combine(branches):
    """Gated mix of NSA branch outputs, in float64: out[t, h, :] = sum over the (o, g) pairs of
    g[t, h] * o[t, h, :] — the Flash-Sparse-Attention module's combination of its compressed, selected
    and sliding-window branches per token and head ("Relaxed-System-Lab/Flash-Sparse-Attention"
    project page, quick-start; README feature list, "Gated attention").  o: bf16 bit patterns
    (uint16) or floats, (total_q, Hq, d); g: floats (total_q, Hq)."""
    out = None
    for o, g in branches:
        o = np.asarray(o)
        of = (o.astype(np.uint32) << 16).view(np.float32).astype(np.float64) if o.dtype == np.uint16 else \
            o.astype(np.float64)
        term = np.asarray(g, np.float64)[..., None] * of
        out = term if out is None else out + term
    return out


def kv_append(k_cache, v_cache, block_table, cache_seqlens, k_new, v_new):
    """In-place KV-cache append as flash_attn_with_kvcache documents it (flash-attention-npu page,
    "FlashAttention v2" API docstrings): when k / v are given, k_cache / v_cache are updated in place
    with them, the new rows of sequence b going to logical positions cache_seqlens[b],
    cache_seqlens[b] + 1, ...; a paged cache (num_pages, page, Hkv, d) maps logical position j of
    sequence b to page block_table[b, j // page], row j % page.  cache_seqlens itself is left as is
    (the caller tracks lengths).  k_new / v_new: (B, seqlen_new, Hkv, d).  Positions past the block
    table, or whose page id is outside [0, num_pages), are not written (counted in `bad`, the
    reading taken here where the docstring only asks the caller to size the cache).
    Returns (k_cache, v_cache, bad) as new arrays; the inputs are not modified."""
    kc, vc = np.array(k_cache, copy=True), np.array(v_cache, copy=True)
    num_pages, page = kc.shape[0], kc.shape[1]
    B, S = k_new.shape[0], k_new.shape[1]
    bad = 0
    for b in range(B):
        for j in range(S):
            pos = int(cache_seqlens[b]) + j
            blk = pos // page
            if blk >= block_table.shape[1]:
                bad += 1
                continue
            pg = int(block_table[b, blk])
            if not 0 <= pg < num_pages:
                bad += 1
                continue
            kc[pg, pos % page] = k_new[b, j]
            vc[pg, pos % page] = v_new[b, j]
    return kc, vc, bad



def _bf16_f64(a):
    a = np.asarray(a)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64) if a.dtype == np.uint16 else \
        a.astype(np.float64)


def decode_kvcache(q, k_cache, v_cache, cache_seqlens, sel, cache_batch_idx, Hkv, scale, wl=-1):
    """Top-k decode over a non-paged cache, in float64, as flash_attn_with_kvcache documents its
    cache_batch_idx argument (flash-attention-npu page, "FlashAttention v2" API docstrings): k_cache /
    v_cache are (batch_cache, seqlen_cache, Hkv, d) and cache_batch_idx (B,) says which of their
    batch entries sequence b uses, so its row j is k_cache[cache_batch_idx[b], j].  For query head h
    (kv head h // G) the kept positions are the distinct entries j >= 0 of sel[b, h // G] below
    L = min(cache_seqlens[b], seqlen_cache) (and >= L - 1 - wl when wl >= 0); out is the softmax of
    scale * q . k_j over them applied to the v_j, lse the natural log of its normaliser.  No kept
    position, or an index outside [0, batch_cache): out 0, lse -inf.  Other negative or too large
    positions are counted in `bad` and skipped.
    q: (B, Hq, d); sel: (B, Hkv, topk).  Returns (out (B, Hq, d), lse (B, Hq), bad)."""
    qf, kf, vf = _bf16_f64(q), _bf16_f64(k_cache), _bf16_f64(v_cache)
    B, Hq, d = qf.shape
    batch_cache, seqlen_cache = kf.shape[0], kf.shape[1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, d), np.float64)
    lse = np.full((B, Hq), -np.inf, np.float64)
    bad = 0
    for b in range(B):
        L = min(int(cache_seqlens[b]), seqlen_cache)
        c = int(cache_batch_idx[b])
        for hk in range(Hkv):
            row = [int(j) for j in sel[b, hk]]
            bad += sum(1 for j in row if j != -1 and not 0 <= j < L)
            keep = sorted({j for j in row if 0 <= j < L and (wl < 0 or j >= L - 1 - wl)})
            if not keep or not 0 <= c < batch_cache:
                continue
            K, V = kf[c, keep, hk], vf[c, keep, hk]
            for h in range(hk * G, (hk + 1) * G):
                s_ = scale * (K @ qf[b, h])
                m = s_.max()
                e = np.exp(s_ - m)
                out[b, h] = e @ V / e.sum()
                lse[b, h] = m + np.log(e.sum())
    return out, lse, bad


def kv_append_kvcache(k_cache, v_cache, cache_batch_idx, cache_seqlens, k_new, v_new):
    """In-place append to a non-paged cache (flash_attn_with_kvcache with cache_batch_idx, same
    docstrings): row j of k_new[b] goes to k_cache[cache_batch_idx[b], cache_seqlens[b] + j].  Rows past
    seqlen_cache, or of a sequence whose index is outside [0, batch_cache), are not written (counted in
    `bad`).  Returns (k_cache, v_cache, bad) as new arrays."""
    kc, vc = np.array(k_cache, copy=True), np.array(v_cache, copy=True)
    batch_cache, seqlen_cache = kc.shape[0], kc.shape[1]
    bad = 0
    for b in range(k_new.shape[0]):
        c = int(cache_batch_idx[b])
        for j in range(k_new.shape[1]):
            pos = int(cache_seqlens[b]) + j
            if not (0 <= c < batch_cache and pos < seqlen_cache):
                bad += 1
                continue
            kc[c, pos] = k_new[b, j]
            vc[c, pos] = v_new[b, j]
    return kc, vc, bad

# ---------------------------------------------------------------------------------------------------
# Index producer for the decode: a Lightning-Indexer-style scan ("Sparse FlashAttention" on Ascend,
# ggplus blog post, section "那个叫Lightning Indexer的家伙": the indexer scores the current query
# against every key with FP8-quantized dot products and keeps the top-k token indices, which then
# crop K and V for the sparse attention; its cost is one O(L) pass over the keys).
# ---------------------------------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_round(x):
    """Round float values to the FP8 E4M3 format (1 sign, 4 exponent bits with bias 7, 3 mantissa
    bits; largest finite 448, smallest subnormal 2^-9, no infinities): round to nearest, ties to an
    even mantissa, magnitudes past 448 saturated to 448.  Returns float64 values of the format."""
    x = np.asarray(x, np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    # exponent of the format's spacing at |a|: 2^(e - 3) for normals (e >= -6), 2^-9 below 2^-6
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)
    q = 2.0 ** (e - 3)
    r = np.round(a / q) * q  # numpy rounds halves to even
    return np.sign(x) * np.minimum(r, E4M3_MAX)


def index_topk(q, k_cache, block_table, cache_seqlens, Hkv, topk, n_local=0):
    """Top-k token positions per (sequence, kv head) for the paged top-k decode.

    Readings taken where the page is silent:
      * the group's G query heads share one selection (one list per kv head, as the decode takes it),
        scored by the sum of their dot products: score_j = sum_g e4m3(q_g) . e4m3(k_j);
      * FP8 is E4M3 with round-to-nearest-even and saturation, no scale factors (N(0,1) data fit);
      * every cache position j < cache_seqlens[b] is a candidate, the last n_local positions are kept
        whatever their score, the rest are the highest scores, a tie going to the lower position;
      * the result is a set: ascending positions, -1 padded when fewer than topk exist;
      * a position whose page id is outside [0, num_pages) is no candidate (counted in `bad`), as the
        decode drops such tokens.
    The scores are exact: the group's summed query values (G values of the format, magnitudes from 2^-9
    to G * 448) need at most 24 significant bits, a product with a key value of the format at most 28,
    and every partial sum of the d products stays within 53 bits, so float64 computes them without
    rounding, in any order.

    q: (B, Hq, d) bf16 bits (uint16) or floats; k_cache: (num_pages, page, Hkv, d) likewise.
    Returns (sel int32 (B, Hkv, topk), scores: list over b of float64 (Hkv, L_b), bad)."""
    def f(a):
        a = np.asarray(a)
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64) if a.dtype == np.uint16 else \
            a.astype(np.float64)
    qf, kf = e4m3_round(f(q)), e4m3_round(f(k_cache))
    B, Hq, d = qf.shape
    G = Hq // Hkv
    page = kf.shape[1]
    sel = np.full((B, Hkv, topk), -1, np.int32)
    scores = []
    bad = 0
    num_pages = kf.shape[0]
    for b in range(B):
        L = int(cache_seqlens[b])
        pos = np.arange(L)
        pg = block_table[b, pos // page]
        ok = (pg >= 0) & (pg < num_pages)
        bad += int((~ok).sum())
        rows = kf[np.where(ok, pg, 0), pos % page]  # (L, Hkv, d): logical order
        sb = np.zeros((Hkv, L), np.float64)
        for hk in range(Hkv):
            qs = qf[b, hk * G:(hk + 1) * G].sum(axis=0)      # exact: G values of the format
            sb[hk] = rows[:, hk, :] @ qs
            nl = min(n_local, L, topk)
            keep = [j for j in range(L - nl, L) if ok[j]]
            rest = [j for j in sorted(range(L - nl), key=lambda j: (-sb[hk, j], j)) if ok[j]][:topk - nl]
            chosen = np.sort(np.array(keep + rest, np.int64))
            sel[b, hk, :chosen.size] = chosen
        scores.append(sb)
    return sel, scores, bad


def e4m3_decode(codes):
    """Values of FP8 E4M3 codes (uint8) as float64, from the format's definition: sign bit 7,
    exponent field E = bits 6..3 (bias 7), mantissa field M = bits 2..0; E = 0 gives M * 2^-9
    (subnormals), otherwise (1 + M / 8) * 2^(E - 7); E = 15 with M = 7 is not a number."""
    c = np.asarray(codes, np.uint8).astype(np.int64)
    s = np.where((c >> 7) & 1, -1.0, 1.0)
    E = (c >> 3) & 15
    M = c & 7
    mag = np.where(E == 0, M * 2.0 ** -9, (1.0 + M / 8.0) * np.exp2(E - 7.0))
    return np.where((E == 15) & (M == 7), np.nan, s * mag)


def decode_fp8(case, sel=None):
    """Paged top-k decode over FP8 caches, in float64: the attention of decode() with every cached
    value equal to e4m3_decode(code) * descale of its (sequence, kv head) (the k_descale / v_descale
    arguments of the FlashAttention-3 docstrings, per batch entry and kv head).  The key set per
    (sequence, kv head) is decode()'s: distinct positions p of the selection with 0 <= p < L (and
    p >= L - 1 - window_left when a window is given) whose page id is inside the cache.
    Returns (out (B, Hq, d), lse (B, Hq), bad = [bad token ids, bad pages])."""
    sel = np.asarray(case.sel if sel is None else sel)
    q = (np.asarray(case.q, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    kc, vc = case.k_cache, case.v_cache  # codes; only the gathered rows are decoded
    B, Hq, d = q.shape
    Hkv, page, num_pages = case.Hkv, case.page, kc.shape[0]
    G = Hq // Hkv
    scale = case.scale if case.scale > 0 else 1.0 / np.sqrt(d)
    out = np.zeros((B, Hq, d))
    lse = np.full((B, Hq), -np.inf)
    bad = np.zeros(2, np.int64)
    for b in range(B):
        L = int(case.cache_seqlens[b])
        for hk in range(Hkv):
            ids = sel[b, hk]
            bad[0] += int(((ids != -1) & ((ids < 0) | (ids >= L))).sum())
            pos = np.unique(ids[(ids >= 0) & (ids < L)])
            if case.wl >= 0:
                pos = pos[pos >= L - 1 - case.wl]
            pg = case.block_table[b, pos // page]
            okp = (pg >= 0) & (pg < num_pages)
            bad[1] += int((~okp).sum())
            pos, pg = pos[okp], pg[okp]
            if pos.size == 0:
                continue
            K = e4m3_decode(kc[pg, pos % page, hk]) * float(case.k_descale[b, hk])
            V = e4m3_decode(vc[pg, pos % page, hk]) * float(case.v_descale[b, hk])
            for g in range(G):
                h = hk * G + g
                s = scale * (K @ q[b, h])
                m = s.max()
                w = np.exp(s - m)
                Z = w.sum()
                out[b, h] = (w @ V) / Z
                lse[b, h] = m + np.log(Z)
    return out, lse, bad
