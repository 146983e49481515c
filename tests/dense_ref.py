"""Brute-force dense masked attention in numpy fp64 (an independent pin for the oracle).

It builds the full (sq x sk) score matrix per sequence and head with matrix products,
applies the mask as a boolean matrix, and normalises with a whole-row softmax.  It
knows nothing of blocks or selections: the sparse oracle must agree with it whenever
the selection covers every block that holds a kept key.
"""
import numpy as np

from sfa_workloads import bf16_bits_to_f32


def mask_matrix(sq, sk, causal, wl, wr):
    i = np.arange(sq)[:, None]
    j = np.arange(sk)[None, :]
    d = sk - sq
    keep = np.ones((sq, sk), dtype=bool)
    if causal:
        keep &= j <= i + d
    if wl >= 0:
        keep &= j >= i + d - wl
    if wr >= 0:
        keep &= j <= i + d + wr
    return keep


def dense_attention(case):
    """out (total_q, Hq, d) and lse (Hq, total_q), fp64."""
    q = bf16_bits_to_f32(case.q).astype(np.float64)
    k = bf16_bits_to_f32(case.k).astype(np.float64)
    v = bf16_bits_to_f32(case.v).astype(np.float64)
    G = case.Hq // case.Hkv
    out = np.zeros(q.shape, np.float64)
    lse = np.full((case.Hq, case.total_q), -np.inf)
    scale = case.softmax_scale
    for b in range(case.batch):
        q0, q1 = case.cu_q[b], case.cu_q[b + 1]
        k0, k1 = case.cu_k[b], case.cu_k[b + 1]
        keep = mask_matrix(q1 - q0, k1 - k0, case.causal, case.wl, case.wr)
        for h in range(case.Hq):
            s = (q[q0:q1, h, :] @ k[k0:k1, h // G, :].T) * scale
            s = np.where(keep, s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            full = np.isfinite(m[:, 0])
            e = np.where(keep, np.exp(s - np.where(np.isfinite(m), m, 0.0)), 0.0)
            z = e.sum(axis=1, keepdims=True)
            o = np.where(full[:, None], (e / np.where(z > 0, z, 1.0)) @ v[k0:k1, h // G, :], 0.0)
            out[q0:q1, h, :] = o
            lse[h, q0:q1] = np.where(full, m[:, 0] + np.log(np.where(z[:, 0] > 0, z[:, 0], 1.0)), -np.inf)
    return out, lse


def dense_decode(case):
    """Decode by explicit gather through the block table, then a plain softmax; fp64."""
    q = bf16_bits_to_f32(case.q).astype(np.float64)
    kc = bf16_bits_to_f32(case.k_cache).astype(np.float64)
    vc = bf16_bits_to_f32(case.v_cache).astype(np.float64)
    G = case.Hq // case.Hkv
    out = np.zeros(q.shape, np.float64)
    lse = np.full((case.B, case.Hq), -np.inf)
    for b in range(case.B):
        L = int(case.cache_seqlens[b])
        for hk in range(case.Hkv):
            toks = sorted({int(j) for j in case.sel[b, hk] if 0 <= j < L and (case.wl < 0 or j >= L - 1 - case.wl)})
            if not toks:
                continue
            toks = np.asarray(toks)
            pages = case.block_table[b, toks // case.page]
            K = kc[pages, toks % case.page, hk, :]
            V = vc[pages, toks % case.page, hk, :]
            for g in range(G):
                h = hk * G + g
                s = K @ q[b, h] * case.softmax_scale
                m = s.max()
                e = np.exp(s - m)
                out[b, h] = e @ V / e.sum()
                lse[b, h] = m + np.log(e.sum())
    return out, lse
