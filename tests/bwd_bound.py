"""Per-element error bound for the prefill backward, derived from the arithmetic of the kernels.

The backward of the selected attention (the FlashAttentionScoreGrad case study of the Ascend
"Sparse FlashAttention" article: P from the forward's lse, dP = dO V^T, D = rowsum(dO o O),
dS = P o (dP - D), dQ = scale dS K; dK = scale dS^T Q and dV = P^T dO by the same chain rule) is
computed by the kernels with these roundings, and by the oracle exactly in fp64:

  * D is formed from the forward's bf16 output O~ (the case study's D = rowsum(dO o O) on the output
    the forward actually produced), so D~_i - D_i = sum_c dO_ic (O~_ic - O_ic) exactly, to the fp32
    rounding of that sum.  This input error is known exactly here (O~ is the GPU forward output, O
    the oracle's), so its effect on each gradient element is carried with its sign:
        dq_ic:  -scale * dD_i * sum_j P_ij k_jc
        dk_jc:  -scale * sum_i P_ij dD_i q_ic
  * P is recomputed from the forward's lse, whose error dl_i = lse~_i - lse_i is known exactly too:
    P~_ij = P_ij exp(-dl_i), carried with its sign through dS (dq, dk) and P (dv).
  * P and dS are rounded to bf16 before they enter the tensor cores, and S = scale q.k, dP = dO.v are
    fp32 sums of exact bf16 products.  These rounding errors are independent, zero-mean, and at most
    2^-8 relative (bf16 round to nearest even), so their standard deviation is at most 2^-7/sqrt(12)
    relative.  Their effect on a gradient element is a sum of independent terms; the bound takes
    Z = 6 standard deviations of that sum, element by element (over the ~10^6 elements a test checks,
    a Gaussian sum passes this with probability above 1 - 10^-3).
  * The signed terms above are first-order; they are taken with a factor 1 + 2^-6, which covers the
    second-order products (a 2^-8 rounding of P times the D shift, and the like).
  * D's own fp32 sum: at most 2^-22 sum_c |dO_ic O~_ic| (worst case), carried as P_ij times that
    through the same products without sign.
  * fp32 accumulation inside the tensor cores and the reductions: 2^-20 times the sum of the
    element's absolute terms (a deterministic allowance far above the fp32 unit roundoff per add).
  * The outputs dq, dk, dv are rounded to bf16: 2^-8 of the element's magnitude.

Nothing here is fitted to measurements: every term is the stated rounding model applied to the
element's own terms.  An element with no terms (a key no row keeps, a row that keeps no key) gets a
bound of exactly 0."""
import numpy as np

Z = 6.0                              # standard deviations of the random rounding terms
SIG = 2.0 ** -7 / np.sqrt(12.0)      # std of a bf16 round-to-nearest relative error (bound)
U = 2.0 ** -8                        # bf16 unit roundoff of the outputs
ACC = 2.0 ** -20                     # fp32 accumulation allowance per absolute term
SRE = 2.0 ** -22                     # relative error of fp32 score sums and the exp (per |term|)
DET = 1.0 + 2.0 ** -6                # the signed first-order terms, with room for the second-order ones


def kept_keys(c, sel_c, t_idx, hk, sk, sq, delta):
    """Boolean (len(t_idx), sk): key j kept by token t (selected block and inside the mask)."""
    nblk = (sk + c.bs - 1) // c.bs
    selb = np.zeros((len(t_idx), nblk + 1), bool)
    ids = sel_c[t_idx, hk, :]
    rows = np.repeat(np.arange(len(t_idx)), ids.shape[1])
    flat = ids.reshape(-1)
    ok = flat >= 0
    selb[rows[ok], flat[ok]] = True
    j = np.arange(sk)
    keep = selb[:, j // c.bs]
    return keep


def bwd_bounds(c, dout, out_gpu, lse_gpu, out_ref, lse_ref, sel_c, chunk=64):
    """Bounds (bq, bk, bv) shaped like dq, dk, dv, without the output rounding of dk and dv (which
    assert_within_bound adds from the values).  All inputs float64 (bf16-valued where bf16):
    dout (total_q, Hq, d); out_gpu / out_ref (total_q, Hq, d); lse_gpu / lse_ref (Hq, total_q);
    sel_c the canonical block lists (total_q, Hkv, topk)."""
    q = _f(c.q)
    k = _f(c.k)
    v = _f(c.v)
    G = c.Hq // c.Hkv
    sc = float(c.scale if c.scale > 0 else 1.0 / np.sqrt(c.d))
    bq = np.zeros((c.total_q, c.Hq, c.d))
    bk_det = np.zeros((c.total_k, c.Hkv, c.d))   # signed deterministic terms
    bv_det = np.zeros((c.total_k, c.Hkv, c.d))
    bk_var = np.zeros((c.total_k, c.Hkv, c.d))   # variance of the random terms
    bv_var = np.zeros((c.total_k, c.Hkv, c.d))
    bk_abs = np.zeros((c.total_k, c.Hkv, c.d))   # sums of absolute terms
    bv_abs = np.zeros((c.total_k, c.Hkv, c.d))
    bk_ext = np.zeros((c.total_k, c.Hkv, c.d))   # unsigned worst-case terms (D's fp32 sum)
    for b in range(c.batch):
        q0, q1 = int(c.cu_q[b]), int(c.cu_q[b + 1])
        k0, k1 = int(c.cu_k[b]), int(c.cu_k[b + 1])
        sq, sk = q1 - q0, k1 - k0
        delta = sk - sq
        for hk in range(c.Hkv):
            K = k[k0:k1, hk]
            V = v[k0:k1, hk]
            aK, aV = np.abs(K), np.abs(V)
            for t0 in range(0, sq, chunk):
                t1 = min(sq, t0 + chunk)
                i = np.arange(t0, t1)
                keep = kept_keys(c, sel_c, q0 + i, hk, sk, sq, delta)
                j = np.arange(sk)
                lo = np.zeros(len(i), np.int64)
                hi = np.full(len(i), sk - 1)
                if c.wl >= 0:
                    lo = np.maximum(lo, i + delta - c.wl)
                if c.causal:
                    hi = np.minimum(hi, i + delta)
                if c.wr >= 0:
                    hi = np.minimum(hi, i + delta + c.wr)
                keep &= (j[None, :] >= lo[:, None]) & (j[None, :] <= hi[:, None])
                if not keep.any():
                    continue
                for g in range(G):
                    h = hk * G + g
                    rows = q0 + i
                    Q = q[rows, h]
                    dO = dout[rows, h]
                    S = sc * (Q @ K.T)
                    L = lse_ref[h, rows]
                    with np.errstate(invalid="ignore", over="ignore"):
                        P = np.where(keep, np.exp(np.where(keep, S, 0.0) - np.where(np.isfinite(L), L, 0.0)[:, None]),
                                     0.0)
                    dP = dO @ V.T
                    D = (P * dP).sum(axis=1)
                    dS = P * (dP - D[:, None])
                    # known input errors, carried with their signs
                    dD = (dO * (out_gpu[rows, h] - out_ref[rows, h])).sum(axis=1)
                    dl = np.where(np.isfinite(L), lse_gpu[h, rows] - L, 0.0)
                    dS_det = -P * dD[:, None] - dl[:, None] * dS      # first-order change of dS
                    P_det = -dl[:, None] * P
                    # D's own fp32 sum (worst case, two bits of slack): a shift of dS by at most P * eD
                    eD = SRE * (np.abs(dO) * np.abs(out_gpu[rows, h])).sum(axis=1)
                    # relative error of P from the fp32 score and the exp: a random term per pair
                    sre = SRE * (sc * (np.abs(Q) @ aK.T) + 1.0)
                    # random terms: dS rounded to bf16; P's own errors inside dS; dP's fp32 sum
                    absPdPD = P * np.abs(dP - D[:, None])
                    var_ds = (SIG * dS) ** 2 + ((SIG + sre) * absPdPD) ** 2 + \
                        (P * SRE * (np.abs(dO) @ aV.T)) ** 2
                    var_p = ((SIG + sre) * P) ** 2
                    abs_ds = np.abs(dS)
                    # dq_ic = scale sum_j dS_ij k_jc
                    det_q = sc * (dS_det @ K)
                    eD_q = sc * eD[:, None] * (P @ aK)
                    var_q = sc * sc * (var_ds @ (K * K))
                    abs_q = sc * (abs_ds @ aK)
                    dq = sc * (dS @ K)
                    bq[rows, h] = DET * np.abs(det_q) + eD_q + Z * np.sqrt(var_q) + ACC * abs_q + U * np.abs(dq)
                    # dk_jc = scale sum_i dS_ij q_ic ; dv_jc = sum_i P_ij dO_ic (over every row i)
                    bk_det[k0:k1, hk] += sc * (dS_det.T @ Q)
                    bk_var[k0:k1, hk] += sc * sc * (var_ds.T @ (Q * Q))
                    bk_abs[k0:k1, hk] += sc * (abs_ds.T @ np.abs(Q))
                    bk_ext[k0:k1, hk] += sc * ((P * eD[:, None]).T @ np.abs(Q))
                    bv_det[k0:k1, hk] += P_det.T @ dO
                    bv_var[k0:k1, hk] += var_p.T @ (dO * dO)
                    bv_abs[k0:k1, hk] += P.T @ np.abs(dO)
    bk = DET * np.abs(bk_det) + bk_ext + Z * np.sqrt(bk_var) + ACC * bk_abs
    bv = DET * np.abs(bv_det) + Z * np.sqrt(bv_var) + ACC * bv_abs
    return bq, bk, bv


def _f(bits):
    a = np.asarray(bits)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def assert_within_bound(gpu, ref, bound, what, add_rounding=False):
    g = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert g.shape == ref.shape == bound.shape, (what, g.shape, ref.shape, bound.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    err = np.abs(g - ref)
    # bf16 rounding of the output, of the larger of the two magnitudes (the GPU value is the rounded one);
    # bq already holds U * |dq|, the rest is the rounding of the part above |ref|
    b = bound + U * np.maximum(np.abs(g), np.abs(ref)) if add_rounding else \
        bound + U * np.maximum(np.abs(g) - np.abs(ref), 0.0)
    excess = err - b
    worst = np.unravel_index(np.argmax(excess), excess.shape)
    assert excess.max() <= 0.0, (f"{what}: |gpu - ref| {err[worst]:.4g} above its bound {b[worst]:.4g} at {worst}: "
                                 f"gpu {g[worst]} ref {ref[worst]}")
