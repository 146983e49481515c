"""The backward's per-element error bound (tests/bwd_bound.py) on the CPU.

Two properties, checked against the fp64 oracle on a small NSA case (G 4, a 2-key row, a 1-token
sequence, a row cut by the causal edge):
  * sound: gradients computed with the roundings the bound models — a bf16 forward output entering
    D, an lse off by up to 1e-6, P and dS rounded to bf16 before their products, bf16 results — stay
    within it element by element;
  * sharp: a planted mistake (one row's term dropped from one key's dV; a sixteenth of the rows
    dropped from a block-0 key's dK, what a lost piece of a long row would do; a sign error in one
    row's dQ) lands outside it."""
import numpy as np
import pytest

import sfa_workloads as W
from tests import bwd_bound as BB

torch = pytest.importorskip("torch")


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


def _emulate(c, dout, out_g, lse_g, sel_c):
    """dq, dk, dv with the kernels' roundings, in numpy (the mask and selection as in the bound)."""
    q, k, v = BB._f(c.q), BB._f(c.k), BB._f(c.v)
    G = c.Hq // c.Hkv
    sc = c.scale if c.scale > 0 else 1 / np.sqrt(c.d)
    dq = np.zeros((c.total_q, c.Hq, c.d))
    dk = np.zeros((c.total_k, c.Hkv, c.d))
    dv = np.zeros_like(dk)
    for b in range(c.batch):
        q0, q1, k0, k1 = int(c.cu_q[b]), int(c.cu_q[b + 1]), int(c.cu_k[b]), int(c.cu_k[b + 1])
        sq, sk = q1 - q0, k1 - k0
        i = np.arange(sq)
        for hk in range(c.Hkv):
            K, V = k[k0:k1, hk], v[k0:k1, hk]
            keep = BB.kept_keys(c, sel_c, q0 + i, hk, sk, sq, sk - sq)
            keep &= np.arange(sk)[None, :] <= (i + sk - sq)[:, None]
            for g in range(G):
                h, rows = hk * G + g, q0 + i
                Q, dO = q[rows, h], dout[rows, h]
                S = (sc * (Q @ K.T)).astype(np.float32).astype(np.float64)
                L = lse_g[h, rows]
                P = np.where(keep, np.exp(np.where(keep, S, 0) - np.where(np.isfinite(L), L, 0)[:, None]), 0)
                P = P.astype(np.float32).astype(np.float64)
                dP = (dO @ V.T).astype(np.float32).astype(np.float64)
                D = (dO * out_g[rows, h]).sum(1).astype(np.float32).astype(np.float64)
                dS = _bf16(P * (dP - D[:, None]))
                dq[rows, h] = _bf16(sc * (dS @ K))
                dk[k0:k1, hk] += sc * (dS.T @ Q)
                dv[k0:k1, hk] += _bf16(P).T @ dO
    return dq, _bf16(dk), _bf16(dv)


@pytest.fixture(scope="module")
def case(oracle_lib):
    c = W.make_nsa_prefill(21, [700, 300, 64, 1], 8, 2, 128, 64, 6, 1, 2)
    rng = np.random.default_rng(3)
    dout_bits = W.f32_to_bf16_bits(rng.standard_normal((c.total_q, c.Hq, c.d), dtype=np.float32))
    dout = BB._f(dout_bits)
    ro, rl, _ = oracle_lib.fwd(c)
    out_g = _bf16(ro * (1 + rng.uniform(-2 ** -9, 2 ** -9, ro.shape)))  # a perturbed, bf16 forward output
    lse_g = (rl + rng.uniform(-1e-6, 1e-6, rl.shape)).astype(np.float32).astype(np.float64)
    rq, rk, rv, bad = oracle_lib.bwd(c, dout_bits)
    assert bad == 0
    sel_c, _, _ = oracle_lib.fwd_index(c)
    got = _emulate(c, dout, out_g, lse_g, sel_c)
    bq, bk, bv = BB.bwd_bounds(c, dout, out_g, lse_g, ro, rl, sel_c)
    return dict(c=c, dout=dout, ro=ro, rl=rl, ref=(rq, rk, rv), got=got, bound=(bq, bk, bv))


def test_bound_holds_for_modelled_roundings(case):
    (rq, rk, rv), (gq, gk, gv), (bq, bk, bv) = case["ref"], case["got"], case["bound"]
    BB.assert_within_bound(gq, rq, bq, "dq")
    BB.assert_within_bound(gk, rk, bk, "dk", add_rounding=True)
    BB.assert_within_bound(gv, rv, bv, "dv", add_rounding=True)
    # elements with no terms have bound 0 and must be exactly equal
    assert (gk[bk == 0] == rk[bk == 0]).all()


def _outside(g, r, b, what, add_rounding=False):
    with pytest.raises(AssertionError):
        BB.assert_within_bound(g, r, b, what, add_rounding=add_rounding)


def test_bound_rejects_planted_mistakes(case):
    c = case["c"]
    (rq, rk, rv), (gq, gk, gv), (bq, bk, bv) = case["ref"], case["got"], case["bound"]
    q, k, v = BB._f(c.q), BB._f(c.k), BB._f(c.v)
    sc = 1 / np.sqrt(c.d)
    ro, rl, dout = case["ro"], case["rl"], case["dout"]
    # one row's term dropped from one key's dV (token 705 of the second sequence, head 0, key 3)
    t, h, j = 705, 0, 3
    p = np.exp(sc * q[t, h] @ k[j, 0] - rl[h, t])
    gv2 = gv.copy()
    gv2[j, 0] -= p * dout[t, h]
    _outside(gv2, rv, bv, "dv", True)
    # a sixteenth of the first sequence's rows dropped from the dK of key 10 (block 0, kept by all)
    gk2 = gk.copy()
    for t in range(10, 700, 16):
        for h in range(c.Hq // c.Hkv):
            p = np.exp(sc * q[t, h] @ k[10, 0] - rl[h, t])
            ds = p * (dout[t, h] @ v[10, 0] - (ro[t, h] * dout[t, h]).sum())
            gk2[10, 0] -= sc * ds * q[t, h]
    _outside(gk2, rk, bk, "dk", True)
    # dQ of one row with its largest key term's sign flipped
    t, h = 400, 1
    gq2 = gq.copy()
    j = int(np.argmax(np.abs(sc * q[t, h] @ k[:64, 0].T)))  # a key of block 0, which every row keeps
    p = np.exp(sc * q[t, h] @ k[j, 0] - rl[h, t])
    ds = p * (dout[t, h] @ v[j, 0] - (ro[t, h] * dout[t, h]).sum())
    gq2[t, h] -= 2 * sc * ds * k[j, 0]
    _outside(gq2, rq, bq, "dq")
