"""Pins for the backward oracle (oracle.bwd), each independent of the oracle's own arithmetic:
a worked example whose gradients follow by hand from the sigmoid, PyTorch autograd (float64, CPU)
through a dense masked softmax attention, and closed-form invariants of the softmax Jacobian."""
import numpy as np
import pytest

import sfa_workloads as W

torch = pytest.importorskip("torch")


def _bits(x):
    return W.f32_to_bf16_bits(np.asarray(x, np.float32))


def _case(q, k, v, cu_q, cu_k, sel, Hq, Hkv, d, bs, causal=1, wl=-1, wr=-1):
    sel = np.asarray(sel, np.int32)
    return W.PrefillCase("b", np.asarray(q, np.uint16), np.asarray(k, np.uint16), np.asarray(v, np.uint16),
                         np.asarray(cu_q, np.int32), np.asarray(cu_k, np.int32), sel, Hq, Hkv, d, bs, sel.shape[-1],
                         causal, wl, wr, 0.0)


def test_bwd_two_key_worked_example(oracle_lib):
    """One query (q = 1), two keys (k = 0, 1), values 1 and 3, d = 1 (scale 1), dout = 1.
    p1 = sigmoid(q (k1 - k0)) = e / (1 + e), p0 = 1 - p1, out = p0 + 3 p1, so by hand
    d out / d q = 2 p0 p1, d out / d k0 = -2 p0 p1, d out / d k1 = 2 p0 p1, d out / d v = (p0, p1)."""
    c = _case(_bits([[[1.0]]]), _bits([[[0.0]], [[1.0]]]), _bits([[[1.0]], [[3.0]]]), [0, 1], [0, 2],
              [[[0]]], 1, 1, 1, 2)
    dq, dk, dv, bad = oracle_lib.bwd(c, _bits([[[1.0]]]))
    e = np.e
    p1 = e / (1 + e)
    p0 = 1 - p1
    assert bad == 0
    np.testing.assert_allclose(dq.ravel(), [2 * p0 * p1], rtol=1e-14)
    np.testing.assert_allclose(dk.ravel(), [-2 * p0 * p1, 2 * p0 * p1], rtol=1e-14)
    np.testing.assert_allclose(dv.ravel(), [p0, p1], rtol=1e-14)


def _keep(c):
    """Boolean (total_q, Hkv, max_sk) of kept keys, from the selection read as a set of blocks and
    the bottom-right causal / window mask — written per element, without the oracle."""
    nk = int(np.diff(c.cu_k).max())
    keep = np.zeros((c.total_q, c.Hkv, nk), bool)
    for b in range(c.batch):
        sq, sk = int(c.cu_q[b + 1] - c.cu_q[b]), int(c.cu_k[b + 1] - c.cu_k[b])
        nblk = -(-sk // c.bs)
        for i in range(sq):
            t = int(c.cu_q[b]) + i
            for hk in range(c.Hkv):
                blocks = {int(s) for s in c.sel[t, hk] if 0 <= s < nblk}
                for j in range(sk):
                    ok = j // c.bs in blocks
                    if c.causal:
                        ok &= j <= i + sk - sq
                    if c.wl >= 0:
                        ok &= j >= i + sk - sq - c.wl
                    if c.wr >= 0:
                        ok &= j <= i + sk - sq + c.wr
                    keep[t, hk, j] = ok
    return keep


def _autograd(c, dout_bits):
    f = lambda a: torch.from_numpy(W.bf16_bits_to_f32(a).astype(np.float64))
    q, k, v, do = f(c.q).requires_grad_(), f(c.k).requires_grad_(), f(c.v).requires_grad_(), f(dout_bits)
    keep = torch.from_numpy(_keep(c))
    G, scale = c.Hq // c.Hkv, 1.0 / np.sqrt(c.d)
    loss = 0.0
    for b in range(c.batch):
        q0, q1, k0, k1 = (int(x) for x in (c.cu_q[b], c.cu_q[b + 1], c.cu_k[b], c.cu_k[b + 1]))
        for h in range(c.Hq):
            m = keep[q0:q1, h // G, :k1 - k0]
            s = (q[q0:q1, h] @ k[k0:k1, h // G].T) * scale
            s = s.masked_fill(~m, float("-inf"))
            live = m.any(dim=1, keepdim=True)
            p = torch.softmax(torch.where(live, s, torch.zeros_like(s)), dim=1) * m * live
            loss = loss + (do[q0:q1, h] * (p @ v[k0:k1, h // G])).sum()
    loss.backward()
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


@pytest.mark.parametrize("causal,wl,wr,lq,lk", [(1, -1, -1, [23, 9], [23, 9]), (1, 6, 0, [11, 17], [30, 17]),
                                                (0, 5, 3, [14], [19]), (0, -1, -1, [7, 12], [12, 5])])
def test_bwd_matches_autograd(oracle_lib, causal, wl, wr, lq, lk):
    """Selections with duplicates, -1 slots and one out-of-range id; GQA 4 / 2; rows with no kept
    key (the causal limit before the first selected block) included."""
    rng = np.random.default_rng(sum(lq) * 31 + sum(lk))
    Hq, Hkv, d, bs, topk = 4, 2, 16, 4, 3
    tq, tk = sum(lq), sum(lk)
    q = _bits(rng.standard_normal((tq, Hq, d)))
    k = _bits(rng.standard_normal((tk, Hkv, d)))
    v = _bits(rng.standard_normal((tk, Hkv, d)))
    nblk = -(-max(lk) // bs)
    sel = rng.integers(-1, nblk, size=(tq, Hkv, topk)).astype(np.int32)
    sel[0, 0, 1] = sel[0, 0, 0]   # a duplicate
    sel[1, 1, 2] = nblk + 5       # out of range: counted, ignored
    c = _case(q, k, v, np.r_[0, np.cumsum(lq)], np.r_[0, np.cumsum(lk)], sel, Hq, Hkv, d, bs, causal, wl, wr)
    dout = _bits(rng.standard_normal((tq, Hq, d)))
    dq, dk, dv, bad = oracle_lib.bwd(c, dout)
    gq, gk, gv = _autograd(c, dout)
    assert bad >= 1
    np.testing.assert_allclose(dq, gq, rtol=0, atol=1e-11)
    np.testing.assert_allclose(dk, gk, rtol=0, atol=1e-11)
    np.testing.assert_allclose(dv, gv, rtol=0, atol=1e-11)


def test_bwd_invariants(oracle_lib):
    """Softmax rows sum to 1 and shifting every score of a row by a constant changes nothing, so
    per (sequence, kv head): sum over keys of dk = 0, and sum over keys of dv = sum of dout over the
    rows that keep a key.  With every value row equal, dP is constant along each row and
    dq = dk = 0."""
    c = W.small_config(2)
    rng = np.random.default_rng(5)
    dout = _bits(rng.standard_normal((c.total_q, c.Hq, c.d)))
    dq, dk, dv, _ = oracle_lib.bwd(c, dout)
    _, lse, _ = oracle_lib.fwd(c)
    G = c.Hq // c.Hkv
    do = W.bf16_bits_to_f32(dout).astype(np.float64)
    live = np.isfinite(lse.T)  # (total_q, Hq)
    for b in range(c.batch):
        k0, k1, q0, q1 = c.cu_k[b], c.cu_k[b + 1], c.cu_q[b], c.cu_q[b + 1]
        for hk in range(c.Hkv):
            np.testing.assert_allclose(dk[k0:k1, hk].sum(0), 0.0, atol=1e-9)
            hs = slice(hk * G, hk * G + G)
            want = (do[q0:q1, hs] * live[q0:q1, hs, None]).sum((0, 1))
            np.testing.assert_allclose(dv[k0:k1, hk].sum(0), want, rtol=1e-12, atol=1e-9)
    row = _bits(rng.standard_normal((1, 1, c.d)))
    cu = W.PrefillCase(**{**c.__dict__, "v": np.broadcast_to(row, c.v.shape).copy()})
    dq2, dk2, _, _ = oracle_lib.bwd(cu, dout)
    assert np.abs(dq2).max() < 1e-12 and np.abs(dk2).max() < 1e-12
