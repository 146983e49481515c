"""GPU parity of the prefill backward (sfa_bwd) against the fp64 oracle (oracle.bwd), through the C ABI.

The forward's out / lse come from sfa_fwd on the same inputs; dout is seeded.  Every element of dq,
dk and dv must lie within its own error bound, derived from the kernels' arithmetic in
tests/bwd_bound.py: the exactly known effect of the bf16 forward output on D = rowsum(dO o O) and of
the forward's lse error, carried with their signs; six standard deviations of the independent bf16
roundings of P and dS over the element's own terms; fp32 accumulation; bf16 rounding of the result.
There is no tensor-wide term: a wrong value on a key that few rows keep is judged against that key's
own terms.  An element with no terms must be exactly 0.
"""
import dataclasses

import numpy as np
import pytest

import sfa_workloads as W
from tests import bwd_bound as BB
from tests.parity import upload_prefill, dev_tensor

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sfa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_flashattention_b200 as m
    return m


def _run(sfa, c, dd, dout, status=None, with_fwd=False):
    kw = dict(cu_seqlens_k=dd["cu_k"], max_seqlen_q=c.max_sq, max_seqlen_k=c.max_sk, causal=bool(c.causal),
              window=(c.wl, c.wr))
    out, lse = sfa.fwd(dd["q"], dd["k"], dd["v"], dd["cu_q"], dd["sel"], c.bs, **kw)
    dq, dk, dv = sfa.bwd(dd["q"], dd["k"], dd["v"], out, dout, lse, dd["cu_q"], dd["sel"], c.bs, status=status, **kw)
    return (dq, dk, dv, out, lse) if with_fwd else (dq, dk, dv)


def check_grads(oracle_lib, c, dout_bits, grads, out, lse, ref=None):
    """Every element of dq, dk, dv within its derived bound (tests/bwd_bound.py)."""
    rq, rk, rv, bad = oracle_lib.bwd(c, dout_bits) if ref is None else ref
    assert bad == 0
    ro, rl, _ = oracle_lib.fwd(c)
    sel_c, _, _ = oracle_lib.fwd_index(c)
    og = out.float().cpu().numpy().astype(np.float64)
    lg = lse.cpu().numpy().astype(np.float64)
    bq, bk, bv = BB.bwd_bounds(c, BB._f(dout_bits), og, lg, ro, rl, sel_c, chunk=128)
    dq, dk, dv = (x.float().cpu().numpy().astype(np.float64) for x in grads)
    BB.assert_within_bound(dq, rq, bq, "dq")
    BB.assert_within_bound(dk, rk, bk, "dk", add_rounding=True)
    BB.assert_within_bound(dv, rv, bv, "dv", add_rounding=True)


BWD_CASES = {
    # NSA selection, G 4; block 0 of the 1100-token sequence is selected by every token: a row cut
    # into three pieces summed through the running partial.
    "nsa_g4": lambda: W.make_nsa_prefill(21, [1100, 300, 64, 1], 8, 2, 128, 64, 6, 1, 2),
    # G 8 (16 tokens per chunk), init 1 / local 2 of topk 8.
    "nsa_g8": lambda: W.make_nsa_prefill(22, [700, 50], 16, 2, 128, 64, 8, 1, 2),
    # G 1 (128 tokens per chunk), sq != sk, two-sided window without causal.
    "window_g1": lambda: W.make_window_prefill(23, 2, 150, 260, 2, 2, 128, 64, 100, 20, causal=0),
    # causal window, sq < sk (bottom-right), G 2.
    "window_g2": lambda: W.make_window_prefill(24, 1, 200, 640, 4, 2, 128, 64, 256, 0, causal=1),
    # the tiny configuration's shape: d 64, block 32, G 4, top-4 with block 0 and the own block forced
    "tiny_d64_bs32": lambda: W.config1(),
    # d 128, block 32: 35 chunks of 32 tokens select block 0 (a row of three pieces)
    "nsa_d128_bs32": lambda: W.make_nsa_prefill(41, [1100, 130], 8, 2, 128, 32, 8, 1, 2),
    # d 64, block 64, G 1 (128 tokens per chunk)
    "nsa_d64_bs64_g1": lambda: W.make_nsa_prefill(42, [900, 77], 4, 4, 64, 64, 6, 1, 2),
    # d 64, block 32, G 3, causal window with sq < sk
    "window_d64_bs32_g3": lambda: W.make_window_prefill(43, 1, 300, 500, 6, 2, 64, 32, 100, 0, causal=1),
}


@pytest.mark.parametrize("name", sorted(BWD_CASES))
def test_bwd_parity(sfa, oracle_lib, name):
    c = BWD_CASES[name]()
    rng = np.random.default_rng(len(name))
    dout_bits = W.f32_to_bf16_bits(rng.standard_normal((c.total_q, c.Hq, c.d), dtype=np.float32))
    dd = upload_prefill(c)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq, dk, dv, out, lse = _run(sfa, c, dd, dev_tensor(dout_bits, torch.bfloat16), status, with_fwd=True)
    assert sfa.last_launch_count() == 7
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    check_grads(oracle_lib, c, dout_bits, (dq, dk, dv), out, lse)


def test_bwd_full_length_sequence(sfa, oracle_lib):
    """The backward at the length the benchmark runs it: one 8192-token NSA sequence, Hq 4 / Hkv 1
    (G 4, 32 tokens per chunk), d 128, block 64, top-16 with init 1 / local 2.  Block 0 is selected
    by all 8192 tokens, so its (block, kv head) row is cut into the largest number of pieces the
    piece scheme makes (16), summed in piece order.  Every element of dq, dk and dv is checked."""
    c = W.make_nsa_prefill(26, [8192], 4, 1, 128, 64, 16, 1, 2)
    rng = np.random.default_rng(9)
    dout_bits = W.f32_to_bf16_bits(rng.standard_normal((c.total_q, c.Hq, c.d), dtype=np.float32))
    dd = upload_prefill(c)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq, dk, dv, out, lse = _run(sfa, c, dd, dev_tensor(dout_bits, torch.bfloat16), status, with_fwd=True)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    check_grads(oracle_lib, c, dout_bits, (dq, dk, dv), out, lse)


def test_bwd_deterministic_and_empty_rows(sfa, oracle_lib):
    """Tokens whose selection is all -1 keep no key: dq exactly 0 there.  Two calls give the same
    bits (the multi-piece rows are summed in piece order)."""
    c = W.make_nsa_prefill(25, [1500, 90], 8, 2, 128, 64, 4, 1, 1)
    sel = c.sel.copy()
    sel[5:40] = -1
    sel[1500 + 10] = -1
    c = dataclasses.replace(c, sel=sel)
    rng = np.random.default_rng(7)
    dout_bits = W.f32_to_bf16_bits(rng.standard_normal((c.total_q, c.Hq, c.d), dtype=np.float32))
    dd = upload_prefill(c)
    dout = dev_tensor(dout_bits, torch.bfloat16)
    a = _run(sfa, c, dd, dout, with_fwd=True)
    b = _run(sfa, c, dd, dout, with_fwd=True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    dq = a[0]
    assert (dq[5:40] == 0).all() and (dq[1510] == 0).all()
    check_grads(oracle_lib, c, dout_bits, a[:3], a[3], a[4])


def test_bwd_no_queries_zero_key_grads(sfa):
    """total_q = 0 with keys present: dk = dv = 0 and no kernel runs."""
    k = torch.randn((64, 2, 128), device="cuda").to(torch.bfloat16)
    q = torch.zeros((0, 4, 128), dtype=torch.bfloat16, device="cuda")
    cu_q = torch.zeros(2, dtype=torch.int32, device="cuda")
    cu_k = torch.tensor([0, 64], dtype=torch.int32, device="cuda")
    sel = torch.zeros((0, 2, 4), dtype=torch.int32, device="cuda")
    lse = torch.zeros((4, 0), dtype=torch.float32, device="cuda")
    dk = torch.full_like(k, 7.0)
    dv = torch.full_like(k, 7.0)
    sfa.bwd(q, k, k, q, q, lse, cu_q, sel, 64, cu_seqlens_k=cu_k, max_seqlen_q=0, max_seqlen_k=64, dk=dk, dv=dv)
    assert (dk == 0).all() and (dv == 0).all()


def test_bwd_unsupported_shapes_rejected(sfa):
    """A head dimension outside {64, 128} or a block size outside {32, 64}: an error, no launch."""
    cu = torch.tensor([0, 8], dtype=torch.int32, device="cuda")
    sel = torch.zeros((8, 2, 1), dtype=torch.int32, device="cuda")
    lse = torch.zeros((2, 8), dtype=torch.float32, device="cuda")
    q = torch.zeros((8, 2, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sfa.SfaError):
        sfa.bwd(q, q, q, q, q, lse, cu, sel, 64)
    q = torch.zeros((8, 2, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sfa.SfaError):
        sfa.bwd(q, q, q, q, q, lse, cu, sel, 16)
