"""GPU parity of the prefill backward (sfa_bwd) against the fp64 oracle (oracle.bwd), through the C ABI.

The forward's out / lse come from sfa_fwd on the same inputs; dout is seeded.  Tolerance, from the
arithmetic of the kernels: P and dS enter the tensor cores as bf16 (unit roundoff 2^-8), and
D = rowsum(dO o O) is taken, as the FlashAttentionScoreGrad case study prescribes, from the forward's
output — bf16 here — while the oracle sums p dP exactly.  Each gradient element therefore carries an
error of a few 2^-8 times the size of the terms it sums; where those terms cancel (a row with two
keys, a key that few rows keep) the element is small and the error is not.  The check, per tensor:
  - every element: |gpu - ref| <= 2e-2 |ref| + 8e-2 rms(ref)
  - 99.9 % of the elements: |gpu - ref| - 2e-2 |ref| <= 1.5e-2 rms(ref)
  - relative Frobenius error below 1e-2.
(Measured on B200: worst element 4.2 % of rms, 99.9th percentile 0.5 %, Frobenius 0.25 %; a wrong
sign, a dropped term or a misplaced row is an O(1) Frobenius error.)"""
import dataclasses

import numpy as np
import pytest

import sfa_workloads as W
from tests.parity import upload_prefill, dev_tensor

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sfa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_flashattention_b200 as m
    return m


def assert_grad_close(gpu, ref, what):
    g = gpu.float().cpu().numpy().astype(np.float64)
    ref = np.asarray(ref, np.float64)
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    if ref.size == 0:
        return
    rms = float(np.sqrt(np.mean(ref * ref)))
    excess = np.abs(g - ref) - 2e-2 * np.abs(ref)
    worst = np.unravel_index(np.argmax(excess), excess.shape)
    assert excess.max() <= 8e-2 * rms, \
        f"{what}: excess {excess.max():.4g} (rms {rms:.4g}) at {worst}: gpu {g[worst]} ref {ref[worst]}"
    p999 = np.percentile(np.maximum(excess, 0), 99.9)
    assert p999 <= 1.5e-2 * rms, f"{what}: 99.9th percentile excess {p999:.4g} (rms {rms:.4g})"
    rel = np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-30)
    assert rel < 1e-2, f"{what}: relative Frobenius error {rel:.4g}"


def _run(sfa, c, dd, dout, status=None):
    kw = dict(cu_seqlens_k=dd["cu_k"], max_seqlen_q=c.max_sq, max_seqlen_k=c.max_sk, causal=bool(c.causal),
              window=(c.wl, c.wr))
    out, lse = sfa.fwd(dd["q"], dd["k"], dd["v"], dd["cu_q"], dd["sel"], c.bs, **kw)
    dq, dk, dv = sfa.bwd(dd["q"], dd["k"], dd["v"], out, dout, lse, dd["cu_q"], dd["sel"], c.bs, status=status, **kw)
    return dq, dk, dv


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
}


@pytest.mark.parametrize("name", sorted(BWD_CASES))
def test_bwd_parity(sfa, oracle_lib, name):
    c = BWD_CASES[name]()
    rng = np.random.default_rng(len(name))
    dout_bits = W.f32_to_bf16_bits(rng.standard_normal((c.total_q, c.Hq, c.d), dtype=np.float32))
    dd = upload_prefill(c)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq, dk, dv = _run(sfa, c, dd, dev_tensor(dout_bits, torch.bfloat16), status)
    assert sfa.last_launch_count() == 7
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rq, rk, rv, bad = oracle_lib.bwd(c, dout_bits)
    assert bad == 0
    assert_grad_close(dq, rq, "dq")
    assert_grad_close(dk, rk, "dk")
    assert_grad_close(dv, rv, "dv")


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
    a = _run(sfa, c, dd, dout)
    b = _run(sfa, c, dd, dout)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    dq = a[0]
    assert (dq[5:40] == 0).all() and (dq[1510] == 0).all()
    rq, rk, rv, _ = oracle_lib.bwd(c, dout_bits)
    assert_grad_close(a[0], rq, "dq")
    assert_grad_close(a[1], rk, "dk")
    assert_grad_close(a[2], rv, "dv")


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
    """d = 64 or block_size = 32 are outside the backward of this build: an error, no launch."""
    q = torch.zeros((8, 2, 64), dtype=torch.bfloat16, device="cuda")
    cu = torch.tensor([0, 8], dtype=torch.int32, device="cuda")
    sel = torch.zeros((8, 2, 1), dtype=torch.int32, device="cuda")
    lse = torch.zeros((2, 8), dtype=torch.float32, device="cuda")
    with pytest.raises(sfa.SfaError):
        sfa.bwd(q, q, q, q, q, lse, cu, sel, 64)
