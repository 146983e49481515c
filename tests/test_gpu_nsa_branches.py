"""GPU parity of the NSA branches beside the selected attention, through the C ABI: the sliding-window
branch (sfa_window_fwd) against the fp64 oracle given every block of the sequence (the oracle then
computes plain attention under the causal / window mask), and bitwise against sfa_fwd on that same
all-blocks selection; the gated mix (sfa_gated_combine) against the oracle's float64 sum."""
import dataclasses

import numpy as np
import pytest

import sfa_workloads as W
from tests.parity import assert_empty_rows_exact, assert_lse_close, assert_out_close, dev_tensor, upload_prefill

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sfa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_flashattention_b200 as m
    return m


def _case(seqlens_q, seqlens_k, Hq, Hkv, d, causal, wl, wr, seed):
    """Random q/k/v and, for the oracle and sfa_fwd, a selection of every 64-key block."""
    rng = np.random.default_rng(seed)
    tq, tk = int(sum(seqlens_q)), int(sum(seqlens_k))
    q = W.f32_to_bf16_bits(rng.standard_normal((tq, Hq, d), dtype=np.float32))
    k = W.f32_to_bf16_bits(rng.standard_normal((tk, Hkv, d), dtype=np.float32))
    v = W.f32_to_bf16_bits(rng.standard_normal((tk, Hkv, d), dtype=np.float32))
    nblk = (max(seqlens_k) + 63) // 64
    sel = np.broadcast_to(np.arange(nblk, dtype=np.int32), (tq, Hkv, nblk)).copy()
    return W.PrefillCase("w", q, k, v, W._cu(seqlens_q), W._cu(seqlens_k), sel, Hq, Hkv, d, 64, nblk, causal, wl, wr,
                         0.0)


WINDOW_CASES = [
    # lengths q, lengths k, Hq, Hkv, d, causal, window_left, window_right
    ([1024, 517, 300, 77], [1024, 517, 300, 77], 16, 4, 128, 1, 512, 0),  # the NSA window branch
    ([1024, 517, 300, 77], [1024, 517, 300, 77], 16, 4, 128, 1, -1, -1),  # plain causal attention
    ([200, 64], [700, 64], 8, 2, 128, 1, 128, 0),                         # sq != sk, bottom-right
    ([333], [333], 6, 2, 64, 0, 64, 32),                                   # two-sided local window, G 3
    ([129, 1], [129, 1], 4, 4, 128, 0, -1, -1),                            # full attention, G 1
    ([5], [2], 2, 1, 64, 1, -1, -1),                                       # docstring example: rows 0-2 empty
]


@pytest.mark.parametrize("lq,lk,Hq,Hkv,d,causal,wl,wr", WINDOW_CASES)
def test_window_fwd_parity(sfa, oracle_lib, lq, lk, Hq, Hkv, d, causal, wl, wr):
    c = _case(lq, lk, Hq, Hkv, d, causal, wl, wr, seed=sum(lq) + Hq + d + wl)
    dd = upload_prefill(c)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = sfa.window_fwd(dd["q"], dd["k"], dd["v"], dd["cu_q"], cu_seqlens_k=dd["cu_k"], max_seqlen_q=max(lq),
                              max_seqlen_k=max(lk), causal=bool(causal), window=(wl, wr), status=status)
    assert sfa.last_launch_count() == 1
    ro, rl, _ = oracle_lib.fwd(c)
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
    ninf = np.isneginf(rl)
    if ninf.any():
        h, t = np.where(ninf)
        assert_empty_rows_exact(out[torch.as_tensor(t), torch.as_tensor(h)], lse[torch.as_tensor(h), torch.as_tensor(t)])
    assert int(status.item()) == 0
    # The same attention through the selected path, every block selected: same blocks, same masks.
    o2, l2 = sfa.fwd(dd["q"], dd["k"], dd["v"], dd["cu_q"], dd["sel"], 64, cu_seqlens_k=dd["cu_k"],
                     max_seqlen_q=max(lq), max_seqlen_k=max(lk), causal=bool(causal), window=(wl, wr))
    assert torch.equal(out, o2) and torch.equal(lse, l2)


def test_window_fwd_empty_batch(sfa):
    q = torch.zeros((0, 4, 64), dtype=torch.bfloat16, device="cuda")
    cu = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = sfa.window_fwd(q, q[:, :1], q[:, :1], cu, max_seqlen_q=0, max_seqlen_k=0)
    assert out.shape == (0, 4, 64) and lse.shape == (4, 0)


@pytest.mark.parametrize("d,nb", [(128, 3), (64, 2)])
def test_gated_combine_parity(sfa, oracle_lib, d, nb):
    rng = np.random.default_rng(d + nb)
    total_q, Hq = 777, 16
    os_ = [W.f32_to_bf16_bits(rng.standard_normal((total_q, Hq, d), dtype=np.float32)) for _ in range(nb)]
    gs = [rng.random((total_q, Hq), dtype=np.float32) for _ in range(nb)]
    br = [(dev_tensor(o, torch.bfloat16), dev_tensor(g)) for o, g in zip(os_, gs)]
    if nb == 2:
        br = [None] + br  # compressed branch left out
    out = sfa.gated_combine(br)
    assert sfa.last_launch_count() == 1
    assert_out_close(out, oracle_lib.gated_combine(list(zip(os_, gs))))


def test_gated_combine_one_hot_is_the_branch(sfa):
    rng = np.random.default_rng(3)
    total_q, Hq, d = 100, 8, 128
    os_ = [dev_tensor(W.f32_to_bf16_bits(rng.standard_normal((total_q, Hq, d), dtype=np.float32)), torch.bfloat16)
           for _ in range(3)]
    zero = torch.zeros((total_q, Hq), dtype=torch.float32, device="cuda")
    one = torch.ones((total_q, Hq), dtype=torch.float32, device="cuda")
    out = sfa.gated_combine([(os_[0], zero), (os_[1], one), (os_[2], zero)])
    assert torch.equal(out, os_[1])


FLEX_CASES = [
    # lengths q, lengths k, Hq, Hkv, d, causal, per-head left windows, per-head right windows (None: scalar -1)
    ([700, 130, 64], [700, 130, 64], 8, 2, 128, 1, [0, 16, 64, 512, -1, 100, 7, 300], None),
    ([257, 90], [400, 90], 6, 2, 64, 0, [0, 33, -1, 64, 5, 128], [0, 5, -1, 70, 64, 1]),
    ([300], [300], 4, 4, 128, 0, None, [0, 64, 200, -1]),
]


@pytest.mark.parametrize("lq,lk,Hq,Hkv,d,causal,wlh,wrh", FLEX_CASES)
def test_window_fwd_per_head_windows(sfa, oracle_lib, lq, lk, Hq, Hkv, d, causal, wlh, wrh):
    """Flex local windows: each query head takes its own window; head h must equal the oracle run
    with head h's window for every head."""
    c = _case(lq, lk, Hq, Hkv, d, causal, -1, -1, seed=sum(lq) + Hq + 7)
    dd = upload_prefill(c)
    wl = torch.tensor(wlh, dtype=torch.int32, device="cuda") if wlh is not None else None
    wr = torch.tensor(wrh, dtype=torch.int32, device="cuda") if wrh is not None else None
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = sfa.window_fwd(dd["q"], dd["k"], dd["v"], dd["cu_q"], cu_seqlens_k=dd["cu_k"], max_seqlen_q=max(lq),
                              max_seqlen_k=max(lk), causal=bool(causal), window_per_head=(wl, wr), status=status)
    assert int(status.item()) == 0
    for h in range(Hq):
        ch = dataclasses.replace(c, wl=wlh[h] if wlh is not None else -1, wr=wrh[h] if wrh is not None else -1)
        ro, rl, _ = oracle_lib.fwd(ch)
        assert_out_close(out[:, h:h + 1], ro[:, h:h + 1])
        assert_lse_close(lse[h:h + 1], rl[h:h + 1])


def test_window_fwd_uniform_per_head_equals_scalar(sfa):
    """Per-head arrays holding one value for every head give the scalar-window result bit for bit."""
    c = _case([600, 77], [600, 77], 8, 2, 128, 1, 256, 0, seed=11)
    dd = upload_prefill(c)
    kw = dict(cu_seqlens_k=dd["cu_k"], max_seqlen_q=600, max_seqlen_k=600, causal=True)
    o1, l1 = sfa.window_fwd(dd["q"], dd["k"], dd["v"], dd["cu_q"], window=(256, 0), **kw)
    wl = torch.full((8,), 256, dtype=torch.int32, device="cuda")
    wr = torch.zeros(8, dtype=torch.int32, device="cuda")
    o2, l2 = sfa.window_fwd(dd["q"], dd["k"], dd["v"], dd["cu_q"], window_per_head=(wl, wr), **kw)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
