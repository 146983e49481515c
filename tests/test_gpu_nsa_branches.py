"""GPU parity of the NSA branches beside the selected attention, through the C ABI: the sliding-window
branch (sfa_window_fwd) against the fp64 oracle given every block of the sequence (the oracle then
computes plain attention under the causal / window mask), and bitwise against sfa_fwd on that same
all-blocks selection; the gated mix (sfa_gated_combine) against the oracle's float64 sum."""
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
