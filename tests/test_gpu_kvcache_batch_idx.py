"""GPU parity of the non-paged cache entry points (sfa_decode_kvcache, sfa_kv_append_kvcache): caches
(batch_cache, seqlen_cache, Hkv, d) addressed through cache_batch_idx, as flash_attn_with_kvcache takes
them, against oracle.decode_kvcache / oracle.kv_append_kvcache, and bit for bit against the paged decode
of the same rows repacked into randomly placed pages."""
import numpy as np
import pytest

import oracle
import sfa_workloads as W
from tests.parity import assert_lse_close, assert_out_close, dev_tensor

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sfa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_flashattention_b200 as m
    return m


def _upload(c):
    return dict(q=dev_tensor(c.q, torch.bfloat16), k=dev_tensor(c.k_cache, torch.bfloat16),
                v=dev_tensor(c.v_cache, torch.bfloat16), idx=dev_tensor(c.cache_batch_idx),
                lens=dev_tensor(c.cache_seqlens), sel=dev_tensor(c.sel))


@pytest.mark.parametrize("B,batch_cache,seqlen_cache,Hq,Hkv,d,lo,hi,topk,last,wl", [
    (4, 7, 900, 8, 2, 64, 1, 900, 96, 8, -1),        # seqlen_cache not a power of two
    (3, 3, 2048, 32, 8, 128, 1500, 2048, 256, 32, 100),
    (2, 5, 4096, 4, 1, 128, 3000, 4096, 3000, 64, -1),  # selections past 2048 positions: the prep kernel
])
def test_decode_kvcache_parity(sfa, B, batch_cache, seqlen_cache, Hq, Hkv, d, lo, hi, topk, last, wl):
    c = W.make_decode_kvcache(70 + d + B, B, batch_cache, seqlen_cache, Hq, Hkv, d, lo, hi, topk, last)
    c.wl = wl
    t = _upload(c)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = sfa.decode_kvcache(t["q"], t["k"], t["v"], t["lens"], t["sel"], cache_batch_idx=t["idx"],
                                  window_left=wl, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ro, rl, bad = oracle.decode_kvcache(c.q, c.k_cache, c.v_cache, c.cache_seqlens, c.sel, c.cache_batch_idx,
                                        c.Hkv, c.softmax_scale, wl=wl)
    assert bad == 0
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
    # the same rows in pages of 64 at random places: the paged decode gives the same bits
    pc = W.kvcache_as_paged(c, 64, seed=B)
    po, pl = sfa.decode(t["q"], dev_tensor(pc.k_cache, torch.bfloat16), dev_tensor(pc.v_cache, torch.bfloat16),
                        dev_tensor(pc.block_table), t["lens"], t["sel"], window_left=wl)
    assert torch.equal(out, po) and torch.equal(lse, pl)


def test_decode_kvcache_default_index_and_bad_entry(sfa):
    c = W.make_decode_kvcache(81, 3, 3, 512, 8, 2, 64, 100, 512, 64, 4)
    t = _upload(c)
    # None: sequence b on entry b
    out, lse = sfa.decode_kvcache(t["q"], t["k"], t["v"], t["lens"], t["sel"])
    ident = np.arange(3, dtype=np.int32)
    ro, rl, _ = oracle.decode_kvcache(c.q, c.k_cache, c.v_cache, c.cache_seqlens, c.sel, ident, c.Hkv,
                                      c.softmax_scale)
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
    # an entry outside the cache: that sequence's rows are dropped and flagged
    idx = torch.tensor([0, 7, 2], dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = sfa.decode_kvcache(t["q"], t["k"], t["v"], t["lens"], t["sel"], cache_batch_idx=idx, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & 2  # SFA_DEV_BAD_PAGE
    assert bool((out[1] == 0).all()) and bool(torch.isneginf(lse[1]).all())
    ro, rl, _ = oracle.decode_kvcache(c.q, c.k_cache, c.v_cache, c.cache_seqlens, c.sel, idx.cpu().numpy(),
                                      c.Hkv, c.softmax_scale)
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


def test_kv_append_kvcache_bit_exact(sfa):
    c = W.make_decode_kvcache(91, 3, 5, 300, 8, 2, 128, 10, 280, 8, 2)
    rng = np.random.default_rng(5)
    kn = W.f32_to_bf16_bits(rng.standard_normal((3, 40, 2, 128), dtype=np.float32))
    vn = W.f32_to_bf16_bits(rng.standard_normal((3, 40, 2, 128), dtype=np.float32))
    t = _upload(c)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sfa.kv_append_kvcache(dev_tensor(kn, torch.bfloat16), dev_tensor(vn, torch.bfloat16), t["k"], t["v"],
                          t["lens"], cache_batch_idx=t["idx"], status=st)
    torch.cuda.synchronize()
    wk, wv, bad = oracle.kv_append_kvcache(c.k_cache, c.v_cache, c.cache_batch_idx, c.cache_seqlens, kn, vn)
    np.testing.assert_array_equal(t["k"].view(torch.int16).cpu().numpy().view(np.uint16), wk)
    np.testing.assert_array_equal(t["v"].view(torch.int16).cpu().numpy().view(np.uint16), wv)
    assert (int(st.item()) != 0) == (bad > 0)
