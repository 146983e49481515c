"""GPU parity of sfa_index_topk: bit-exact
selections against oracle.index_topk (exact scores make the set unique), and the decode fed by the
indexer against the oracle decode with the oracle's selection."""
import dataclasses

import numpy as np
import pytest

import oracle
import sfa_workloads as W
from tests.parity import assert_lse_close, assert_out_close, dev_tensor, run_decode, upload_decode

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sfa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_flashattention_b200 as m
    return m


@pytest.mark.parametrize("B,Hq,Hkv,d,page,lo,hi,topk,nl,keys", [
    (3, 8, 2, 64, 16, 10, 700, 64, 4, "normal"),
    (2, 32, 8, 128, 256, 700, 3000, 256, 32, "normal"),
    (4, 4, 4, 128, 64, 1, 300, 300, 0, "normal"),     # topk >= L for some sequences
    (2, 8, 2, 128, 16, 100, 900, 50, 3, "ties"),      # many exact ties
    (2, 8, 2, 128, 64, 500, 2000, 100, 4, "tiny"),    # keys mostly E4M3 subnormals (below 2^-6)
    (2, 8, 2, 64, 64, 500, 2000, 100, 4, "huge"),     # keys often past 448: saturated
    (3, 8, 4, 128, 100, 300, 2500, 128, 8, "normal"), # page not a multiple of a warp's 8 rows
])
def test_index_topk_bitwise(sfa, B, Hq, Hkv, d, page, lo, hi, topk, nl, keys):
    c = W.make_decode(200 + topk, B, Hq, Hkv, d, page, lo, hi, 8, 2)
    scale = {"normal": None, "ties": None, "tiny": 2.0 ** -8, "huge": 300.0}[keys]
    kf = W.bf16_bits_to_f32(c.k_cache)
    if keys == "ties":
        c = dataclasses.replace(c, k_cache=W.f32_to_bf16_bits(np.round(kf)))
    elif scale is not None:
        c = dataclasses.replace(c, k_cache=W.f32_to_bf16_bits(kf * np.float32(scale)))
    dd = upload_decode(c)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sel = sfa.index_topk(dd["q"], dd["k_cache"], dd["block_table"], dd["cache_seqlens"], topk, n_local=nl, status=st)
    assert sfa.last_launch_count() == 2 and int(st.item()) == 0
    want, _, bad = oracle.index_topk(c.q, c.k_cache, c.block_table, c.cache_seqlens, Hkv, topk, n_local=nl)
    assert bad == 0
    np.testing.assert_array_equal(sel.cpu().numpy(), want)


def test_indexer_then_decode(sfa):
    c = W.make_decode(300, 4, 32, 8, 128, 256, 700, 3000, 256, 32)
    dd = upload_decode(c)
    sel = sfa.index_topk(dd["q"], dd["k_cache"], dd["block_table"], dd["cache_seqlens"], 256, n_local=32)
    out, lse = run_decode(sfa, c, dd, sel=sel)
    want, _, _ = oracle.index_topk(c.q, c.k_cache, c.block_table, c.cache_seqlens, c.Hkv, 256, n_local=32)
    ro, rl, _ = oracle.decode(dataclasses.replace(c, sel=want))
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


def test_index_topk_full_length(sfa):
    """At the cache lengths the benchmark scores (L ~ U[100000, 131072], page 256, d 128, G 4): 25 to
    32 scoring CTAs per (sequence, kv head), and a selection CTA whose 1024 threads take about 128
    positions each per pass: the selection is still the oracle's, bit for bit."""
    c = W.make_decode(410, 2, 8, 2, 128, 256, 100000, 131072, 8, 2)
    assert int(np.asarray(c.cache_seqlens).min()) >= 100000
    dd = upload_decode(c)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sel = sfa.index_topk(dd["q"], dd["k_cache"], dd["block_table"], dd["cache_seqlens"], 2048, n_local=128, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    want, _, bad = oracle.index_topk(c.q, c.k_cache, c.block_table, c.cache_seqlens, c.Hkv, 2048, n_local=128)
    assert bad == 0
    np.testing.assert_array_equal(sel.cpu().numpy(), want)
