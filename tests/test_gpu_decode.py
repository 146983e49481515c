"""GPU parity of the paged top-k decode path (sfa_decode through the C ABI) against the oracle."""
import numpy as np
import pytest

import sfa_workloads as W
from tests.parity import assert_empty_rows_exact, assert_lse_close, assert_out_close, dev_tensor, run_decode, upload_decode

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sfa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_flashattention_b200 as m
    return m


def _parity(sfa, oracle_lib, c, status_expect=0, **kw):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = run_decode(sfa, c, status=status, **kw)
    ro, rl, _ = oracle_lib.decode(c)
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
    assert int(status.item()) == status_expect
    return out, lse


def test_small_decode_parity(sfa, oracle_lib):
    _parity(sfa, oracle_lib, W.small_config(5))


def test_decode_prep_bit_exact(sfa, oracle_lib):
    c = W.small_config(5)
    d = upload_decode(c)
    _, tok_c, cnt = sfa.decode_prep(d["cache_seqlens"], d["sel"], Hq=c.Hq, d=c.d, max_pages_per_seq=c.max_pages,
                                    page_size=c.page)
    rt, rc, _ = oracle_lib.decode_index(c)
    np.testing.assert_array_equal(cnt.cpu().numpy(), rc)
    np.testing.assert_array_equal(tok_c.cpu().numpy(), rt)


@pytest.mark.parametrize("splits", [1, 2, 3, 4, 8, 16])
def test_split_count_invariance(sfa, oracle_lib, splits):
    """Any number of key chunks merged through their LSEs gives the unsplit result."""
    c = W.small_config(5)
    out, lse = _parity(sfa, oracle_lib, c, num_splits=splits)


@pytest.mark.parametrize("B,Hq,Hkv,d,page,lo,hi,topk,last", [(3, 8, 8, 128, 64, 10, 900, 200, 16),
                                                              (5, 16, 2, 64, 16, 1, 333, 100, 8),
                                                              (2, 16, 1, 128, 256, 3000, 5000, 1000, 64),
                                                              (4, 4, 4, 64, 1, 5, 300, 64, 4)])
def test_decode_shapes(sfa, oracle_lib, B, Hq, Hkv, d, page, lo, hi, topk, last):
    c = W.make_decode(B * 7 + d + page, B, Hq, Hkv, d, page, lo, hi, topk, last)
    _parity(sfa, oracle_lib, c)


def test_decode_window(sfa, oracle_lib):
    c = W.small_config(5)
    c = W.DecodeCase(**{**c.__dict__, "wl": 500})
    _parity(sfa, oracle_lib, c)


def test_paging_invariance_bitwise(sfa):
    """The seeded permuted block table over the permuted pool == the identity table over
    contiguous pages, bit for bit."""
    c = W.small_config(5)
    out, lse = run_decode(sfa, c)
    npg = c.max_pages
    kc = np.zeros((c.B * npg, c.page, c.Hkv, c.d), np.uint16)
    vc = np.zeros_like(kc)
    bt = np.full((c.B, npg), -1, np.int32)
    for b in range(c.B):
        for p in range(npg):
            if c.block_table[b, p] >= 0:
                kc[b * npg + p] = c.k_cache[c.block_table[b, p]]
                vc[b * npg + p] = c.v_cache[c.block_table[b, p]]
                bt[b, p] = b * npg + p
    c2 = W.DecodeCase(**{**c.__dict__, "k_cache": kc, "v_cache": vc, "block_table": bt})
    o2, l2 = run_decode(sfa, c2)
    assert torch.equal(out, o2) and torch.equal(lse, l2)


def test_bad_page_and_bad_ids(sfa, oracle_lib):
    c = W.small_config(5)
    bt = c.block_table.copy()
    bt[1, 0] = c.num_pages + 3
    c2 = W.DecodeCase(**{**c.__dict__, "block_table": bt})
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = run_decode(sfa, c2, status=status)
    ro, rl, bad = oracle_lib.decode(c2)
    assert bad[1] > 0 and int(status.item()) & 2  # SFA_DEV_BAD_PAGE
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
    sel = c.sel.copy()
    sel[0, 0, 0] = c.cache_seqlens[0] + 5
    sel[2, 1, 3] = -9
    c3 = W.DecodeCase(**{**c.__dict__, "sel": sel})
    status.zero_()
    out, lse = run_decode(sfa, c3, status=status)
    ro, rl, bad = oracle_lib.decode(c3)
    assert bad[0] == 2 and int(status.item()) & 1
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


def test_all_padding_decode(sfa):
    c = W.small_config(5)
    out, lse = run_decode(sfa, c, sel=dev_tensor(np.full_like(c.sel, -1)))
    assert_empty_rows_exact(out, lse)


def _split_launches(sfa, c, num_splits=0):
    # split kernel, plus the combine kernel when the splits of a (sequence, kv head) span CTAs
    S = sfa.decode_num_splits(c.q.shape[0], c.Hq, c.Hkv, c.d, c.sel.shape[2], num_splits)
    return 1 if S <= 6 else 2


@pytest.mark.parametrize("splits", [0, 4, 6, 7, 16])
def test_decode_launch_count(sfa, splits):
    c = W.small_config(5)  # 256 positions per (sequence, kv head): deduplicated in the split kernel
    run_decode(sfa, c, num_splits=splits)
    assert sfa.last_launch_count() == _split_launches(sfa, c, splits)


def test_long_selection_goes_through_prep(sfa, oracle_lib):
    """More than 2048 selected positions per (sequence, kv head): prep kernel, then split + combine."""
    c = W.make_decode(77, 2, 8, 2, 128, 64, 6000, 9000, 3000, 64)
    _parity(sfa, oracle_lib, c)
    assert sfa.last_launch_count() == 1 + _split_launches(sfa, c)


@pytest.mark.parametrize("splits", [0, 3, 8])
def test_stages_equal_fused_call_bitwise(sfa, splits):
    """sfa_decode_prep + sfa_decode_attend (canonical sets through the workspace) and sfa_decode
    (deduplicated inside the split kernel) split the same sorted lists the same way: the outputs
    are bit-identical."""
    c = W.small_config(5)
    d = upload_decode(c)
    out1, lse1 = run_decode(sfa, c, d=d, num_splits=splits)
    ws = torch.empty(sfa.decode_workspace_size(c.q.shape[0], c.Hq, c.Hkv, c.d, c.sel.shape[2], splits),
                     dtype=torch.uint8, device="cuda")
    sfa.decode_prep(d["cache_seqlens"], d["sel"], Hq=c.Hq, d=c.d, max_pages_per_seq=c.max_pages, page_size=c.page,
                    window_left=c.wl, num_splits=splits, workspace=ws)
    out2, lse2 = sfa.decode_attend(d["q"], d["k_cache"], d["v_cache"], d["block_table"], ws, topk_tok=c.sel.shape[2],
                                   scale=c.scale if c.scale > 0 else None, num_splits=splits)
    torch.cuda.synchronize()
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    assert torch.equal(lse1, lse2)


def test_full_size_decode(sfa, oracle_lib):
    """The paged decode workload at full size (B32, Hq32/Hkv8, L up to 131072, 2048 tokens per
    (sequence, kv head)), in the launch configuration the benchmark times: every output row
    against the oracle, and the canonical token sets bit-exact."""
    c = W.config5()
    d = upload_decode(c)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = run_decode(sfa, c, d=d, status=status)
    ro, rl, _ = oracle_lib.decode(c)
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
    assert int(status.item()) == 0
    _, tok_c, cnt = sfa.decode_prep(d["cache_seqlens"], d["sel"], Hq=c.Hq, d=c.d, max_pages_per_seq=c.max_pages,
                                    page_size=c.page)
    rt, rc, _ = oracle_lib.decode_index(c)
    np.testing.assert_array_equal(cnt.cpu().numpy(), rc)
    np.testing.assert_array_equal(tok_c.cpu().numpy(), rt)


@pytest.mark.parametrize("d,L", [(64, 900000), (128, 1000000)])
def test_long_cache_dedupe_in_several_ranges(sfa, oracle_lib, d, L):
    """Caches close to the 2^20-position limit: the split kernel deduplicates the selection one
    position range at a time (several ranges at these lengths)."""
    c = W.make_decode(d + 3, 1, 4, 1, d, 256, L, L, 2048, 64, parallel_values=True)
    _parity(sfa, oracle_lib, c)


def test_largest_selection(sfa, oracle_lib):
    """topk_tok = 65536, the largest this build takes (prep kernel path)."""
    c = W.make_decode(11, 1, 2, 1, 64, 128, 70000, 70000, 65536, 128, parallel_values=True)
    _parity(sfa, oracle_lib, c)


def test_decode_captured_in_cuda_graph(sfa):
    """The decode call allocates nothing and never synchronises the host, so it can be captured in a
    CUDA graph (as the Flash-Sparse-Attention README's decode example does) and replayed: the replay
    gives the eager call's bits, also after the inputs change in place."""
    c = W.small_config(5)
    d = upload_decode(c)
    B, Hq, dd = c.q.shape
    ws = torch.empty(sfa.decode_workspace_size(B, Hq, c.Hkv, dd, c.sel.shape[2]), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(d["q"])
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")

    def call():
        sfa.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["cache_seqlens"], d["sel"], out=out,
                   lse=lse, workspace=ws, window_left=c.wl, scale=c.scale if c.scale > 0 else None)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(2):
            call()
    torch.cuda.current_stream().wait_stream(s)
    ref_out, ref_lse = out.clone(), lse.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
    assert torch.equal(lse, ref_lse)
    # new query values in place: the replay follows them
    d["q"].copy_(torch.flip(d["q"], dims=[0]))
    call()
    torch.cuda.synchronize()
    eager = out.clone()
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), eager.view(torch.int16))
