"""GPU parity of the in-place paged KV-cache append (sfa_kv_append) against oracle.kv_append: bit-exact
cache contents (a copy, no arithmetic); a decode over the appended cache against the oracle decode
of the oracle-appended cache; positions past the block table and invalid page ids flagged and not
written."""
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


def _new_rows(rng, B, S, Hkv, d):
    return W.f32_to_bf16_bits(rng.standard_normal((B, S, Hkv, d), dtype=np.float32))


@pytest.mark.parametrize("S,d,page", [(3, 128, 256), (1, 64, 16), (5, 128, 64)])
def test_kv_append_bitwise(sfa, S, d, page):
    c = W.make_decode(31 + S, 5, 8, 2, d, page, 40, 900, 32, 4)
    rng = np.random.default_rng(S)
    kn, vn = _new_rows(rng, c.B, S, c.Hkv, d), _new_rows(rng, c.B, S, c.Hkv, d)
    lens = np.maximum(c.cache_seqlens - S, 0).astype(np.int32)  # rewrite each sequence's last S positions
    dd = upload_decode(c)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sfa.kv_append(dev_tensor(kn, torch.bfloat16), dev_tensor(vn, torch.bfloat16), dd["k_cache"], dd["v_cache"],
                  dd["block_table"], dev_tensor(lens), status=st)
    assert sfa.last_launch_count() == 1
    rk, rv, bad = oracle.kv_append(c.k_cache, c.v_cache, c.block_table, lens, kn, vn)
    assert bad == 0 and int(st.item()) == 0
    np.testing.assert_array_equal(dd["k_cache"].view(torch.int16).cpu().numpy().view(np.uint16), rk)
    np.testing.assert_array_equal(dd["v_cache"].view(torch.int16).cpu().numpy().view(np.uint16), rv)


def test_decode_after_append(sfa):
    """Decode step with append: the new token's key / value written at position L - 1 (the query's own
    position), then the decode over length L sees them."""
    c = W.make_decode(41, 4, 32, 8, 128, 256, 700, 3000, 256, 32)
    rng = np.random.default_rng(9)
    kn, vn = _new_rows(rng, c.B, 1, c.Hkv, c.d), _new_rows(rng, c.B, 1, c.Hkv, c.d)
    pos = (c.cache_seqlens - 1).astype(np.int32)
    dd = upload_decode(c)
    sfa.kv_append(dev_tensor(kn, torch.bfloat16), dev_tensor(vn, torch.bfloat16), dd["k_cache"], dd["v_cache"],
                  dd["block_table"], dev_tensor(pos))
    out, lse = run_decode(sfa, c, dd)
    rk, rv, _ = oracle.kv_append(c.k_cache, c.v_cache, c.block_table, pos, kn, vn)
    ro, rl, bad = oracle.decode(dataclasses.replace(c, k_cache=rk, v_cache=rv))
    assert not np.asarray(bad).any()
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


def test_kv_append_out_of_table_and_bad_page(sfa):
    """A position past the block table sets SFA_DEV_BAD_SEQLEN (8), a page id outside [0, num_pages)
    sets SFA_DEV_BAD_PAGE (2); neither is written, the other rows are."""
    c = W.make_decode(51, 3, 4, 2, 64, 16, 40, 60, 8, 2)
    bt = c.block_table.copy()
    assert bt.shape[1] == 4
    bt[0, 3] = bt[0, 0]  # a valid page for sequence 0's last table entry (its row 15 is otherwise unused here)
    lens = np.array([4 * 16 - 1, 0, 0], np.int32)  # sequence 0: its 2nd new row is past the table
    bt[2, 0] = c.num_pages + 7                                          # sequence 2: invalid page id
    rng = np.random.default_rng(3)
    kn, vn = _new_rows(rng, 3, 2, 2, 64), _new_rows(rng, 3, 2, 2, 64)
    dd = upload_decode(c)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sfa.kv_append(dev_tensor(kn, torch.bfloat16), dev_tensor(vn, torch.bfloat16), dd["k_cache"], dd["v_cache"],
                  dev_tensor(bt), dev_tensor(lens), status=st)
    rk, rv, bad = oracle.kv_append(c.k_cache, c.v_cache, bt, lens, kn, vn)
    assert bad == 3  # one row of sequence 0, both rows of sequence 2
    assert int(st.item()) == 8 | 2
    np.testing.assert_array_equal(dd["k_cache"].view(torch.int16).cpu().numpy().view(np.uint16), rk)
    np.testing.assert_array_equal(dd["v_cache"].view(torch.int16).cpu().numpy().view(np.uint16), rv)
