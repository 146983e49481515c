"""GPU parity of the prefill path (sfa_fwd through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest

import sfa_workloads as W
from tests.parity import (assert_empty_rows_exact, assert_lse_close, assert_out_close, dev_tensor, run_fwd,
                          upload_prefill)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sfa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_flashattention_b200 as m
    return m


def _case(seqlens_q, seqlens_k, Hq, Hkv, d, bs, sel, seed, causal=1, wl=-1, wr=-1, scale=0.0):
    rng = np.random.default_rng(seed)
    tq, tk = int(sum(seqlens_q)), int(sum(seqlens_k))
    q = W.f32_to_bf16_bits(rng.standard_normal((tq, Hq, d), dtype=np.float32))
    k = W.f32_to_bf16_bits(rng.standard_normal((tk, Hkv, d), dtype=np.float32))
    v = W.f32_to_bf16_bits(rng.standard_normal((tk, Hkv, d), dtype=np.float32))
    return W.PrefillCase("t", q, k, v, W._cu(seqlens_q), W._cu(seqlens_k), np.asarray(sel, np.int32), Hq, Hkv, d, bs,
                         sel.shape[-1], causal, wl, wr, scale)


def _all_blocks(total_q, Hkv, nblk, rng=None):
    s = np.broadcast_to(np.arange(nblk, dtype=np.int32), (total_q, Hkv, nblk)).copy()
    if rng is not None:
        s = W._shuffle_rows(rng, s.reshape(-1, nblk)).reshape(s.shape)
    return s


def _full_parity(sfa, oracle_lib, c):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = run_fwd(sfa, c, status=status)
    ro, rl, bad = oracle_lib.fwd(c)
    status_expect = 1 if bad else 0  # SFA_DEV_BAD_INDEX iff the oracle met out-of-range ids
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
    ninf = np.isneginf(rl)  # (Hq, total_q)
    if ninf.any():
        h, t = np.where(ninf)
        assert_empty_rows_exact(out[torch.as_tensor(t), torch.as_tensor(h)], lse[torch.as_tensor(h), torch.as_tensor(t)])
    assert int(status.item()) == status_expect
    return out, lse


@pytest.mark.parametrize("n", [1, 2, 3, 4])
def test_small_configs_full_parity(sfa, oracle_lib, n):
    """Oracle-sized versions of the four prefill workloads: every output element."""
    _full_parity(sfa, oracle_lib, W.small_config(n))


@pytest.mark.parametrize("n", [1, 2, 3, 4])
def test_index_prep_bit_exact(sfa, oracle_lib, n):
    c = W.small_config(n)
    d = upload_prefill(c)
    _, sel_c, cnt = sfa.fwd_prep(d["cu_q"], d["sel"], Hq=c.Hq, d=c.d, block_size=c.bs, cu_seqlens_k=d["cu_k"],
                                 max_seqlen_q=c.max_sq, max_seqlen_k=c.max_sk, causal=bool(c.causal),
                                 window=(c.wl, c.wr))
    rs, rc, _ = oracle_lib.fwd_index(c)
    np.testing.assert_array_equal(sel_c.cpu().numpy(), rs)
    np.testing.assert_array_equal(cnt.cpu().numpy(), rc)


def _sample_rows(c, n, seed):
    rng = np.random.default_rng(seed)
    rows = set(rng.integers(0, c.total_q * c.Hq, size=n).tolist())
    for b in range(c.batch):  # first and last token of every sequence, every head
        for t in (c.cu_q[b], c.cu_q[b + 1] - 1):
            rows.update(int(t) * c.Hq + h for h in range(c.Hq))
    return np.asarray(sorted(rows), np.int64)


FULL = {1: W.config1, 2: W.config2, 3: W.config3, 4: W.config4}


@pytest.mark.parametrize("n", [1, 2, 3, 4])
def test_full_size_configs_sampled(sfa, oracle_lib, n):
    """The four prefill workloads at full size, in the launch configuration the benchmark
    times: every row computed on the GPU, a sample of rows (plus every sequence's first and
    last token) checked against the oracle; the whole canonical index set bit-exact."""
    c = FULL[n]()
    d = upload_prefill(c)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = run_fwd(sfa, c, d=d, status=status)
    rows = _sample_rows(c, 3000, n)
    ro, rl, _ = oracle_lib.fwd(c, rows=rows)
    t, h = rows // c.Hq, rows % c.Hq
    assert_out_close(out.view(-1, c.d)[torch.as_tensor(rows, device="cuda")], ro)
    assert_lse_close(lse[torch.as_tensor(h, device="cuda"), torch.as_tensor(t, device="cuda")], rl)
    assert int(status.item()) == 0
    _, sel_c, cnt = sfa.fwd_prep(d["cu_q"], d["sel"], Hq=c.Hq, d=c.d, block_size=c.bs, cu_seqlens_k=d["cu_k"],
                                 max_seqlen_q=c.max_sq, max_seqlen_k=c.max_sk, causal=bool(c.causal),
                                 window=(c.wl, c.wr))
    rs, rc, _ = oracle_lib.fwd_index(c)
    np.testing.assert_array_equal(cnt.cpu().numpy(), rc)
    np.testing.assert_array_equal(sel_c.cpu().numpy(), rs)
    o = out.float()
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()


@pytest.mark.parametrize("sq,sk", [(2, 5), (5, 2), (70, 200), (200, 70)])
def test_bottom_right_causal_and_empty_rows(sfa, oracle_lib, sq, sk):
    """Unequal lengths (the printed 2x5 and 5x2 examples and larger ones): rows whose causal
    limit is below key 0 output exactly 0 with lse -inf."""
    bs = 32
    nblk = -(-sk // bs)
    c = _case([sq, sq], [sk, sk], 4, 2, 64, bs, _all_blocks(2 * sq, 2, nblk, np.random.default_rng(0)), 3)
    _full_parity(sfa, oracle_lib, c)


@pytest.mark.parametrize("Hq,Hkv,d,bs", [(6, 2, 64, 32), (6, 2, 128, 64), (8, 8, 128, 64), (16, 2, 64, 64),
                                         (32, 2, 128, 32), (1, 1, 64, 64), (128, 1, 64, 32)])
def test_gqa_groups_and_shapes(sfa, oracle_lib, Hq, Hkv, d, bs):
    """GQA groups G = 3 (the 6->2 example), 1, 8, 16, 128 with d 64/128 and block 32/64, on
    ragged sequences with an NSA selection."""
    lens = [300, 1, 77, 129]
    c = W.make_nsa_prefill(Hq * 100 + Hkv + d + bs, lens, Hq, Hkv, d, bs, 6, 1, 2)
    _full_parity(sfa, oracle_lib, c)


@pytest.mark.parametrize("causal,wl,wr", [(0, -1, -1), (0, 40, 30), (1, 100, 0), (0, 0, 0), (1, 0, -1)])
def test_windows(sfa, oracle_lib, causal, wl, wr):
    sq, sk, bs = 150, 260, 64
    nblk = -(-sk // bs)
    c = _case([sq, 90], [sk, 100], 8, 2, 128, bs, _all_blocks(sq + 90, 2, nblk, np.random.default_rng(1)), 5,
              causal=causal, wl=wl, wr=wr)
    _full_parity(sfa, oracle_lib, c)


def test_window_minus1_0_equals_causal_bitwise(sfa):
    c = W.small_config(2)
    a, la = run_fwd(sfa, c)
    c2 = W.PrefillCase(**{**c.__dict__, "causal": 0, "wl": -1, "wr": 0})
    b, lb = run_fwd(sfa, c2)
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_selection_is_a_set_bitwise(sfa, oracle_lib):
    """Permuted and duplicated slots give bit-identical outputs (the kernel sees only the
    canonical set)."""
    c = W.small_config(4)
    base, lbase = run_fwd(sfa, c)
    rng = np.random.default_rng(3)
    sel = W._shuffle_rows(rng, c.sel.reshape(-1, c.topk)).reshape(c.sel.shape).copy()
    flat = sel.reshape(-1, c.topk)
    for r in range(flat.shape[0]):
        valid = flat[r][flat[r] >= 0]
        pads = np.where(flat[r] < 0)[0]
        if valid.size and pads.size:
            flat[r, pads] = rng.choice(valid, size=pads.size)
    out, lse = run_fwd(sfa, c, sel=dev_tensor(sel))
    assert torch.equal(out, base) and torch.equal(lse, lbase)


def test_bad_ids_flagged_and_ignored(sfa, oracle_lib):
    c = W.small_config(2)
    base, lbase = run_fwd(sfa, c)
    sel = c.sel.copy()
    idx = np.argwhere(sel == -1)[:50]
    sel[idx[:, 0], idx[:, 1], idx[:, 2]] = np.where(np.arange(len(idx)) % 2 == 0, 10 ** 6, -7)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = run_fwd(sfa, c, sel=dev_tensor(sel), status=status)
    assert int(status.item()) & 1  # SFA_DEV_BAD_INDEX
    assert torch.equal(out, base) and torch.equal(lse, lbase)


def test_all_padding_rows(sfa):
    """A selection of only -1 slots: every row is empty."""
    c = W.small_config(2)
    sel = np.full_like(c.sel, -1)
    out, lse = run_fwd(sfa, c, sel=dev_tensor(sel))
    assert_empty_rows_exact(out, lse)


def test_rows_sum_to_one(sfa):
    """v == 1: every non-empty row outputs 1 within the bf16 tolerance."""
    c = W.small_config(4)
    c = W.PrefillCase(**{**c.__dict__, "v": np.full_like(c.v, 0x3F80)})
    out, _ = run_fwd(sfa, c)
    assert_out_close(out, np.ones(out.shape))


def test_empty_batch_and_explicit_scale(sfa, oracle_lib):
    c = W.small_config(1)
    c = W.PrefillCase(**{**c.__dict__, "scale": 0.3})
    _full_parity(sfa, oracle_lib, c)
    q = torch.empty((0, 4, 64), dtype=torch.bfloat16, device="cuda")
    cu = torch.zeros(2, dtype=torch.int32, device="cuda")
    sel = torch.empty((0, 1, 4), dtype=torch.int32, device="cuda")
    out, lse = sfa.fwd(q, q[:, :1], q[:, :1], cu, sel, 32, max_seqlen_q=0, max_seqlen_k=0)
    assert out.shape == (0, 4, 64) and lse.shape == (4, 0)


@pytest.mark.parametrize("n", [1, 2, 3])
def test_launch_count_and_stages(sfa, oracle_lib, n):
    """sfa_fwd without the block-major schedule is one kernel that canonicalizes the selections
    itself; with it, prep (3 kernels) + attend (3: query-major, block-major, merge).  The split-stage
    calls (prep kernel, then attention on its canonical sets) give bitwise the same result, and the
    same status word."""
    c = W.small_config(n)
    d = upload_prefill(c)
    st1 = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = run_fwd(sfa, c, d=d, status=st1)
    assert sfa.last_launch_count() == 1  # these sequences hold at most 10*topk blocks: no block-major plan
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    kw = dict(cu_seqlens_k=d["cu_k"], max_seqlen_q=c.max_sq, max_seqlen_k=c.max_sk, causal=bool(c.causal),
              window=(c.wl, c.wr), status=st2)
    ws, _, _ = sfa.fwd_prep(d["cu_q"], d["sel"], Hq=c.Hq, d=c.d, block_size=c.bs, **kw)
    o2, l2 = sfa.fwd_attend(d["q"], d["k"], d["v"], d["cu_q"], ws, topk=c.topk, block_size=c.bs,
                            scale=c.scale if c.scale > 0 else None, **kw)
    assert torch.equal(out, o2) and torch.equal(lse, l2)
    assert int(st1.item()) == int(st2.item())


def _block_major_windows(c, oracle_lib):
    """How many (window, sequence, kv head) groups the prep will send to the block-major kernel:
    the union of a window's query-tile block sets exceeds 4x the window's selected blocks."""
    sel_c, cnt, _ = oracle_lib.fwd_index(c)
    G = c.Hq // c.Hkv
    Tq = 128 // G
    W = Tq * 64
    n = 0
    for b in range(c.batch):
        q0, sq = c.cu_q[b], c.cu_q[b + 1] - c.cu_q[b]
        for hk in range(c.Hkv):
            for w0 in range(0, sq, W):
                useful = int(cnt[q0 + w0:q0 + min(sq, w0 + W), hk].sum())
                union = 0
                for t0 in range(w0, min(sq, w0 + W), Tq):
                    t1 = min(sq, t0 + Tq)
                    blocks = set(sel_c[q0 + t0:q0 + t1, hk].ravel().tolist()) - {-1}
                    union += len(blocks) * (t1 - t0)
                n += union > 4 * useful
    return n


@pytest.mark.parametrize("Hq,Hkv,d,bs,topk,lens", [(16, 4, 128, 64, 6, [12000, 300]),
                                                   (2, 2, 64, 32, 6, [9000, 77]),
                                                   (8, 2, 128, 32, 8, [8000]),
                                                   (6, 2, 64, 64, 5, [10000, 1000]),
                                                   (8, 2, 64, 32, 40, [20000])])
def test_block_major_windows(sfa, oracle_lib, Hq, Hkv, d, bs, topk, lens):
    """Long sequences with a small random top-k: late windows' query tiles select unions of
    blocks over 10x their selected work, so those windows go to the block-major kernel (items of
    one block and the tokens that selected it, bf16 partials, merge kernel) while early windows
    stay query-major.  The blocks most of a block-major tile selects (the forced initial and local
    ones) run query-major for the tile and join the merge as one more partial; with topk 40 (over
    32) that split is off.  Every element against the oracle, ragged lengths included."""
    c = W.make_nsa_prefill(Hq + 7 * d + bs + topk, lens, Hq, Hkv, d, bs, topk, 1, 2)
    assert _block_major_windows(c, oracle_lib) > 0
    _full_parity(sfa, oracle_lib, c)
    out, lse = run_fwd(sfa, c)
    out2, lse2 = run_fwd(sfa, c)  # a repeated call on fresh buffers gives the same bits
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


@pytest.mark.parametrize("topk,lens,bs,d", [(48, [3000, 700], 32, 64), (128, [5000], 32, 128)])
def test_long_selections_sorted_in_shared_memory(sfa, oracle_lib, topk, lens, bs, d):
    """topk above 32: the prep sorts each selection in shared memory instead of registers;
    topk = 128 is the largest this build takes."""
    c = W.make_nsa_prefill(topk + bs + d, lens, 8, 2, d, bs, topk, 1, 2)
    _full_parity(sfa, oracle_lib, c)
    rs, rc, _ = oracle_lib.fwd_index(c)
    d_ = upload_prefill(c)
    _, sel_c, cnt = sfa.fwd_prep(d_["cu_q"], d_["sel"], Hq=c.Hq, d=c.d, block_size=c.bs, cu_seqlens_k=d_["cu_k"],
                                 max_seqlen_q=c.max_sq, max_seqlen_k=c.max_sk)
    np.testing.assert_array_equal(sel_c.cpu().numpy(), rs)
    np.testing.assert_array_equal(cnt.cpu().numpy(), rc)


@pytest.mark.parametrize("sk,bs,topk,Hq,Hkv", [(100000, 32, 16, 8, 2), (131072, 64, 32, 2, 2)])
def test_many_key_blocks_short_queries(sfa, oracle_lib, sk, bs, topk, Hq, Hkv):
    """64 queries over 100000 keys (bs 32: 3125 blocks, more than the block-major schedule takes),
    blocks drawn per (token, kv head) from the bottom-right causal range.  The second case (one q
    head per kv head, 128-token tiles, top-32 of 2048 blocks) gives tile unions of up to 2048 blocks,
    too many for the pipelined query-major kernel's shared memory: the one-tile kernel runs it."""
    sq = 64
    rng = np.random.default_rng(5)
    sel = np.full((sq, Hkv, topk), -1, np.int32)
    for i in range(sq):
        nb = (i + sk - sq) // bs + 1
        for h in range(Hkv):
            sel[i, h] = rng.choice(nb, size=topk, replace=False)
    c = _case([sq], [sk], Hq, Hkv, 128, bs, sel, 6)
    _full_parity(sfa, oracle_lib, c)


def test_prefill_captured_in_cuda_graph(sfa):
    """sfa_fwd (prep, attend and, when eligible, the block-major kernels, chained with programmatic
    dependent launch) captured in a CUDA graph and replayed gives the eager call's bits."""
    c = W.small_config(2)
    d = upload_prefill(c)
    ws = torch.empty(sfa.fwd_workspace_size(c.batch, c.max_sq, c.max_sk, c.total_q, c.Hq, c.Hkv, c.d, c.topk, c.bs),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty_like(d["q"])
    lse = torch.empty((c.Hq, c.total_q), dtype=torch.float32, device="cuda")

    def call():
        run_fwd(sfa, c, d=d, out=out, lse=lse, workspace=ws)

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
    for _ in range(3):
        out.zero_()
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
    assert torch.equal(lse, ref_lse)
