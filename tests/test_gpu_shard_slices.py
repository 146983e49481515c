"""The splits a multi-GPU caller makes of this path reproduce the full call bit for bit.

Every (sequence, kv head) of the prefill and every (sequence, kv head) of the decode is an
independent problem (the flash-attention-npu varlen docstrings: sequences packed by cu_seqlens,
query head h reading kv head h / (Hq/Hkv)), so a caller can shard a call across GPUs by kv heads
(each GPU takes Hkv/N kv heads with their G query heads, the K/V columns and the selection columns)
or by sequences, with no exchange between GPUs.  Run on one GPU here: each slice, passed to the
same entry point as its own call, must equal the matching slice of the full call exactly.

The host-side bounds that size the work stay those of the full call (max_seqlen_q/k for the
prefill, num_splits for the decode), as a caller sharding one batch passes them; with them the
kernels see the same tiles, schedule and splits per problem, so equality is bitwise."""
import dataclasses

import numpy as np
import pytest

import sfa_workloads as W
from tests.parity import run_decode, upload_prefill

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sfa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_flashattention_b200 as m
    return m


def _bits_equal(a, b):
    ia = a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32)
    ib = b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32)
    return torch.equal(ia, ib)


def _kv_slice(c, h0, h1):
    G = c.Hq // c.Hkv
    return dataclasses.replace(c, q=np.ascontiguousarray(c.q[:, h0 * G:h1 * G]),
                               k=np.ascontiguousarray(c.k[:, h0:h1]), v=np.ascontiguousarray(c.v[:, h0:h1]),
                               sel=np.ascontiguousarray(c.sel[:, h0:h1]), Hq=(h1 - h0) * G, Hkv=h1 - h0)


def _seq_subset(c, seqs):
    qi = np.concatenate([np.arange(c.cu_q[b], c.cu_q[b + 1]) for b in seqs]).astype(np.int64)
    ki = np.concatenate([np.arange(c.cu_k[b], c.cu_k[b + 1]) for b in seqs]).astype(np.int64)
    lq = [int(c.cu_q[b + 1] - c.cu_q[b]) for b in seqs]
    lk = [int(c.cu_k[b + 1] - c.cu_k[b]) for b in seqs]
    return dataclasses.replace(c, q=c.q[qi], k=c.k[ki], v=c.v[ki], sel=c.sel[qi], cu_q=W._cu(lq), cu_k=W._cu(lk)), qi


PREFILL = {
    # query-major (no sequence long enough for the block-major schedule)
    "nsa_varlen": lambda: W.small_config(2),
    # block-major windows in the long sequence, query-major elsewhere
    "nsa_block_major": lambda: W.make_nsa_prefill(31, [12000, 300, 900], 16, 4, 128, 64, 6, 1, 2),
    # dense window with sq != sk
    "window": lambda: W.small_config(3),
}


def _fwd(sfa, c, full):
    d = upload_prefill(c)
    return sfa.fwd(d["q"], d["k"], d["v"], d["cu_q"], d["sel"], c.bs, cu_seqlens_k=d["cu_k"],
                   max_seqlen_q=full.max_sq, max_seqlen_k=full.max_sk, causal=bool(c.causal), window=(c.wl, c.wr))


@pytest.mark.parametrize("name", sorted(PREFILL))
def test_prefill_kv_head_shards(sfa, name):
    c = PREFILL[name]()
    out, lse = _fwd(sfa, c, c)
    G = c.Hq // c.Hkv
    for h0, h1 in [(0, 1), (1, c.Hkv), (c.Hkv // 2, c.Hkv)]:
        o, l = _fwd(sfa, _kv_slice(c, h0, h1), c)
        assert _bits_equal(o, out[:, h0 * G:h1 * G].contiguous()), (name, h0, h1)
        assert _bits_equal(l, lse[h0 * G:h1 * G].contiguous()), (name, h0, h1)


@pytest.mark.parametrize("name", sorted(PREFILL))
def test_prefill_sequence_shards(sfa, name):
    c = PREFILL[name]()
    out, lse = _fwd(sfa, c, c)
    B = c.batch
    for seqs in ([0], list(range(1, B)), list(range(B - 1, -1, -2))):
        s, qi = _seq_subset(c, seqs)
        o, l = _fwd(sfa, s, c)
        idx = torch.as_tensor(qi, device="cuda")
        assert _bits_equal(o, out.index_select(0, idx)), (name, seqs)
        assert _bits_equal(l, lse.index_select(1, idx)), (name, seqs)


DECODE = {
    "decode_small": lambda: W.small_config(5),
    "decode_prep_path": lambda: W.make_decode(33, 6, 16, 4, 128, 64, 3000, 7000, 2600, 64),  # topk > 2048
}


@pytest.mark.parametrize("name", sorted(DECODE))
def test_decode_batch_and_kv_head_shards(sfa, name):
    c = DECODE[name]()
    S = sfa.decode_num_splits(c.B, c.Hq, c.Hkv, c.d, c.topk, 0)
    out, lse = run_decode(sfa, c, num_splits=S)
    # by sequence
    for bsel in ([0], list(range(1, c.B)), list(range(c.B - 1, -1, -2))):
        s = dataclasses.replace(c, q=c.q[bsel], block_table=c.block_table[bsel], cache_seqlens=c.cache_seqlens[bsel],
                                sel=c.sel[bsel])
        o, l = run_decode(sfa, s, num_splits=S)
        idx = torch.as_tensor(bsel, device="cuda")
        assert _bits_equal(o, out.index_select(0, idx)), (name, bsel)
        assert _bits_equal(l, lse.index_select(0, idx)), (name, bsel)
    # by kv head (each shard holds its kv heads' columns of the cache)
    G = c.Hq // c.Hkv
    for h0, h1 in [(0, 1), (1, c.Hkv)]:
        s = dataclasses.replace(c, q=np.ascontiguousarray(c.q[:, h0 * G:h1 * G]),
                                k_cache=np.ascontiguousarray(c.k_cache[:, :, h0:h1]),
                                v_cache=np.ascontiguousarray(c.v_cache[:, :, h0:h1]),
                                sel=np.ascontiguousarray(c.sel[:, h0:h1]), Hq=(h1 - h0) * G, Hkv=h1 - h0)
        o, l = run_decode(sfa, s, num_splits=S)
        assert _bits_equal(o, out[:, h0 * G:h1 * G].contiguous()), (name, h0, h1)
        assert _bits_equal(l, lse[:, h0 * G:h1 * G].contiguous()), (name, h0, h1)
