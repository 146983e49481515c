"""The bench's algorithmic work count: kept (query, key) pairs taken from the selections as given.

It must equal, for every workload shape, the pairs the oracle's canonical index sets keep (ascending
distinct in-range blocks with at least one key under the mask), and for the NSA recipe the seed-free
closed form; -1 slots, duplicates and out-of-range ids add nothing."""
import dataclasses

import numpy as np
import pytest

import bench
import sfa_workloads as W


def _pairs_from_canonical(c, oracle_lib):
    sel_c, cnt, _ = oracle_lib.fwd_index(c)
    tot = 0
    for b in range(c.batch):
        q0, q1 = int(c.cu_q[b]), int(c.cu_q[b + 1])
        sq, sk = q1 - q0, int(c.cu_k[b + 1] - c.cu_k[b])
        for t in range(q0, q1):
            i = t - q0
            lo, hi = 0, sk - 1
            if c.causal:
                hi = min(hi, i + sk - sq)
            if c.wr >= 0:
                hi = min(hi, i + sk - sq + c.wr)
            if c.wl >= 0:
                lo = max(lo, i + sk - sq - c.wl)
            for hk in range(c.Hkv):
                for s in sel_c[t, hk, :cnt[t, hk]]:
                    a, z = max(lo, s * c.bs), min(hi, min(s * c.bs + c.bs, sk) - 1)
                    tot += max(0, z - a + 1)
    return tot


@pytest.mark.parametrize("n", [1, 2, 3, 4])
def test_kept_pairs_match_canonical_sets(oracle_lib, n):
    c = W.small_config(n)
    assert bench.kept_pairs(c) == _pairs_from_canonical(c, oracle_lib)


def test_kept_pairs_nsa_closed_form():
    for c in (W.small_config(2), W.small_config(4), W.config1()):
        per_head = W.kept_pairs_nsa(np.diff(c.cu_q).tolist(), c.bs, c.topk)
        assert bench.kept_pairs(c) == per_head * c.Hkv
        assert bench.prefill_flops(c) == 4.0 * c.d * c.Hq * per_head


def test_kept_pairs_ignore_padding_duplicates_and_bad_ids(oracle_lib):
    c = W.small_config(2)
    base = bench.kept_pairs(c)
    sel = c.sel.copy()
    sel = np.concatenate([sel, sel[:, :, :3], np.full(sel.shape[:2] + (2,), -1, np.int32),
                          np.full(sel.shape[:2] + (1,), 10 ** 6, np.int32)], axis=2)
    c2 = dataclasses.replace(c, sel=sel, topk=sel.shape[2])
    assert bench.kept_pairs(c2) == base == _pairs_from_canonical(c2, oracle_lib)


def test_full_size_workload_counts():
    """Config 4 (the benchmark's headline workload) against the closed form at full size."""
    c = W.config4()
    per_head = W.kept_pairs_nsa(np.diff(c.cu_q).tolist(), c.bs, c.topk)
    assert bench.prefill_flops(c) == 4.0 * c.d * c.Hq * per_head
    assert abs(bench.prefill_flops(c) / 1e9 - 197.8) < 0.1
