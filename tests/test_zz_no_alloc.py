"""sfa_decode_noalloc, the decode entry point for callers that cannot allocate device memory
(for example a serving engine whose memory pool is frozen before serving starts, or a plugin
hook handed only input and output pointers).  It keeps its scratch in a static device array
instead of a caller workspace.

These tests call it through the C ABI.  The cases are chosen so that the scratch array is
really used: selections longer than 2048 positions go through the prep kernel, whose canonical
token lists live in the scratch, and more than six splits make the split kernel write its fp32
partials there for a separate combine kernel.  A larger call runs before a smaller one, so the
smaller call starts on an array the larger call left full.  Each result must equal sfa_decode
(caller workspace, same split count) bit for bit, the same kernels on the same inputs, and the
fp64 oracle within the decode tolerance.  The file name makes pytest collect it last."""
import ctypes

import numpy as np
import pytest

import sfa_workloads as W
from tests.parity import assert_lse_close, assert_out_close, upload_decode

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_flashattention_b200 as sfa
    l = ctypes.CDLL(sfa.lib_path())
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    l.sfa_decode_noalloc.restype = I
    l.sfa_decode_noalloc.argtypes = [P, P, P, P, I, I, I, P, P, I, I, I, I, I, I, F, I, P, P, P, P]
    return l


def _noalloc(lib, c, d, splits, out, lse, status, q=None):
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return lib.sfa_decode_noalloc(p(d["q"] if q is None else q), p(d["k_cache"]), p(d["v_cache"]),
                                  p(d["block_table"]), c.max_pages, c.num_pages, c.page, p(d["cache_seqlens"]),
                                  p(d["sel"]), c.topk, c.B, c.Hq, c.Hkv, c.d, c.wl, 0.0, splits, p(status), p(out),
                                  p(lse), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


# (case, num_splits): larger scratch users first, then smaller ones, then the first again.
def _cases():
    big = W.make_decode(91, 4, 16, 4, 128, 64, 5000, 9000, 3000, 64)    # topk 3000 > 2048: prep kernel
    mid = W.make_decode(92, 3, 8, 2, 64, 32, 2500, 4000, 2100, 32)      # d 64, prep kernel
    small = W.small_config(5)                                            # in-kernel dedupe
    return [(big, 12), (mid, 8), (small, 9), (small, 0), (big, 12)]


def test_noalloc_decode_matches_workspace_decode_and_oracle(lib, oracle_lib):
    import sparse_flashattention_b200 as sfa
    refs = {}
    for c, splits in _cases():
        d = upload_decode(c)
        assert sfa.decode_workspace_size(c.B, c.Hq, c.Hkv, c.d, c.topk, splits) <= (8 << 20)
        ws_out, ws_lse = sfa.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["cache_seqlens"],
                                    d["sel"], num_splits=splits)
        key = id(c)
        if key not in refs:
            refs[key] = oracle_lib.decode(c)[:2]
        ro, rl = refs[key]
        for _ in range(2):  # two calls in a row on the shared scratch
            out = torch.full_like(ws_out, float("nan"))
            lse = torch.full_like(ws_lse, float("nan"))
            status = torch.zeros(1, dtype=torch.int32, device="cuda")
            assert _noalloc(lib, c, d, splits, out, lse, status) == 0
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            assert torch.equal(out.view(torch.int16), ws_out.view(torch.int16)), "out differs from sfa_decode"
            assert torch.equal(lse.view(torch.int32), ws_lse.view(torch.int32)), "lse differs from sfa_decode"
            assert_out_close(out, ro)
            assert_lse_close(lse, rl)


def test_noalloc_rejects_oversized_calls(lib):
    """A call whose workspace would exceed the fixed 8 MiB scratch is refused before any launch."""
    c = W.small_config(5)
    d = upload_decode(c)
    big_topk = 1 << 16  # (B * Hkv * topk) int32 token lists alone exceed 8 MiB for B=4, Hkv=8
    import sparse_flashattention_b200 as sfa
    assert sfa.decode_workspace_size(c.B, c.Hq, c.Hkv, c.d, big_topk) > (8 << 20)
    sel = torch.full((c.B, c.Hkv, big_topk), -1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(d["q"])
    lse = torch.empty((c.B, c.Hq), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    d2 = dict(d, sel=sel)
    c2 = W.DecodeCase(**{**c.__dict__, "sel": np.full((c.B, c.Hkv, big_topk), -1, np.int32)})
    assert _noalloc(lib, c2, d2, 0, out, lse, status) == 3  # SFA_ERR_WORKSPACE_TOO_SMALL


def test_noalloc_rejects_host_pointers(lib):
    """q must be device memory of the current device; a host buffer is refused before any launch."""
    c = W.small_config(5)
    d = upload_decode(c)
    out = torch.empty_like(d["q"])
    lse = torch.empty((c.B, c.Hq), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q_host = d["q"].cpu()
    assert _noalloc(lib, c, d, 0, out, lse, status, q=q_host) == 1  # SFA_ERR_INVALID_ARG
