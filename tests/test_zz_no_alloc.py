"""sfa_decode_noalloc, the decode entry point for callers that cannot allocate device memory
(for example a serving engine whose memory pool is frozen before serving starts, or a plugin
hook handed only input and output pointers).  It keeps its scratch in a static device array
instead of a caller workspace.  This test calls it through the C ABI and checks it against
sfa_decode, which uses a caller workspace, on two calls in a row (the second call reuses the
array the first one left behind).  The file name makes pytest collect it last."""
import ctypes

import numpy as np
import pytest

import sfa_workloads as W
from tests.parity import OUT_ATOL, OUT_RTOL, LSE_ATOL, upload_decode

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


def _noalloc(lib, c, d, out, lse, status):
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return lib.sfa_decode_noalloc(p(d["q"]), p(d["k_cache"]), p(d["v_cache"]), p(d["block_table"]), c.max_pages,
                                  c.num_pages, c.page, p(d["cache_seqlens"]), p(d["sel"]), c.topk, c.B, c.Hq, c.Hkv,
                                  c.d, c.wl, 0.0, 0, p(status), p(out), p(lse),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _close(a, b, alse, blse):
    a, b = a.float().cpu().numpy(), b.float().cpu().numpy()
    assert (np.abs(a - b) <= OUT_ATOL + OUT_RTOL * np.abs(b)).all()
    al, bl = alse.cpu().numpy(), blse.cpu().numpy()
    np.testing.assert_array_equal(np.isneginf(al), np.isneginf(bl))
    fin = np.isfinite(bl)
    assert np.abs(al[fin] - bl[fin]).max(initial=0.0) <= LSE_ATOL


def test_noalloc_decode_matches_workspace_decode(lib):
    import sparse_flashattention_b200 as sfa
    cases = [W.small_config(5), W.make_decode(77, 6, 16, 4, 128, 64, 50, 4000, 512, 32)]
    for c in cases:
        d = upload_decode(c)
        ref, ref_lse = sfa.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["cache_seqlens"], d["sel"])
        for _ in range(2):  # two calls in a row on the shared scratch
            out = torch.full_like(ref, float("nan"))
            lse = torch.full_like(ref_lse, float("nan"))
            status = torch.zeros(1, dtype=torch.int32, device="cuda")
            assert _noalloc(lib, c, d, out, lse, status) == 0
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            _close(out, ref, lse, ref_lse)


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
    assert _noalloc(lib, c2, d2, out, lse, status) == 3  # SFA_ERR_WORKSPACE_TOO_SMALL
