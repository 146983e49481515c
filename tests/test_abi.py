"""The C ABI without a GPU: the library loads, exports every function include/sfa.h declares,
and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sfa.h")


@pytest.fixture(scope="module")
def lib():
    from sparse_flashattention_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sfa_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert "sfa_fwd" in names and "sfa_decode" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/sfa.h but not exported"


def test_status_strings(lib):
    lib.sfa_status_string.restype = ctypes.c_char_p
    for code in range(5):
        assert lib.sfa_status_string(code).decode().startswith("SFA_")


P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
FAKE = ctypes.c_void_p(1 << 20)  # 16-byte aligned, never dereferenced: validation fails first


def _fwd(lib, **over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, cu_q=FAKE, cu_k=None, batch=1, max_sq=128, max_sk=128, total_q=128,
             total_k=128, Hq=4, Hkv=1, d=64, sel=FAKE, topk=4, bs=32, causal=1, wl=-1, wr=-1, scale=0.0,
             ws=FAKE, ws_bytes=0, status=None, out=FAKE, lse=FAKE, stream=None)
    a.update(over)
    lib.sfa_fwd.restype = I
    lib.sfa_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, I, P, I, I, I, I, I, F, P, Z, P, P, P, P]
    return lib.sfa_fwd(*a.values())


def test_fwd_host_validation(lib):
    lib.sfa_fwd_workspace_size.restype = Z
    lib.sfa_fwd_workspace_size.argtypes = [I] * 9
    need = lib.sfa_fwd_workspace_size(1, 128, 128, 128, 4, 1, 64, 4, 32)
    assert need > 0
    assert lib.sfa_fwd_workspace_size(1, 0, 0, 0, 4, 1, 64, 4, 32) == 0
    assert _fwd(lib, Hq=6, Hkv=4) == 1          # Hq % Hkv != 0 -> SFA_ERR_INVALID_ARG
    assert _fwd(lib, d=96) == 2                  # unsupported head dim
    assert _fwd(lib, bs=48) == 2                 # unsupported block size
    assert _fwd(lib, topk=0) == 1
    assert _fwd(lib, topk=129) == 2
    assert _fwd(lib, causal=2) == 1
    assert _fwd(lib, wl=-2) == 1
    assert _fwd(lib, q=ctypes.c_void_p((1 << 20) + 8)) == 1   # misaligned base
    assert _fwd(lib, sel=None) == 1
    assert _fwd(lib, total_k=100) == 1           # cu_k NULL but total_k != total_q
    assert _fwd(lib, ws_bytes=need - 1) == 3     # SFA_ERR_WORKSPACE_TOO_SMALL
    assert _fwd(lib, ws=ctypes.c_void_p((1 << 20) + 16), ws_bytes=need) == 1  # workspace off a 256-byte boundary
    assert _fwd(lib, total_q=0, total_k=0) == 0   # nothing to do: OK without launching


def test_decode_host_validation(lib):
    lib.sfa_decode.restype = I
    lib.sfa_decode.argtypes = [P, P, P, P, I, I, I, P, P, I, I, I, I, I, I, F, I, P, Z, P, P, P, P]
    lib.sfa_decode_workspace_size.restype = Z
    lib.sfa_decode_workspace_size.argtypes = [I] * 6

    def call(**over):
        a = dict(q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, maxp=4, npages=8, page=256, lens=FAKE, sel=FAKE, topk=64, B=2,
                 Hq=8, Hkv=2, d=128, wl=-1, scale=0.0, splits=0, ws=FAKE, ws_bytes=0, status=None, out=FAKE,
                 lse=FAKE, stream=None)
        a.update(over)
        return lib.sfa_decode(*a.values())

    need = lib.sfa_decode_workspace_size(2, 8, 2, 128, 64, 0)
    assert need > 0
    assert call(Hq=8, Hkv=3) == 1
    assert call(Hq=64, Hkv=2) == 2               # G = 32 > 16 unsupported
    assert call(d=80) == 2
    assert call(page=0) == 1
    assert call(bt=None) == 1
    assert call(wl=-5) == 1
    assert call(ws_bytes=need - 1) == 3
    assert call(ws=ctypes.c_void_p((1 << 20) + 16), ws_bytes=need) == 1  # workspace off a 256-byte boundary
    assert call(B=0) == 0


def test_decode_split_heuristic(lib):
    lib.sfa_decode_num_splits.restype = I
    lib.sfa_decode_num_splits.argtypes = [I] * 6
    assert lib.sfa_decode_num_splits(32, 32, 8, 128, 2048, 5) == 5
    s = lib.sfa_decode_num_splits(32, 32, 8, 128, 2048, 0)
    assert 1 <= s <= 16
    assert lib.sfa_decode_num_splits(1, 8, 8, 128, 100, 0) == 1


def _bwd(lib, **over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, dout=FAKE, lse=FAKE, cu_q=FAKE, cu_k=None, batch=1, max_sq=128,
             max_sk=128, total_q=128, total_k=128, Hq=4, Hkv=1, d=128, sel=FAKE, topk=4, bs=64, causal=1, wl=-1,
             wr=-1, scale=0.0, ws=FAKE, ws_bytes=0, status=None, dq=FAKE, dk=FAKE, dv=FAKE, stream=None)
    a.update(over)
    lib.sfa_bwd.restype = I
    lib.sfa_bwd.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, I, I, I, I, I, F, P, Z, P, P, P, P, P]
    return lib.sfa_bwd(*a.values())


def test_bwd_host_validation(lib):
    """Backward: sizes outside this build (d != 128, block_size != 64) and bad arguments are rejected
    on the host; the workspace grows with the token bitmaps and the token lists."""
    lib.sfa_bwd_workspace_size.restype = Z
    lib.sfa_bwd_workspace_size.argtypes = [I] * 9
    base = lib.sfa_bwd_workspace_size(1, 128, 128, 128, 4, 1, 128, 4, 64)
    assert base > 0
    assert lib.sfa_bwd_workspace_size(1, 128, 128, 128, 4, 1, 64, 4, 64) > 0     # d 64
    assert lib.sfa_bwd_workspace_size(1, 128, 128, 128, 4, 1, 128, 4, 32) > 0    # block 32
    assert lib.sfa_bwd_workspace_size(1, 128, 128, 128, 4, 1, 96, 4, 64) == 0    # d 96: unsupported
    assert lib.sfa_bwd_workspace_size(1, 0, 0, 0, 4, 1, 128, 4, 64) == 0         # no query
    assert lib.sfa_bwd_workspace_size(1, 4096, 4096, 4096, 4, 1, 128, 4, 64) > \
        lib.sfa_bwd_workspace_size(1, 1024, 4096, 1024, 4, 1, 128, 4, 64) > base
    assert _bwd(lib, d=96) == 2                   # SFA_ERR_UNSUPPORTED
    assert _bwd(lib, bs=48) == 2
    assert _bwd(lib, Hq=6, Hkv=4) == 1            # SFA_ERR_INVALID_ARG
    assert _bwd(lib, dout=None) == 1
    assert _bwd(lib, dk=None) == 1
    assert _bwd(lib, wl=-3) == 1
    assert _bwd(lib, ws_bytes=16) == 3            # SFA_ERR_WORKSPACE_TOO_SMALL
    assert _bwd(lib, ws=ctypes.c_void_p((1 << 20) + 16), ws_bytes=1 << 40) == 1  # workspace off a 256-byte boundary
    assert _bwd(lib, q=ctypes.c_void_p((1 << 20) + 8)) == 1  # misaligned
    # G 1 (128 tokens per tile) with topk 128 over 8192 blocks: a tile's union of up to 8192 blocks
    # (two copies, 64 KB) does not fit beside the dQ kernel's rings
    big = dict(Hq=1, Hkv=1, topk=128, max_sq=1 << 19, max_sk=1 << 19, total_q=1 << 19, total_k=1 << 19,
               ws_bytes=1 << 62)
    assert _bwd(lib, **big) == 2


def test_kv_append_host_validation(lib):
    lib.sfa_kv_append.restype = I
    lib.sfa_kv_append.argtypes = [P, P, I, P, P, P, I, I, I, P, I, I, I, P, P]

    def call(**over):
        a = dict(kn=FAKE, vn=FAKE, S=1, kc=FAKE, vc=FAKE, bt=FAKE, max_pages=4, num_pages=8, page=16, lens=FAKE,
                 B=2, Hkv=2, d=128, status=None, stream=None)
        a.update(over)
        return lib.sfa_kv_append(*a.values())

    assert call(d=12) == 2        # not a multiple of 8
    assert call(B=0) == 0         # nothing to append: no launch
    assert call(S=0) == 0
    assert call(page=0) == 1
    assert call(bt=None) == 1
    assert call(kc=ctypes.c_void_p((1 << 20) + 4)) == 1


def test_index_topk_host_validation(lib):
    lib.sfa_index_topk_workspace_size.restype = Z
    lib.sfa_index_topk_workspace_size.argtypes = [I] * 4
    assert lib.sfa_index_topk_workspace_size(2, 4, 8, 16) == 2 * 4 * 8 * 16 * 8
    assert lib.sfa_index_topk_workspace_size(0, 4, 8, 16) == 0
    lib.sfa_index_topk.restype = I
    lib.sfa_index_topk.argtypes = [P, P, P, I, I, I, P, I, I, I, I, I, I, P, Z, P, P, P]

    def call(**over):
        a = dict(q=FAKE, kc=FAKE, bt=FAKE, max_pages=8, num_pages=16, page=16, lens=FAKE, B=2, Hq=8, Hkv=4, d=128,
                 topk=32, n_local=0, ws=FAKE, ws_bytes=1 << 20, status=None, out=FAKE, stream=None)
        a.update(over)
        return lib.sfa_index_topk(*a.values())

    assert call(d=96) == 2                 # SFA_ERR_UNSUPPORTED
    assert call(Hq=6) == 1                 # Hq % Hkv
    assert call(Hq=4 * 1025) == 2          # groups past 1024 query heads: scores no longer exact in fp64
    assert call(topk=0) == 1
    assert call(n_local=-1) == 1
    assert call(out=None) == 1
    assert call(ws_bytes=8) == 3           # SFA_ERR_WORKSPACE_TOO_SMALL
    assert call(ws=ctypes.c_void_p((1 << 20) + 16)) == 1  # workspace off a 256-byte boundary
    assert call(max_pages=1 << 16, page=32) == 2  # more than 2^20 positions per sequence
    assert call(B=0) == 0


def test_window_and_gated_combine_host_validation(lib):
    lib.sfa_window_fwd.restype = I
    lib.sfa_window_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, I, I, I, I, P, P, F, P, Z, P, P, P, P]

    def win(**over):
        a = dict(q=FAKE, k=FAKE, v=FAKE, cu_q=FAKE, cu_k=None, batch=1, max_sq=128, max_sk=128, total_q=128,
                 total_k=128, Hq=4, Hkv=1, d=128, causal=1, wl=512, wr=0, wlh=None, wrh=None, scale=0.0, ws=FAKE,
                 ws_bytes=256, status=None, out=FAKE, lse=FAKE, stream=None)
        a.update(over)
        return lib.sfa_window_fwd(*a.values())

    assert win(d=96) == 2
    assert win(wl=-2) == 1
    assert win(causal=2) == 1
    assert win(out=None) == 1
    assert win(ws_bytes=4) == 3
    assert win(total_q=0, total_k=0) == 0     # nothing to compute
    assert win(total_q=0) == 1                # k lengths must match q's when cu_seqlens_k is NULL

    lib.sfa_gated_combine.restype = I
    lib.sfa_gated_combine.argtypes = [P, P, P, P, P, P, I, I, I, P, P]

    def mix(**over):
        a = dict(o1=FAKE, g1=FAKE, o2=None, g2=None, o3=None, g3=None, total_q=16, Hq=4, d=128, out=FAKE,
                 stream=None)
        a.update(over)
        return lib.sfa_gated_combine(*a.values())

    assert mix(d=96) == 2
    assert mix(o1=None) == 1                      # no branch left
    assert mix(o1=ctypes.c_void_p((1 << 20) + 2)) == 1
    assert mix(out=None) == 1
    assert mix(total_q=0) == 0


def test_kvcache_entries_host_validation(lib):
    """The non-paged entries are the paged ones with block_table = cache_batch_idx, one page of
    seqlen_cache rows per cache entry: the same host checks apply."""
    lib.sfa_decode_kvcache.restype = I
    lib.sfa_decode_kvcache.argtypes = [P, P, P, I, I, P, P, P, I, I, I, I, I, I, F, I, P, Z, P, P, P, P]

    def dec(**over):
        a = dict(q=FAKE, kc=FAKE, vc=FAKE, batch_cache=4, seqlen_cache=1024, idx=FAKE, lens=FAKE, sel=FAKE,
                 topk=64, B=2, Hq=8, Hkv=2, d=128, wl=-1, scale=0.0, splits=0, ws=FAKE, ws_bytes=1 << 30,
                 status=None, out=FAKE, lse=FAKE, stream=None)
        a.update(over)
        return lib.sfa_decode_kvcache(*a.values())

    assert dec(idx=None) == 1                          # cache_batch_idx is required
    assert dec(seqlen_cache=0) == 1
    assert dec(seqlen_cache=(1 << 20) + 64) == 2       # more than 2^20 rows per sequence
    assert dec(d=96) == 2
    assert dec(ws_bytes=8) == 3
    assert dec(B=0) == 0

    lib.sfa_kv_append_kvcache.restype = I
    lib.sfa_kv_append_kvcache.argtypes = [P, P, I, P, P, I, I, P, P, I, I, I, P, P]

    def app(**over):
        a = dict(kn=FAKE, vn=FAKE, S=4, kc=FAKE, vc=FAKE, batch_cache=4, seqlen_cache=1024, idx=FAKE, lens=FAKE,
                 B=2, Hkv=2, d=128, status=None, stream=None)
        a.update(over)
        return lib.sfa_kv_append_kvcache(*a.values())

    assert app(idx=None) == 1
    assert app(seqlen_cache=0) == 1
    assert app(d=12) == 2
    assert app(S=0) == 0
