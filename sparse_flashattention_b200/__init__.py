"""Top-k sparse FlashAttention forward for NVIDIA B200 (sm_100a).

A thin ctypes binding over libsfa.so (C ABI in include/sfa.h).  This module only marshals
arguments: it checks dtypes/shapes, takes device pointers from torch tensors, allocates
outputs and workspaces with torch when the caller does not pass them, and passes the
current CUDA stream.  Every step of the computation runs in the library's CUDA kernels;
there is no CPU or PyTorch fallback, and importing fails loudly if the library is missing.

    out, lse = fwd(q, k, v, cu_seqlens_q, sel_idx, block_size=64, max_seqlen_q=...)
    out, lse = decode(q, k_cache, v_cache, block_table, cache_seqlens, sel_tok_idx)
"""
from __future__ import annotations

import ctypes
import functools
import math
import os
from typing import Optional, Tuple

import torch

__all__ = ["SfaError", "lib_path", "fwd", "fwd_prep", "fwd_attend", "fwd_workspace_size", "window_fwd",
           "gated_combine", "decode", "decode_prep",
           "decode_attend", "decode_noalloc", "decode_fp8", "decode_workspace_size", "decode_num_splits", "last_launch_count",
           "DEV_BAD_INDEX", "DEV_BAD_PAGE", "DEV_TIMEOUT"]

DEV_BAD_INDEX, DEV_BAD_PAGE, DEV_TIMEOUT = 1, 2, 4

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsfa.so")


class SfaError(RuntimeError):
    pass


def lib_path() -> str:
    return _LIB_PATH


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with `python sparse_flashattention_b200/build.py` "
                          "(there is no fallback implementation)")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    sig = {
        "sfa_fwd_workspace_size": (Z, [I, I, I, I, I, I, I, I, I]),
        "sfa_fwd_workspace_offsets": (I, [I, I, I, I, I, I, I, I, I, P, P]),
        "sfa_fwd": (I, [P, P, P, P, P, I, I, I, I, I, I, I, I, P, I, I, I, I, I, F, P, Z, P, P, P, P]),
        "sfa_fwd_prep": (I, [P, P, I, I, I, I, I, I, I, P, I, I, I, I, I, P, Z, P, P]),
        "sfa_fwd_attend": (I, [P, P, P, P, P, I, I, I, I, I, I, I, I, I, I, I, I, I, F, P, Z, P, P, P, P]),
        "sfa_decode_num_splits": (I, [I, I, I, I, I, I]),
        "sfa_decode_workspace_size": (Z, [I, I, I, I, I, I]),
        "sfa_decode_workspace_offsets": (I, [I, I, I, I, I, I, P, P]),
        "sfa_decode": (I, [P, P, P, P, I, I, I, P, P, I, I, I, I, I, I, F, I, P, Z, P, P, P, P]),
        "sfa_decode_prep": (I, [P, P, I, I, I, I, I, I, I, I, I, P, Z, P, P]),
        "sfa_decode_attend": (I, [P, P, P, P, I, I, I, I, I, I, I, I, F, I, P, Z, P, P, P, P]),
        "sfa_decode_noalloc": (I, [P, P, P, P, I, I, I, P, P, I, I, I, I, I, I, F, I, P, P, P, P]),
        "sfa_decode_fp8": (I, [P, P, P, P, P, P, I, I, I, P, P, I, I, I, I, I, I, F, I, P, Z, P, P, P, P]),
        "sfa_window_fwd_workspace_size": (Z, []),
        "sfa_window_fwd": (I, [P, P, P, P, P, I, I, I, I, I, I, I, I, I, I, I, P, P, F, P, Z, P, P, P, P]),
        "sfa_gated_combine": (I, [P, P, P, P, P, P, I, I, I, P, P]),
        "sfa_kv_append": (I, [P, P, I, P, P, P, I, I, I, P, I, I, I, P, P]),
        "sfa_decode_kvcache": (I, [P, P, P, I, I, P, P, P, I, I, I, I, I, I, F, I, P, Z, P, P, P, P]),
        "sfa_kv_append_kvcache": (I, [P, P, I, P, P, I, I, P, P, I, I, I, P, P]),
        "sfa_index_topk_workspace_size": (Z, [I, I, I, I]),
        "sfa_index_topk": (I, [P, P, P, I, I, I, P, I, I, I, I, I, I, P, Z, P, P, P]),
        "sfa_bwd_workspace_size": (Z, [I, I, I, I, I, I, I, I, I]),
        "sfa_bwd": (I, [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, I, I, I, I, I, F, P, Z, P, P, P, P, P]),
        "sfa_status_string": (ctypes.c_char_p, [I]),
        "sfa_last_launch_count": (I, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def _check(rc: int):
    if rc != 0:
        raise SfaError(_lib.sfa_status_string(rc).decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _first_cuda_tensor(args, kwargs):
    for a in list(args) + list(kwargs.values()):
        items = a if isinstance(a, (list, tuple)) else [a]
        for x in items:
            for y in (x if isinstance(x, (list, tuple)) else [x]):
                if isinstance(y, torch.Tensor) and y.is_cuda:
                    return y
    return None


def _on_tensor_device(fn):
    """Run a call with the device of its first CUDA tensor current: the library launches on the
    current device and the default stream is that device's current stream."""
    @functools.wraps(fn)
    def wrapper(*args, **kwargs):
        t = _first_cuda_tensor(args, kwargs)
        if t is None or t.device == torch.device("cuda", torch.cuda.current_device()):
            return fn(*args, **kwargs)
        with torch.cuda.device(t.device):
            return fn(*args, **kwargs)
    return wrapper


def _need(t: torch.Tensor, name: str, dtype, ndim: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _scale(scale):
    return 0.0 if scale is None else float(scale)


def last_launch_count() -> int:
    """Kernel launches made by the last successful call on this thread."""
    return int(_lib.sfa_last_launch_count())


# ---------------------------------------------------------------------------------------
# Prefill
# ---------------------------------------------------------------------------------------

def _seq_bounds(cu: torch.Tensor) -> int:
    c = cu.detach().to("cpu", torch.int64)
    return int((c[1:] - c[:-1]).max()) if c.numel() > 1 else 0


def fwd_workspace_size(batch, max_seqlen_q, max_seqlen_k, total_q, Hq, Hkv, d, topk, block_size) -> int:
    return int(_lib.sfa_fwd_workspace_size(batch, max_seqlen_q, max_seqlen_k, total_q, Hq, Hkv, d, topk,
                                           block_size))


class _FwdArgs:
    def __init__(self, q, k, v, cu_seqlens_q, sel_idx, block_size, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                 causal, window, scale, topk=None):
        _need(q, "q", torch.bfloat16, 3)
        _need(k, "k", torch.bfloat16, 3)
        _need(v, "v", torch.bfloat16, 3)
        _need(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
        if cu_seqlens_k is not None:
            _need(cu_seqlens_k, "cu_seqlens_k", torch.int32, 1)
        if sel_idx is not None:
            _need(sel_idx, "sel_idx", torch.int32, 3)
        if k.shape != v.shape:
            raise ValueError("k and v must have the same shape")
        self.total_q, self.Hq, self.d = q.shape
        self.total_k, self.Hkv, dk = k.shape
        if dk != self.d:
            raise ValueError("q and k head dims differ")
        self.batch = cu_seqlens_q.numel() - 1
        self.max_sq = _seq_bounds(cu_seqlens_q) if max_seqlen_q is None else int(max_seqlen_q)
        if max_seqlen_k is None:
            max_seqlen_k = self.max_sq if cu_seqlens_k is None else _seq_bounds(cu_seqlens_k)
        self.max_sk = int(max_seqlen_k)
        self.topk = int(sel_idx.shape[2]) if sel_idx is not None else int(topk)
        if sel_idx is not None and tuple(sel_idx.shape[:2]) != (self.total_q, self.Hkv):
            raise ValueError(f"sel_idx must be (total_q, Hkv, topk) = ({self.total_q}, {self.Hkv}, *)")
        self.bs = int(block_size)
        self.causal = 1 if causal else 0
        self.wl, self.wr = (int(window[0]), int(window[1]))
        self.scale = _scale(scale)
        self.ws_bytes = fwd_workspace_size(self.batch, self.max_sq, self.max_sk, self.total_q, self.Hq, self.Hkv,
                                           self.d, self.topk, self.bs)

    def geom(self):
        return (self.batch, self.max_sq, self.max_sk, self.total_q, self.Hq, self.Hkv, self.d, self.topk, self.bs)


def _workspace(ws, nbytes, device):
    if ws is None:
        return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)
    if ws.numel() * ws.element_size() < nbytes:
        raise ValueError(f"workspace has {ws.numel() * ws.element_size()} bytes, needs {nbytes}")
    return ws


@_on_tensor_device
def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens_q: torch.Tensor, sel_idx: torch.Tensor,
        block_size: int, *, cu_seqlens_k: Optional[torch.Tensor] = None, max_seqlen_q: Optional[int] = None,
        max_seqlen_k: Optional[int] = None, causal: bool = True, window: Tuple[int, int] = (-1, -1),
        scale: Optional[float] = None, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
        workspace: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
        stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Varlen top-k sparse attention forward (sfa_fwd).

    q (total_q, Hq, d), k/v (total_k, Hkv, d) bf16; cu_seqlens int32 (batch+1);
    sel_idx int32 (total_q, Hkv, topk) block ids, -1 = unused.  Returns out (total_q, Hq, d)
    bf16 and lse (Hq, total_q) fp32.  Pass max_seqlen_q/k to avoid a device->host read of
    cu_seqlens.  status (int32, 1 element, on the device) accumulates SFA_DEV_* bits."""
    a = _FwdArgs(q, k, v, cu_seqlens_q, sel_idx, block_size, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal,
                 window, scale)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((a.Hq, a.total_q), dtype=torch.float32, device=q.device) if lse is None else lse
    ws = _workspace(workspace, a.ws_bytes, q.device)
    rc = _lib.sfa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), a.batch, a.max_sq, a.max_sk,
                      a.total_q, a.total_k, a.Hq, a.Hkv, a.d, _ptr(sel_idx), a.topk, a.bs, a.causal, a.wl, a.wr,
                      a.scale, _ptr(ws), ws.numel() * ws.element_size(), _ptr(status), _ptr(out), _ptr(lse),
                      _stream(stream))
    _check(rc)
    return out, lse


def index_topk_workspace_size(B, Hkv, max_pages_per_seq, page_size) -> int:
    return int(_lib.sfa_index_topk_workspace_size(B, Hkv, max_pages_per_seq, page_size))


@_on_tensor_device
def index_topk(q: torch.Tensor, k_cache: torch.Tensor, block_table: torch.Tensor, cache_seqlens: torch.Tensor,
               topk: int, *, n_local: int = 0, out: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    """Decode index producer (sfa_index_topk): per (sequence, kv head) the top-k cache positions by exact
    FP8 (E4M3) dot products of the group's query heads with every key, the last n_local always kept.
    Returns int32 (B, Hkv, topk), ascending, -1 padded — the sel_tok_idx argument of decode."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(cache_seqlens, "cache_seqlens", torch.int32, 1)
    B, Hq, d = q.shape
    num_pages, page, Hkv, d2 = k_cache.shape
    if d2 != d or block_table.shape[0] != B or cache_seqlens.numel() != B:
        raise ValueError("inconsistent shapes")
    out = torch.empty((B, Hkv, topk), dtype=torch.int32, device=q.device) if out is None else out
    ws = _workspace(workspace, int(_lib.sfa_index_topk_workspace_size(B, Hkv, block_table.shape[1], page)), q.device)
    rc = _lib.sfa_index_topk(_ptr(q), _ptr(k_cache), _ptr(block_table), block_table.shape[1], num_pages, page,
                             _ptr(cache_seqlens), B, Hq, Hkv, d, int(topk), int(n_local), _ptr(ws),
                             ws.numel() * ws.element_size(), _ptr(status), _ptr(out), _stream(stream))
    _check(rc)
    return out


@_on_tensor_device
def kv_append(k_new: torch.Tensor, v_new: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
              block_table: torch.Tensor, cache_seqlens: torch.Tensor, status: Optional[torch.Tensor] = None,
              stream=None) -> None:
    """In-place paged KV-cache append (sfa_kv_append): k_new / v_new (B, seqlen_new, Hkv, d) bf16 go to
    logical positions cache_seqlens[b] + j of k_cache / v_cache (num_pages, page, Hkv, d).
    cache_seqlens is not updated."""
    for t, name in ((k_new, "k_new"), (v_new, "v_new"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, name, torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(cache_seqlens, "cache_seqlens", torch.int32, 1)
    if k_new.shape != v_new.shape or k_cache.shape != v_cache.shape:
        raise ValueError("k / v shapes differ")
    B, S, Hkv, d = k_new.shape
    num_pages, page, hk2, d2 = k_cache.shape
    if (hk2, d2) != (Hkv, d) or block_table.shape[0] != B or cache_seqlens.numel() != B:
        raise ValueError("inconsistent shapes")
    rc = _lib.sfa_kv_append(_ptr(k_new), _ptr(v_new), S, _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                            block_table.shape[1], num_pages, page, _ptr(cache_seqlens), B, Hkv, d, _ptr(status),
                            _stream(stream))
    _check(rc)


def _batch_idx(cache_batch_idx, B, device):
    if cache_batch_idx is None:
        return torch.arange(B, dtype=torch.int32, device=device)
    _need(cache_batch_idx, "cache_batch_idx", torch.int32, 1)
    if cache_batch_idx.numel() != B:
        raise ValueError("cache_batch_idx must have one entry per sequence")
    return cache_batch_idx


@_on_tensor_device
def decode_kvcache(q, k_cache, v_cache, cache_seqlens, sel_tok_idx, *, cache_batch_idx=None, window_left: int = -1,
                   scale=None, num_splits: int = 0, out=None, lse=None, workspace=None, status=None, stream=None):
    """Top-k decode over non-paged caches (sfa_decode_kvcache): k_cache / v_cache (batch_cache,
    seqlen_cache, Hkv, d); sequence b reads row j at k_cache[cache_batch_idx[b], j] (None = 0..B-1,
    the flash_attn_with_kvcache default).  Other arguments and the result as decode()."""
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(q, "q", torch.bfloat16, 3)
    _need(cache_seqlens, "cache_seqlens", torch.int32, 1)
    _need(sel_tok_idx, "sel_tok_idx", torch.int32, 3)
    if k_cache.shape != v_cache.shape:
        raise ValueError("k_cache and v_cache must have the same shape")
    B, Hq, d = q.shape
    batch_cache, seqlen_cache, Hkv, dk = k_cache.shape
    if dk != d:
        raise ValueError("q and cache head dims differ")
    idx = _batch_idx(cache_batch_idx, B, q.device)
    topk = sel_tok_idx.shape[2]
    nbytes = decode_workspace_size(B, Hq, Hkv, d, topk, num_splits)
    ws = _workspace(workspace, nbytes, q.device)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if lse is None else lse
    rc = _lib.sfa_decode_kvcache(_ptr(q), _ptr(k_cache), _ptr(v_cache), batch_cache, seqlen_cache, _ptr(idx),
                                 _ptr(cache_seqlens), _ptr(sel_tok_idx), topk, B, Hq, Hkv, d, int(window_left),
                                 _scale(scale), int(num_splits), _ptr(ws), ws.numel() * ws.element_size(),
                                 _ptr(status), _ptr(out), _ptr(lse), _stream(stream))
    _check(rc)
    return out, lse


@_on_tensor_device
def kv_append_kvcache(k_new: torch.Tensor, v_new: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                      cache_seqlens: torch.Tensor, cache_batch_idx: Optional[torch.Tensor] = None,
                      status: Optional[torch.Tensor] = None, stream=None) -> None:
    """In-place append to non-paged caches (sfa_kv_append_kvcache): row j of k_new[b] goes to
    k_cache[cache_batch_idx[b], cache_seqlens[b] + j] (None = 0..B-1).  cache_seqlens is not updated."""
    for t, name in ((k_new, "k_new"), (v_new, "v_new"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, name, torch.bfloat16, 4)
    _need(cache_seqlens, "cache_seqlens", torch.int32, 1)
    if k_new.shape != v_new.shape or k_cache.shape != v_cache.shape:
        raise ValueError("k / v shapes differ")
    B, S, Hkv, d = k_new.shape
    batch_cache, seqlen_cache, hk2, d2 = k_cache.shape
    if (hk2, d2) != (Hkv, d) or cache_seqlens.numel() != B:
        raise ValueError("inconsistent shapes")
    idx = _batch_idx(cache_batch_idx, B, k_new.device)
    rc = _lib.sfa_kv_append_kvcache(_ptr(k_new), _ptr(v_new), S, _ptr(k_cache), _ptr(v_cache), batch_cache,
                                    seqlen_cache, _ptr(idx), _ptr(cache_seqlens), B, Hkv, d, _ptr(status),
                                    _stream(stream))
    _check(rc)


def bwd_workspace_size(batch, max_seqlen_q, max_seqlen_k, total_q, Hq, Hkv, d, topk, block_size) -> int:
    return int(_lib.sfa_bwd_workspace_size(batch, max_seqlen_q, max_seqlen_k, total_q, Hq, Hkv, d, topk,
                                           block_size))


@_on_tensor_device
def bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor, dout: torch.Tensor,
        lse: torch.Tensor, cu_seqlens_q: torch.Tensor, sel_idx: torch.Tensor, block_size: int, *,
        cu_seqlens_k: Optional[torch.Tensor] = None, max_seqlen_q: Optional[int] = None,
        max_seqlen_k: Optional[int] = None, causal: bool = True, window: Tuple[int, int] = (-1, -1),
        scale: Optional[float] = None, dq: Optional[torch.Tensor] = None, dk: Optional[torch.Tensor] = None,
        dv: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
        status: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Backward of fwd (sfa_bwd): given the forward's out and lse and the gradient dout of the loss
    with respect to out, returns dq (total_q, Hq, d), dk and dv (total_k, Hkv, d), bf16.  The other
    arguments are fwd's."""
    a = _FwdArgs(q, k, v, cu_seqlens_q, sel_idx, block_size, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal,
                 window, scale)
    for t, name in ((out, "out"), (dout, "dout")):
        _need(t, name, torch.bfloat16, 3)
        if t.shape != q.shape:
            raise ValueError(f"{name} must have q's shape {tuple(q.shape)}")
    _need(lse, "lse", torch.float32, 2)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    nbytes = bwd_workspace_size(*a.geom())
    ws = _workspace(workspace, nbytes, q.device)
    rc = _lib.sfa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), _ptr(cu_seqlens_q),
                      _ptr(cu_seqlens_k), a.batch, a.max_sq, a.max_sk, a.total_q, a.total_k, a.Hq, a.Hkv, a.d,
                      _ptr(sel_idx), a.topk, a.bs, a.causal, a.wl, a.wr, a.scale, _ptr(ws),
                      ws.numel() * ws.element_size(), _ptr(status), _ptr(dq), _ptr(dk), _ptr(dv), _stream(stream))
    _check(rc)
    return dq, dk, dv


@_on_tensor_device
def window_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens_q: torch.Tensor, *,
               cu_seqlens_k: Optional[torch.Tensor] = None, max_seqlen_q: Optional[int] = None,
               max_seqlen_k: Optional[int] = None, causal: bool = True, window: Tuple[int, int] = (-1, -1),
               window_per_head: Optional[Tuple[Optional[torch.Tensor], Optional[torch.Tensor]]] = None,
               scale: Optional[float] = None, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
               stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Sliding-window branch (sfa_window_fwd): every query attends to all keys its causal / window
    mask keeps.  Layouts as fwd, no selection.  window_per_head: optional (left, right) int32 (Hq)
    device tensors (either may be None) overriding `window` per query head.  Returns out
    (total_q, Hq, d) bf16, lse (Hq, total_q)."""
    a = _FwdArgs(q, k, v, cu_seqlens_q, None, 64, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal, window, scale,
                 topk=1)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((a.Hq, a.total_q), dtype=torch.float32, device=q.device) if lse is None else lse
    ws = _workspace(workspace, int(_lib.sfa_window_fwd_workspace_size()), q.device)
    wlh, wrh = window_per_head if window_per_head is not None else (None, None)
    for t, name in ((wlh, "window_left_per_head"), (wrh, "window_right_per_head")):
        if t is not None:
            _need(t, name, torch.int32, 1)
            if t.numel() != a.Hq:
                raise ValueError(f"{name} must have Hq = {a.Hq} elements")
    rc = _lib.sfa_window_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), a.batch, a.max_sq,
                             a.max_sk, a.total_q, a.total_k, a.Hq, a.Hkv, a.d, a.causal, a.wl, a.wr, _ptr(wlh),
                             _ptr(wrh), a.scale, _ptr(ws), ws.numel() * ws.element_size(), _ptr(status), _ptr(out),
                             _ptr(lse), _stream(stream))
    _check(rc)
    return out, lse


@_on_tensor_device
def gated_combine(branches, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Gated mix (sfa_gated_combine): out = sum over (o, g) in branches of g[..., None] * o, for up to
    three (o, g) pairs in the order (compressed, selected, window); None entries are left out.
    o bf16 (total_q, Hq, d), g fp32 (total_q, Hq)."""
    pairs = list(branches) + [None] * (3 - len(branches))
    if len(pairs) != 3:
        raise ValueError("at most three branches")
    ref = next((o for o, _ in (x for x in pairs if x is not None)), None)
    if ref is None:
        raise ValueError("no branch given")
    _need(ref, "o", torch.bfloat16, 3)
    total_q, Hq, d = ref.shape
    args = []
    for x in pairs:
        if x is None:
            args += [None, None]
            continue
        o, g = x
        _need(o, "o", torch.bfloat16, 3)
        _need(g, "g", torch.float32, 2)
        if tuple(o.shape) != (total_q, Hq, d) or tuple(g.shape) != (total_q, Hq):
            raise ValueError("branch shapes differ")
        args += [o, g]
    out = torch.empty_like(ref) if out is None else out
    rc = _lib.sfa_gated_combine(*[_ptr(t) for t in args], total_q, Hq, d, _ptr(out), _stream(stream))
    _check(rc)
    return out


@_on_tensor_device
def fwd_prep(cu_seqlens_q, sel_idx, *, Hq: int, d: int, block_size: int, cu_seqlens_k=None, max_seqlen_q=None,
             max_seqlen_k=None, causal=True, window=(-1, -1), workspace=None, status=None, stream=None):
    """Stage 1 (sfa_fwd_prep).  Returns (workspace, sel_c, cnt): sel_c (total_q, Hkv, topk) and
    cnt (total_q, Hkv) are int32 views into the workspace holding the canonical selection."""
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    _need(sel_idx, "sel_idx", torch.int32, 3)
    total_q, Hkv, topk = sel_idx.shape
    batch = cu_seqlens_q.numel() - 1
    max_sq = _seq_bounds(cu_seqlens_q) if max_seqlen_q is None else int(max_seqlen_q)
    if max_seqlen_k is None:
        max_seqlen_k = max_sq if cu_seqlens_k is None else _seq_bounds(cu_seqlens_k)
    geom = (batch, max_sq, int(max_seqlen_k), total_q, int(Hq), Hkv, int(d), topk, int(block_size))
    nbytes = fwd_workspace_size(*geom)
    ws = _workspace(workspace, nbytes, sel_idx.device)
    rc = _lib.sfa_fwd_prep(_ptr(cu_seqlens_q), _ptr(cu_seqlens_k), batch, max_sq, int(max_seqlen_k), total_q, int(Hq),
                           Hkv, int(d), _ptr(sel_idx), topk, int(block_size), 1 if causal else 0, int(window[0]),
                           int(window[1]), _ptr(ws), ws.numel() * ws.element_size(), _ptr(status), _stream(stream))
    _check(rc)
    off_sel = ctypes.c_size_t()
    off_cnt = ctypes.c_size_t()
    _check(_lib.sfa_fwd_workspace_offsets(*geom, ctypes.byref(off_sel), ctypes.byref(off_cnt)))
    flat = ws.view(torch.uint8).reshape(-1)
    sel_c = flat[off_sel.value:off_sel.value + total_q * Hkv * topk * 4].view(torch.int32).view(total_q, Hkv, topk)
    cnt = flat[off_cnt.value:off_cnt.value + total_q * Hkv * 4].view(torch.int32).view(total_q, Hkv)
    return ws, sel_c, cnt


@_on_tensor_device
def fwd_attend(q, k, v, cu_seqlens_q, workspace, *, topk: int, block_size: int, cu_seqlens_k=None,
               max_seqlen_q=None, max_seqlen_k=None, causal=True, window=(-1, -1), scale=None, out=None, lse=None,
               status=None, stream=None):
    """Stage 2 (sfa_fwd_attend) on a workspace filled by fwd_prep with the same arguments."""
    a = _FwdArgs(q, k, v, cu_seqlens_q, None, block_size, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal, window,
                 scale, topk=topk)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((a.Hq, a.total_q), dtype=torch.float32, device=q.device) if lse is None else lse
    rc = _lib.sfa_fwd_attend(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), a.batch, a.max_sq,
                             a.max_sk, a.total_q, a.total_k, a.Hq, a.Hkv, a.d, a.topk, a.bs, a.causal, a.wl, a.wr,
                             a.scale, _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
                             _ptr(out), _ptr(lse), _stream(stream))
    _check(rc)
    return out, lse


# ---------------------------------------------------------------------------------------
# Decode
# ---------------------------------------------------------------------------------------

def decode_num_splits(B, Hq, Hkv, d, topk_tok, num_splits=0) -> int:
    return int(_lib.sfa_decode_num_splits(B, Hq, Hkv, d, topk_tok, num_splits))


def decode_workspace_size(B, Hq, Hkv, d, topk_tok, num_splits=0) -> int:
    return int(_lib.sfa_decode_workspace_size(B, Hq, Hkv, d, topk_tok, num_splits))


def _dec_checks(q, k_cache, v_cache, block_table, cache_seqlens, sel_tok_idx, cache_dtype=torch.bfloat16):
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", cache_dtype, 4)
    _need(v_cache, "v_cache", cache_dtype, 4)
    _need(block_table, "block_table", torch.int32, 2)
    if cache_seqlens is not None:
        _need(cache_seqlens, "cache_seqlens", torch.int32, 1)
    if sel_tok_idx is not None:
        _need(sel_tok_idx, "sel_tok_idx", torch.int32, 3)
    if k_cache.shape != v_cache.shape:
        raise ValueError("k_cache and v_cache must have the same shape")
    B, Hq, d = q.shape
    num_pages, page, Hkv, dk = k_cache.shape
    if dk != d:
        raise ValueError("q and cache head dims differ")
    return B, Hq, d, num_pages, page, Hkv


@_on_tensor_device
def decode(q, k_cache, v_cache, block_table, cache_seqlens, sel_tok_idx, *, window_left: int = -1, scale=None,
           num_splits: int = 0, out=None, lse=None, workspace=None, status=None, stream=None):
    """Paged top-k decode (sfa_decode): q (B, Hq, d); caches (num_pages, page, Hkv, d);
    block_table (B, max_pages) int32; cache_seqlens (B,) int32; sel_tok_idx (B, Hkv, topk_tok)
    int32 positions, -1 = unused.  Returns out (B, Hq, d) bf16 and lse (B, Hq) fp32."""
    B, Hq, d, num_pages, page, Hkv = _dec_checks(q, k_cache, v_cache, block_table, cache_seqlens, sel_tok_idx)
    topk = sel_tok_idx.shape[2]
    nbytes = decode_workspace_size(B, Hq, Hkv, d, topk, num_splits)
    ws = _workspace(workspace, nbytes, q.device)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if lse is None else lse
    rc = _lib.sfa_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), block_table.shape[1], num_pages,
                         page, _ptr(cache_seqlens), _ptr(sel_tok_idx), topk, B, Hq, Hkv, d, int(window_left),
                         _scale(scale), int(num_splits), _ptr(ws), ws.numel() * ws.element_size(), _ptr(status),
                         _ptr(out), _ptr(lse), _stream(stream))
    _check(rc)
    return out, lse


@_on_tensor_device
def decode_fp8(q, k_cache, v_cache, block_table, cache_seqlens, sel_tok_idx, *, k_descale=None, v_descale=None,
               window_left: int = -1, scale=None, num_splits: int = 0, out=None, lse=None, workspace=None,
               status=None, stream=None):
    """Paged top-k decode over FP8 caches (sfa_decode_fp8): k_cache / v_cache hold E4M3 codes as uint8
    (num_pages, page, Hkv, d); k_descale / v_descale fp32 (B, Hkv) or None (1).  Otherwise as decode()."""
    B, Hq, d, num_pages, page, Hkv = _dec_checks(q, k_cache, v_cache, block_table, cache_seqlens, sel_tok_idx,
                                                 cache_dtype=torch.uint8)
    for name, t in (("k_descale", k_descale), ("v_descale", v_descale)):
        if t is not None:
            _need(t, name, torch.float32, 2)
            if tuple(t.shape) != (B, Hkv):
                raise ValueError(f"{name} must have shape (B, Hkv)")
    topk = sel_tok_idx.shape[2]
    nbytes = decode_workspace_size(B, Hq, Hkv, d, topk, num_splits)
    ws = _workspace(workspace, nbytes, q.device)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if lse is None else lse
    rc = _lib.sfa_decode_fp8(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_descale), _ptr(v_descale),
                             _ptr(block_table), block_table.shape[1], num_pages, page, _ptr(cache_seqlens),
                             _ptr(sel_tok_idx), topk, B, Hq, Hkv, d, int(window_left), _scale(scale), int(num_splits),
                             _ptr(ws), ws.numel() * ws.element_size(), _ptr(status), _ptr(out), _ptr(lse),
                             _stream(stream))
    _check(rc)
    return out, lse


@_on_tensor_device
def decode_prep(cache_seqlens, sel_tok_idx, *, Hq: int, d: int, max_pages_per_seq: int, page_size: int,
                window_left=-1, num_splits=0, workspace=None, status=None, stream=None):
    """Stage 1 (sfa_decode_prep).  Returns (workspace, tok_c, cnt) with int32 views into the
    workspace: tok_c (B, Hkv, topk_tok) canonical ascending positions, cnt (B, Hkv)."""
    _need(cache_seqlens, "cache_seqlens", torch.int32, 1)
    _need(sel_tok_idx, "sel_tok_idx", torch.int32, 3)
    B, Hkv, topk = sel_tok_idx.shape
    nbytes = decode_workspace_size(B, Hq, Hkv, d, topk, num_splits)
    ws = _workspace(workspace, nbytes, sel_tok_idx.device)
    rc = _lib.sfa_decode_prep(_ptr(cache_seqlens), _ptr(sel_tok_idx), topk, int(max_pages_per_seq), int(page_size), B,
                              int(Hq), Hkv, int(d), int(window_left), int(num_splits), _ptr(ws),
                              ws.numel() * ws.element_size(), _ptr(status), _stream(stream))
    _check(rc)
    off_t, off_c = ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib.sfa_decode_workspace_offsets(B, int(Hq), Hkv, int(d), topk, int(num_splits), ctypes.byref(off_t),
                                             ctypes.byref(off_c)))
    flat = ws.view(torch.uint8).reshape(-1)
    tok_c = flat[off_t.value:off_t.value + B * Hkv * topk * 4].view(torch.int32).view(B, Hkv, topk)
    cnt = flat[off_c.value:off_c.value + B * Hkv * 4].view(torch.int32).view(B, Hkv)
    return ws, tok_c, cnt


@_on_tensor_device
def decode_attend(q, k_cache, v_cache, block_table, workspace, *, topk_tok: int, scale=None, num_splits=0, out=None,
                  lse=None, status=None, stream=None):
    """sfa_decode_attend: the split kernel (and, beyond six splits, the combine kernel) on the
    canonical sets decode_prep wrote into the workspace."""
    B, Hq, d, num_pages, page, Hkv = _dec_checks(q, k_cache, v_cache, block_table, None, None)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if lse is None else lse
    rc = _lib.sfa_decode_attend(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), block_table.shape[1],
                                num_pages, page, int(topk_tok), B, Hq, Hkv, d, _scale(scale), int(num_splits),
                                _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
                                _ptr(out), _ptr(lse), _stream(stream))
    _check(rc)
    return out, lse


@_on_tensor_device
def decode_noalloc(q, k_cache, v_cache, block_table, cache_seqlens, sel_tok_idx, *, window_left: int = -1,
                   scale=None, num_splits: int = 0, out=None, lse=None, status=None, stream=None):
    """sfa_decode_noalloc: the same decode without a workspace, for callers that may not
    allocate device memory at call time.  Its scratch is a static 8 MiB device array shared by
    every call on the device (calls must not overlap on the GPU); the first call on a device
    should come before any stream capture.  Pass out/lse to avoid allocating them here."""
    B, Hq, d, num_pages, page, Hkv = _dec_checks(q, k_cache, v_cache, block_table, cache_seqlens, sel_tok_idx)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if lse is None else lse
    rc = _lib.sfa_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), block_table.shape[1],
                                 num_pages, page, _ptr(cache_seqlens), _ptr(sel_tok_idx), sel_tok_idx.shape[2], B, Hq,
                                 Hkv, d, int(window_left), _scale(scale), int(num_splits), _ptr(status), _ptr(out),
                                 _ptr(lse), _stream(stream))
    _check(rc)
    return out, lse
