"""Helpers shared by the GPU parity tests: upload seeded inputs, compare with the oracle.

Tolerances (fixed by the benchmark spec of the problem): bf16 outputs within
|gpu - ref| <= 2e-2 + 2e-2 * |ref| element-wise; fp32 LSE within 1e-3 absolute; a row with
no kept key must be exactly 0 with lse exactly -inf; canonical index sets bit-exact.
"""
import numpy as np
import torch

from sfa_workloads import dev_tensor, upload_decode, upload_prefill  # noqa: F401 (re-exported)

OUT_ATOL = 2e-2
OUT_RTOL = 2e-2
LSE_ATOL = 1e-3


def run_fwd(sfa, c, d=None, status=None, sel=None, **kw):
    d = d or upload_prefill(c)
    return sfa.fwd(d["q"], d["k"], d["v"], d["cu_q"], d["sel"] if sel is None else sel, c.bs, cu_seqlens_k=d["cu_k"],
                   max_seqlen_q=c.max_sq, max_seqlen_k=c.max_sk, causal=bool(c.causal), window=(c.wl, c.wr),
                   scale=c.scale if c.scale > 0 else None, status=status, **kw)


def run_decode(sfa, c, d=None, status=None, sel=None, block_table=None, **kw):
    d = d or upload_decode(c)
    return sfa.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"] if block_table is None else block_table,
                      d["cache_seqlens"], d["sel"] if sel is None else sel, window_left=c.wl,
                      scale=c.scale if c.scale > 0 else None, status=status, **kw)


def assert_out_close(gpu, ref, what="out"):
    g = gpu.float().cpu().numpy().astype(np.float64) if isinstance(gpu, torch.Tensor) else gpu
    ref = np.asarray(ref, np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    excess = np.abs(g - ref) - (OUT_ATOL + OUT_RTOL * np.abs(ref))
    worst = np.unravel_index(np.argmax(excess), excess.shape)
    assert excess.max() <= 0, f"{what}: max excess {excess.max():.4g} at {worst}: gpu {g[worst]} ref {ref[worst]}"


def assert_lse_close(gpu, ref, what="lse"):
    g = gpu.cpu().numpy().astype(np.float64) if isinstance(gpu, torch.Tensor) else gpu
    ref = np.asarray(ref, np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    ninf = np.isneginf(ref)
    np.testing.assert_array_equal(np.isneginf(g), ninf, err_msg=f"{what}: -inf pattern differs")
    fin = ~ninf
    if fin.any():
        err = np.abs(g[fin] - ref[fin])
        assert err.max() <= LSE_ATOL, f"{what}: max |dlse| {err.max():.4g}"


def assert_empty_rows_exact(out_rows, lse_rows):
    """Rows with no kept key: exactly zero output and lse exactly -inf."""
    o = out_rows.float().cpu().numpy()
    assert (o == 0).all(), "empty row output is not exactly 0"
    assert np.isneginf(lse_rows.cpu().numpy()).all(), "empty row lse is not -inf"
