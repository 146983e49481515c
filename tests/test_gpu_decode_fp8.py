"""GPU parity of the FP8 KV-cache decode (sfa_decode_fp8) through the C ABI.

The caches hold FP8 E4M3 codes with a descale per (sequence, kv head); the oracle (oracle.decode_fp8)
dequantizes exactly in fp64.  The kernel computes with the cached values themselves (E4M3 values are
exact in bf16), so the tolerance is the decode's own: |gpu - ref| <= 2e-2 + 2e-2 |ref| for out,
|dlse| <= 1e-3, empty rows exactly 0 / -inf.  With unit descales the FP8 call must equal sfa_decode on
a bf16 cache holding the same values bit for bit: the same kernel arithmetic after the conversion."""
import dataclasses

import numpy as np
import pytest

import oracle
import sfa_workloads as W
from tests.parity import assert_empty_rows_exact, assert_lse_close, assert_out_close, dev_tensor, upload_decode

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sfa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_flashattention_b200 as m
    return m


def _upload_fp8(c):
    d = upload_decode(dataclasses.replace(c, k_cache=np.zeros(1, np.uint16), v_cache=np.zeros(1, np.uint16)))
    d["k_cache"] = dev_tensor(c.k_cache)
    d["v_cache"] = dev_tensor(c.v_cache)
    d["kd"] = dev_tensor(np.ascontiguousarray(c.k_descale, np.float32))
    d["vd"] = dev_tensor(np.ascontiguousarray(c.v_descale, np.float32))
    return d


def _run(sfa, c, d, **kw):
    return sfa.decode_fp8(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["cache_seqlens"], d["sel"],
                          k_descale=d["kd"], v_descale=d["vd"], window_left=c.wl,
                          scale=c.scale if c.scale > 0 else None, **kw)


CASES = {
    "b4_hq32_d128": lambda: W.make_decode_fp8(71, 4, 32, 8, 128, 256, 700, 3000, 256, 32),
    "b3_hq8_d64_page32": lambda: W.make_decode_fp8(72, 3, 8, 2, 64, 32, 300, 1500, 200, 16),
    "window": lambda: dataclasses.replace(W.make_decode_fp8(73, 4, 16, 4, 128, 64, 500, 2500, 300, 8), wl=700),
    "long_selection_prep": lambda: W.make_decode_fp8(74, 2, 8, 2, 128, 64, 6000, 9000, 3000, 64),
}


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("splits", [0, 9])
def test_decode_fp8_parity(sfa, name, splits):
    c = CASES[name]()
    d = _upload_fp8(c)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = _run(sfa, c, d, num_splits=splits, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ro, rl, bad = oracle.decode_fp8(c)
    assert list(bad) == [0, 0]
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


def test_unit_descale_equals_bf16_decode_bitwise(sfa):
    c = W.make_decode_fp8(75, 4, 32, 8, 128, 256, 700, 3000, 256, 32)
    c = dataclasses.replace(c, k_descale=np.ones_like(c.k_descale), v_descale=np.ones_like(c.v_descale))
    d = _upload_fp8(c)
    out8, lse8 = _run(sfa, c, d)
    kb = W.f32_to_bf16_bits(oracle.e4m3_decode(c.k_cache).astype(np.float32))
    vb = W.f32_to_bf16_bits(oracle.e4m3_decode(c.v_cache).astype(np.float32))
    cb = dataclasses.replace(c, k_cache=kb, v_cache=vb, k_descale=None, v_descale=None)
    db = upload_decode(cb)
    outb, lseb = sfa.decode(db["q"], db["k_cache"], db["v_cache"], db["block_table"], db["cache_seqlens"], db["sel"])
    torch.cuda.synchronize()
    assert torch.equal(out8.view(torch.int16), outb.view(torch.int16))
    assert torch.equal(lse8.view(torch.int32), lseb.view(torch.int32))
    # no descale arrays: the same as unit descales
    o2, l2 = sfa.decode_fp8(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["cache_seqlens"], d["sel"])
    assert torch.equal(o2.view(torch.int16), out8.view(torch.int16)) and torch.equal(l2, lse8)


def test_decode_fp8_bad_page_padding_and_empty(sfa):
    c = W.make_decode_fp8(76, 4, 8, 2, 128, 64, 300, 900, 100, 8)
    bt = c.block_table.copy()
    bt[1, 0] = c.num_pages + 2
    sel = c.sel.copy()
    sel[2] = -1  # a sequence with nothing selected: out 0, lse -inf
    c2 = dataclasses.replace(c, block_table=bt, sel=sel)
    d = _upload_fp8(c2)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = _run(sfa, c2, d, status=status)
    torch.cuda.synchronize()
    ro, rl, bad = oracle.decode_fp8(c2)
    assert bad[1] > 0 and int(status.item()) & 2
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
    assert_empty_rows_exact(out[2], lse[2])


def test_decode_fp8_full_size(sfa):
    """The paged decode workload at full size (B32, Hq32/Hkv8, L up to 131072, 2048 tokens per
    (sequence, kv head)) with its caches quantized to E4M3 on the device (per (sequence, kv head)
    descale = max |value| / 448, round to nearest even, as the workload generator does), in the
    launch configuration the benchmark times: every output row against the oracle."""
    c = W.config5()
    d = upload_decode(c)
    kq, vq, kd, vd = W.quantize_cache_e4m3_device(c, d)
    out, lse = sfa.decode_fp8(d["q"], kq, vq, d["block_table"], d["cache_seqlens"], d["sel"], k_descale=kd,
                              v_descale=vd)
    torch.cuda.synchronize()
    cf = dataclasses.replace(c, k_cache=kq.cpu().numpy(), v_cache=vq.cpu().numpy(), k_descale=kd.cpu().numpy(),
                             v_descale=vd.cpu().numpy())
    ro, rl, bad = oracle.decode_fp8(cf)
    assert list(bad) == [0, 0]
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
