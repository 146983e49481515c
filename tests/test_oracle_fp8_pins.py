"""Pins of the FP8 KV-cache decode oracle (oracle.decode_fp8) and of the E4M3 codes it reads.

The cache format is FP8 E4M3 with a descale per (sequence, kv head), as the k_descale / v_descale
arguments of the FlashAttention-3 docstrings (flash-attention-npu page) take it, and FP8 caches are a
feature of the Flash-Sparse-Attention README ("Fused Quant").  Pinned here:
  * the code tables: the workload's encoder and the oracle's decoder against PyTorch's float8_e4m3fn;
  * with unit descales the FP8 decode is the bf16 decode of the same values (every E4M3 value is a
    bf16 value), checked against the C oracle;
  * the descales act where the definition puts them: k_descale scales the scores (the same as scaling
    q), v_descale scales the output and leaves the LSE;
  * a two-token closed form;
  * the generator's quantisation error is within half a spacing of the format.
"""
import dataclasses

import numpy as np
import pytest

import oracle
import sfa_workloads as W

torch = pytest.importorskip("torch")


def test_e4m3_encoder_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(200000).astype(np.float32) * np.float32(60),
                        rng.standard_normal(20000).astype(np.float32) * np.float32(0.01),
                        np.array([0.0, -0.0, 448, 449, 464, 465, 1e9, -1e9, 2 ** -9, 2 ** -10, 3 * 2 ** -11,
                                  2 ** -6, 0.0625 * 1.0625, 15 * 2 ** -10], np.float32)])
    want = torch.from_numpy(x).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(W.f32_to_e4m3_bits(x), want)


def test_e4m3_decoder_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_decode(codes)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(want)
    assert nan.sum() == 2 and (np.isnan(got) == nan).all()
    np.testing.assert_array_equal(got[~nan], want[~nan])
    # spot values of the format: 1.0, 448, the smallest subnormal, the largest subnormal
    assert got[0x38] == 1.0 and got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x07] == 7 * 2.0 ** -9


def _as_bf16_case(c):
    """The same cached values as bf16 bit patterns (exact: E4M3 values are bf16 values)."""
    kb = W.f32_to_bf16_bits((oracle.e4m3_decode(c.k_cache) * 1.0).astype(np.float32))
    vb = W.f32_to_bf16_bits((oracle.e4m3_decode(c.v_cache) * 1.0).astype(np.float32))
    return dataclasses.replace(c, k_cache=kb, v_cache=vb, k_descale=None, v_descale=None)


def test_unit_descale_equals_bf16_decode(oracle_lib):
    c = W.make_decode_fp8(61, 3, 8, 2, 64, 32, 300, 900, 200, 16)
    c = dataclasses.replace(c, k_descale=np.ones_like(c.k_descale), v_descale=np.ones_like(c.v_descale),
                            wl=400)
    o8, l8, b8 = oracle_lib.decode_fp8(c)
    ob, lb, bb = oracle_lib.decode(_as_bf16_case(c))
    np.testing.assert_allclose(o8, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l8, lb, rtol=0, atol=1e-12)
    assert list(b8) == list(bb)


def test_descales_act_on_scores_and_outputs(oracle_lib):
    c = W.make_decode_fp8(62, 2, 8, 2, 128, 64, 200, 600, 150, 8)
    base_o, base_l, _ = oracle_lib.decode_fp8(c)
    # k_descale x 2 == the scores x 2 == q x 2 (bf16 doubling is exact)
    c2 = dataclasses.replace(c, k_descale=c.k_descale * np.float32(2))
    qf = W.bf16_bits_to_f32(c.q) * np.float32(2)
    c3 = dataclasses.replace(c, q=W.f32_to_bf16_bits(qf))
    o2, l2, _ = oracle_lib.decode_fp8(c2)
    o3, l3, _ = oracle_lib.decode_fp8(c3)
    np.testing.assert_allclose(o2, o3, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(l2, l3, rtol=1e-12, atol=1e-12)
    # v_descale x 4 (exact in float32): outputs x 4, lse unchanged
    c4 = dataclasses.replace(c, v_descale=c.v_descale * np.float32(4))
    o4, l4, _ = oracle_lib.decode_fp8(c4)
    np.testing.assert_allclose(o4, 4 * base_o, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(l4, base_l)


def test_two_token_closed_form(oracle_lib):
    """One sequence, one kv head, two selected tokens: out = (e^s0 v0 + e^s1 v1) / (e^s0 + e^s1)."""
    d, page = 64, 16
    rng = np.random.default_rng(5)
    q = W.f32_to_bf16_bits(rng.standard_normal((1, 1, d)).astype(np.float32))
    kc = W.f32_to_e4m3_bits(rng.standard_normal((1, page, 1, d)).astype(np.float32) * 30)
    vc = W.f32_to_e4m3_bits(rng.standard_normal((1, page, 1, d)).astype(np.float32) * 30)
    kd, vd = np.array([[0.05]], np.float32), np.array([[0.02]], np.float32)
    c = W.DecodeCase("two", q, kc, vc, np.array([[0]], np.int32), np.array([10], np.int32),
                     np.array([[[7, 3, 7, -1]]], np.int32), 1, 1, d, page, k_descale=kd, v_descale=vd)
    out, lse, bad = oracle_lib.decode_fp8(c)
    qv = W.bf16_bits_to_f32(q)[0, 0].astype(np.float64)
    K = oracle.e4m3_decode(kc)[0, [3, 7], 0] * float(kd[0, 0])
    V = oracle.e4m3_decode(vc)[0, [3, 7], 0] * float(vd[0, 0])
    s = (K @ qv) / np.sqrt(d)
    w = np.exp(s - s.max())
    np.testing.assert_allclose(out[0, 0], (w @ V) / w.sum(), rtol=1e-13, atol=1e-15)
    assert abs(lse[0, 0] - (s.max() + np.log(w.sum()))) < 1e-13
    assert list(bad) == [0, 0]


def test_generator_quantisation_within_half_spacing():
    c = W.make_decode_fp8(63, 2, 4, 2, 64, 32, 100, 300, 50, 4)
    src = W.make_decode(63, 2, 4, 2, 64, 32, 100, 300, 50, 4)
    for b in range(c.B):
        pages = c.block_table[b][c.block_table[b] >= 0]
        for h in range(c.Hkv):
            for codes, raw, ds in ((c.k_cache, src.k_cache, c.k_descale), (c.v_cache, src.v_cache, c.v_descale)):
                x = W.bf16_bits_to_f32(raw[pages, :, h]).astype(np.float64) / float(ds[b, h])
                y = oracle.e4m3_decode(codes[pages, :, h])
                assert np.abs(x).max() <= 448.0 * (1 + 1e-6)
                # half a spacing: 2^-4 relative for normals, 2^-10 absolute in the subnormal range
                assert (np.abs(y - x) <= np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10) + 1e-12).all()
