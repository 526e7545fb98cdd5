"""Pins of the oracle's e4m3 codec, per-head FP8 quantiser and FP8-input attention.

The codec is written from the OCP 8-bit floating-point definition (E4M3: one
sign bit, four exponent bits with bias 7, three mantissa bits, subnormals at
exponent field 0, no infinities, S.1111.111 = NaN, largest finite 448); the
FP8 operands are those of FlashAttention-3 ("FlashAttention-2 (TH)", section
on FlashAttention-3).  Pins: torch's float8_e4m3fn type (a library routine),
closed-form code values, round-to-nearest-even ties, the quantiser's scale
invariances, and reduction of FP8 attention to the bf16 definition when every
dequantised value is a bf16 number.
"""
import math

import numpy as np
import pytest

import oracle
from tiled_attention_23_b200 import synthetic as syn

torch = pytest.importorskip("torch")


def torch_decode(codes):
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def test_decode_matches_library_for_every_code():
    c = np.arange(256, dtype=np.uint8)
    v, t = oracle.e4m3_decode(c), torch_decode(c)
    assert np.array_equal(np.isnan(v), np.isnan(t))
    assert np.isnan(v).sum() == 2                      # 0x7F and 0xFF only
    assert np.array_equal(v[~np.isnan(v)], t[~np.isnan(t)])


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6), (0x38, 1.0), (0x39, 1.125),
    (0x3F, 1.875), (0x40, 2.0), (0x7E, 448.0), (0x77, 240.0), (0xB8, -1.0), (0xFE, -448.0),
])
def test_decode_closed_forms(code, value):
    assert oracle.e4m3_decode(np.array([code], np.uint8))[0] == value


def test_negative_zero_and_nan():
    v = oracle.e4m3_decode(np.array([0x80, 0x7F, 0xFF], np.uint8))
    assert v[0] == 0.0 and math.copysign(1.0, v[0]) < 0
    assert np.isnan(v[1]) and np.isnan(v[2])


def test_encode_inverts_decode_on_every_finite_code():
    c = np.array([i for i in range(256) if i not in (0x7F, 0xFF)], np.uint8)
    v = oracle.e4m3_decode(c).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(v), c)


def test_encode_ties_go_to_even_mantissa():
    # midpoints between neighbouring positive codes (exact in float32)
    c = np.arange(0x00, 0x7E, dtype=np.uint8)
    lo, hi = oracle.e4m3_decode(c), oracle.e4m3_decode(c + 1)
    mid = ((lo + hi) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (lo + hi) / 2)
    got = oracle.e4m3_encode(mid)
    want = np.where(c % 2 == 0, c, c + 1).astype(np.uint8)   # the even code of the pair
    assert np.array_equal(got, want)
    assert np.array_equal(oracle.e4m3_encode(-mid), want | 0x80)


def test_encode_matches_library_rounding_in_range():
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.normal(0, 30, 20000), rng.normal(0, 0.01, 5000), rng.uniform(-447, 447, 5000)])
    x = x.astype(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(x), want)


def test_encode_saturates():
    x = np.array([448.0, 460.0, 464.0, 500.0, 1e30, np.inf, -1e9, -np.inf], np.float32)
    assert list(oracle.e4m3_encode(x)) == [0x7E] * 6 + [0xFE] * 2


def test_quantiser_maps_the_head_maximum_to_448_and_bounds_the_error():
    x = syn.normal_bf16((2, 300, 3, 64), 11, syn.STREAM_Q)
    codes, descale = oracle.quantize_fp8(x)
    xv = oracle.bf16_bits_to_f64(x)
    amax = np.abs(xv).max(axis=(1, 3))                       # [B, H]
    assert np.array_equal(descale, (amax.astype(np.float32) / np.float32(448)).astype(np.float32))
    vals = oracle.e4m3_decode(codes)
    assert np.abs(vals).max() == 448.0
    for b in range(2):
        for h in range(3):
            assert np.abs(vals[b, :, h]).max() == 448.0
            y = xv[b, :, h] * (448.0 / amax[b, h])            # exact-scale image of x
            err = np.abs(vals[b, :, h] - y)
            # half an e4m3 step: 2^-4 relative for normals, 2^-10 absolute below 2^-6,
            # plus the fp32 rounding of inv and of the product
            bound = np.maximum(np.abs(y) * 2.0 ** -4, 2.0 ** -10) + np.abs(y) * 2.0 ** -22
            assert (err <= bound).all()


def test_quantiser_is_invariant_to_power_of_two_head_scaling():
    x = syn.normal_bf16((1, 200, 2, 64), 12, syn.STREAM_K)
    x2 = syn.normal_bf16((1, 200, 2, 64), 12, syn.STREAM_K, pow2=3)   # the same values times 8
    c1, d1 = oracle.quantize_fp8(x)
    c2, d2 = oracle.quantize_fp8(x2)
    assert np.array_equal(c1, c2)
    assert np.array_equal(d2, d1 * np.float32(8))


def test_quantiser_all_zero_head():
    x = syn.normal_bf16((1, 64, 2, 64), 13, syn.STREAM_V)
    x[:, :, 1, :] = 0
    codes, descale = oracle.quantize_fp8(x)
    assert descale[0, 1] == 1.0 and not codes[:, :, 1, :].any()
    assert descale[0, 0] != 1.0


def bf16_bits_of(v):
    """bf16 bit patterns of float64 values that are bf16 numbers (checked)."""
    f = v.astype(np.float32)
    bits = (f.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(oracle.bf16_bits_to_f64(bits), v)
    return bits


@pytest.mark.parametrize("causal,G", [(False, 1), (True, 2)])
def test_fp8_attention_reduces_to_the_definition_on_bf16_values(causal, G):
    # power-of-two descales keep code * descale a bf16 number (3 mantissa bits)
    B, L, Hq, D = 2, 150, 4, 64
    Hkv = Hq // G
    q8 = oracle.quantize_fp8(syn.normal_bf16((B, L, Hq, D), 14, syn.STREAM_Q))[0]
    k8 = oracle.quantize_fp8(syn.normal_bf16((B, L, Hkv, D), 14, syn.STREAM_K))[0]
    v8 = oracle.quantize_fp8(syn.normal_bf16((B, L, Hkv, D), 14, syn.STREAM_V))[0]
    qd = np.full((B, Hq), 2.0 ** -7, np.float32)
    kd = np.full((B, Hkv), 2.0 ** -6, np.float32)
    vd = np.full((B, Hkv), 2.0 ** -8, np.float32)
    vd[1] *= 4
    O8, L8 = oracle.attention_fp8(q8, k8, v8, qd, kd, vd, 0.125, causal)
    q = bf16_bits_of(oracle.e4m3_decode(q8) * 2.0 ** -7)
    k = bf16_bits_of(oracle.e4m3_decode(k8) * 2.0 ** -6)
    v = bf16_bits_of(oracle.e4m3_decode(v8) * vd[:, None, :, None].astype(np.float64))
    O, Lr = oracle.attention(q, k, v, 0.125, causal)
    assert np.allclose(O8, O, rtol=0, atol=1e-12)
    assert np.allclose(L8, Lr, rtol=0, atol=1e-12)


def test_fp8_attention_brute_force_with_general_descales():
    B, L, H, D = 1, 40, 2, 64
    q8 = oracle.quantize_fp8(syn.normal_bf16((B, L, H, D), 15, syn.STREAM_Q))[0]
    k8 = oracle.quantize_fp8(syn.normal_bf16((B, L, H, D), 15, syn.STREAM_K))[0]
    v8 = oracle.quantize_fp8(syn.normal_bf16((B, L, H, D), 15, syn.STREAM_V))[0]
    qd = np.array([[0.0071, 0.0093]], np.float32)
    kd = np.array([[0.0113, 0.0057]], np.float32)
    vd = np.array([[0.0311, 0.0029]], np.float32)
    O8, L8 = oracle.attention_fp8(q8, k8, v8, qd, kd, vd, 0.3, True)
    qv = oracle.e4m3_decode(q8) * qd[:, None, :, None]
    kv = oracle.e4m3_decode(k8) * kd[:, None, :, None]
    vv = oracle.e4m3_decode(v8) * vd[:, None, :, None]
    for h in range(H):
        s = 0.3 * qv[0, :, h] @ kv[0, :, h].T
        s[np.triu_indices(L, 1)] = -np.inf
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        assert np.allclose(O8[0, :, h], (p @ vv[0, :, h]) / p.sum(axis=1, keepdims=True), rtol=1e-12, atol=1e-14)
        assert np.allclose(L8[0, h], (m[:, 0] + np.log(p.sum(axis=1))), rtol=1e-12, atol=1e-12)


def test_quantiser_tiny_head_keeps_unit_factors():
    # bf16 subnormals: amax < 2^-110, so inv = descale = 1 and every code is e4m3(x) = +-0
    x = syn.normal_bf16((1, 64, 2, 64), 16, syn.STREAM_V)
    x[:, :, 1, :] &= 0x807F
    codes, descale = oracle.quantize_fp8(x)
    assert descale[0, 1] == 1.0
    assert set(np.unique(codes[:, :, 1, :]).tolist()) <= {0x00, 0x80}
    neg = (x[:, :, 1, :] & 0x8000) != 0
    assert np.array_equal(codes[:, :, 1, :] == 0x80, neg)
