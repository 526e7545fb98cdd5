"""Pins of the KV-INT8 quantiser and int8-cache decode oracle (CPU only).

Quantiser: codes stay in [-127, 127], every non-zero row uses the full range,
an all-zero row gets scale 0, reconstruction is within half a step, and
values that are already a scale times an integer come back exactly.
Decode: with power-of-two scales the dequantised cache is exactly
representable in bf16, so the int8 oracle must equal the pinned bf16 decode
definition on that cache; a tiny case is checked against a 40-digit decimal
brute force.
"""
from decimal import Decimal, getcontext

import numpy as np
import pytest

import oracle
from tiled_attention_23_b200 import synthetic as syn


def test_quantiser_properties():
    x = syn.normal_bf16((2, 33, 3, 64), 5, 12, pow2=2)
    x[1, 7, 2] = 0                                   # an all-zero row
    codes, scales = oracle.quantize_kv_int8(x)
    assert codes.dtype == np.int8 and scales.shape == (2, 3, 33)
    assert codes.min() >= -127 and codes.max() <= 127
    xf = oracle.bf16_bits_to_f64(x)
    s = scales.transpose(0, 2, 1)[..., None].astype(np.float64)      # [B, L, H, 1]
    nz = np.abs(xf).max(axis=-1) > 0
    assert np.all(np.abs(codes).max(axis=-1)[nz] == 127)
    assert scales[1, 2, 7] == 0 and np.all(codes[1, 7, 2] == 0)
    err = np.abs(xf - s * codes)
    # half a step, plus the fp32 rounding of x / scale (|x / scale| <= 127, so <= 2^-17)
    assert np.all(err <= s * (0.5 + 2.0 ** -17) + 1e-30)


def test_quantiser_round_trips_scaled_integers():
    rng = np.random.default_rng(0)
    c = rng.integers(-127, 128, (1, 20, 2, 16))
    c[..., 0] = 127                                  # the row maximum is 127 * 2^-3
    x = (c.astype(np.float32) / 8.0).view(np.uint32) >> 16
    codes, scales = oracle.quantize_kv_int8(x.astype(np.uint16))
    np.testing.assert_array_equal(codes, c)
    assert np.all(scales == np.float32(0.125))


def tie_row(D):
    """A row whose maximum is 127 * 2^-3, so scale = 0.125 exactly, with entries
    at exact half steps 0.5, 1.5, 2.5, -2.5, 3.5 (all bf16 numbers).  Round half
    to even (the stated reading) gives codes 0, 2, 2, -2, 4; rounding half away
    from zero would give 1, 2, 3, -3, 4."""
    vals = np.zeros(D, np.float32)
    vals[0] = 127 * 0.125
    vals[1:6] = np.array([0.5, 1.5, 2.5, -2.5, 3.5], np.float32) * 0.125
    bits = vals.view(np.uint32)
    assert np.all(bits & 0xFFFF == 0)
    return (bits >> 16).astype(np.uint16)


def test_quantiser_rounds_exact_half_steps_to_even():
    x = np.zeros((1, 2, 1, 16), np.uint16)
    x[0, 0, 0] = tie_row(16)
    x[0, 1, 0] = tie_row(16) ^ np.uint16(0x8000) * (tie_row(16) != 0)   # the negated row
    codes, scales = oracle.quantize_kv_int8(x)
    assert np.all(scales == np.float32(0.125))
    np.testing.assert_array_equal(codes[0, 0, 0, :6], [127, 0, 2, 2, -2, 4])
    np.testing.assert_array_equal(codes[0, 1, 0, :6], [-127, 0, -2, -2, 2, -4])
    assert np.all(codes[0, :, 0, 6:] == 0)


def int8_cache(B, L, H, D, seed):
    rng = np.random.default_rng(seed)
    codes = rng.integers(-127, 128, (B, L, H, D)).astype(np.int8)
    scales = (2.0 ** rng.integers(-9, -2, (B, H, L))).astype(np.float32)
    deq = codes.astype(np.float32) * scales.transpose(0, 2, 1)[..., None]
    bits = (deq.view(np.uint32) >> 16).astype(np.uint16)
    assert np.all(deq.view(np.uint32) & 0xFFFF == 0)   # exactly representable in bf16
    return codes, scales, bits


@pytest.mark.parametrize("v_int8", [False, True])
def test_int8_decode_equals_bf16_decode_on_the_dequantised_cache(v_int8):
    B, Hq, Hkv, D, Lmax = 3, 8, 2, 32, 90
    q = syn.normal_bf16((B, 1, Hq, D), 3, 11)
    kc, ks, kb = int8_cache(B, Lmax, Hkv, D, 1)
    vc, vs, vb = int8_cache(B, Lmax, Hkv, D, 2)
    lens = np.array([1, 45, 90], np.int32)
    O, L = oracle.decode_int8(q, kc, ks, vc if v_int8 else vb, vs if v_int8 else None, lens, 0.3)
    Or, Lr = oracle.decode(q, kb, vb, lens, 0.3)
    np.testing.assert_allclose(O, Or, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Lr, rtol=0, atol=1e-12)


def test_tiny_int8_decode_against_decimal_brute_force():
    getcontext().prec = 40
    rng = np.random.default_rng(9)
    B, Hq, Hkv, D, Lmax = 1, 2, 1, 3, 5
    q = syn.normal_bf16((B, 1, Hq, D), 4, 11)
    kc = rng.integers(-127, 128, (B, Lmax, Hkv, D)).astype(np.int8)
    vc = rng.integers(-127, 128, (B, Lmax, Hkv, D)).astype(np.int8)
    ks = rng.uniform(0.001, 0.05, (B, Hkv, Lmax)).astype(np.float32)
    vs = rng.uniform(0.001, 0.05, (B, Hkv, Lmax)).astype(np.float32)
    lens = np.array([4], np.int32)
    O, L = oracle.decode_int8(q, kc, ks, vc, vs, lens, 0.9)
    qd = oracle.bf16_bits_to_f64(q)
    dec = lambda x: Decimal(repr(float(x)))
    for h in range(Hq):
        s = [dec(0.9) * sum(dec(qd[0, 0, h, d]) * dec(ks[0, 0, j]) * Decimal(int(kc[0, j, 0, d])) for d in range(D))
             for j in range(4)]
        m = max(s)
        e = [(x - m).exp() for x in s]
        z = sum(e)
        for d in range(D):
            ref = sum(e[j] * dec(vs[0, 0, j]) * Decimal(int(vc[0, j, 0, d])) for j in range(4)) / z
            assert abs(float(ref) - O[0, h, d]) < 1e-13
        assert abs(float(m + z.ln()) - L[0, h]) < 1e-13
