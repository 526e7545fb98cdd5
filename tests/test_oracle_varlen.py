"""Pins of the variable-length (packed, block-diagonal) oracle (CPU only).

``oracle.attention_varlen`` walks a packed batch through its own code path.
Each sequence must equal the fixed-shape definition (pinned in
test_oracle_pins.py) run on that sequence alone, for Lq = Lk and for fewer
queries than keys (bottom-right causal alignment per sequence); rows with no
allowed key follow the stated convention (O = 0, L = -inf); and a tiny packed
case is checked against a 40-digit decimal brute force.
"""
from decimal import Decimal, getcontext

import numpy as np
import pytest

import oracle
from tiled_attention_23_b200 import synthetic as syn


def packed(lens_q, lens_k, Hq=4, Hkv=2, D=8, seed=40):
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    q = syn.normal_bf16((int(cu_q[-1]), Hq, D), seed, 11)
    k = syn.normal_bf16((max(int(cu_k[-1]), 1), Hkv, D), seed, 12)[: int(cu_k[-1])]
    v = syn.normal_bf16((max(int(cu_k[-1]), 1), Hkv, D), seed, 13)[: int(cu_k[-1])]
    return q, k, v, cu_q, cu_k


@pytest.mark.parametrize("causal", [False, True])
def test_each_sequence_equals_the_fixed_shape_definition(causal):
    lens_q = [5, 1, 17, 9]
    lens_k = [5, 3, 17, 20] if causal else [7, 3, 2, 20]
    q, k, v, cu_q, cu_k = packed(lens_q, lens_k)
    O, L = oracle.attention_varlen(q, k, v, cu_q, cu_k, 0.3, causal)
    for b in range(4):
        qs = q[cu_q[b]:cu_q[b + 1]][None]
        ks, vs = k[cu_k[b]:cu_k[b + 1]][None], v[cu_k[b]:cu_k[b + 1]][None]
        Or, Lr = oracle.attention(qs, ks, vs, 0.3, causal)
        np.testing.assert_allclose(O[cu_q[b]:cu_q[b + 1]], Or[0], rtol=0, atol=1e-13)
        np.testing.assert_allclose(L[:, cu_q[b]:cu_q[b + 1]], Lr[0], rtol=0, atol=1e-13)


def test_rows_without_keys_follow_the_convention():
    # sequence 0: no keys at all; sequence 1: causal with 5 queries over 3 keys
    q, k, v, cu_q, cu_k = packed([4, 5], [0, 3])
    O, L = oracle.attention_varlen(q, k, v, cu_q, cu_k, 0.5, True)
    assert np.all(O[0:4] == 0) and np.all(L[:, 0:4] == -np.inf)
    assert np.all(O[4:6] == 0) and np.all(L[:, 4:6] == -np.inf)     # rows 0, 1 of sequence 1
    Or, Lr = oracle.attention(q[6:9][None], k[0:3][None], v[0:3][None], 0.5, True)
    np.testing.assert_allclose(O[6:9], Or[0], rtol=0, atol=1e-13)
    np.testing.assert_allclose(L[:, 6:9], Lr[0], rtol=0, atol=1e-13)


def test_tiny_packed_against_decimal_brute_force():
    getcontext().prec = 40
    lens_q, lens_k = [3, 2], [4, 2]
    q, k, v, cu_q, cu_k = packed(lens_q, lens_k, Hq=2, Hkv=1, D=3, seed=41)
    O, L = oracle.attention_varlen(q, k, v, cu_q, cu_k, 0.6, True)
    qd, kd, vd = (oracle.bf16_bits_to_f64(x) for x in (q, k, v))
    dec = lambda x: Decimal(repr(float(x)))
    for b in range(2):
        Lq, Lk = lens_q[b], lens_k[b]
        for i in range(Lq):
            t = cu_q[b] + i
            keys = [cu_k[b] + j for j in range(Lk) if j <= i + Lk - Lq]
            for h in range(2):
                s = [dec(0.6) * sum(dec(qd[t, h, d]) * dec(kd[j, 0, d]) for d in range(3)) for j in keys]
                m = max(s)
                e = [(x - m).exp() for x in s]
                z = sum(e)
                for d in range(3):
                    ref = sum(ei * dec(vd[j, 0, d]) for ei, j in zip(e, keys)) / z
                    assert abs(float(ref) - O[t, h, d]) < 1e-13
                assert abs(float(m + z.ln()) - L[h, t]) < 1e-13


def test_rows_subset_matches_full():
    q, k, v, cu_q, cu_k = packed([6, 11, 3], [6, 11, 3])
    O, L = oracle.attention_varlen(q, k, v, cu_q, cu_k, 0.2, True)
    rows = np.array([0, 5, 17, 30, 79], np.int64)
    Os, Ls = oracle.attention_varlen(q, k, v, cu_q, cu_k, 0.2, True, rows=rows)
    np.testing.assert_array_equal(Os, O.reshape(-1, O.shape[-1])[rows])
    np.testing.assert_array_equal(Ls, L.T.reshape(-1)[rows])
