"""Pins of the paged-cache decode oracle (CPU only).

``oracle.decode_paged`` gathers keys through a block table; it shares no code
path with ``oracle.decode`` (the contiguous-cache definition, pinned in
test_oracle_pins.py).  A page layout that holds the same keys must give the
same result, whatever the physical order of the pages; pages and rows that no
key uses (filled with NaN) must never be read; and a tiny case is checked
against a 40-digit decimal brute force of the gathered keys.
"""
from decimal import Decimal, getcontext

import numpy as np
import pytest

import oracle
from tiled_attention_23_b200 import synthetic as syn


def case(B=4, Hq=8, Hkv=2, D=16, Lmax=200, lens=(1, 17, 64, 199), seed=30):
    w = syn.DecodeWorkload("t", B, Hq, Hkv, D, 1, Lmax, 1, seed=seed)
    q, kc, vc, _ = w.inputs()
    return q, kc, vc, np.array(lens, np.int32)


@pytest.mark.parametrize("page_size", [1, 7, 16, 64, 256])
def test_paged_equals_contiguous(page_size):
    q, kc, vc, lens = case()
    kp, vp, table = syn.paginate(kc, vc, lens, page_size, seed=page_size, spare_pages=3)
    O, L = oracle.decode_paged(q, kp, vp, table, lens, 0.25)
    Or, Lr = oracle.decode(q, kc, vc, lens, 0.25)
    np.testing.assert_allclose(O, Or, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Lr, rtol=0, atol=1e-12)
    assert np.all(np.isfinite(O)) and np.all(np.isfinite(L))   # NaN pages / tail rows untouched


def test_page_order_does_not_matter():
    q, kc, vc, lens = case(seed=31)
    a = oracle.decode_paged(q, *syn.paginate(kc, vc, lens, 16, seed=1), lens, 0.3)
    b = oracle.decode_paged(q, *syn.paginate(kc, vc, lens, 16, seed=2, spare_pages=5), lens, 0.3)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_tiny_paged_against_decimal_brute_force():
    getcontext().prec = 40
    q, kc, vc, lens = case(B=2, Hq=4, Hkv=2, D=3, Lmax=9, lens=(9, 4), seed=32)
    kp, vp, table = syn.paginate(kc, vc, lens, 2, seed=5, spare_pages=1)
    O, L = oracle.decode_paged(q, kp, vp, table, lens, 0.7)
    qd, kd, vd = (oracle.bf16_bits_to_f64(x) for x in (q, kp, vp))
    for b in range(2):
        for h in range(4):
            g = h // 2
            rows = [(table[b, j // 2], j % 2) for j in range(lens[b])]
            s = [Decimal(repr(0.7)) * sum(Decimal(repr(float(qd[b, 0, h, d]))) * Decimal(repr(float(kd[pg, r, g, d])))
                                          for d in range(3)) for pg, r in rows]
            m = max(s)
            e = [(x - m).exp() for x in s]
            z = sum(e)
            for d in range(3):
                ref = sum(ei * Decimal(repr(float(vd[pg, r, g, d]))) for ei, (pg, r) in zip(e, rows)) / z
                assert abs(float(ref) - O[b, h, d]) < 1e-13
            assert abs(float(m + z.ln()) - L[b, h]) < 1e-13


def test_rejects_table_entries_out_of_range():
    q, kc, vc, lens = case()
    kp, vp, table = syn.paginate(kc, vc, lens, 16)
    bad = table.copy()
    bad[3, 0] = kp.shape[0]
    with pytest.raises(ValueError):
        oracle.decode_paged(q, kp, vp, bad, lens, 0.25)
