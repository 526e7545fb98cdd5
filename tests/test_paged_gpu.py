"""Parity of fa_decode_paged (CUDA, sm_100a) with the fp64 paged-cache oracle.

Pages are laid out in a seeded random order with spare pages, and every page
or row that no key uses holds NaN, so a read of the wrong page shows up.  The
kernel must match the oracle within the parity tolerances, and match the
contiguous-cache kernel bit for bit (same chunks, same arithmetic).  The
full-size decode workload (64 sequences, lengths in [512, 32768]) is run with
64-key pages exactly as the benchmark runs it.
"""
import numpy as np
import pytest

import oracle
from tiled_attention_23_b200 import synthetic as syn
from tiled_attention_23_b200 import attention as A
from _helpers import assert_close

pytestmark = pytest.mark.gpu


def _dev(q, kc, vc, lens):
    import torch
    return (*(A.to_device_bf16(x) for x in (q, kc, vc)),
            torch.from_numpy(np.ascontiguousarray(lens, dtype=np.int32)).cuda())


def run_paged(q, kp, vp, table, lens, scale, splits):
    import torch
    dq, dk, dv, dl = _dev(q, kp, vp, lens)
    dt = torch.from_numpy(np.ascontiguousarray(table, dtype=np.int32)).cuda()
    o, lse = A.decode_paged(dq, dk, dv, dt, dl, splits, scale=scale)
    torch.cuda.synchronize()
    assert A.device_status() == A.FA_OK
    return A.to_f64(o)[:, 0], lse.cpu().double().numpy()


def run_contiguous(q, kc, vc, lens, scale, splits):
    import torch
    dq, dk, dv, dl = _dev(q, kc, vc, lens)
    o, lse = A.decode_splitkv(dq, dk, dv, dl, splits, scale=scale)
    torch.cuda.synchronize()
    assert A.device_status() == A.FA_OK
    return A.to_f64(o)[:, 0], lse.cpu().double().numpy()


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("G", [1, 4, 8])
@pytest.mark.parametrize("page_size", [16, 48, 64, 256])
def test_small_paged_parity(D, G, page_size):
    Hkv = 2
    w = syn.DecodeWorkload("t", 4, Hkv * G, Hkv, D, 1, 300, 1, seed=D + G + page_size)
    q, kc, vc, _ = w.inputs()
    lens = np.array([1, 77, 300, 64], np.int32)
    kp, vp, table = syn.paginate(kc, vc, lens, page_size, seed=page_size, spare_pages=2)
    scale = 1.0 / np.sqrt(D)
    Or, Lr = oracle.decode_paged(q, kp, vp, table, lens, scale)
    for splits in (1, 3, 8):
        O, L = run_paged(q, kp, vp, table, lens, scale, splits)
        assert_close(O, L, Or, Lr, f"D={D} G={G} page={page_size} splits={splits}")
        Oc, Lc = run_contiguous(q, kc, vc, lens, scale, splits)
        np.testing.assert_array_equal(O, Oc)
        np.testing.assert_array_equal(L, Lc)


def test_full_decode_workload_paged():
    w = syn.DECODE
    q, kc, vc, lens = w.inputs()
    kp, vp, table = syn.paginate(kc, vc, lens, syn.DECODE_PAGE_SIZE, seed=7, spare_pages=16)
    O, L = run_paged(q, kp, vp, table, lens, w.scale, w.num_splits)
    Or, Lr = oracle.decode_paged(q, kp, vp, table, lens, w.scale)
    assert_close(O, L, Or, Lr, w.name + " paged")
    Oc, Lc = run_contiguous(q, kc, vc, lens, w.scale, w.num_splits)
    np.testing.assert_array_equal(O, Oc)
    np.testing.assert_array_equal(L, Lc)
