"""Parity of fa_decode_splitkv (CUDA, sm_100a) with the fp64 oracle.

The full-size decode workload (64 sequences, KV lengths drawn uniformly from
[512, 32768], 32 query heads over 8 KV heads, head_dim 128, 8 splits) is run
exactly as the benchmark runs it and compared on every output row.  Small
cases cover head_dim 64/128/256, GQA groups 1/2/4/8, split counts, empty
chunks, sequences of one key and cache rows past the sequence end that hold
non-finite values.
"""
import numpy as np
import pytest

import oracle
from tiled_attention_23_b200 import synthetic as syn
from tiled_attention_23_b200 import attention as A
from _helpers import assert_close

pytestmark = pytest.mark.gpu


def run_decode(q, kc, vc, lens, scale, splits):
    import torch
    dq, dk, dv = (A.to_device_bf16(x) for x in (q, kc, vc))
    dl = torch.from_numpy(np.ascontiguousarray(lens, dtype=np.int32)).cuda()
    o, lse = A.decode_splitkv(dq, dk, dv, dl, splits, scale=scale)
    torch.cuda.synchronize()
    assert A.device_status() == A.FA_OK
    return A.to_f64(o)[:, 0], lse.cpu().double().numpy()


def small_case(B, Hq, Hkv, D, Lmax, lens, seed):
    w = syn.DecodeWorkload("t", B, Hq, Hkv, D, 1, Lmax, 1, seed=seed)
    q, kc, vc, _ = w.inputs()
    return q, kc, vc, np.array(lens, np.int32)


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_small_parity(D, G):
    Hkv = 2
    lens = [1, 77, 300, 64]
    q, kc, vc, lens = small_case(4, Hkv * G, Hkv, D, 300, lens, seed=D + G)
    scale = 1.0 / np.sqrt(D)
    for splits in (1, 3, 8):
        O, L = run_decode(q, kc, vc, lens, scale, splits)
        Or, Lr = oracle.decode(q, kc, vc, lens, scale)
        assert_close(O, L, Or, Lr, f"D={D} G={G} splits={splits}")


def test_many_splits_and_empty_chunks():
    q, kc, vc, lens = small_case(3, 8, 2, 128, 2000, [5, 1999, 640], seed=11)
    for splits in (16, 64):
        O, L = run_decode(q, kc, vc, lens, 0.09, splits)
        Or, Lr = oracle.decode(q, kc, vc, lens, 0.09)
        assert_close(O, L, Or, Lr, f"splits={splits}")


def test_garbage_past_sequence_end_is_ignored():
    q, kc, vc, lens = small_case(3, 8, 2, 128, 512, [17, 300, 511], seed=12)
    O, L = run_decode(q, kc, vc, lens, 0.088, 4)
    kc2, vc2 = kc.copy(), vc.copy()
    for b, n in enumerate(lens):
        kc2[b, n:] = 0x7FC0   # NaN
        vc2[b, n:] = 0x7F80   # +inf
    O2, L2 = run_decode(q, kc2, vc2, lens, 0.088, 4)
    np.testing.assert_array_equal(O, O2)
    np.testing.assert_array_equal(L, L2)


def test_decode_matches_last_row_of_prefill():
    """The decode query at position len-1 equals the last row of a causal prefill."""
    import torch
    from tiled_attention_23_b200 import attention as Am
    q, kc, vc, lens = small_case(1, 8, 2, 128, 700, [700], seed=13)
    O, L = run_decode(q, kc, vc, lens, 0.1, 8)
    qp = np.zeros((1, 700, 8, 128), np.uint16)
    qp[:, -1] = q[:, 0]
    dq, dk, dv = (Am.to_device_bf16(x) for x in (qp, kc, vc))
    o, lse = Am.fwd(dq, dk, dv, causal=True, scale=0.1)
    torch.cuda.synchronize()
    Op = Am.to_f64(o)[:, -1]
    Lp = lse.cpu().double().numpy()[:, :, -1]
    assert np.max(np.abs(O - Op)) <= 2e-2
    assert np.max(np.abs(L - Lp)) <= 5e-3


def test_full_decode_workload_all_rows():
    w = syn.DECODE
    q, kc, vc, lens = w.inputs()
    O, L = run_decode(q, kc, vc, lens, w.scale, w.num_splits)
    Or, Lr = oracle.decode(q, kc, vc, lens, w.scale)
    assert_close(O, L, Or, Lr, w.name)
    # the split count changes rounding only
    O1, L1 = run_decode(q, kc, vc, lens, w.scale, 1)
    assert_close(O1, L1, Or, Lr, w.name + " splits=1")
