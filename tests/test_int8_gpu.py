"""Parity of the KV-INT8 path (CUDA, sm_100a) with the fp64 oracle.

fa_quantize_kv_int8 must reproduce the oracle's fp32 quantiser bit for bit
(codes are integer results decided in fp32 on both sides).  fa_decode_int8 is
fed codes and scales made by the oracle's quantiser (never by the CUDA path)
and must match the oracle's int8-cache decode within the parity tolerances,
for int8 K with bf16 V and for int8 K and V, head_dim 64/128/256, GQA groups
1/4/8 and several split counts; the full decode workload is compared on every
row in both modes.
"""
import numpy as np
import pytest

import oracle
from tiled_attention_23_b200 import synthetic as syn
from tiled_attention_23_b200 import attention as A
from _helpers import assert_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("D", [64, 128, 256])
def test_quantiser_is_bit_exact(D):
    from test_oracle_int8 import tie_row
    import torch
    x = syn.normal_bf16((3, 37, 4, D), D, 12, pow2=1)
    x[1, 5, 2] = 0                                    # all-zero row
    x[2, 9, 1, :] = 0x3F80                            # constant row of 1.0
    x[0, 3, 0] = tie_row(D)                           # exact half steps: round half to even
    codes_r, scales_r = oracle.quantize_kv_int8(x)
    codes, scales = A.quantize_kv_int8(A.to_device_bf16(x))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(codes.cpu().numpy(), codes_r)
    np.testing.assert_array_equal(scales.cpu().numpy(), scales_r)


def quantised_case(B, Hq, Hkv, D, Lmax, lens, seed):
    w = syn.DecodeWorkload("t", B, Hq, Hkv, D, 1, Lmax, 1, seed=seed)
    q, kc, vc, _ = w.inputs()
    kq, ks = oracle.quantize_kv_int8(kc)
    vq, vs = oracle.quantize_kv_int8(vc)
    return q, kc, vc, kq, ks, vq, vs, np.array(lens, np.int32)


def run_int8(q, kq, ks, v, vs, lens, scale, splits):
    import torch
    dq = A.to_device_bf16(q)
    dk, dks = torch.from_numpy(kq).cuda(), torch.from_numpy(ks).cuda()
    if vs is None:
        dv, dvs = A.to_device_bf16(v), None
    else:
        dv, dvs = torch.from_numpy(v).cuda(), torch.from_numpy(vs).cuda()
    dl = torch.from_numpy(np.ascontiguousarray(lens, dtype=np.int32)).cuda()
    o, lse = A.decode_int8(dq, dk, dks, dv, dvs, dl, splits, scale=scale)
    torch.cuda.synchronize()
    assert A.device_status() == A.FA_OK
    return A.to_f64(o)[:, 0], lse.cpu().double().numpy()


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("G", [1, 4, 8])
@pytest.mark.parametrize("v_int8", [False, True])
def test_small_int8_parity(D, G, v_int8):
    Hkv = 2
    q, kc, vc, kq, ks, vq, vs, lens = quantised_case(4, Hkv * G, Hkv, D, 300, [1, 77, 300, 64], seed=D + G)
    scale = 1.0 / np.sqrt(D)
    v, vsc = (vq, vs) if v_int8 else (vc, None)
    Or, Lr = oracle.decode_int8(q, kq, ks, v, vsc, lens, scale)
    for splits in (1, 3, 8):
        O, L = run_int8(q, kq, ks, v, vsc, lens, scale, splits)
        assert_close(O, L, Or, Lr, f"D={D} G={G} v_int8={v_int8} splits={splits}")


def test_nonfinite_bf16_v_past_the_end_is_ignored():
    q, kc, vc, kq, ks, vq, vs, lens = quantised_case(3, 8, 2, 128, 512, [17, 300, 511], seed=12)
    O, L = run_int8(q, kq, ks, vc, None, lens, 0.088, 4)
    vc2, ks2 = vc.copy(), ks.copy()
    for b, n in enumerate(lens):
        vc2[b, n:] = 0x7F80          # +inf in bf16 V rows past the end
        ks2[b, :, n:] = np.nan       # NaN K scales past the end
    O2, L2 = run_int8(q, kq, ks2, vc2, None, lens, 0.088, 4)
    np.testing.assert_array_equal(O, O2)
    np.testing.assert_array_equal(L, L2)


@pytest.mark.parametrize("v_int8", [False, True])
def test_full_decode_workload_int8(v_int8):
    w = syn.DECODE
    q, kc, vc, lens = w.inputs()
    kq, ks = oracle.quantize_kv_int8(kc)
    if v_int8:
        v, vsc = oracle.quantize_kv_int8(vc)
    else:
        v, vsc = vc, None
    O, L = run_int8(q, kq, ks, v, vsc, lens, w.scale, w.num_splits)
    Or, Lr = oracle.decode_int8(q, kq, ks, v, vsc, lens, w.scale)
    assert_close(O, L, Or, Lr, f"{w.name} int8 v_int8={v_int8}")
