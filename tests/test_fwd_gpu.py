"""Parity of fa_fwd (CUDA, sm_100a) with the fp64 oracle, plus GPU invariants.

Small problems are compared element by element over every output; the
full-size workloads (the sizes the benchmark times, in the same launch
configuration) are compared on sampled rows that the oracle computes one by
one, and checked for properties that hold at any size.  Tolerances:
max|O - O_ref| <= 2e-2 and max|L - L_ref| <= 5e-3.
"""
import math

import numpy as np
import pytest

import oracle
from tiled_attention_23_b200 import synthetic as syn
from tiled_attention_23_b200 import attention as A
from _helpers import assert_close, gather_rows, oracle_rows, run_fwd, sample_rows

pytestmark = pytest.mark.gpu


def case(B, Lq, Lk, Hq, Hkv, D, seed=1, pow2=0):
    w = syn.PrefillWorkload("t", B, Lq, Lk, Hq, Hkv, D, False, k_pow2=pow2, seed=seed)
    return w.inputs()


def test_tiny_bidirectional_workload_full():
    w = syn.TINY_BIDIR
    q, k, v = w.inputs()
    O, L = run_fwd(q, k, v, w.scale, w.causal)
    Or, Lr = oracle.attention(q, k, v, w.scale, w.causal)
    assert O.shape == (1, 256, 2, 64) and L.shape == (1, 2, 256)
    assert_close(O, L, Or, Lr, w.name)


SMALL = [
    # B, Lq, Lk, Hq, Hkv, D
    (2, 300, 300, 4, 4, 64),     # 3 query tiles, ragged tail
    (1, 257, 257, 2, 2, 128),
    (1, 200, 333, 4, 2, 128),    # Lq < Lk, GQA 2
    (1, 130, 130, 4, 1, 256),    # GQA 4, head_dim 256
    (1, 192, 192, 8, 1, 256),    # GQA 8
    (2, 1, 77, 2, 2, 128),       # one query row
    (1, 64, 1000, 2, 2, 128),    # long ragged key range
    (1, 384, 384, 2, 2, 64),     # whole tiles only
    (1, 129, 129, 16, 2, 128),   # GQA 8, D 128
]


# Shapes large enough for the persistent form of the head_dim 64/128 kernel (one
# CTA per SM walking couples of query-tile pairs): an odd number of pairs (the
# middle pair has no partner), a tail pair whose second tile is past the end
# (Lq = 1100: pairs of 256 rows, the last one holds rows 1024-1099), GQA, fewer
# queries than keys, and head_dim 64.
PERSISTENT = [
    # B, Lq, Lk, Hq, Hkv, D
    (4, 1280, 1280, 32, 32, 128),   # 5 pairs per head: an unpartnered middle pair
    (4, 1100, 1100, 32, 8, 128),    # tail pair with an empty second tile, GQA 4
    (6, 900, 1300, 32, 16, 128),    # Lq < Lk, GQA 2
    (4, 1100, 1100, 32, 32, 64),    # head_dim 64
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", PERSISTENT)
def test_persistent_schedule_full_parity(shape, causal):
    B, Lq, Lk, Hq, Hkv, D = shape
    q, k, v = case(*shape, seed=sum(shape) + 7)
    scale = 1.0 / math.sqrt(D)
    O, L = run_fwd(q, k, v, scale, causal)
    Or, Lr = oracle.attention(q, k, v, scale, causal)
    assert_close(O, L, Or, Lr, f"persistent {shape} causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", SMALL)
def test_small_full_parity(shape, causal):
    B, Lq, Lk, Hq, Hkv, D = shape
    q, k, v = case(*shape, seed=sum(shape))
    scale = 1.0 / math.sqrt(D)
    O, L = run_fwd(q, k, v, scale, causal)
    Or, Lr = oracle.attention(q, k, v, scale, causal)
    assert_close(O, L, Or, Lr, f"{shape} causal={causal}")


def test_single_key_bidirectional():
    q, k, v = case(1, 5, 1, 2, 2, 64, seed=3)
    O, L = run_fwd(q, k, v, 0.125, False)
    Or, Lr = oracle.attention(q, k, v, 0.125, False)
    assert_close(O, L, Or, Lr, "Lk=1")


def test_sharpened_scores():
    """K scaled by 2 (as in the Llama-shaped workload) and a large scale."""
    q, k, v = case(1, 256, 256, 2, 2, 128, seed=4, pow2=1)
    for scale in (1.0 / math.sqrt(128), 0.5):
        for causal in (False, True):
            O, L = run_fwd(q, k, v, scale, causal)
            Or, Lr = oracle.attention(q, k, v, scale, causal)
            assert_close(O, L, Or, Lr, f"scale={scale} causal={causal}")


def test_zero_scale_gives_mean_of_allowed_values():
    q, k, v = case(1, 140, 140, 2, 2, 64, seed=5)
    O, L = run_fwd(q, k, v, 0.0, True)
    Or, Lr = oracle.attention(q, k, v, 0.0, True)
    assert_close(O, L, Or, Lr, "scale=0")


def test_causal_first_row_is_v0_bitwise_and_runs_are_deterministic():
    import torch
    q, k, v = case(2, 512, 512, 4, 2, 128, seed=6)
    dq, dk, dv = (A.to_device_bf16(x) for x in (q, k, v))
    o1, l1 = A.fwd(dq, dk, dv, causal=True)
    o2, l2 = A.fwd(dq, dk, dv, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    # row 0 sees key 0 only: p = 1, O = v0 exactly
    v0 = dv[:, 0].repeat_interleave(2, dim=1)
    assert torch.equal(o1[:, 0], v0)


def test_gqa_equals_mha_on_repeated_kv_bitwise():
    import torch
    q, k, v = case(1, 300, 300, 8, 2, 128, seed=7)
    dq, dk, dv = (A.to_device_bf16(x) for x in (q, k, v))
    o1, l1 = A.fwd(dq, dk, dv, causal=True)
    o2, l2 = A.fwd(dq, dk.repeat_interleave(4, dim=2).contiguous(), dv.repeat_interleave(4, dim=2).contiguous(),
                   causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_lse_optional():
    import torch
    q, k, v = case(1, 200, 200, 2, 2, 64, seed=8)
    dq, dk, dv = (A.to_device_bf16(x) for x in (q, k, v))
    o1, _ = A.fwd(dq, dk, dv, causal=False, want_lse=False)
    o2, _ = A.fwd(dq, dk, dv, causal=False)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


FULL = [syn.MID_CAUSAL, syn.LLAMA_PREFILL] + [syn.LONG_GQA[g] for g in (1, 2, 4, 8)]


@pytest.mark.parametrize("w", FULL, ids=[w.name for w in FULL])
def test_full_size_sampled_rows(w):
    """The benchmarked sizes: every output finite, sampled rows match the oracle,
    causal row 0 equals v0 bitwise."""
    import torch
    q, k, v = w.inputs()
    dq, dk, dv = (A.to_device_bf16(x) for x in (q, k, v))
    o, lse = A.fwd(dq, dk, dv, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    assert A.device_status() == A.FA_OK
    assert bool(torch.isfinite(o).all()) and bool(torch.isfinite(lse).all())
    rows = sample_rows(w.B, w.Lq, w.Hq, 384, seed=w.B + w.Hkv)
    Or, Lr = oracle_rows(q, k, v, w.scale, w.causal, rows)
    O = A.to_f64(o)
    L = lse.cpu().double().numpy()
    Og, Lg = gather_rows(O, L, rows, w.Lq, w.Hq)
    assert_close(Og, Lg, Or, Lr, w.name)
    if w.causal:
        G = w.Hq // w.Hkv
        assert torch.equal(o[:, 0], dv[:, 0].repeat_interleave(G, dim=1))
