"""The FP8 forward's error bound, checked on a CPU model of its arithmetic.

The bound used by the GPU parity tests (FP8 support of FlashAttention-3, named
on the "FlashAttention-2 (TH)" page; the derivation is the design notes'
reading of the FP8 path):

    |O - O_ref| <= (2^-4 + 2^-9) sum_j p_j |v_j| + n_keys 2^-16 max|v| + 2^-8 |O_ref| + 1e-5

Here a plain numpy model takes the kernel's rounding steps - fp32 scores, the
online softmax over 128-key tiles with a stale reference max (slack 2, base 2),
P scaled by 2^6 and rounded to e4m3 (the oracle's encoder), the row sum of the
unrounded P - and the test checks that the bound holds for it and is not
vacuous.  bf16 output rounding is left out of the model (its 2^-8 |O| term is
kept in the bound, as on the GPU).
"""
import numpy as np
import pytest

import oracle
from tiled_attention_23_b200 import synthetic as syn

THRESHOLD, P_EXP, TILE = 2.0, 6.0, 128


def model_row(s_row, v, sl2):
    """One query row: s_row [n] fp32 scores, v [n, D] fp64 values."""
    m = -np.inf
    l = np.float32(0)
    o = np.zeros(v.shape[1])
    for k0 in range(0, s_row.shape[0], TILE):
        t = s_row[k0:k0 + TILE].astype(np.float32) * np.float32(sl2)
        t_max = np.float32(t.max())
        alpha = np.float32(1)
        if m == -np.inf:
            m = t_max
        elif t_max > m + THRESHOLD:
            alpha = np.exp2(np.float32(m - t_max))
            m = t_max
        p = np.exp2(t - np.float32(m - P_EXP)).astype(np.float32)
        p8 = oracle.e4m3_decode(oracle.e4m3_encode(p))
        l = np.float32(l * alpha + p.sum(dtype=np.float32))
        o = o * float(alpha) + p8 @ v[k0:k0 + TILE]
    return o / float(l)


@pytest.mark.parametrize("seed,kscale", [(1, 0), (2, 2), (3, 4)])
def test_bound_holds_on_a_model_of_the_kernel(seed, kscale):
    B, L, H, D = 1, 700, 2, 64
    q8, qd = oracle.quantize_fp8(syn.normal_bf16((B, L, H, D), seed, syn.STREAM_Q))
    k8, kd = oracle.quantize_fp8(syn.normal_bf16((B, L, H, D), seed, syn.STREAM_K, kscale))
    v8, vd = oracle.quantize_fp8(syn.normal_bf16((B, L, H, D), seed, syn.STREAM_V))
    scale = D ** -0.5
    rows = np.arange(B * H * L, dtype=np.int64)[::7]
    Or, _ = oracle.attention_fp8(q8, k8, v8, qd, kd, vd, scale, False, rows=rows)
    Oa, _ = oracle.attention_fp8(q8, k8, v8 & np.uint8(0x7F), qd, kd, vd, scale, False, rows=rows)
    qv, kv, vv = (oracle.e4m3_decode(a) for a in (q8, k8, v8))
    worst = 0.0
    for n, r in enumerate(rows):
        i, h = r % L, (r // L) % H
        s = (qv[0, i, h] @ kv[0, :, h].T).astype(np.float32)          # exact products, fp32 sum
        sl2 = scale * float(qd[0, h]) * float(kd[0, h]) * np.log2(np.e)
        o = model_row(s, vv[0, :, h] * float(vd[0, h]), sl2)
        vmax = np.abs(vv[0, :, h]).max() * float(vd[0, h])
        bound = (2.0 ** -4 + 2.0 ** -9) * Oa[n] + L * 2.0 ** -16 * vmax + 2.0 ** -8 * np.abs(Or[n]) + 1e-5
        err = np.abs(o - Or[n])
        assert (err <= bound).all(), f"row {r}: max err/bound {float((err / bound).max()):.3f}"
        worst = max(worst, float((err / bound).max()))
    # the bound is not vacuous: the rounding of P uses a visible share of it
    assert worst > 0.05


def test_exponent_offset_keeps_p_in_the_normal_range():
    # with the offset, the largest p of a tile lies in [2^6, 2^8]: below 448 and far above e4m3's subnormals
    t = np.linspace(-3.0, 0.0, 1000, dtype=np.float32)       # t - m in [-slack - 1, 0]
    for slack in (0.0, 1.0, THRESHOLD):
        p = np.exp2(t + np.float32(slack + P_EXP))
        assert p.max() <= 2.0 ** 8 * (1 + 1e-6) and oracle.e4m3_decode(oracle.e4m3_encode(p)).max() <= 448
        assert np.exp2(np.float32(P_EXP)) >= 2.0 ** -6 * 2 ** 12          # row max is 2^12 above the subnormal edge
