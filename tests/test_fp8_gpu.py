"""FP8 (e4m3) prefill and its per-head quantiser on the GPU against the oracle.

The FP8 path is FlashAttention-3's low-precision forward, named on the
"FlashAttention-2 (TH)" page (section on FlashAttention-3).  The quantiser is
compared bit for bit.  The attention result is the fp64 definition on the
dequantised inputs; its tolerance follows from the arithmetic (derived in the
design notes and restated in fp8_tolerance below): P enters the P V product
rounded to e4m3, so each probability carries up to 2^-4 relative error
(normal range) or 2^-10 absolute (subnormal range, where the kernel's
exponent offset keeps every p below 2^-12 of the row maximum and the row sum
at least 2^6).
"""
import numpy as np
import pytest

import oracle
from tiled_attention_23_b200 import synthetic as syn
from tiled_attention_23_b200 import attention as A
from _helpers import L_TOL, sample_rows

pytestmark = pytest.mark.gpu


def fp8_tolerance(q8, k8, v8, qd, kd, vd, scale, causal, rows, Or, Lq, Lk, Hq, Hkv):
    """Per-element bound on |O - O_ref| for rows (flat (b*Hq+h)*Lq+i):
    (2^-4 + 2^-9) sum_j p_j |v_j| + n_keys 2^-16 max|v| + 2^-8 |O_ref| + 1e-5."""
    A_abs, _ = oracle.attention_fp8(q8, k8, v8 & np.uint8(0x7F), qd, kd, vd, scale, causal, rows=rows)
    i = rows % Lq
    h = (rows // Lq) % Hq
    b = rows // (Lq * Hq)
    g = h // (Hq // Hkv)
    n_keys = np.minimum(Lk, i + (Lk - Lq) + 1) if causal else np.full(rows.shape, Lk)
    vmax = np.abs(oracle.e4m3_decode(v8)).max(axis=(1, 3)) * vd      # [B, Hkv]
    vmax_r = vmax[b, g]
    return ((2.0 ** -4 + 2.0 ** -9) * A_abs + (n_keys * 2.0 ** -16 * vmax_r)[:, None]
            + 2.0 ** -8 * np.abs(Or) + 1e-5)


def quantized_inputs(B, Lq, Lk, Hq, Hkv, D, seed, k_pow2=0):
    q8, qd = oracle.quantize_fp8(syn.normal_bf16((B, Lq, Hq, D), seed, syn.STREAM_Q))
    k8, kd = oracle.quantize_fp8(syn.normal_bf16((B, Lk, Hkv, D), seed, syn.STREAM_K, k_pow2))
    v8, vd = oracle.quantize_fp8(syn.normal_bf16((B, Lk, Hkv, D), seed, syn.STREAM_V))
    return q8, k8, v8, qd, kd, vd


def run_fp8(q8, k8, v8, qd, kd, vd, scale, causal):
    import torch
    dev = [torch.from_numpy(np.ascontiguousarray(x)).cuda() for x in (q8, k8, v8, qd, kd, vd)]
    o, lse = A.fwd_fp8(*dev, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert A.device_status() == A.FA_OK
    return A.to_f64(o), lse.cpu().double().numpy()


def check(q8, k8, v8, qd, kd, vd, scale, causal, what):
    B, Lq, Hq, D = q8.shape
    Lk, Hkv = k8.shape[1], k8.shape[2]
    O, L = run_fp8(q8, k8, v8, qd, kd, vd, scale, causal)
    assert np.isfinite(O).all() and np.isfinite(L).all(), what
    rows = np.arange(B * Hq * Lq, dtype=np.int64)
    Or, Lr = oracle.attention_fp8(q8, k8, v8, qd, kd, vd, scale, causal, rows=rows)
    i, h, b = rows % Lq, (rows // Lq) % Hq, rows // (Lq * Hq)
    Og, Lg = O[b, i, h], L[b, h, i]
    tol = fp8_tolerance(q8, k8, v8, qd, kd, vd, scale, causal, rows, Or, Lq, Lk, Hq, Hkv)
    err = np.abs(Og - Or)
    worst = float((err / tol).max())
    assert worst <= 1.0, f"{what}: max |O - O_ref| / tol = {worst:.3f} (max err {err.max():.3e})"
    el = float(np.abs(Lg - Lr).max())
    assert el <= L_TOL, f"{what}: max|L - L_ref| = {el:.3e}"
    return err.max(), worst


@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,causal", [
    (1, 256, 256, 2, 2, False),     # two query tiles, two key tiles
    (2, 300, 300, 4, 2, True),      # ragged tail, GQA 2
    (1, 200, 700, 8, 1, True),      # Lq < Lk (bottom-right causal), GQA 8
    (1, 1000, 1000, 4, 1, False),   # eight key tiles, ragged
    (2, 1, 129, 4, 4, False),       # one query row, key tail of one
    (1, 129, 129, 2, 1, True),      # second query tile of one row
])
def test_fp8_small_full_parity(B, Lq, Lk, Hq, Hkv, causal):
    q8, k8, v8, qd, kd, vd = quantized_inputs(B, Lq, Lk, Hq, Hkv, 128, seed=Lq + Lk + Hq)
    check(q8, k8, v8, qd, kd, vd, 128 ** -0.5, causal, f"fp8 B{B} Lq{Lq} Lk{Lk} Hq{Hq} Hkv{Hkv} c{causal}")


@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,causal", [
    (1, 256, 256, 2, 2, False),     # two query tiles, two key tiles
    (2, 300, 300, 4, 2, True),      # ragged tail, GQA 2
    (1, 200, 700, 8, 1, True),      # Lq < Lk, GQA 8
    (1, 1000, 1000, 4, 4, False),   # eight key tiles, ragged
])
def test_fp8_head_dim_64_parity(B, Lq, Lk, Hq, Hkv, causal):
    q8, k8, v8, qd, kd, vd = quantized_inputs(B, Lq, Lk, Hq, Hkv, 64, seed=Lq + 3 * Lk + Hq)
    check(q8, k8, v8, qd, kd, vd, 64 ** -0.5, causal, f"fp8 D64 B{B} Lq{Lq} Lk{Lk} Hq{Hq} Hkv{Hkv} c{causal}")


@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,causal", [
    (1, 256, 256, 2, 2, False),     # four 64-key tiles
    (2, 300, 300, 4, 2, True),      # ragged tail, GQA 2
    (1, 200, 700, 8, 1, True),      # Lq < Lk, GQA 8
    (1, 129, 129, 2, 1, True),      # second query tile of one row
])
def test_fp8_head_dim_256_parity(B, Lq, Lk, Hq, Hkv, causal):
    q8, k8, v8, qd, kd, vd = quantized_inputs(B, Lq, Lk, Hq, Hkv, 256, seed=Lq + 2 * Lk + Hq)
    check(q8, k8, v8, qd, kd, vd, 256 ** -0.5, causal, f"fp8 D256 B{B} Lq{Lq} Lk{Lk} Hq{Hq} Hkv{Hkv} c{causal}")


def test_fp8_sharp_scores_and_extreme_codes():
    # raw codes over the whole finite range (subnormals, +-448, signed zeros)
    # with descales that make the softmax sharp (P near one-hot)
    B, L, H, D = 1, 384, 2, 128

    def codes(stream):
        c = syn.uniform_int(B * L * H * D, 21, stream, 0, 253).astype(np.uint8)
        c[c >= 0x7F] += 1                       # no NaN code (0x7F; 0xFF is out of range)
        return c.reshape(B, L, H, D)

    q8, k8, v8 = codes(syn.STREAM_Q), codes(syn.STREAM_K), codes(syn.STREAM_V)
    qd = np.full((B, H), 1 / 448, np.float32)
    kd = np.full((B, H), 1 / 64, np.float32)
    vd = np.array([[1 / 448, 1.0]], np.float32)
    check(q8, k8, v8, qd, kd, vd, 0.5, True, "fp8 raw codes")


@pytest.mark.parametrize("shape", [(2, 300, 3, 128), (1, 1000, 2, 64), (1, 130, 4, 256), (3, 64, 1, 128)])
def test_quantizer_bit_exact(shape):
    import torch
    x = syn.normal_bf16(shape, 31, syn.STREAM_K, pow2=-3)
    x[0, :, 0, :] = 0                          # an all-zero head
    if shape[2] > 1:
        x[-1, :, 1, :] &= 0x807F               # a head of tiny (exponent-stripped) values
    codes, ds = A.quantize_fp8(A.to_device_bf16(x))
    torch.cuda.synchronize()
    c_ref, d_ref = oracle.quantize_fp8(x)
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    assert np.array_equal(ds.cpu().numpy(), d_ref)


def test_fp8_runs_are_deterministic():
    import torch
    q8, k8, v8, qd, kd, vd = quantized_inputs(1, 512, 512, 4, 2, 128, seed=5)
    dev = [torch.from_numpy(np.ascontiguousarray(x)).cuda() for x in (q8, k8, v8, qd, kd, vd)]
    o1, _ = A.fwd_fp8(*dev, causal=True)
    o2, _ = A.fwd_fp8(*dev, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


FULL = [syn.LLAMA_PREFILL, syn.LONG_GQA[4]]


@pytest.mark.parametrize("w", FULL, ids=[w.name for w in FULL])
def test_fp8_full_size_sampled_rows(w):
    """The benchmarked Llama-shaped causal prefill (B32 H32 L4096 D128, K x 2) and
    the long GQA prefill (B2 Hq32 Hkv8 L8192 D256): quantised on the device,
    codes of the sampled heads equal the oracle's, and sampled rows match the
    oracle within the FP8 bound."""
    import torch
    q, k, v = w.inputs()
    xs = [A.to_device_bf16(x) for x in (q, k, v)]
    (q8d, qdd), (k8d, kdd), (v8d, vdd) = (A.quantize_fp8(x) for x in xs)
    o, lse = A.fwd_fp8(q8d, k8d, v8d, qdd, kdd, vdd, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    assert A.device_status() == A.FA_OK
    assert bool(torch.isfinite(o).all()) and bool(torch.isfinite(lse).all())
    rows = sample_rows(w.B, w.Lq, w.Hq, 96, seed=17)
    G = w.Hq // w.Hkv
    worst = 0.0
    for bh in sorted(set((rows // w.Lq).tolist())):
        b, h = divmod(bh, w.Hq)
        g = h // G
        sl = lambda a, hh: np.ascontiguousarray(a[b:b + 1, :, hh:hh + 1, :])
        q8, qd = oracle.quantize_fp8(sl(q, h))
        k8, kd = oracle.quantize_fp8(sl(k, g))
        v8, vd = oracle.quantize_fp8(sl(v, g))
        assert np.array_equal(q8d[b, :, h].cpu().numpy(), q8[0, :, 0])
        assert np.array_equal(k8d[b, :, g].cpu().numpy(), k8[0, :, 0])
        assert np.array_equal(v8d[b, :, g].cpu().numpy(), v8[0, :, 0])
        assert qdd[b, h].item() == qd[0, 0] and kdd[b, g].item() == kd[0, 0] and vdd[b, g].item() == vd[0, 0]
        ii = np.array(sorted(r % w.Lq for r in rows if r // w.Lq == bh), dtype=np.int64)
        Or, Lr = oracle.attention_fp8(q8, k8, v8, qd, kd, vd, w.scale, w.causal, rows=ii)
        Og = o[b, ii, h].double().cpu().numpy()
        Lg = lse[b, h, ii].double().cpu().numpy()
        tol = fp8_tolerance(q8, k8, v8, qd, kd, vd, w.scale, w.causal, ii, Or, w.Lq, w.Lk, 1, 1)
        worst = max(worst, float((np.abs(Og - Or) / tol).max()))
        assert float(np.abs(Lg - Lr).max()) <= L_TOL
    assert worst <= 1.0, f"max |O - O_ref| / tol = {worst:.3f}"
