"""Parity of fa_bwd (CUDA, sm_100a) with the fp64 backward oracle.

The forward runs on the GPU (its O and lse feed the backward, as in training);
dQ, dK, dV are compared with the oracle's exact gradients of the definition.
Tolerance: every product runs in bf16 with fp32 accumulation; P and dS enter
their products rounded to bf16 and each output is rounded to bf16 (at most
2^-9 relative each), and Delta = rowsum(dO o O) uses the bf16 O (2^-9 on O).
Those four roundings bound each gradient's error by about 4 * 2^-9 = 0.8 % of
its largest magnitude; the test holds it to 1 % (max|g - g_ref| <= 1e-2 *
max|g_ref|), against a measured worst case of 0.52 %.  Cases cover head_dim 64/128/256, GQA
groups 1/4, causal and bidirectional, tails that are not tile multiples and
fewer queries than keys, and the benchmarked Llama-shaped size on sampled
heads; the backward is also bitwise deterministic.
"""
import numpy as np
import pytest

import oracle
from tiled_attention_23_b200 import synthetic as syn
from tiled_attention_23_b200 import attention as A

pytestmark = pytest.mark.gpu

REL_TOL = 1e-2


def run(q, k, v, do, scale, causal):
    import torch
    dq_, dk_, dv_, ddo = (A.to_device_bf16(x) for x in (q, k, v, do))
    o, lse = A.fwd(dq_, dk_, dv_, causal=causal, scale=scale)
    gq, gk, gv = A.bwd(dq_, dk_, dv_, o, lse, ddo, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert A.device_status() == A.FA_OK
    return A.to_f64(gq), A.to_f64(gk), A.to_f64(gv)


def case(B, Lq, Lk, Hq, Hkv, D, seed):
    q = syn.normal_bf16((B, Lq, Hq, D), seed, 11)
    k = syn.normal_bf16((B, Lk, Hkv, D), seed, 12)
    v = syn.normal_bf16((B, Lk, Hkv, D), seed, 13)
    do = syn.normal_bf16((B, Lq, Hq, D), seed, 14)
    return q, k, v, do


def check(got, ref, what):
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        assert np.all(np.isfinite(g)), f"{what} {name}: non-finite"
        err = float(np.max(np.abs(g - r)))
        mag = float(np.max(np.abs(r)))
        assert err <= REL_TOL * mag, f"{what} {name}: max err {err:.3e} > {REL_TOL} * {mag:.3e}"


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("G", [1, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_small_backward_parity(D, G, causal):
    Hkv = 2
    q, k, v, do = case(2, 300, 300, Hkv * G, Hkv, D, seed=D + G + causal)
    scale = 1.0 / np.sqrt(D)
    got = run(q, k, v, do, scale, causal)
    ref = oracle.attention_backward(q, k, v, do, scale, causal)
    check(got, ref, f"D={D} G={G} causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_fewer_queries_than_keys(causal):
    q, k, v, do = case(1, 200, 333, 8, 2, 128, seed=60)
    got = run(q, k, v, do, 0.1, causal)
    ref = oracle.attention_backward(q, k, v, do, 0.1, causal)
    check(got, ref, f"Lq<Lk causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_head_dim_256_fewer_queries_than_keys_and_ragged_tails(causal):
    """head_dim 256 runs on 64-row tiles (64-key tiles in the dQ walk, 64-row
    query tiles in the separate dV and dK walks): tails that are not multiples
    of 64 on either side, fewer queries than keys, GQA group 2."""
    q, k, v, do = case(1, 193, 261, 4, 2, 256, seed=62)
    got = run(q, k, v, do, 1.0 / 16, causal)
    ref = oracle.attention_backward(q, k, v, do, 1.0 / 16, causal)
    check(got, ref, f"D=256 Lq<Lk causal={causal}")


def test_head_dim_256_long_gqa_sampled_heads():
    """The long-context GQA shape (B2 Hq32 Hkv8 L8192 D256, causal) at a quarter
    of its length: every gradient finite, and two query heads' dQ plus their
    K/V head's dK and dV (summed over its group of 4 query heads) against the
    oracle on that group."""
    import torch
    w = syn.LONG_GQA[4].with_(Lq=2048, Lk=2048)
    q, k, v = w.inputs()
    do = syn.normal_bf16((w.B, w.Lq, w.Hq, w.D), w.seed, syn.STREAM_Q + 10)
    gq, gk, gv, gdo = (A.to_device_bf16(x) for x in (q, k, v, do))
    o, lse = A.fwd(gq, gk, gv, causal=w.causal, scale=w.scale)
    dq, dk, dv = A.bwd(gq, gk, gv, o, lse, gdo, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    assert A.device_status() == A.FA_OK
    for t in (dq, dk, dv):
        assert bool(torch.isfinite(t).all())
    G = w.Hq // w.Hkv
    for b, hk in ((0, 0), (1, 5)):
        hs = slice(hk * G, (hk + 1) * G)
        ref = oracle.attention_backward(np.ascontiguousarray(q[b:b + 1, :, hs, :]),
                                        np.ascontiguousarray(k[b:b + 1, :, hk:hk + 1, :]),
                                        np.ascontiguousarray(v[b:b + 1, :, hk:hk + 1, :]),
                                        np.ascontiguousarray(do[b:b + 1, :, hs, :]), w.scale, w.causal)
        got = [A.to_f64(dq[b:b + 1, :, hs, :].contiguous()), A.to_f64(dk[b:b + 1, :, hk:hk + 1, :].contiguous()),
               A.to_f64(dv[b:b + 1, :, hk:hk + 1, :].contiguous())]
        check(got, ref, f"long GQA b={b} kv head={hk}")


def test_mid_size_causal_and_determinism():
    q, k, v, do = case(1, 1024, 1024, 8, 2, 128, seed=61)
    scale = 1.0 / np.sqrt(128)
    got = run(q, k, v, do, scale, True)
    ref = oracle.attention_backward(q, k, v, do, scale, True)
    check(got, ref, "mid causal")
    again = run(q, k, v, do, scale, True)
    for a, b in zip(got, again):
        np.testing.assert_array_equal(a, b)


def test_full_size_sampled_heads():
    """The benchmarked backward: the Llama-shaped causal prefill (B32 H32 L4096
    D128, K x 2) as timed by the benchmark; every gradient finite, and three
    (batch, head) slices - all of their rows - against the oracle (MHA: a head's
    dQ, dK, dV depend on that head alone)."""
    import torch
    w = syn.LLAMA_PREFILL
    q, k, v = w.inputs()
    do = syn.normal_bf16((w.B, w.Lq, w.Hq, w.D), w.seed, syn.STREAM_Q + 10)
    gq, gk, gv, gdo = (A.to_device_bf16(x) for x in (q, k, v, do))
    o, lse = A.fwd(gq, gk, gv, causal=w.causal, scale=w.scale)
    dq, dk, dv = A.bwd(gq, gk, gv, o, lse, gdo, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    assert A.device_status() == A.FA_OK
    for t in (dq, dk, dv):
        assert bool(torch.isfinite(t).all())
    assert w.Hq == w.Hkv
    for b, h in ((0, 0), (17, 21), (31, 31)):
        sl = lambda a: np.ascontiguousarray(a[b:b + 1, :, h:h + 1, :])
        ref = oracle.attention_backward(sl(q), sl(k), sl(v), sl(do), w.scale, w.causal)
        got = [A.to_f64(t[b:b + 1, :, h:h + 1, :].contiguous()) for t in (dq, dk, dv)]
        check(got, ref, f"full size b={b} h={h}")
