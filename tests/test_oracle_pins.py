"""Pins of the fp64 oracle against what the mathematics fixes (CPU only).

Each test checks the oracle against something other than itself: an
independent high-precision brute force on tiny inputs (Python ``decimal``),
closed forms (constant V, zero Q, a single key, the first causal row, two-key
sigmoid cases from the golden fixture), invariants (rows of P sum to one,
permutation invariance, GQA as MHA with repeated K/V), a library routine for a
special case (``scipy.special.logsumexp`` on scores built with numpy), and the
pages' own claim that the tiled online softmax gives the standard result
("FlashAttention in Ascend CANN ops-transformer", section 二, step 2).
A dropped term, a wrong sign, an off-by-one causal limit, a wrong GQA head map
or a transposed operand fails at least one of them.
"""
import json
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest
from scipy.special import logsumexp

import oracle
from tiled_attention_23_b200 import synthetic as syn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f64(bits):
    return oracle.bf16_bits_to_f64(bits)


def bf16_bits(x):
    """Exact fp64 -> bf16 bits for values that are representable (test helper)."""
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "value not exactly representable in bf16"
    return (u >> 16).astype(np.uint16)


def rand_case(B, Lq, Lk, Hq, Hkv, D, seed, pow2=0):
    q = syn.normal_bf16((B, Lq, Hq, D), seed, 11)
    k = syn.normal_bf16((B, Lk, Hkv, D), seed, 12, pow2)
    v = syn.normal_bf16((B, Lk, Hkv, D), seed, 13)
    return q, k, v


# ----------------------------------------------------------------------------
# Independent brute force in 40-digit decimal arithmetic.
# ----------------------------------------------------------------------------
def brute_force_decimal(q, k, v, scale, causal):
    getcontext().prec = 40
    qd, kd, vd = f64(q), f64(k), f64(v)
    B, Lq, Hq, D = q.shape
    _, Lk, Hkv, _ = k.shape
    G = Hq // Hkv
    sc = Decimal(repr(scale))
    O = np.zeros((B, Lq, Hq, D))
    L = np.zeros((B, Hq, Lq))
    for b in range(B):
        for h in range(Hq):
            g = h // G
            for i in range(Lq):
                keys = [j for j in range(Lk) if (not causal) or j <= i + (Lk - Lq)]
                scores = []
                for j in keys:
                    acc = Decimal(0)
                    for d in range(D):
                        acc += Decimal(repr(float(qd[b, i, h, d]))) * Decimal(repr(float(kd[b, j, g, d])))
                    scores.append(sc * acc)
                m = max(scores)
                ws = [(s - m).exp() for s in scores]
                tot = sum(ws)
                for d in range(D):
                    num = sum(w * Decimal(repr(float(vd[b, j, g, d]))) for w, j in zip(ws, keys))
                    O[b, i, h, d] = float(num / tot)
                L[b, h, i] = float(m + tot.ln())
    return O, L


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(2, 3, 5, 4, 2, 3), (1, 5, 5, 2, 1, 4), (1, 1, 6, 2, 2, 2),
                                   (2, 4, 7, 8, 1, 3)])
def test_matches_decimal_brute_force(shape, causal):
    B, Lq, Lk, Hq, Hkv, D = shape
    q, k, v = rand_case(B, Lq, Lk, Hq, Hkv, D, seed=hash(shape) & 0xFFFF)
    scale = 0.7
    O, L = oracle.attention(q, k, v, scale, causal)
    Ob, Lb = brute_force_decimal(q, k, v, scale, causal)
    np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-13)
    np.testing.assert_allclose(L, Lb, rtol=0, atol=1e-13)


def test_large_scores_do_not_overflow():
    """K scaled by 2**5 and scale 1: scores in the hundreds; exp must not overflow."""
    q, k, v = rand_case(1, 4, 6, 2, 2, 4, seed=7, pow2=5)
    O, L = oracle.attention(q, k, v, 1.0, False)
    Ob, Lb = brute_force_decimal(q, k, v, 1.0, False)
    assert np.all(np.isfinite(O)) and np.all(np.isfinite(L))
    np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Lb, rtol=1e-14, atol=1e-12)


# ----------------------------------------------------------------------------
# Softmax invariants.
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_prob_rows_sum_to_one_and_mask_is_zero(causal):
    q, k, _ = rand_case(2, 9, 13, 4, 2, 8, seed=3)
    P = oracle.probs(q, k, 0.5, causal)
    np.testing.assert_allclose(P.sum(-1), 1.0, atol=1e-12)
    assert np.all(P >= 0)
    if causal:
        Lq, Lk = 9, 13
        for i in range(Lq):
            assert np.all(P[..., i, i + (Lk - Lq) + 1:] == 0.0)
            assert np.all(P[..., i, : i + (Lk - Lq) + 1] > 0.0)


@pytest.mark.parametrize("causal", [False, True])
def test_probs_times_v_is_the_attention_output(causal):
    """P of oracle.probs, applied to V through the GQA head map, reproduces the
    (independently pinned) attention output; a wrong scale or mask in probs
    changes P and fails this."""
    B, Lq, Lk, Hq, Hkv, D = 2, 9, 13, 4, 2, 8
    q, k, v = rand_case(B, Lq, Lk, Hq, Hkv, D, seed=21)
    for scale in (0.5, 1.7):
        P = oracle.probs(q, k, scale, causal)
        O, _ = oracle.attention(q, k, v, scale, causal)
        vf = oracle.bf16_bits_to_f64(v)                               # [B, Lk, Hkv, D]
        G = Hq // Hkv
        vh = np.repeat(vf, G, axis=2)                                 # [B, Lk, Hq, D]
        O_p = np.einsum("bhij,bjhd->bihd", P, vh)
        np.testing.assert_allclose(O_p, O, rtol=0, atol=1e-12)
    P1 = oracle.probs(q, k, 0.5, causal)
    P2 = oracle.probs(q, k, 1.7, causal)
    assert np.max(np.abs(P1 - P2)) > 1e-3


@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_gives_constant_o(causal):
    q, k, _ = rand_case(1, 8, 11, 2, 2, 16, seed=4)
    v = np.full((1, 11, 2, 16), bf16_bits(np.float32(1.75)), dtype=np.uint16)
    O, _ = oracle.attention(q, k, v, 0.25, causal)
    np.testing.assert_allclose(O, 1.75, rtol=1e-15, atol=0)


def test_causal_first_row_is_v0():
    q, k, v = rand_case(2, 16, 16, 4, 4, 8, seed=5)
    scale = 0.35
    O, L = oracle.attention(q, k, v, scale, True)
    np.testing.assert_array_equal(O[:, 0], f64(v)[:, 0])
    s00 = scale * np.einsum("bhd,bhd->bh", f64(q)[:, 0], f64(k)[:, 0])
    np.testing.assert_allclose(L[:, :, 0], s00, rtol=0, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_q_closed_form(causal):
    """Q = 0: all allowed scores are 0, so O_i = mean of allowed V rows, L_i = ln(#allowed)."""
    B, Lq, Lk, H, D = 1, 5, 9, 2, 4
    q = np.zeros((B, Lq, H, D), np.uint16)
    _, k, v = rand_case(B, Lq, Lk, H, H, D, seed=6)
    O, L = oracle.attention(q, k, v, 1.0, causal)
    vd = f64(v)
    for i in range(Lq):
        n = (i + (Lk - Lq) + 1) if causal else Lk
        np.testing.assert_allclose(O[:, i], vd[:, :n].mean(axis=1), rtol=0, atol=1e-15)
        np.testing.assert_allclose(L[:, :, i], math.log(n), rtol=0, atol=1e-15)


def test_single_key_returns_v0():
    q, k, v = rand_case(1, 3, 1, 2, 2, 8, seed=8)
    O, L = oracle.attention(q, k, v, 0.9, False)
    np.testing.assert_array_equal(O, np.broadcast_to(f64(v)[:, :1], O.shape))
    s = 0.9 * np.einsum("bihd,bhd->bhi", f64(q), f64(k)[:, 0])
    np.testing.assert_allclose(L, s, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_lse_equals_library_logsumexp(causal):
    q, k, v = rand_case(2, 12, 17, 4, 2, 8, seed=9)
    scale = 0.3
    _, L = oracle.attention(q, k, v, scale, causal)
    kd = np.repeat(f64(k), 2, axis=2)
    S = scale * np.einsum("bihd,bjhd->bhij", f64(q), kd)
    if causal:
        i = np.arange(12)[:, None]
        j = np.arange(17)[None, :]
        S = np.where(j <= i + 5, S, -np.inf)
    np.testing.assert_allclose(L, logsumexp(S, axis=-1), rtol=0, atol=1e-13)


def test_golden_closed_forms():
    """Two-key and three-key cases whose softmax is a sigmoid / closed form."""
    with open(os.path.join(GOLDEN, "closed_forms.json")) as f:
        cases = json.load(f)["cases"]
    assert len(cases) >= 3
    for c in cases:
        q = bf16_bits(np.array(c["q"], np.float32))
        k = bf16_bits(np.array(c["k"], np.float32))
        v = bf16_bits(np.array(c["v"], np.float32))
        O, L = oracle.attention(q, k, v, c["scale"], c["causal"])
        np.testing.assert_allclose(O, np.array(c["o"]), rtol=0, atol=1e-14, err_msg=c["name"])
        np.testing.assert_allclose(L, np.array(c["lse"]), rtol=0, atol=1e-14, err_msg=c["name"])


# ----------------------------------------------------------------------------
# Structure: scale placement, causal alignment, GQA, permutations.
# ----------------------------------------------------------------------------
def test_scale_multiplies_scores():
    """softmax(scale * q k^T): doubling q (exact in bf16) equals doubling scale."""
    q, k, v = rand_case(1, 6, 10, 2, 2, 8, seed=10)
    q2 = bf16_bits(2.0 * f64(q).astype(np.float32))
    O1, L1 = oracle.attention(q, k, v, 0.8, True)
    O2, L2 = oracle.attention(q2, k, v, 0.4, True)
    np.testing.assert_allclose(O1, O2, atol=1e-15)
    np.testing.assert_allclose(L1, L2, atol=1e-14)


def test_causal_is_bottom_right_aligned():
    """Causal row i with Lq < Lk sees exactly keys 0 .. i + (Lk - Lq)."""
    B, Lq, Lk, H, D = 1, 4, 9, 2, 8
    q, k, v = rand_case(B, Lq, Lk, H, H, D, seed=11)
    O, L = oracle.attention(q, k, v, 0.5, True)
    for i in range(Lq):
        n = i + (Lk - Lq) + 1
        Oi, Li = oracle.attention(q[:, i:i + 1].copy(), k[:, :n].copy(), v[:, :n].copy(), 0.5, False)
        np.testing.assert_allclose(O[:, i], Oi[:, 0], atol=1e-15)
        np.testing.assert_allclose(L[:, :, i], Li[:, :, 0], atol=1e-15)


def test_causal_rejects_more_queries_than_keys():
    q, k, v = rand_case(1, 5, 4, 1, 1, 4, seed=12)
    with pytest.raises(ValueError):
        oracle.attention(q, k, v, 1.0, True)


@pytest.mark.parametrize("G", [2, 4, 8])
def test_gqa_equals_mha_with_repeated_kv(G):
    Hkv = 2
    q, k, v = rand_case(2, 6, 9, Hkv * G, Hkv, 8, seed=13 + G)
    O, L = oracle.attention(q, k, v, 0.4, True)
    kr = np.repeat(k, G, axis=2)
    vr = np.repeat(v, G, axis=2)
    Om, Lm = oracle.attention(q, kr, vr, 0.4, True)
    np.testing.assert_array_equal(O, Om)
    np.testing.assert_array_equal(L, Lm)
    # and not the other plausible map (h % Hkv)
    kt = np.tile(k, (1, 1, G, 1))
    vt = np.tile(v, (1, 1, G, 1))
    Ot, _ = oracle.attention(q, kt, vt, 0.4, True)
    assert np.max(np.abs(Ot - O)) > 1e-3


def test_bidirectional_is_key_permutation_invariant():
    q, k, v = rand_case(1, 7, 12, 2, 2, 8, seed=14)
    perm = np.random.default_rng(0).permutation(12)
    O1, L1 = oracle.attention(q, k, v, 0.6, False)
    O2, L2 = oracle.attention(q, k[:, perm].copy(), v[:, perm].copy(), 0.6, False)
    np.testing.assert_allclose(O1, O2, atol=1e-14)
    np.testing.assert_allclose(L1, L2, atol=1e-14)


def test_rows_subset_matches_full():
    q, k, v = rand_case(2, 8, 8, 4, 2, 8, seed=15)
    O, L = oracle.attention(q, k, v, 0.5, True)
    rows = np.array([0, 5, 17, 33, 63], np.int64)
    Or, Lr = oracle.attention(q, k, v, 0.5, True, rows=rows)
    B, Lq, Hq = 2, 8, 4
    for n, r in enumerate(rows):
        i, bh = r % Lq, r // Lq
        h, b = bh % Hq, bh // Hq
        np.testing.assert_array_equal(Or[n], O[b, i, h])
        assert Lr[n] == L[b, h, i]


# ----------------------------------------------------------------------------
# The tiled online softmax (the pages' algorithm) equals the definition.
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("block", [1, 7, 64, 200])
def test_online_softmax_equals_definition(block, causal):
    q, k, v = rand_case(1, 150, 200, 2, 1, 16, seed=16, pow2=1)
    O, L = oracle.attention(q, k, v, 0.25, causal)
    Ob, Lb = oracle.online_attention(q, k, v, 0.25, causal, block)
    np.testing.assert_allclose(Ob, O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Lb, L, rtol=0, atol=1e-12)


def test_lse_merge_of_two_halves_equals_full():
    """Attention over keys [0,a) and [a,n) separately, merged by LSE, equals attention over all n."""
    q, k, v = rand_case(1, 3, 20, 1, 1, 8, seed=17)
    O, L = oracle.attention(q, k, v, 0.5, False)
    for a in (1, 7, 19):
        Oa, La = oracle.attention(q, k[:, :a].copy(), v[:, :a].copy(), 0.5, False)
        Ob, Lb = oracle.attention(q, k[:, a:].copy(), v[:, a:].copy(), 0.5, False)
        for i in range(3):
            om, lm = oracle.lse_merge(np.stack([Oa[0, i, 0], Ob[0, i, 0]]), np.array([La[0, 0, i], Lb[0, 0, i]]))
            np.testing.assert_allclose(om, O[0, i, 0], atol=1e-14)
            assert abs(lm - L[0, 0, i]) < 1e-14


def test_lse_merge_ignores_empty_chunks():
    o_parts = np.array([[1.0, 2.0], [0.0, 0.0], [3.0, -1.0]])
    l_parts = np.array([0.0, -np.inf, 0.0])
    o, lse = oracle.lse_merge(o_parts, l_parts)
    np.testing.assert_allclose(o, [2.0, 0.5], atol=1e-15)
    assert abs(lse - math.log(2.0)) < 1e-15


# ----------------------------------------------------------------------------
# Decode.
# ----------------------------------------------------------------------------
def _decode_case(B=3, Hq=8, Hkv=2, D=16, Lmax=300, seed=20):
    q = syn.normal_bf16((B, 1, Hq, D), seed, 21)
    kc = syn.normal_bf16((B, Lmax, Hkv, D), seed, 22)
    vc = syn.normal_bf16((B, Lmax, Hkv, D), seed, 23)
    lens = np.array([1, 77, 300][:B], np.int32)
    return q, kc, vc, lens


def test_decode_equals_last_row_of_causal_prefill():
    q, kc, vc, lens = _decode_case()
    O, L = oracle.decode(q, kc, vc, lens, 0.25)
    for b, n in enumerate(lens):
        Op, Lp = oracle.attention(q[b:b + 1].copy(), kc[b:b + 1, :n].copy(), vc[b:b + 1, :n].copy(), 0.25, True)
        np.testing.assert_array_equal(O[b], Op[0, 0])
        np.testing.assert_array_equal(L[b], Lp[0, :, 0])


@pytest.mark.parametrize("splits", [1, 2, 3, 8, 64])
def test_decode_split_merge_equals_unsplit(splits):
    q, kc, vc, lens = _decode_case()
    O, L = oracle.decode(q, kc, vc, lens, 0.25)
    Os, Ls = oracle.decode(q, kc, vc, lens, 0.25, num_splits=splits)
    np.testing.assert_allclose(Os, O, atol=1e-14)
    np.testing.assert_allclose(Ls, L, atol=1e-13)


def test_decode_ignores_keys_past_length():
    q, kc, vc, lens = _decode_case()
    O, L = oracle.decode(q, kc, vc, lens, 0.25)
    kc2, vc2 = kc.copy(), vc.copy()
    for b, n in enumerate(lens):
        kc2[b, n:] = 0x7F80  # +inf in bf16: must never be read
        vc2[b, n:] = 0x7F80
    O2, L2 = oracle.decode(q, kc2, vc2, lens, 0.25)
    np.testing.assert_array_equal(O, O2)
    np.testing.assert_array_equal(L, L2)
