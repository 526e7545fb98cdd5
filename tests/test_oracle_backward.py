"""Pins of the fp64 backward oracle (CPU only).

``oracle.attention_backward`` (C) is checked against what fixes the gradient
independently: PyTorch autograd in float64 on the same values (a library
routine for the special case of dense attention), central finite differences
of a numpy float64 forward, and invariants of the softmax Jacobian (the rows
of dS sum to zero, so dK summed over keys vanishes; P rows sum to one, so dV
summed over keys equals dO summed over queries).
"""
import numpy as np
import pytest

import oracle
from tiled_attention_23_b200 import synthetic as syn

torch = pytest.importorskip("torch")


def case(B, Lq, Lk, Hq, Hkv, D, seed):
    q = syn.normal_bf16((B, Lq, Hq, D), seed, 11)
    k = syn.normal_bf16((B, Lk, Hkv, D), seed, 12)
    v = syn.normal_bf16((B, Lk, Hkv, D), seed, 13)
    do = syn.normal_bf16((B, Lq, Hq, D), seed, 14)
    return q, k, v, do


def torch_grads(q, k, v, do, scale, causal):
    f = lambda a: torch.from_numpy(oracle.bf16_bits_to_f64(a))
    tq, tk, tv, tdo = f(q).requires_grad_(), f(k).requires_grad_(), f(v).requires_grad_(), f(do)
    B, Lq, Hq, D = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    kk = tk.repeat_interleave(G, dim=2)
    vv = tv.repeat_interleave(G, dim=2)
    s = torch.einsum("bihd,bjhd->bhij", tq, kk) * scale
    if causal:
        i = torch.arange(Lq)[:, None]
        j = torch.arange(Lk)[None, :]
        s = s.masked_fill(j > i + (Lk - Lq), float("-inf"))
    o = torch.einsum("bhij,bjhd->bihd", torch.softmax(s, dim=-1), vv)
    (o * tdo).sum().backward()
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


@pytest.mark.parametrize("shape,causal", [((2, 5, 7, 4, 2, 8), False), ((1, 6, 6, 2, 2, 4), True),
                                          ((1, 3, 9, 8, 1, 4), True), ((2, 9, 9, 4, 4, 16), True)])
def test_matches_torch_autograd(shape, causal):
    B, Lq, Lk, Hq, Hkv, D = shape
    q, k, v, do = case(B, Lq, Lk, Hq, Hkv, D, sum(shape))
    dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.4, causal)
    tq, tk, tv = torch_grads(q, k, v, do, 0.4, causal)
    for a, b in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12)


def test_matches_finite_differences():
    B, Lq, Lk, Hq, Hkv, D = 1, 4, 5, 2, 1, 3
    q, k, v, do = case(B, Lq, Lk, Hq, Hkv, D, 7)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.7, True)
    Q, K, V, DO = (oracle.bf16_bits_to_f64(a) for a in (q, k, v, do))

    def loss(Q, K, V):   # numpy float64 forward of the definition, summed against dO
        out = 0.0
        for h in range(Hq):
            g = h // (Hq // Hkv)
            for i in range(Lq):
                s = np.array([0.7 * Q[0, i, h] @ K[0, j, g] if j <= i + (Lk - Lq) else -np.inf for j in range(Lk)])
                p = np.exp(s - s.max())
                p /= p.sum()
                out += float((p @ V[0, :, g]) @ DO[0, i, h])
        return out

    eps = 1e-6
    for (arr, grad, idx) in ((Q, dq, (0, 2, 1, 1)), (K, dk, (0, 3, 0, 2)), (V, dv, (0, 1, 0, 0)),
                             (K, dk, (0, 0, 0, 0)), (Q, dq, (0, 3, 0, 2))):
        a0 = arr[idx]
        arr[idx] = a0 + eps
        up = loss(Q, K, V)
        arr[idx] = a0 - eps
        dn = loss(Q, K, V)
        arr[idx] = a0
        assert abs((up - dn) / (2 * eps) - grad[idx]) < 1e-7


@pytest.mark.parametrize("causal", [False, True])
def test_jacobian_invariants(causal):
    q, k, v, do = case(2, 12, 12, 4, 2, 16, 9)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.25, causal)
    # rows of dS sum to zero: the gradient is blind to adding a constant to a
    # score row, so dK summed over keys is zero for every (b, kv head, d)
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)
    # rows of P sum to one: dV summed over keys = dO summed over queries of the group
    DO = oracle.bf16_bits_to_f64(do)
    G = 2
    want = DO.reshape(2, 12, 2, G, 16).sum(axis=(1, 3))
    np.testing.assert_allclose(dv.sum(axis=1), want, atol=1e-12)
