"""Parity of fa_fwd_varlen (CUDA, sm_100a) with the fp64 variable-length oracle.

Packed batches mix sequence lengths that are not multiples of the tiles,
empty sequences, a sequence with no keys, fewer queries than keys (bottom-right
causal alignment per sequence) and more queries than keys (rows with no key).
Each sequence must also match the fixed-shape kernel run on that sequence
alone, bit for bit (same tiles, same arithmetic; keys of the next sequence are
masked out with probability exactly 0).  The benchmark's packed workload (32
sequences, lengths in [256, 8192]) is compared on sampled rows.
"""
import numpy as np
import pytest

import oracle
from tiled_attention_23_b200 import synthetic as syn
from tiled_attention_23_b200 import attention as A
from _helpers import assert_close, run_fwd

pytestmark = pytest.mark.gpu


def run_varlen(q, k, v, cu_q, cu_k, scale, causal, max_q=None):
    import torch
    dq, dk, dv = (A.to_device_bf16(x) for x in (q, k, v))
    dcq = torch.from_numpy(np.ascontiguousarray(cu_q, dtype=np.int32)).cuda()
    dck = torch.from_numpy(np.ascontiguousarray(cu_k, dtype=np.int32)).cuda()
    if max_q is None:
        max_q = max(1, int(np.max(np.diff(cu_q))))
    o, lse = A.fwd_varlen(dq, dk, dv, dcq, dck, max_q, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert A.device_status() == A.FA_OK
    return A.to_f64(o), lse.cpu().double().numpy()


def packed(lens_q, lens_k, Hq, Hkv, D, seed):
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    q = syn.normal_bf16((int(cu_q[-1]), Hq, D), seed, 11)
    k = syn.normal_bf16((int(cu_k[-1]), Hkv, D), seed, 12)
    v = syn.normal_bf16((int(cu_k[-1]), Hkv, D), seed, 13)
    return q, k, v, cu_q, cu_k


def check(q, k, v, cu_q, cu_k, scale, causal, what):
    O, L = run_varlen(q, k, v, cu_q, cu_k, scale, causal)
    Or, Lr = oracle.attention_varlen(q, k, v, cu_q, cu_k, scale, causal)
    empty = ~np.isfinite(Lr)
    assert np.all(L[empty] == -np.inf) and np.all(O.transpose(1, 0, 2)[empty] == 0), what
    assert_close(O.transpose(1, 0, 2)[~empty], L[~empty], Or.transpose(1, 0, 2)[~empty], Lr[~empty], what)
    return O, L


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("G", [1, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_small_varlen_parity(D, G, causal):
    Hkv = 2
    lens_q = [1, 300, 0, 129, 256, 77]
    lens_k = [1, 300, 5, 129, 256, 77]
    q, k, v, cu_q, cu_k = packed(lens_q, lens_k, Hkv * G, Hkv, D, seed=D + G + causal)
    O, L = check(q, k, v, cu_q, cu_k, 1.0 / np.sqrt(D), causal, f"D={D} G={G} causal={causal}")
    # each sequence equals the fixed-shape kernel on that sequence alone, bit for bit
    for b, n in enumerate(lens_q):
        if n == 0:
            continue
        sl_q, sl_k = slice(cu_q[b], cu_q[b + 1]), slice(cu_k[b], cu_k[b + 1])
        Od, Ld = run_fwd(q[sl_q][None], k[sl_k][None], v[sl_k][None], 1.0 / np.sqrt(D), causal)
        np.testing.assert_array_equal(O[sl_q], Od[0])
        np.testing.assert_array_equal(L[:, sl_q], Ld[0])


@pytest.mark.parametrize("causal", [False, True])
def test_fewer_and_more_queries_than_keys(causal):
    # chunked-prefill shape (queries are the last part of the keys), a sequence
    # without keys, and (causal) more queries than keys: rows with no key
    lens_q = [100, 7, 300, 20]
    lens_k = [1000, 0, 333, 3]
    q, k, v, cu_q, cu_k = packed(lens_q, lens_k, 8, 2, 128, seed=50 + causal)
    check(q, k, v, cu_q, cu_k, 0.09, causal, f"causal={causal}")


def test_full_varlen_workload_sampled_rows():
    w = syn.VARLEN_PREFILL
    q, k, v, cu = w.inputs()
    O, L = run_varlen(q, k, v, cu, cu, w.scale, w.causal)
    total = int(cu[-1])
    rng = np.random.default_rng(3)
    ends = np.concatenate([cu[1:] - 1, cu[:-1], cu[:-1] + 127, cu[:-1] + 128])
    toks = np.unique(np.concatenate([ends[ends < total], rng.integers(0, total, 400)]))
    heads = rng.integers(0, w.Hq, toks.shape[0])
    rows = toks.astype(np.int64) * w.Hq + heads
    Or, Lr = oracle.attention_varlen(q, k, v, cu, cu, w.scale, w.causal, rows=rows)
    assert_close(O[toks, heads], L[heads, toks], Or, Lr, w.name)
