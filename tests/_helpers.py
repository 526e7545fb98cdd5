"""Shared helpers for the GPU parity tests (inputs, sampling, comparison)."""
import numpy as np

import oracle
from tiled_attention_23_b200 import attention as A

# Tolerances of the parity bar: bf16 inputs and output, fp32 accumulation.
O_TOL = 2e-2
L_TOL = 5e-3


def run_fwd(q, k, v, scale, causal):
    """Upload bf16 bit arrays, run fa_fwd, return (O, L) as float64 numpy."""
    import torch
    dq, dk, dv = A.to_device_bf16(q), A.to_device_bf16(k), A.to_device_bf16(v)
    o, lse = A.fwd(dq, dk, dv, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert A.device_status() == A.FA_OK
    return A.to_f64(o), lse.cpu().double().numpy()


def sample_rows(B, Lq, Hq, n, seed=0):
    """Flat row indices (b*Hq + h)*Lq + i: tile edges, first/last rows, and random ones."""
    rng = np.random.default_rng(seed)
    special_i = sorted({0, 1, 63, 64, 127, 128, 129, 255, 256, Lq // 2, Lq - 129, Lq - 128, Lq - 2, Lq - 1} &
                       set(range(Lq)))
    rows = set()
    for i in special_i:
        b, h = int(rng.integers(B)), int(rng.integers(Hq))
        rows.add((b * Hq + h) * Lq + i)
    while len(rows) < n:
        rows.add(int(rng.integers(B * Hq * Lq)))
    return np.array(sorted(rows), dtype=np.int64)


def gather_rows(O, L, rows, Lq, Hq):
    """Pick rows (flat (b*Hq+h)*Lq+i) out of O [B,Lq,Hq,D] and L [B,Hq,Lq]."""
    i = rows % Lq
    bh = rows // Lq
    h = bh % Hq
    b = bh // Hq
    return O[b, i, h], L[b, h, i]


def assert_close(O, L, Or, Lr, what=""):
    eo = float(np.max(np.abs(O - Or))) if O.size else 0.0
    el = float(np.max(np.abs(L - Lr))) if L.size else 0.0
    assert np.all(np.isfinite(O)) and np.all(np.isfinite(L)), f"{what}: non-finite output"
    assert eo <= O_TOL, f"{what}: max|O - O_ref| = {eo:.3e} > {O_TOL}"
    assert el <= L_TOL, f"{what}: max|L - L_ref| = {el:.3e} > {L_TOL}"
    return eo, el


def oracle_rows(q, k, v, scale, causal, rows):
    return oracle.attention(q, k, v, scale, causal, rows=rows)
