"""fa_decode_splitkv_noalloc: split-KV decode for callers that cannot allocate.

Some callers cannot call cudaMalloc: a plug-in inside a host process whose own
allocator has reserved the GPU's memory up front, or a latency-critical decode
loop where an allocation could synchronise the device.  This entry point takes
no workspace and keeps its split partials in a fixed scratch buffer the library
holds on each GPU.  The test calls it through the C ABI twice in a row, on two
different problems, and compares each result with the fp64 oracle and with the
ordinary fa_decode_splitkv (caller-provided workspace) within the decode parity
tolerances; it also checks the size limit.  This file is collected last.
"""
import numpy as np
import pytest

import oracle
from tiled_attention_23_b200 import attention as A
from tiled_attention_23_b200 import synthetic as syn
from _helpers import L_TOL, O_TOL

pytestmark = pytest.mark.gpu


def _host_inputs(B, Hq, Hkv, D, Lmax, lens, seed):
    w = syn.DecodeWorkload("noalloc", B, Hq, Hkv, D, 1, Lmax, 1, seed=seed)
    q, kc, vc, _ = w.inputs()
    return q, kc, vc, np.asarray(lens, dtype=np.int32)


def _device(q, kc, vc, lens):
    import torch
    return A.to_device_bf16(q), A.to_device_bf16(kc), A.to_device_bf16(vc), torch.from_numpy(lens).cuda()


def _noalloc_raw(q, kc, vc, lens, splits, scale):
    """Direct C-ABI call of fa_decode_splitkv_noalloc (no workspace argument)."""
    import torch
    B, _, Hq, D = q.shape
    _, Lmax, Hkv, _ = kc.shape
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=q.device)
    rc = A.lib().fa_decode_splitkv_noalloc(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), lens.data_ptr(),
                                           o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, D, Lmax, splits,
                                           float(scale), int(torch.cuda.current_stream().cuda_stream))
    return rc, o, lse


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    import torch
    problems = [
        dict(B=64, Hq=32, Hkv=8, D=128, Lmax=4096, lens=syn.uniform_int(64, 3, 4, 1, 4096), seed=21, splits=8),
        dict(B=5, Hq=16, Hkv=2, D=64, Lmax=1000, lens=[1, 999, 64, 500, 1000], seed=22, splits=3),
    ]
    for pb in problems:
        hq, hk, hv, hl = _host_inputs(pb["B"], pb["Hq"], pb["Hkv"], pb["D"], pb["Lmax"], pb["lens"], pb["seed"])
        q, kc, vc, lens = _device(hq, hk, hv, hl)
        scale = 1.0 / np.sqrt(pb["D"])
        rc, o1, l1 = _noalloc_raw(q, kc, vc, lens, pb["splits"], scale)
        assert rc == A.FA_OK, A.status_string(rc)
        o2, l2 = A.decode_splitkv(q, kc, vc, lens, pb["splits"], scale=scale)
        torch.cuda.synchronize()
        assert A.device_status() == A.FA_OK
        assert bool(torch.isfinite(o1.float()).all()) and bool(torch.isfinite(l1).all())
        Or, Lr = oracle.decode(hq, hk, hv, hl, scale)
        assert float(np.abs(A.to_f64(o1).reshape(Or.shape) - Or).max()) <= O_TOL
        assert float(np.abs(l1.cpu().double().numpy().reshape(Lr.shape) - Lr).max()) <= L_TOL
        assert float((o1.float() - o2.float()).abs().max()) <= O_TOL
        assert float((l1 - l2).abs().max()) <= L_TOL


def test_noalloc_rejects_requests_beyond_its_scratch():
    import torch
    # Small tensors whose shapes match the dimensions passed, but 64 splits of
    # 64 query heads x 64 sequences need 64*64*64*(64+1)*4 bytes (68 MB) of
    # scratch, more than the fixed buffer: refused before anything is enqueued.
    B, Hq, Hkv, D, Lmax, splits = 64, 64, 16, 64, 64, 64
    q, kc, vc, lens = _device(*_host_inputs(B, Hq, Hkv, D, Lmax, [Lmax] * B, seed=23))
    need = A.decode_workspace_bytes(B, Hq, D, splits)
    assert need > A.NOALLOC_SCRATCH_BYTES
    o = torch.zeros_like(q)
    lse = torch.zeros((B, Hq), dtype=torch.float32, device=q.device)
    rc = A.lib().fa_decode_splitkv_noalloc(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), lens.data_ptr(),
                                           o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, D, Lmax, splits, 0.125,
                                           int(torch.cuda.current_stream().cuda_stream))
    assert rc == A.FA_ERR_NO_SPACE
    assert A.status_string(rc) == "FA_ERR_NO_SPACE"
    torch.cuda.synchronize()
    assert int(torch.count_nonzero(o)) == 0 and int(torch.count_nonzero(lse)) == 0   # nothing was written
