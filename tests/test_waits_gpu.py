"""The bounded device-side waits give up, report and leave the device usable.

Every mbarrier wait in the kernels is bounded; a wait that gives up records a
status that fa_device_status() returns as FA_ERR_TIMEOUT (and clears), and sets
its block's abort flag so the block's other waits return at once.  The
self-test entry point runs that code path on purpose with a 1 ms limit: one
warp waits on a barrier that nothing completes.  Nothing faults or hangs; the
next forward on the same device still matches the fp64 oracle.
"""
import numpy as np
import pytest

import oracle
from tiled_attention_23_b200 import attention as A
from tiled_attention_23_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


def test_wait_gives_up_reports_timeout_and_clears():
    import torch
    assert A.device_status() == A.FA_OK          # nothing pending from earlier tests
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    A.selftest_wait_timeout(1000)                # 1 ms limit
    end.record()
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    # the first wait gives up after ~1 ms; the second returns at once (abort flag)
    assert 0.9 <= ms < 50.0, ms
    assert A.device_status() == A.FA_ERR_TIMEOUT
    assert A.device_status() == A.FA_OK          # the record was cleared


def test_forward_after_a_timeout_matches_the_oracle():
    A.selftest_wait_timeout(200)
    assert A.device_status() == A.FA_ERR_TIMEOUT
    w = syn.PrefillWorkload("after_timeout", 1, 300, 300, 4, 2, 128, True, seed=17)
    q, k, v = w.inputs()
    o, lse = A.fwd(A.to_device_bf16(q), A.to_device_bf16(k), A.to_device_bf16(v), causal=True, scale=w.scale)
    assert A.device_status() == A.FA_OK
    Or, Lr = oracle.attention(q, k, v, w.scale, True)
    assert np.max(np.abs(A.to_f64(o) - Or)) <= 2e-2
    assert np.max(np.abs(lse.cpu().double().numpy() - Lr)) <= 5e-3
