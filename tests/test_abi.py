"""The C-ABI boundary on the host (no GPU needed).

The library must build for sm_100a, load, export every entry point that
``include/ta23.h`` declares, and reject invalid arguments synchronously without
touching the device.
"""
import ctypes
import os
import re
import subprocess

import pytest

from tiled_attention_23_b200 import attention as A
from tiled_attention_23_b200 import _build

HEADER = os.path.join(_build.INCLUDE, "ta23.h")

# Well-aligned fake device addresses: validation rejects the call before any
# of them is dereferenced.
P = 1 << 20


def declared_entry_points():
    txt = open(HEADER).read()
    return re.findall(r"TA23_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", txt)


def test_header_declares_the_boundary():
    names = declared_entry_points()
    for n in ("fa_fwd", "fa_decode_splitkv", "fa_decode_workspace_bytes", "fa_device_status",
              "fa_status_string", "fa_build_info"):
        assert n in names
    assert set(names) <= set(A.SIGNATURES)


def test_library_exports_every_declared_symbol():
    lib = A.lib()
    for n in declared_entry_points():
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", _build.LIB_CUDA], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert set(declared_entry_points()) <= exported
    # nothing else with the fa_ prefix leaks out
    assert {s for s in exported if s.startswith("fa_")} == set(declared_entry_points())


def test_library_is_built_for_sm100a_only():
    out = subprocess.run(["cuobjdump", "--list-elf", _build.LIB_CUDA], capture_output=True, text=True)
    if out.returncode != 0:
        pytest.skip("cuobjdump not available")
    assert "sm_100a" in out.stdout
    assert all("sm_100a" in l for l in out.stdout.splitlines() if "sm_" in l)


def test_status_strings_and_build_info():
    assert A.status_string(0) == "FA_OK"
    assert A.status_string(4) == "FA_ERR_TIMEOUT"
    info = A.build_info()
    assert "sm_100a" in info and "256" in info


def fwd(**kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, B=1, Lq=128, Lk=128, Hq=4, Hkv=4, D=128, scale=0.1, causal=1, stream=None)
    a.update(kw)
    return A.lib().fa_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Lq"], a["Lk"], a["Hq"], a["Hkv"],
                          a["D"], a["scale"], a["causal"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), A.FA_ERR_INVALID_ARG),
    (dict(o=None), A.FA_ERR_INVALID_ARG),
    (dict(k=P + 8), A.FA_ERR_INVALID_ARG),          # misaligned
    (dict(lse=P + 2), A.FA_ERR_INVALID_ARG),
    (dict(B=0), A.FA_ERR_INVALID_ARG),
    (dict(Lq=0), A.FA_ERR_INVALID_ARG),
    (dict(Lk=-3), A.FA_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), A.FA_ERR_INVALID_ARG),      # Hq % Hkv != 0
    (dict(scale=float("nan")), A.FA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), A.FA_ERR_INVALID_ARG),
    (dict(scale=-1.0), A.FA_ERR_INVALID_ARG),
    (dict(Lq=200, Lk=100), A.FA_ERR_INVALID_ARG),   # causal row with no key
    (dict(D=96), A.FA_ERR_UNSUPPORTED),
    (dict(D=32), A.FA_ERR_UNSUPPORTED),
    (dict(Hq=48, Hkv=4), A.FA_ERR_UNSUPPORTED),     # group 12
    (dict(Hq=16, Hkv=1), A.FA_ERR_UNSUPPORTED),     # group 16
])
def test_fwd_rejects_invalid_arguments(kw, code):
    assert fwd(**kw) == code


def decode(**kw):
    a = dict(q=P, kc=P, vc=P, lens=P, o=P, lse=P, B=2, Hq=8, Hkv=2, D=128, Lmax=1024, S=8, scale=0.1,
             ws=P, wsb=1 << 30, stream=None)
    a.update(kw)
    return A.lib().fa_decode_splitkv(a["q"], a["kc"], a["vc"], a["lens"], a["o"], a["lse"], a["B"], a["Hq"],
                                     a["Hkv"], a["D"], a["Lmax"], a["S"], a["scale"], a["ws"], a["wsb"],
                                     a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), A.FA_ERR_INVALID_ARG),
    (dict(lens=None), A.FA_ERR_INVALID_ARG),
    (dict(ws=None), A.FA_ERR_INVALID_ARG),
    (dict(lens=P + 2), A.FA_ERR_INVALID_ARG),
    (dict(kc=P + 4), A.FA_ERR_INVALID_ARG),
    (dict(S=0), A.FA_ERR_INVALID_ARG),
    (dict(S=65), A.FA_ERR_INVALID_ARG),
    (dict(wsb=100), A.FA_ERR_INVALID_ARG),
    (dict(Hq=8, Hkv=3), A.FA_ERR_INVALID_ARG),
    (dict(Lmax=0), A.FA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), A.FA_ERR_INVALID_ARG),
    (dict(D=80), A.FA_ERR_UNSUPPORTED),
    (dict(Hq=32, Hkv=2), A.FA_ERR_UNSUPPORTED),
])
def test_decode_rejects_invalid_arguments(kw, code):
    assert decode(**kw) == code


def test_selftest_rejects_out_of_range_limits():
    L = A.lib()
    assert L.fa_selftest_wait_timeout(0, None) == A.FA_ERR_INVALID_ARG
    assert L.fa_selftest_wait_timeout(1000001, None) == A.FA_ERR_INVALID_ARG


def test_workspace_size():
    lib = A.lib()
    n = lib.fa_decode_workspace_bytes(64, 32, 128, 8)
    assert n >= 64 * 32 * 8 * (128 + 1) * 4
    assert n % 256 == 0
    assert lib.fa_decode_workspace_bytes(0, 32, 128, 8) == 0


def test_binding_refuses_cpu_tensors():
    torch = pytest.importorskip("torch")
    q = torch.zeros((1, 8, 2, 64), dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        A.fwd(q, q, q, causal=False)
    # every entry point marshals device pointers only: host tensors never reach the library
    q8 = torch.zeros((1, 8, 2, 128), dtype=torch.uint8)
    d = torch.ones((1, 2), dtype=torch.float32)
    with pytest.raises(TypeError):
        A.fwd_fp8(q8, q8, q8, d, d, d, causal=True)
    with pytest.raises(TypeError):
        A.quantize_fp8(torch.zeros((1, 8, 2, 128), dtype=torch.bfloat16))
    lse = torch.zeros((1, 2, 8), dtype=torch.float32)
    with pytest.raises(TypeError):
        A.bwd(q, q, q, q, lse, q, causal=True)


def paged(**kw):
    a = dict(q=P, kp=P, vp=P, table=P, lens=P, o=P, lse=P, B=2, Hq=8, Hkv=2, D=128, pages=64, ps=64, maxp=16,
             S=8, scale=0.1, ws=P, wsb=1 << 30, stream=None)
    a.update(kw)
    return A.lib().fa_decode_paged(a["q"], a["kp"], a["vp"], a["table"], a["lens"], a["o"], a["lse"], a["B"],
                                   a["Hq"], a["Hkv"], a["D"], a["pages"], a["ps"], a["maxp"], a["S"], a["scale"],
                                   a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(table=None), A.FA_ERR_INVALID_ARG),
    (dict(table=P + 2), A.FA_ERR_INVALID_ARG),
    (dict(kp=P + 8), A.FA_ERR_INVALID_ARG),
    (dict(pages=0), A.FA_ERR_INVALID_ARG),
    (dict(maxp=0), A.FA_ERR_INVALID_ARG),
    (dict(ps=8), A.FA_ERR_INVALID_ARG),        # not a multiple of 16
    (dict(ps=40), A.FA_ERR_INVALID_ARG),
    (dict(ps=1 << 17), A.FA_ERR_INVALID_ARG),
    (dict(S=0), A.FA_ERR_INVALID_ARG),
    (dict(wsb=64), A.FA_ERR_INVALID_ARG),
    (dict(scale=-0.5), A.FA_ERR_INVALID_ARG),
    (dict(D=96), A.FA_ERR_UNSUPPORTED),
    (dict(Hq=6, Hkv=2), A.FA_ERR_UNSUPPORTED),   # group 3
])
def test_paged_decode_rejects_invalid_arguments(kw, code):
    assert paged(**kw) == code


def varlen(**kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, cuq=P, cuk=P, B=4, maxq=512, tq=1024, tk=1024, Hq=8, Hkv=2, D=128,
             scale=0.1, causal=1, stream=None)
    a.update(kw)
    return A.lib().fa_fwd_varlen(a["q"], a["k"], a["v"], a["o"], a["lse"], a["cuq"], a["cuk"], a["B"], a["maxq"],
                                 a["tq"], a["tk"], a["Hq"], a["Hkv"], a["D"], a["scale"], a["causal"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(cuq=None), A.FA_ERR_INVALID_ARG),
    (dict(cuk=P + 2), A.FA_ERR_INVALID_ARG),
    (dict(q=P + 8), A.FA_ERR_INVALID_ARG),
    (dict(B=0), A.FA_ERR_INVALID_ARG),
    (dict(maxq=0), A.FA_ERR_INVALID_ARG),
    (dict(maxq=2048), A.FA_ERR_INVALID_ARG),    # longer than the packed tensor
    (dict(tq=0), A.FA_ERR_INVALID_ARG),
    (dict(tk=0), A.FA_ERR_INVALID_ARG),
    (dict(Hq=8, Hkv=3), A.FA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), A.FA_ERR_INVALID_ARG),
    (dict(D=48), A.FA_ERR_UNSUPPORTED),
    (dict(Hq=24, Hkv=2), A.FA_ERR_UNSUPPORTED),  # group 12
])
def test_varlen_rejects_invalid_arguments(kw, code):
    assert varlen(**kw) == code


def dec_i8(**kw):
    a = dict(q=P, k=P, ks=P, v=P, vs=P, lens=P, o=P, lse=P, B=2, Hq=8, Hkv=2, D=128, Lmax=1024, S=8, scale=0.1,
             ws=P, wsb=1 << 30, stream=None)
    a.update(kw)
    return A.lib().fa_decode_int8(a["q"], a["k"], a["ks"], a["v"], a["vs"], a["lens"], a["o"], a["lse"], a["B"],
                                  a["Hq"], a["Hkv"], a["D"], a["Lmax"], a["S"], a["scale"], a["ws"], a["wsb"],
                                  a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(k=None), A.FA_ERR_INVALID_ARG),
    (dict(ks=None), A.FA_ERR_INVALID_ARG),
    (dict(ks=P + 4), A.FA_ERR_INVALID_ARG),
    (dict(vs=P + 8), A.FA_ERR_INVALID_ARG),
    (dict(Lmax=1022), A.FA_ERR_INVALID_ARG),    # scale rows must be 16-byte aligned
    (dict(S=70), A.FA_ERR_INVALID_ARG),
    (dict(wsb=16), A.FA_ERR_INVALID_ARG),
    (dict(D=32), A.FA_ERR_UNSUPPORTED),
    (dict(Hq=6, Hkv=2), A.FA_ERR_UNSUPPORTED),
])
def test_int8_decode_rejects_invalid_arguments(kw, code):
    assert dec_i8(**kw) == code


@pytest.mark.parametrize("args,code", [
    ((None, P, P, 1, 8, 2, 128), A.FA_ERR_INVALID_ARG),
    ((P, P + 4, P, 1, 8, 2, 128), A.FA_ERR_INVALID_ARG),
    ((P, P, P + 2, 1, 8, 2, 128), A.FA_ERR_INVALID_ARG),
    ((P, P, P, 0, 8, 2, 128), A.FA_ERR_INVALID_ARG),
    ((P, P, P, 1, 8, 2, 96), A.FA_ERR_UNSUPPORTED),
])
def test_quantiser_rejects_invalid_arguments(args, code):
    assert A.lib().fa_quantize_kv_int8(*args, None) == code


def bwd(**kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, do=P, dq=P, dk=P, dv=P, B=1, Lq=128, Lk=128, Hq=4, Hkv=4, D=128,
             scale=0.1, causal=1, ws=P, wsb=1 << 30, stream=None)
    a.update(kw)
    return A.lib().fa_bwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["do"], a["dq"], a["dk"], a["dv"], a["B"],
                          a["Lq"], a["Lk"], a["Hq"], a["Hkv"], a["D"], a["scale"], a["causal"], a["ws"], a["wsb"],
                          a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(lse=None), A.FA_ERR_INVALID_ARG),
    (dict(do=None), A.FA_ERR_INVALID_ARG),
    (dict(dk=P + 8), A.FA_ERR_INVALID_ARG),
    (dict(lse=P + 2), A.FA_ERR_INVALID_ARG),
    (dict(ws=None), A.FA_ERR_INVALID_ARG),
    (dict(wsb=64), A.FA_ERR_INVALID_ARG),
    (dict(Lq=256, Lk=128), A.FA_ERR_INVALID_ARG),   # causal row with no key
    (dict(scale=float("nan")), A.FA_ERR_INVALID_ARG),
    (dict(D=96), A.FA_ERR_UNSUPPORTED),
    (dict(Hq=12, Hkv=4), A.FA_ERR_UNSUPPORTED),
])
def test_bwd_rejects_invalid_arguments(kw, code):
    assert bwd(**kw) == code


def test_bwd_workspace_size():
    lib = A.lib()
    assert lib.fa_bwd_workspace_bytes(2, 4, 300) >= 2 * 4 * 300 * 4
    assert lib.fa_bwd_workspace_bytes(0, 4, 300) == 0


def fwd8(**kw):
    a = dict(q=P, k=P, v=P, qd=P, kd=P, vd=P, o=P, lse=P, B=1, Lq=128, Lk=128, Hq=4, Hkv=4, D=128, scale=0.1,
             causal=1, stream=None)
    a.update(kw)
    return A.lib().fa_fwd_fp8(a["q"], a["k"], a["v"], a["qd"], a["kd"], a["vd"], a["o"], a["lse"], a["B"],
                              a["Lq"], a["Lk"], a["Hq"], a["Hkv"], a["D"], a["scale"], a["causal"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), A.FA_ERR_INVALID_ARG),
    (dict(kd=None), A.FA_ERR_INVALID_ARG),
    (dict(vd=P + 2), A.FA_ERR_INVALID_ARG),
    (dict(v=P + 8), A.FA_ERR_INVALID_ARG),
    (dict(lse=P + 1), A.FA_ERR_INVALID_ARG),
    (dict(Lq=0), A.FA_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), A.FA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), A.FA_ERR_INVALID_ARG),
    (dict(Lq=256, Lk=128), A.FA_ERR_INVALID_ARG),   # causal row with no key
    (dict(D=32), A.FA_ERR_UNSUPPORTED),
    (dict(D=96), A.FA_ERR_UNSUPPORTED),
    (dict(Hq=48, Hkv=4), A.FA_ERR_UNSUPPORTED),
])
def test_fp8_fwd_rejects_invalid_arguments(kw, code):
    assert fwd8(**kw) == code


@pytest.mark.parametrize("args,code", [
    ((None, P, P, 1, 8, 2, 128), A.FA_ERR_INVALID_ARG),
    ((P, P + 4, P, 1, 8, 2, 128), A.FA_ERR_INVALID_ARG),
    ((P, P, P + 2, 1, 8, 2, 128), A.FA_ERR_INVALID_ARG),
    ((P, P, P, 1, 0, 2, 128), A.FA_ERR_INVALID_ARG),
    ((P, P, P, 1, 8, 2, 80), A.FA_ERR_UNSUPPORTED),
])
def test_fp8_quantiser_rejects_invalid_arguments(args, code):
    assert A.lib().fa_quantize_fp8(*args, None) == code
