"""Python binding of the C ABI in ``include/ta23.h`` (argument marshalling only).

Every function here forwards torch tensors' device pointers, sizes and the
current CUDA stream to ``libta23.so``; all arithmetic runs in the library's
sm_100a kernels.  There is no fallback: without the library, a CUDA device or
CUDA tensors the call raises.
"""
from __future__ import annotations

import ctypes
import math
import threading

from ._build import LIB_CUDA, build_cuda

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT, FA_ERR_NO_SPACE = 0, 1, 2, 3, 4, 5
NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024   # FA_NOALLOC_SCRATCH_BYTES

_lock = threading.Lock()
_lib = None

# Entry points of include/ta23.h with their ctypes signatures.
_P, _I, _F, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "fa_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_fwd_varlen": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_fwd_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_quantize_fp8": (_I, [_P, _P, _P, _I, _I, _I, _I, _P]),
    "fa_bwd_workspace_bytes": (_Z, [_I, _I, _I]),
    "fa_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P, _Z, _P]),
    "fa_decode_workspace_bytes": (_Z, [_I, _I, _I, _I]),
    "fa_decode_splitkv": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _Z, _P]),
    "fa_decode_splitkv_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "fa_quantize_kv_int8": (_I, [_P, _P, _P, _I, _I, _I, _I, _P]),
    "fa_decode_int8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _Z, _P]),
    "fa_decode_paged": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P, _Z, _P]),
    "fa_device_status": (_I, []),
    "fa_selftest_wait_timeout": (_I, [ctypes.c_uint, _P]),
    "fa_status_string": (ctypes.c_char_p, [_I]),
    "fa_build_info": (ctypes.c_char_p, []),
}


class FAError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {status_string(code)}")


def lib(build: bool = True):
    """The loaded ``libta23.so`` (built in-tree first when missing or stale)."""
    global _lib
    with _lock:
        if _lib is None:
            path = build_cuda() if build else LIB_CUDA
            h = ctypes.CDLL(path)
            for name, (res, args) in SIGNATURES.items():
                f = getattr(h, name)
                f.restype = res
                f.argtypes = args
            _lib = h
    return _lib


def status_string(code: int) -> str:
    return lib().fa_status_string(int(code)).decode()


def build_info() -> str:
    return lib().fa_build_info().decode()


def device_status() -> int:
    """Synchronise and return FA_OK, or FA_ERR_TIMEOUT if a bounded wait gave up."""
    return int(lib().fa_device_status())


def selftest_wait_timeout(limit_us: int, stream=None) -> None:
    """Enqueue the bounded-wait self-test (a wait that gives up after limit_us);
    the next device_status() then reports FA_ERR_TIMEOUT."""
    rc = lib().fa_selftest_wait_timeout(int(limit_us), _stream_ptr(stream))
    if rc != FA_OK:
        raise FAError("fa_selftest_wait_timeout", rc)


def _stream_ptr(stream) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _check(t, name, dtype=None):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def fwd(q, k, v, causal: bool, scale: float | None = None, o=None, lse=None, want_lse: bool = True,
        stream=None):
    """Attention forward through ``fa_fwd``.

    q [B, Lq, Hq, D], k/v [B, Lk, Hkv, D] bf16 CUDA tensors.  ``scale``
    defaults to 1/sqrt(D) (the ops-transformer page's softmax_scale default).
    Returns (o [B, Lq, Hq, D] bf16, lse [B, Hq, Lq] fp32 or None).
    """
    import torch
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, torch.bfloat16)
    B, Lq, Hq, D = q.shape
    Bk, Lk, Hkv, Dk = k.shape
    if Bk != B or Dk != D or v.shape != k.shape:
        raise ValueError("q, k, v shapes do not agree")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty_like(q)
    _check(o, "o", torch.bfloat16)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _check(lse, "lse", torch.float32)
    rc = lib().fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                      lse.data_ptr() if lse is not None else None,
                      B, Lq, Lk, Hq, Hkv, D, float(scale), int(bool(causal)), _stream_ptr(stream))
    if rc != FA_OK:
        raise FAError("fa_fwd", rc)
    return o, lse


def quantize_fp8(x, out=None, descale=None, stream=None):
    """Per-(batch, head) e4m3 quantisation through ``fa_quantize_fp8``.

    x [B, L, H, D] bf16.  Returns (codes [B, L, H, D] uint8, descale [B, H] fp32).
    """
    import torch
    _check(x, "x", torch.bfloat16)
    B, L, H, D = x.shape
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if descale is None:
        descale = torch.empty((B, H), dtype=torch.float32, device=x.device)
    _check(out, "out", torch.uint8)
    _check(descale, "descale", torch.float32)
    rc = lib().fa_quantize_fp8(x.data_ptr(), out.data_ptr(), descale.data_ptr(), B, L, H, D, _stream_ptr(stream))
    if rc != FA_OK:
        raise FAError("fa_quantize_fp8", rc)
    return out, descale


def fwd_fp8(q8, k8, v8, q_descale, k_descale, v_descale, causal: bool, scale: float | None = None, o=None,
            lse=None, want_lse: bool = True, stream=None):
    """Attention forward on e4m3 inputs through ``fa_fwd_fp8``.

    q8 [B, Lq, Hq, D], k8/v8 [B, Lk, Hkv, D] uint8 e4m3 codes; q_descale
    [B, Hq], k_descale/v_descale [B, Hkv] fp32.  Returns (o bf16, lse or None).
    """
    import torch
    for t, n in ((q8, "q8"), (k8, "k8"), (v8, "v8")):
        _check(t, n, torch.uint8)
    for t, n in ((q_descale, "q_descale"), (k_descale, "k_descale"), (v_descale, "v_descale")):
        _check(t, n, torch.float32)
    B, Lq, Hq, D = q8.shape
    Bk, Lk, Hkv, Dk = k8.shape
    if Bk != B or Dk != D or v8.shape != k8.shape or tuple(q_descale.shape) != (B, Hq) \
            or tuple(k_descale.shape) != (B, Hkv) or tuple(v_descale.shape) != (B, Hkv):
        raise ValueError("fp8 shapes do not agree")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty((B, Lq, Hq, D), dtype=torch.bfloat16, device=q8.device)
    _check(o, "o", torch.bfloat16)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q8.device)
    if lse is not None:
        _check(lse, "lse", torch.float32)
    rc = lib().fa_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), q_descale.data_ptr(),
                          k_descale.data_ptr(), v_descale.data_ptr(), o.data_ptr(),
                          lse.data_ptr() if lse is not None else None,
                          B, Lq, Lk, Hq, Hkv, D, float(scale), int(bool(causal)), _stream_ptr(stream))
    if rc != FA_OK:
        raise FAError("fa_fwd_fp8", rc)
    return o, lse


def fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, causal: bool,
               scale: float | None = None, o=None, lse=None, want_lse: bool = True, stream=None):
    """Attention forward over a packed variable-length batch through ``fa_fwd_varlen``.

    q [total_q, Hq, D], k/v [total_k, Hkv, D] bf16; cu_seqlens_q/k [B+1] int32
    on the device.  Returns (o [total_q, Hq, D] bf16, lse [Hq, total_q] fp32 or None).
    """
    import torch
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, torch.bfloat16)
    _check(cu_seqlens_q, "cu_seqlens_q", torch.int32)
    _check(cu_seqlens_k, "cu_seqlens_k", torch.int32)
    total_q, Hq, D = q.shape
    total_k, Hkv, Dk = k.shape
    B = cu_seqlens_q.shape[0] - 1
    if Dk != D or v.shape != k.shape or cu_seqlens_k.shape != cu_seqlens_q.shape or B < 1:
        raise ValueError("varlen shapes do not agree")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty_like(q)
    _check(o, "o", torch.bfloat16)
    if lse is None and want_lse:
        lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device)
    rc = lib().fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                             lse.data_ptr() if lse is not None else None,
                             cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), B, int(max_seqlen_q),
                             total_q, total_k, Hq, Hkv, D, float(scale), int(bool(causal)), _stream_ptr(stream))
    if rc != FA_OK:
        raise FAError("fa_fwd_varlen", rc)
    return o, lse


def bwd(q, k, v, o, lse, dout, causal: bool, scale: float | None = None, dq=None, dk=None, dv=None,
        workspace=None, stream=None):
    """Attention backward through ``fa_bwd``: returns (dq, dk, dv) bf16.

    q [B, Lq, Hq, D], k/v [B, Lk, Hkv, D], o and dout [B, Lq, Hq, D] bf16, lse
    [B, Hq, Lq] fp32 (fa_fwd's outputs).  ``scale`` defaults to 1/sqrt(D).
    """
    import torch
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _check(t, n, torch.bfloat16)
    _check(lse, "lse", torch.float32)
    B, Lq, Hq, D = q.shape
    Bk, Lk, Hkv, Dk = k.shape
    if (Bk != B or Dk != D or v.shape != k.shape or o.shape != q.shape or dout.shape != q.shape
            or tuple(lse.shape) != (B, Hq, Lq)):
        raise ValueError("backward shapes do not agree")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _check(t, n, torch.bfloat16)
    need = int(lib().fa_bwd_workspace_bytes(B, Hq, Lq))
    if workspace is None:
        workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=q.device)
    _check(workspace, "workspace")
    rc = lib().fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), dout.data_ptr(),
                      dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Lq, Lk, Hq, Hkv, D, float(scale),
                      int(bool(causal)), workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                      _stream_ptr(stream))
    if rc != FA_OK:
        raise FAError("fa_bwd", rc)
    return dq, dk, dv


def decode_workspace_bytes(B: int, Hq: int, D: int, num_splits: int) -> int:
    return int(lib().fa_decode_workspace_bytes(B, Hq, D, num_splits))


def decode_splitkv(q, k_cache, v_cache, seqlens, num_splits: int, scale: float | None = None,
                   o=None, lse=None, workspace=None, want_lse: bool = True, stream=None):
    """Split-KV decode through ``fa_decode_splitkv``.

    q [B, 1, Hq, D]; k_cache/v_cache [B, max_seqlen, Hkv, D] bf16; seqlens [B]
    int32 on the device.  Returns (o [B, 1, Hq, D] bf16, lse [B, Hq] fp32 or None).
    """
    import torch
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _check(t, n, torch.bfloat16)
    _check(seqlens, "seqlens", torch.int32)
    B, one, Hq, D = q.shape
    Bk, Lmax, Hkv, Dk = k_cache.shape
    if one != 1 or Bk != B or Dk != D or v_cache.shape != k_cache.shape or seqlens.shape != (B,):
        raise ValueError("decode shapes do not agree")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    need = decode_workspace_bytes(B, Hq, D, num_splits)
    if workspace is None:
        workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=q.device)
    _check(workspace, "workspace")
    rc = lib().fa_decode_splitkv(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), seqlens.data_ptr(),
                                 o.data_ptr(), lse.data_ptr() if lse is not None else None,
                                 B, Hq, Hkv, D, Lmax, int(num_splits), float(scale),
                                 workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                 _stream_ptr(stream))
    if rc != FA_OK:
        raise FAError("fa_decode_splitkv", rc)
    return o, lse


def decode_paged(q, k_pages, v_pages, block_table, seqlens, num_splits: int, scale: float | None = None,
                 o=None, lse=None, workspace=None, want_lse: bool = True, stream=None):
    """Split-KV decode against a paged cache through ``fa_decode_paged``.

    q [B, 1, Hq, D]; k_pages/v_pages [num_pages, page_size, Hkv, D] bf16;
    block_table [B, max_pages_per_seq] int32 and seqlens [B] int32 on the device.
    Returns (o [B, 1, Hq, D] bf16, lse [B, Hq] fp32 or None).
    """
    import torch
    for t, n in ((q, "q"), (k_pages, "k_pages"), (v_pages, "v_pages")):
        _check(t, n, torch.bfloat16)
    _check(seqlens, "seqlens", torch.int32)
    _check(block_table, "block_table", torch.int32)
    B, one, Hq, D = q.shape
    num_pages, page_size, Hkv, Dk = k_pages.shape
    if (one != 1 or Dk != D or v_pages.shape != k_pages.shape or seqlens.shape != (B,)
            or block_table.dim() != 2 or block_table.shape[0] != B):
        raise ValueError("paged decode shapes do not agree")
    max_pages = block_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    need = decode_workspace_bytes(B, Hq, D, num_splits)
    if workspace is None:
        workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=q.device)
    _check(workspace, "workspace")
    rc = lib().fa_decode_paged(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(), block_table.data_ptr(),
                               seqlens.data_ptr(), o.data_ptr(), lse.data_ptr() if lse is not None else None,
                               B, Hq, Hkv, D, num_pages, page_size, max_pages, int(num_splits), float(scale),
                               workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                               _stream_ptr(stream))
    if rc != FA_OK:
        raise FAError("fa_decode_paged", rc)
    return o, lse


def quantize_kv_int8(x, codes=None, scales=None, stream=None):
    """int8 codes and per-(b, head, token) scales of a bf16 cache through ``fa_quantize_kv_int8``.

    x [B, L, H, D] bf16.  Returns (codes [B, L, H, D] int8, scales [B, H, L] fp32).
    """
    import torch
    _check(x, "x", torch.bfloat16)
    B, L, H, D = x.shape
    if codes is None:
        codes = torch.empty((B, L, H, D), dtype=torch.int8, device=x.device)
    if scales is None:
        scales = torch.empty((B, H, L), dtype=torch.float32, device=x.device)
    _check(codes, "codes", torch.int8)
    _check(scales, "scales", torch.float32)
    rc = lib().fa_quantize_kv_int8(x.data_ptr(), codes.data_ptr(), scales.data_ptr(), B, L, H, D,
                                   _stream_ptr(stream))
    if rc != FA_OK:
        raise FAError("fa_quantize_kv_int8", rc)
    return codes, scales


def decode_int8(q, k_codes, k_scales, v, v_scales, seqlens, num_splits: int, scale: float | None = None,
                o=None, lse=None, workspace=None, want_lse: bool = True, stream=None):
    """Split-KV decode against an int8 cache through ``fa_decode_int8``.

    q [B, 1, Hq, D] bf16; k_codes [B, Lmax, Hkv, D] int8 with k_scales [B, Hkv, Lmax]
    fp32; v either int8 codes with v_scales, or bf16 (v_scales None); seqlens [B]
    int32.  Returns (o [B, 1, Hq, D] bf16, lse [B, Hq] fp32 or None).
    """
    import torch
    _check(q, "q", torch.bfloat16)
    _check(k_codes, "k_codes", torch.int8)
    _check(k_scales, "k_scales", torch.float32)
    _check(v, "v", torch.int8 if v_scales is not None else torch.bfloat16)
    if v_scales is not None:
        _check(v_scales, "v_scales", torch.float32)
    _check(seqlens, "seqlens", torch.int32)
    B, one, Hq, D = q.shape
    Bk, Lmax, Hkv, Dk = k_codes.shape
    if (one != 1 or Bk != B or Dk != D or tuple(v.shape) != tuple(k_codes.shape) or seqlens.shape != (B,)
            or tuple(k_scales.shape) != (B, Hkv, Lmax)
            or (v_scales is not None and tuple(v_scales.shape) != (B, Hkv, Lmax))):
        raise ValueError("int8 decode shapes do not agree")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    need = decode_workspace_bytes(B, Hq, D, num_splits)
    if workspace is None:
        workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=q.device)
    _check(workspace, "workspace")
    rc = lib().fa_decode_int8(q.data_ptr(), k_codes.data_ptr(), k_scales.data_ptr(), v.data_ptr(),
                              v_scales.data_ptr() if v_scales is not None else None, seqlens.data_ptr(),
                              o.data_ptr(), lse.data_ptr() if lse is not None else None,
                              B, Hq, Hkv, D, Lmax, int(num_splits), float(scale),
                              workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    if rc != FA_OK:
        raise FAError("fa_decode_int8", rc)
    return o, lse


def decode_splitkv_noalloc(q, k_cache, v_cache, seqlens, num_splits: int, scale: float | None = None,
                           o=None, lse=None, want_lse: bool = True, stream=None):
    """Split-KV decode through ``fa_decode_splitkv_noalloc``: no workspace.

    For callers that cannot allocate device memory (see the C header): the
    split partials go to the library's fixed scratch buffer, shared by every
    call on the device, so calls that overlap on the GPU race.  Same arguments
    and results as :func:`decode_splitkv`; ``o``/``lse`` are allocated here only
    when not given.
    """
    import torch
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _check(t, n, torch.bfloat16)
    _check(seqlens, "seqlens", torch.int32)
    B, one, Hq, D = q.shape
    Bk, Lmax, Hkv, Dk = k_cache.shape
    if one != 1 or Bk != B or Dk != D or v_cache.shape != k_cache.shape or seqlens.shape != (B,):
        raise ValueError("decode shapes do not agree")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    rc = lib().fa_decode_splitkv_noalloc(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), seqlens.data_ptr(),
                                         o.data_ptr(), lse.data_ptr() if lse is not None else None,
                                         B, Hq, Hkv, D, Lmax, int(num_splits), float(scale), _stream_ptr(stream))
    if rc != FA_OK:
        raise FAError("fa_decode_splitkv_noalloc", rc)
    return o, lse


def to_device_bf16(bits, device="cuda"):
    """numpy uint16 bf16 bit patterns -> bf16 CUDA tensor (input marshalling)."""
    import numpy as np
    import torch
    a = np.ascontiguousarray(bits, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)


def to_f64(t):
    """A CUDA/CPU tensor -> numpy float64 (output marshalling for comparisons)."""
    return t.detach().float().cpu().double().numpy()
