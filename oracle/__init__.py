"""fp64 CPU oracle for exact attention (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path (the CUDA library and its Python
binding) never does, and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, fp64); this module compiles it
with gcc when the shared object is missing or older than the source, and wraps
it with ctypes.  Every function takes bf16 inputs as ``uint16`` bit patterns.
See ``oracle.c`` for the definition and the passages it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` (IEEE fp64, no fast-math).  Returns its path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-fno-fast-math", "-ffp-contract=off", "-Wall", "-Wextra",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I, I64, D = ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.oracle_attention_rows.argtypes = [P, P, P, I, I, I, I, I, I, D, I, P, I64, P, P, I]
            lib.oracle_online_rows.argtypes = [P, P, P, I, I, I, I, I, I, D, I, I64, P, I64, P, P, I]
            lib.oracle_probs.argtypes = [P, P, I, I, I, I, I, I, D, I, P]
            lib.oracle_lse_merge.argtypes = [P, P, I, I, P, P]
            lib.oracle_decode_rows.argtypes = [P, P, P, P, I, I, I, I, I, D, P, I64, P, P, I]
            lib.oracle_decode_split_rows.argtypes = [P, P, P, P, I, I, I, I, I, I, D, P, I64, P, P, I]
            lib.oracle_decode_paged_rows.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, D, P, I64, P, P, I]
            lib.oracle_attention_varlen_rows.argtypes = [P, P, P, P, P, I, I, I, I, I, I, D, I, P, I64, P, P, I]
            lib.oracle_quantize_kv_int8.argtypes = [P, P, P, I, I, I, I]
            lib.oracle_decode_int8_rows.argtypes = [P, P, P, P, P, I, P, I, I, I, I, I, D, P, I64, P, P, I]
            lib.oracle_attention_backward.argtypes = [P, P, P, P, I, I, I, I, I, I, D, I, P, P, P]
            lib.oracle_e4m3_decode.argtypes = [P, I64, P]
            lib.oracle_e4m3_encode.argtypes = [P, I64, P]
            lib.oracle_quantize_fp8.argtypes = [P, P, P, I, I, I, I]
            lib.oracle_attention_fp8_rows.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, D, I, P, I64, P, P, I]
            for f in (lib.oracle_attention_rows, lib.oracle_online_rows, lib.oracle_probs,
                      lib.oracle_lse_merge, lib.oracle_decode_rows, lib.oracle_decode_split_rows,
                      lib.oracle_decode_paged_rows, lib.oracle_attention_varlen_rows,
                      lib.oracle_quantize_kv_int8, lib.oracle_decode_int8_rows,
                      lib.oracle_attention_backward, lib.oracle_e4m3_decode, lib.oracle_e4m3_encode,
                      lib.oracle_quantize_fp8, lib.oracle_attention_fp8_rows):
                f.restype = ctypes.c_int
            _lib = lib
    return _lib


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _bits(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (numpy uint16)")
    return a


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def attention(q, k, v, scale: float, causal: bool, rows=None, nthreads: int | None = None):
    """Exact attention in fp64.

    q: [B, Lq, Hq, D]; k, v: [B, Lk, Hkv, D] (uint16 bf16 bits).
    rows: optional flat indices (b*Hq + h)*Lq + i; default all rows.
    Returns (O, L): with ``rows`` None, O is [B, Lq, Hq, D] and L is [B, Hq, Lq];
    otherwise O is [n, D] and L is [n].
    """
    q, k, v = _bits(q), _bits(k), _bits(v)
    B, Lq, Hq, D = q.shape
    Bk, Lk, Hkv, Dk = k.shape
    if (Bk, Dk) != (B, D) or v.shape != k.shape:
        raise ValueError("shape mismatch")
    full = rows is None
    rows = np.arange(B * Hq * Lq, dtype=np.int64) if full else np.ascontiguousarray(rows, dtype=np.int64)
    n = rows.shape[0]
    o = np.empty((n, D), np.float64)
    lse = np.empty((n,), np.float64)
    rc = _load().oracle_attention_rows(_ptr(q), _ptr(k), _ptr(v), B, Lq, Lk, Hq, Hkv, D,
                                       float(scale), int(bool(causal)), _ptr(rows), n,
                                       _ptr(o), _ptr(lse), nthreads or default_threads())
    if rc:
        raise ValueError(f"oracle_attention_rows rejected its arguments (code {rc})")
    if full:
        return o.reshape(B, Hq, Lq, D).transpose(0, 2, 1, 3).copy(), lse.reshape(B, Hq, Lq)
    return o, lse


def online_attention(q, k, v, scale: float, causal: bool, block: int, rows=None,
                     nthreads: int | None = None):
    """The pages' tiled online-softmax algorithm in fp64, blocks of ``block`` keys.

    Same arguments and return layout as :func:`attention`.
    """
    q, k, v = _bits(q), _bits(k), _bits(v)
    B, Lq, Hq, D = q.shape
    _, Lk, Hkv, _ = k.shape
    full = rows is None
    rows = np.arange(B * Hq * Lq, dtype=np.int64) if full else np.ascontiguousarray(rows, dtype=np.int64)
    n = rows.shape[0]
    o = np.empty((n, D), np.float64)
    lse = np.empty((n,), np.float64)
    rc = _load().oracle_online_rows(_ptr(q), _ptr(k), _ptr(v), B, Lq, Lk, Hq, Hkv, D,
                                    float(scale), int(bool(causal)), int(block), _ptr(rows), n,
                                    _ptr(o), _ptr(lse), nthreads or default_threads())
    if rc:
        raise ValueError(f"oracle_online_rows rejected its arguments (code {rc})")
    if full:
        return o.reshape(B, Hq, Lq, D).transpose(0, 2, 1, 3).copy(), lse.reshape(B, Hq, Lq)
    return o, lse


def probs(q, k, scale: float, causal: bool):
    """Probability matrix P [B, Hq, Lq, Lk] of the definition (small inputs)."""
    q, k = _bits(q), _bits(k)
    B, Lq, Hq, D = q.shape
    _, Lk, Hkv, _ = k.shape
    p = np.empty((B, Hq, Lq, Lk), np.float64)
    rc = _load().oracle_probs(_ptr(q), _ptr(k), B, Lq, Lk, Hq, Hkv, D, float(scale),
                              int(bool(causal)), _ptr(p))
    if rc:
        raise ValueError(f"oracle_probs rejected its arguments (code {rc})")
    return p


def lse_merge(o_parts: np.ndarray, l_parts: np.ndarray):
    """Merge chunk results (O_c [S, D], L_c [S]) through their log-sum-exp."""
    o_parts = np.ascontiguousarray(o_parts, dtype=np.float64)
    l_parts = np.ascontiguousarray(l_parts, dtype=np.float64)
    S, D = o_parts.shape
    o = np.empty((D,), np.float64)
    lse = np.empty((1,), np.float64)
    rc = _load().oracle_lse_merge(_ptr(o_parts), _ptr(l_parts), S, D, _ptr(o), _ptr(lse))
    if rc:
        raise ValueError(f"oracle_lse_merge rejected its arguments (code {rc})")
    return o, float(lse[0])


def decode(q, k_cache, v_cache, seqlens, scale: float, rows=None, num_splits: int | None = None,
           nthreads: int | None = None):
    """One query token per sequence against a KV cache, in fp64.

    q: [B, 1, Hq, D] (or [B, Hq, D]); caches: [B, Lmax, Hkv, D]; seqlens: [B] int32.
    rows: optional flat indices b*Hq + h.  With ``num_splits`` the result is
    computed chunk by chunk and merged through the LSE (the split-KV algorithm);
    without it, by the plain definition.
    Returns (O, L): O [B, Hq, D] and L [B, Hq] (or [n, D], [n] with rows).
    """
    q, k_cache, v_cache = _bits(q), _bits(k_cache), _bits(v_cache)
    seqlens = np.ascontiguousarray(seqlens, dtype=np.int32)
    B, Lmax, Hkv, D = k_cache.shape
    Hq = q.shape[-2]
    full = rows is None
    rows = np.arange(B * Hq, dtype=np.int64) if full else np.ascontiguousarray(rows, dtype=np.int64)
    n = rows.shape[0]
    o = np.empty((n, D), np.float64)
    lse = np.empty((n,), np.float64)
    lib = _load()
    nt = nthreads or default_threads()
    if num_splits is None:
        rc = lib.oracle_decode_rows(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), B, Hq,
                                    Hkv, D, Lmax, float(scale), _ptr(rows), n, _ptr(o), _ptr(lse), nt)
    else:
        rc = lib.oracle_decode_split_rows(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), B,
                                          Hq, Hkv, D, Lmax, int(num_splits), float(scale),
                                          _ptr(rows), n, _ptr(o), _ptr(lse), nt)
    if rc:
        raise ValueError(f"oracle decode rejected its arguments (code {rc})")
    if full:
        return o.reshape(B, Hq, D), lse.reshape(B, Hq)
    return o, lse


def attention_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, scale: float, causal: bool, rows=None,
                     nthreads: int | None = None):
    """Exact attention over a packed batch of variable-length sequences, in fp64.

    q: [total_q, Hq, D]; k, v: [total_k, Hkv, D]; cu_seqlens_q/k: [B+1] int32.
    A query token attends only keys of its own sequence (bottom-right causal
    alignment per sequence); a row with no allowed key gets O = 0, L = -inf.
    rows: optional flat indices t*Hq + h.  Returns (O, L): O [total_q, Hq, D]
    and L [Hq, total_q], or O [n, D] and L [n] with rows.
    """
    q, k, v = _bits(q), _bits(k), _bits(v)
    cu_q = np.ascontiguousarray(cu_seqlens_q, dtype=np.int32)
    cu_k = np.ascontiguousarray(cu_seqlens_k, dtype=np.int32)
    total_q, Hq, D = q.shape
    total_k, Hkv, _ = k.shape
    B = cu_q.shape[0] - 1
    full = rows is None
    rows = np.arange(total_q * Hq, dtype=np.int64) if full else np.ascontiguousarray(rows, dtype=np.int64)
    n = rows.shape[0]
    o = np.empty((n, D), np.float64)
    lse = np.empty((n,), np.float64)
    rc = _load().oracle_attention_varlen_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_q), _ptr(cu_k), B, total_q,
                                              total_k, Hq, Hkv, D, float(scale), int(bool(causal)), _ptr(rows),
                                              n, _ptr(o), _ptr(lse), nthreads or default_threads())
    if rc:
        raise ValueError(f"oracle_attention_varlen_rows rejected its arguments (code {rc})")
    if full:
        return o.reshape(total_q, Hq, D), lse.reshape(total_q, Hq).T.copy()
    return o, lse


def attention_backward(q, k, v, dout, scale: float, causal: bool):
    """Gradients (dQ, dK, dV) of the attention definition for upstream gradient dO, in fp64.

    q, dout: [B, Lq, Hq, D]; k, v: [B, Lk, Hkv, D] (uint16 bf16 bits).  Returns dq
    [B, Lq, Hq, D], dk and dv [B, Lk, Hkv, D] (float64); GQA heads sum into their
    K/V head.  Full P rows per (b, head): for small and mid-size problems.
    """
    q, k, v, dout = _bits(q), _bits(k), _bits(v), _bits(dout)
    B, Lq, Hq, D = q.shape
    _, Lk, Hkv, _ = k.shape
    if dout.shape != q.shape or v.shape != k.shape:
        raise ValueError("shape mismatch")
    dq = np.empty((B, Lq, Hq, D), np.float64)
    dk = np.empty((B, Lk, Hkv, D), np.float64)
    dv = np.empty((B, Lk, Hkv, D), np.float64)
    rc = _load().oracle_attention_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), B, Lq, Lk, Hq, Hkv, D,
                                           float(scale), int(bool(causal)), _ptr(dq), _ptr(dk), _ptr(dv))
    if rc:
        raise ValueError(f"oracle_attention_backward rejected its arguments (code {rc})")
    return dq, dk, dv


def quantize_kv_int8(x):
    """Symmetric int8 quantisation of K or V rows, one scale per (b, token, head).

    x: [B, L, H, D] bf16 bits.  Returns (codes [B, L, H, D] int8, scales
    [B, H, L] float32): scale = max|x| / 127 and code = round-half-even(x /
    scale) clamped to [-127, 127], both in fp32; an all-zero row gets scale 0.
    """
    x = _bits(x)
    B, L, H, D = x.shape
    codes = np.empty((B, L, H, D), np.int8)
    scales = np.empty((B, H, L), np.float32)
    rc = _load().oracle_quantize_kv_int8(_ptr(x), _ptr(codes), _ptr(scales), B, L, H, D)
    if rc:
        raise ValueError(f"oracle_quantize_kv_int8 rejected its arguments (code {rc})")
    return codes, scales


def decode_int8(q, k_codes, k_scales, v, v_scales, seqlens, scale: float, rows=None,
                nthreads: int | None = None):
    """One query token per sequence against an int8 KV cache, in fp64.

    k_codes [B, Lmax, Hkv, D] int8 with k_scales [B, Hkv, Lmax] float32; v is
    either int8 codes with v_scales, or bf16 bits (v_scales None).  The cache is
    dequantised exactly (scale * code) and the plain decode definition applied.
    Returns (O [B, Hq, D], L [B, Hq]) (or [n, D], [n] with rows).
    """
    q = _bits(q)
    k_codes = np.ascontiguousarray(k_codes, dtype=np.int8)
    k_scales = np.ascontiguousarray(k_scales, dtype=np.float32)
    v_int8 = v_scales is not None
    if v_int8:
        v = np.ascontiguousarray(v, dtype=np.int8)
        v_scales = np.ascontiguousarray(v_scales, dtype=np.float32)
    else:
        v = _bits(v)
    seqlens = np.ascontiguousarray(seqlens, dtype=np.int32)
    B, Lmax, Hkv, D = k_codes.shape
    Hq = q.shape[-2]
    full = rows is None
    rows = np.arange(B * Hq, dtype=np.int64) if full else np.ascontiguousarray(rows, dtype=np.int64)
    n = rows.shape[0]
    o = np.empty((n, D), np.float64)
    lse = np.empty((n,), np.float64)
    rc = _load().oracle_decode_int8_rows(_ptr(q), _ptr(k_codes), _ptr(k_scales), _ptr(v),
                                         _ptr(v_scales) if v_int8 else None, int(v_int8), _ptr(seqlens),
                                         B, Hq, Hkv, D, Lmax, float(scale), _ptr(rows), n, _ptr(o), _ptr(lse),
                                         nthreads or default_threads())
    if rc:
        raise ValueError(f"oracle_decode_int8_rows rejected its arguments (code {rc})")
    if full:
        return o.reshape(B, Hq, D), lse.reshape(B, Hq)
    return o, lse


def decode_paged(q, k_pages, v_pages, block_table, seqlens, scale: float, rows=None,
                 nthreads: int | None = None):
    """One query token per sequence against a paged cache, in fp64.

    q: [B, 1, Hq, D] (or [B, Hq, D]); k_pages/v_pages: [num_pages, page_size, Hkv, D];
    block_table: [B, max_pages] int32; seqlens: [B] int32.  Key j of sequence b
    is row j % page_size of page block_table[b, j // page_size].
    Returns (O, L): O [B, Hq, D] and L [B, Hq] (or [n, D], [n] with rows).
    """
    q, k_pages, v_pages = _bits(q), _bits(k_pages), _bits(v_pages)
    table = np.ascontiguousarray(block_table, dtype=np.int32)
    seqlens = np.ascontiguousarray(seqlens, dtype=np.int32)
    num_pages, page_size, Hkv, D = k_pages.shape
    Hq = q.shape[-2]
    B, max_pages = table.shape
    full = rows is None
    rows = np.arange(B * Hq, dtype=np.int64) if full else np.ascontiguousarray(rows, dtype=np.int64)
    n = rows.shape[0]
    o = np.empty((n, D), np.float64)
    lse = np.empty((n,), np.float64)
    rc = _load().oracle_decode_paged_rows(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(table), _ptr(seqlens),
                                          B, Hq, Hkv, D, num_pages, page_size, max_pages, float(scale),
                                          _ptr(rows), n, _ptr(o), _ptr(lse), nthreads or default_threads())
    if rc:
        raise ValueError(f"oracle_decode_paged_rows rejected its arguments (code {rc})")
    if full:
        return o.reshape(B, Hq, D), lse.reshape(B, Hq)
    return o, lse


def e4m3_decode(codes) -> np.ndarray:
    """Values of e4m3 codes (OCP 8-bit float E4M3; NaN for S.1111.111), float64."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, np.float64)
    if _load().oracle_e4m3_decode(_ptr(c), c.size, _ptr(out)):
        raise ValueError("oracle_e4m3_decode rejected its arguments")
    return out


def e4m3_encode(x) -> np.ndarray:
    """e4m3 codes of float32 values: round to nearest even, saturating at +-448."""
    a = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(a.shape, np.uint8)
    if _load().oracle_e4m3_encode(_ptr(a), a.size, _ptr(out)):
        raise ValueError("oracle_e4m3_encode rejected its arguments")
    return out


def quantize_fp8(x):
    """Per-(batch, head) e4m3 quantisation of x [B, L, H, D] (bf16 bits).

    Returns (codes [B, L, H, D] uint8, descale [B, H] float32): amax over the
    head's L x D slice, inv = 448 / amax and descale = amax / 448 in fp32 (both
    1 when amax < 2^-110, e.g. an all-zero slice), code = e4m3(x * inv) with the
    product in fp32.
    """
    x = _bits(x)
    B, L, H, D = x.shape
    codes = np.empty((B, L, H, D), np.uint8)
    descale = np.empty((B, H), np.float32)
    rc = _load().oracle_quantize_fp8(_ptr(x), _ptr(codes), _ptr(descale), B, L, H, D)
    if rc:
        raise ValueError(f"oracle_quantize_fp8 rejected its arguments (code {rc})")
    return codes, descale


def attention_fp8(q8, k8, v8, q_descale, k_descale, v_descale, scale: float, causal: bool, rows=None,
                  nthreads: int | None = None):
    """Exact attention in fp64 on e4m3 inputs, each value code * descale of its head.

    q8 [B, Lq, Hq, D], k8/v8 [B, Lk, Hkv, D] uint8 codes; q_descale [B, Hq],
    k_descale/v_descale [B, Hkv] float32.  Rows and returns as for attention().
    """
    q8, k8, v8 = (np.ascontiguousarray(a, dtype=np.uint8) for a in (q8, k8, v8))
    qd, kd, vd = (np.ascontiguousarray(a, dtype=np.float32) for a in (q_descale, k_descale, v_descale))
    B, Lq, Hq, D = q8.shape
    Bk, Lk, Hkv, Dk = k8.shape
    if (Bk, Dk) != (B, D) or v8.shape != k8.shape or qd.shape != (B, Hq) or kd.shape != (B, Hkv) \
            or vd.shape != (B, Hkv):
        raise ValueError("shape mismatch")
    full = rows is None
    rows = np.arange(B * Hq * Lq, dtype=np.int64) if full else np.ascontiguousarray(rows, dtype=np.int64)
    n = rows.shape[0]
    o = np.empty((n, D), np.float64)
    lse = np.empty((n,), np.float64)
    rc = _load().oracle_attention_fp8_rows(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(qd), _ptr(kd), _ptr(vd),
                                           B, Lq, Lk, Hq, Hkv, D, float(scale), int(bool(causal)),
                                           _ptr(rows), n, _ptr(o), _ptr(lse), nthreads or default_threads())
    if rc:
        raise ValueError(f"oracle_attention_fp8_rows rejected its arguments (code {rc})")
    if full:
        return o.reshape(B, Hq, Lq, D).transpose(0, 2, 1, 3).copy(), lse.reshape(B, Hq, Lq)
    return o, lse


def bf16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    """Exact conversion of bf16 bit patterns to float64 (for tests)."""
    a = np.asarray(a, dtype=np.uint16)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
