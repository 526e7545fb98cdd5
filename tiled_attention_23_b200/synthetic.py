"""Seeded synthetic inputs (random numbers only, no attention arithmetic).

The generator is counter-mode splitmix64 with Box-Muller normals rounded to
bf16; its definition is in ``csrc/synthetic.c``, compiled into its own small
library.  Tests, the benchmark and the smoke check draw every input from here,
then hand the same bits to both the CUDA path and the fp64 oracle.

Workloads are the shapes the attention pages discuss: the tiny bidirectional
exact-check case, a mid-size causal prefill, the Llama-2-7B-shaped causal
prefill (batch 32, 4096 tokens, head_dim 128 — the recommended configuration of
the ops-transformer page, section 四), the long-context GQA prefill (head_dim
256, GQA groups 1/2/4/8 as on the MNN attention_mode page), and the split-KV
decode against KV caches of seeded lengths.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading
from dataclasses import dataclass

import numpy as np

from ._build import build_synth

_lock = threading.Lock()
_lib = None

STREAM_Q, STREAM_K, STREAM_V, STREAM_LENS, STREAM_PAGES = 1, 2, 3, 4, 5
BF16_NAN = 0x7FC0


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build_synth())
            lib.ta23_synth_normal_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64,
                                                   ctypes.c_uint64, ctypes.c_int, ctypes.c_int]
            lib.ta23_synth_normal_bf16.restype = ctypes.c_int
            lib.ta23_synth_uniform_int.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64,
                                                   ctypes.c_uint64, ctypes.c_int32, ctypes.c_int32]
            lib.ta23_synth_uniform_int.restype = ctypes.c_int
            lib.ta23_synth_word.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64]
            lib.ta23_synth_word.restype = ctypes.c_uint64
            _lib = lib
    return _lib


def _threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def normal_bf16(shape, seed: int, stream: int, pow2: int = 0) -> np.ndarray:
    """bf16 bit patterns (numpy uint16) of i.i.d. N(0,1) * 2**pow2 values."""
    out = np.empty(tuple(shape), dtype=np.uint16)
    rc = _load().ta23_synth_normal_bf16(out.ctypes.data_as(ctypes.c_void_p), out.size,
                                        seed & (2**64 - 1), stream, int(pow2), _threads())
    if rc:
        raise ValueError("synthetic normal generator rejected its arguments")
    return out


def uniform_int(n: int, seed: int, stream: int, lo: int, hi: int) -> np.ndarray:
    """int32 values uniform on [lo, hi] (inclusive)."""
    out = np.empty((n,), dtype=np.int32)
    rc = _load().ta23_synth_uniform_int(out.ctypes.data_as(ctypes.c_void_p), n,
                                        seed & (2**64 - 1), stream, int(lo), int(hi))
    if rc:
        raise ValueError("synthetic integer generator rejected its arguments")
    return out


def word(seed: int, stream: int, counter: int) -> int:
    """Raw 64-bit word ``counter`` of stream (seed, stream) (for tests)."""
    return int(_load().ta23_synth_word(seed & (2**64 - 1), stream, counter))


@dataclass(frozen=True)
class PrefillWorkload:
    """An attention forward problem: Q [B,Lq,Hq,D], K/V [B,Lk,Hkv,D]."""
    name: str
    B: int
    Lq: int
    Lk: int
    Hq: int
    Hkv: int
    D: int
    causal: bool
    k_pow2: int = 0          # K multiplied by 2**k_pow2 after bf16 rounding
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def flops(self) -> float:
        """Metric convention: 4*B*Hq*Lq*Lk*D, halved when causal."""
        f = 4.0 * self.B * self.Hq * self.Lq * self.Lk * self.D
        return f / 2 if self.causal else f

    def with_(self, **kw) -> "PrefillWorkload":
        d = dict(self.__dict__)
        d.update(kw)
        return PrefillWorkload(**d)

    def inputs(self, seed_offset: int = 0):
        s = self.seed + seed_offset
        q = normal_bf16((self.B, self.Lq, self.Hq, self.D), s, STREAM_Q)
        k = normal_bf16((self.B, self.Lk, self.Hkv, self.D), s, STREAM_K, self.k_pow2)
        v = normal_bf16((self.B, self.Lk, self.Hkv, self.D), s, STREAM_V)
        return q, k, v


@dataclass(frozen=True)
class DecodeWorkload:
    """One query token per sequence against a KV cache [B, Lmax, Hkv, D]."""
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    len_lo: int
    len_hi: int
    num_splits: int
    seed: int = 0

    @property
    def Lmax(self) -> int:
        return self.len_hi

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def with_(self, **kw) -> "DecodeWorkload":
        d = dict(self.__dict__)
        d.update(kw)
        return DecodeWorkload(**d)

    def seqlens(self, seed_offset: int = 0) -> np.ndarray:
        return uniform_int(self.B, self.seed + seed_offset, STREAM_LENS, self.len_lo, self.len_hi)

    def kv_bytes(self, seqlens: np.ndarray) -> int:
        """Algorithmic KV bytes read: every valid key and value row once."""
        return int(np.sum(seqlens.astype(np.int64))) * self.Hkv * self.D * 2 * 2

    def io_bytes(self, seqlens: np.ndarray) -> int:
        """KV bytes plus q, o (bf16) and lse (fp32)."""
        return self.kv_bytes(seqlens) + self.B * self.Hq * (self.D * 2 * 2 + 4)

    def inputs(self, seed_offset: int = 0):
        s = self.seed + seed_offset
        q = normal_bf16((self.B, 1, self.Hq, self.D), s, STREAM_Q)
        kc = normal_bf16((self.B, self.Lmax, self.Hkv, self.D), s, STREAM_K)
        vc = normal_bf16((self.B, self.Lmax, self.Hkv, self.D), s, STREAM_V)
        return q, kc, vc, self.seqlens(seed_offset)


def permutation(n: int, seed: int, stream: int = STREAM_PAGES) -> np.ndarray:
    """A seeded permutation of range(n) (Fisher-Yates driven by the generator)."""
    w = uniform_int(max(n, 1), seed, stream, 0, 2**31 - 1).astype(np.int64)
    perm = np.arange(n, dtype=np.int32)
    for i in range(n - 1, 0, -1):
        j = int(w[i] % (i + 1))
        perm[i], perm[j] = perm[j], perm[i]
    return perm


def paginate(k_cache, v_cache, seqlens, page_size: int, seed: int = 0, spare_pages: int = 0,
             poison_tail: bool = True):
    """Lay a contiguous cache [B, Lmax, Hkv, D] out as a shuffled page pool.

    Sequence b needs ceil(len_b / page_size) pages; all needed pages plus
    ``spare_pages`` unused ones form the pool, in a seeded random order.
    Returns (k_pages, v_pages [num_pages, page_size, Hkv, D], block_table
    [B, max_pages] int32, with -1 in entries no key uses).  Unused pages, and
    with ``poison_tail`` the rows past each sequence's end, hold bf16 NaN, so a
    kernel that reads them cannot go unnoticed.
    """
    B, Lmax, Hkv, D = k_cache.shape
    seqlens = np.asarray(seqlens, dtype=np.int64)
    need = (seqlens + page_size - 1) // page_size
    max_pages = (Lmax + page_size - 1) // page_size
    total = int(need.sum()) + int(spare_pages)
    perm = permutation(total, seed)
    k_pages = np.full((total, page_size, Hkv, D), BF16_NAN, dtype=np.uint16)
    v_pages = np.full((total, page_size, Hkv, D), BF16_NAN, dtype=np.uint16)
    table = np.full((B, max_pages), -1, dtype=np.int32)
    nxt = 0
    for b in range(B):
        n = int(seqlens[b])
        for lp in range(int(need[b])):
            phys = int(perm[nxt])
            nxt += 1
            table[b, lp] = phys
            lo, hi = lp * page_size, min((lp + 1) * page_size, n if poison_tail else Lmax)
            hi = max(hi, lo)
            k_pages[phys, : hi - lo] = k_cache[b, lo:hi]
            v_pages[phys, : hi - lo] = v_cache[b, lo:hi]
    return k_pages, v_pages, table


@dataclass(frozen=True)
class VarlenWorkload:
    """A packed batch of B self-attention sequences of seeded lengths in
    [len_lo, len_hi]: q [total, Hq, D], k/v [total, Hkv, D], cu_seqlens [B+1]."""
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    len_lo: int
    len_hi: int
    causal: bool
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def with_(self, **kw) -> "VarlenWorkload":
        d = dict(self.__dict__)
        d.update(kw)
        return VarlenWorkload(**d)

    def seqlens(self, seed_offset: int = 0) -> np.ndarray:
        return uniform_int(self.B, self.seed + seed_offset, STREAM_LENS, self.len_lo, self.len_hi)

    def flops(self, seqlens) -> float:
        """Metric convention per sequence: 4*Hq*L*L*D, halved when causal."""
        L = np.asarray(seqlens, dtype=np.float64)
        f = 4.0 * self.Hq * self.D * float(np.sum(L * L))
        return f / 2 if self.causal else f

    def inputs(self, seed_offset: int = 0):
        s = self.seed + seed_offset
        lens = self.seqlens(seed_offset)
        cu = np.zeros((self.B + 1,), np.int32)
        cu[1:] = np.cumsum(lens)
        total = int(cu[-1])
        q = normal_bf16((total, self.Hq, self.D), s, STREAM_Q)
        k = normal_bf16((total, self.Hkv, self.D), s, STREAM_K)
        v = normal_bf16((total, self.Hkv, self.D), s, STREAM_V)
        return q, k, v, cu


TINY_BIDIR = PrefillWorkload("tiny_bidir_B1_H2_L256_D64", 1, 256, 256, 2, 2, 64, False)
MID_CAUSAL = PrefillWorkload("mid_causal_B4_H16_L2048_D128", 4, 2048, 2048, 16, 16, 128, True)
LLAMA_PREFILL = PrefillWorkload("llama2_7b_prefill_B32_H32_L4096_D128", 32, 4096, 4096, 32, 32, 128,
                                True, k_pow2=1)
LONG_GQA = {g: PrefillWorkload(f"long_gqa_B2_Hq32_Hkv{32 // g}_L8192_D256", 2, 8192, 8192, 32, 32 // g,
                               256, True) for g in (1, 2, 4, 8)}
DECODE = DecodeWorkload("decode_splitkv_B64_Hq32_Hkv8_D128_len512-32768_S8", 64, 32, 8, 128, 512,
                        32768, 8)

DECODE_PAGE_SIZE = 64   # page size of the paged-cache variant of DECODE
# Packed variable-length prefill: the Llama-shaped heads (32 x 128) over 32
# sequences of lengths uniform in [256, 8192] (about as many tokens as the
# fixed-shape Llama-shaped batch), causal.
VARLEN_PREFILL = VarlenWorkload("varlen_prefill_B32_H32_D128_len256-8192", 32, 32, 32, 128, 256, 8192, True)

PREFILL_WORKLOADS = [TINY_BIDIR, MID_CAUSAL, LLAMA_PREFILL] + [LONG_GQA[g] for g in (1, 2, 4, 8)]
