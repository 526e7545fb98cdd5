"""B200-native tiled attention: prefill forward (fixed-shape and packed
variable-length, bf16 and e4m3), split-KV decode (contiguous, paged and int8
caches) and the backward pass.

The compute path is the CUDA library ``libta23.so`` (sm_100a) behind the C ABI
declared in ``include/ta23.h``; :mod:`.attention` is a thin ctypes binding with
the same entry-point names (``fwd``, ``fwd_varlen``, ``fwd_fp8``,
``quantize_fp8``, ``decode_splitkv``, ``decode_paged``, ``quantize_kv_int8``,
``decode_int8``, ``decode_splitkv_noalloc``, ``bwd``).  ``synthetic`` holds the
seeded input generators.  Nothing here falls back to a CPU implementation:
calling an entry point without the CUDA library or a GPU raises.

    >>> import torch
    >>> from tiled_attention_23_b200 import attention as A
    >>> q = torch.randn(1, 1024, 8, 128, device="cuda", dtype=torch.bfloat16)
    >>> o, lse = A.fwd(q, q, q, causal=True)        # doctest: +SKIP
"""
__all__ = ["attention", "synthetic"]
