"""B200-native tiled attention forward (prefill and split-KV decode).

The compute path is the CUDA library ``libta23.so`` (sm_100a) behind the C ABI
declared in ``include/ta23.h``; :mod:`.attention` is a thin ctypes binding with
the same entry-point names.  ``synthetic`` holds the seeded input generators.
Nothing here falls back to a CPU implementation: calling an entry point without
the CUDA library or a GPU raises.
"""
__all__ = ["attention", "synthetic"]
