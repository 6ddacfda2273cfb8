"""CSA2 decode step over a globally cached FP4 KV, hand-written CUDA for B200 (sm_100a).

The compute lives in ``libcsa2.so`` (C ABI declared in ``include/csa2.h``); the module
``sparse_attention_fp4_pack_b200.csa2`` is the thin ctypes binding with the same entry
point names.  Importing this package loads nothing; the library is loaded on first use
and a missing or unloadable library raises instead of falling back to anything else.
"""

__all__ = ["csa2"]
