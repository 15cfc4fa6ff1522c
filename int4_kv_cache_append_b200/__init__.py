"""INT4 KV cache for decode attention on B200 (sm_100a): append and paged decode behind a C ABI.

The CUDA library is ``libkv4.so`` (declared in ``include/kv4.h``); ``kv4`` is its ctypes
binding.  Submodules are imported explicitly so that the input generator can be used
without the CUDA library.
"""
__all__ = ["kv4", "workload"]
