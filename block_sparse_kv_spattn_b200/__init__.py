"""Block-sparse decode attention over a paged KV cache, for B200 (sm_100a).

The compute lives in libspattn.so (C ABI, include/spattn.h); ``spattn`` is
its ctypes binding, ``workloads`` draws seeded synthetic inputs, ``build``
compiles the library in-tree.
"""
__all__ = ["spattn", "workloads", "build"]
