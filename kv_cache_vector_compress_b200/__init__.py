"""kv_cache_vector_compress_b200 -- TurboQuant KV-cache vector compression on B200.

The product is the C-ABI library ``libtq.so`` (declared in ``include/tq.h``) built from
``csrc/``; ``tq`` is its thin Python binding over torch tensors and ``synth`` generates
seeded synthetic inputs.  Import ``kv_cache_vector_compress_b200.tq`` to use the library;
it raises if the compiled library is missing.
"""
__all__ = ["tq", "synth"]
