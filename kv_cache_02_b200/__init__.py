"""GQA over a KV cache on B200 (sm_100a): ctypes binding of libgqa.so.

Importing ``kv_cache_02_b200.gqa`` loads the library; it raises if the library
has not been built (``python -m kv_cache_02_b200.build``). There is no other
implementation behind these calls.
"""
