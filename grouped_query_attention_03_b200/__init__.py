"""B200-native grouped-query attention: prefill, split-K decode, KV-cache append.

The compute lives in the CUDA library ``libgqa_b200.so`` (C ABI in
``include/gqa.h``); ``gqa`` is its ctypes binding.  Build with
``grouped_query_attention_03_b200.build.build()``.
"""
from . import build  # noqa: F401
