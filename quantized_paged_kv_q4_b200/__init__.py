"""quantized_paged_kv_q4_b200 -- attention over a Q8_0-K / Q4_0-V paged KV cache on B200.

The compute lives in libkvattn.so (hand-written CUDA for sm_100a, C ABI in include/kvattn.h);
this package only builds it (``build.build()``) and binds it (``kvattn``).
"""
from . import kvattn  # noqa: F401
from .kvattn import KVAttnError  # noqa: F401
