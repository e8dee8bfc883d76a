"""SemKV-style semantic mixed-precision KV-cache quantization: B200 (sm_100a) hot path.

The compute lives in libsemkv.so (CUDA, C ABI in include/semkv.h); this package is its ctypes
binding (`_lib`, same function names as the C entry points), a torch-allocated cache holder
(`cache.SemkvCache`) and the seeded synthetic input generator (`synth`).
"""
from ._lib import (  # noqa: F401
    SemkvError,
    semkv_append_decode,
    semkv_append_token,
    semkv_append_token_running,
    semkv_assign_precision,
    semkv_cache_bytes,
    semkv_capacities,
    semkv_decode_attention,
    semkv_decode_attention_noalloc,
    semkv_dequantize,
    semkv_quantize_pack,
    semkv_p_for_ratio,
    semkv_p_for_ratio_kv,
    semkv_radix_digits,
    semkv_selftest_wait_timeout,
    semkv_workspace_bytes,
    status_string,
)
from .cache import SemkvCache, capacities  # noqa: F401
