"""Chunked KV-cache attention with H2O summed weights, eviction and 8/4-bit
cache quantization on B200 (sm_100a), behind the C ABI of ``include/h2okv.h``.

``binding`` holds the ctypes binding (same names as the C ABI) and ``KVCache``,
a cache whose device buffers torch allocates; ``configs`` and ``synth`` hold the
named synthetic workloads and their seeded inputs.
"""

from .binding import (  # noqa: F401
    EXPORTED,
    CacheShape,
    H2OKVError,
    KVCache,
    attn_chunk_with_scoresum,
    h2o_evict_insert,
    h2okv_abi_version,
    h2okv_last_error,
    kv_cache_create,
    kv_cache_destroy,
    kv_cache_device_status,
    kv_cache_get_fill,
    kv_cache_quantize,
    kv_cache_query_sizes,
    kv_cache_reset,
    kv_cache_set_fill,
    kv_cache_set_wait_timeout,
    lib_path,
    load,
)
