"""B200 (sm_100a) low-bit KV cache: INT4/INT2 quantize-append with Hadamard
rotation (KIVI per-channel keys, values grouped along tokens, attention sinks,
hybrid symmetric/asymmetric groups as options), split-K decode attention over
the packed cache (also over token ranges sharded across GPUs), and XQuant-style
K/V rematerialization on the tensor cores, alone or fused with attention.

The compute lives in libkvq.so (C ABI, include/kvq.h); this package is its
ctypes binding plus helpers that allocate the cache buffers with torch
(`cache`), run the sharded exchange (`sharded`) and capture a decode step as a
CUDA graph (`graph`).
"""
from ._binding import (  # noqa: F401
    BF16, FP16, FP32, PER_TOKEN, PER_CHANNEL,
    DEV_CAPACITY, DEV_TIMEOUT, DEV_SEQLEN,
    DEBUG_WAIT_TIMEOUT_NS, DEBUG_SKIP_TILE,
    OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CAPACITY, ERR_TIMEOUT, ERR_CUDA,
    CacheDesc, KvqError, lib, header_symbols, status_string, check,
    quantize_append, decode_workspace_size, decode_attention, decode_attention_static,
    decode_splitk, decode_merge, decode_merge_partial, merge_partials, partial_buffer, partial_views,
    remat_kv, remat_attention, rope_tables, debug_set, version,
)
from .cache import CacheSpec, KVCache, bf16_cache_desc, sink_view  # noqa: F401
from .graph import DecodeStep  # noqa: F401
