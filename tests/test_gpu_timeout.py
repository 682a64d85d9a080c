"""Failure detection without a GPU fault: every wait in the decode kernel is
bounded. A test hook makes the producer skip staging one tile, so the
consumers' wait on it runs out after a short limit; the kernel must return,
report KVQ_DEV_TIMEOUT in the status word, and leave the context usable."""
import numpy as np
import pytest
import torch

import bit_kv_cache_21_b200 as K
import workloads as W
from gpu_common import D, SCALE, append, assert_close, dev, lens_tensor, oracle_decode_tokens

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    g = np.random.default_rng(31)
    ch = W.outlier_channels(g)
    k = W.finish(W.keys(g, (300, 1, D), ch), "bf16")
    v = W.finish(W.normal(g, (300, 1, D)), "bf16")
    q = W.finish(W.normal(g, (1, 4, D)), "bf16")
    spec = K.CacheSpec(1, 1, hadamard_block_k=128, capacity_tokens=320)
    cache = K.KVCache(spec)
    sl = lens_tensor([0])
    append(cache, [k], [v], sl)
    torch.cuda.synchronize()
    try:
        K.debug_set(K.DEBUG_WAIT_TIMEOUT_NS, 20_000_000)   # 20 ms
        K.debug_set(K.DEBUG_SKIP_TILE, 0)
        K.decode_attention(cache.desc, dev(q, "bf16"), sl, 320, SCALE)
        torch.cuda.synchronize()
    finally:
        K.debug_set(K.DEBUG_SKIP_TILE, -1)
        K.debug_set(K.DEBUG_WAIT_TIMEOUT_NS, 0)
    assert cache.device_status() & K.DEV_TIMEOUT
    cache.clear_status()
    out = K.decode_attention(cache.desc, dev(q, "bf16"), sl, 320, SCALE).cpu().numpy()
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    assert_close(out[0], oracle_decode_tokens(k, v, q[0], spec), "after timeout")
