"""The allocation-free decode call, kvq_decode_attention_static.

It serves callers that cannot hand the library a device workspace (a plain C
host program or a plugin inside a runtime that owns all device memory, or a
decode loop that must not call cudaMalloc). Its workspace is a fixed array the
library declares in device memory. These tests check that it returns what
kvq_decode_attention returns with a caller workspace, on two calls in a row
(the array keeps the previous call's contents), and that a batch whose
workspace would not fit the array is refused before anything runs.
This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import bit_kv_cache_21_b200 as K
import workloads as W
from gpu_common import D, SCALE, append, assert_close, dev, lens_tensor

pytestmark = pytest.mark.gpu


def test_static_workspace_matches_caller_workspace_twice():
    g = np.random.default_rng(2024)
    S, H, gqa = 4, 8, 4
    lens = [1000, 777, 1, 2048]
    ch = W.outlier_channels(g)
    ks = [W.finish(W.keys(g, (t, H, D), ch), "bf16") for t in lens]
    vs = [W.finish(W.normal(g, (t, H, D)), "bf16") for t in lens]
    cache = K.KVCache(K.CacheSpec(S, H, hadamard_block_k=128, capacity_tokens=2048))
    sl = lens_tensor([0] * S)
    append(cache, ks, vs, sl)
    for call in range(2):
        q = dev(W.finish(W.normal(g, (S, H * gqa, D)), "bf16"), "bf16")
        want = K.decode_attention(cache.desc, q, sl, 2048, SCALE)
        got = K.decode_attention_static(cache.desc, q, sl, 2048, SCALE)
        torch.cuda.synchronize()
        assert cache.device_status() == 0
        assert_close(got.cpu().numpy(), want.cpu().numpy(), "call %d" % call)


def test_static_workspace_refuses_oversize_batch():
    # 1024 sequences x 32 query heads need more split workspace than the array
    S, H = 1024, 8
    cache = K.KVCache(K.CacheSpec(S, H, capacity_tokens=64))
    sl = lens_tensor([0] * S)
    q = torch.zeros((S, 4 * H, D), dtype=torch.bfloat16, device="cuda")
    assert K.decode_workspace_size(cache.desc, S, 4 * H, 64) > 16 << 20
    with pytest.raises(K.KvqError) as err:
        K.decode_attention_static(cache.desc, q, sl, 64, SCALE)
    assert err.value.status == K.ERR_CAPACITY
