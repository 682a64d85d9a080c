"""The allocation-free decode call, kvq_decode_attention_static.

It serves callers that cannot hand the library a device workspace (a plain C
host program or a plugin inside a runtime that owns all device memory, or a
decode loop that must not call cudaMalloc). Its workspace is a fixed array the
library declares in device memory. These tests check that it returns what
kvq_decode_attention returns with a caller workspace, bit for bit, on two
calls in a row and after a larger call (the array keeps the previous call's
contents), that an empty context gives zeros, and that a batch whose
workspace would not fit the array is refused before anything runs.
This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import bit_kv_cache_21_b200 as K
import workloads as W
from gpu_common import D, SCALE, append, dev, lens_tensor

pytestmark = pytest.mark.gpu


def _cache(g, lens, H, cap):
    ch = W.outlier_channels(g)
    ks = [W.finish(W.keys(g, (t, H, D), ch), "bf16") for t in lens]
    vs = [W.finish(W.normal(g, (t, H, D)), "bf16") for t in lens]
    cache = K.KVCache(K.CacheSpec(len(lens), H, hadamard_block_k=128, capacity_tokens=cap))
    sl = lens_tensor([0] * len(lens))
    append(cache, ks, vs, sl)
    return cache, sl


def test_static_workspace_matches_caller_workspace_twice():
    # The same kernels on the same inputs: the results must be the same bits
    # as with a caller workspace, on two calls in a row (the array keeps the
    # previous call's partials and item counter).
    g = np.random.default_rng(2024)
    S, H, gqa = 4, 8, 4
    cache, sl = _cache(g, [1000, 777, 1, 2048], H, 2048)
    for call in range(2):
        q = dev(W.finish(W.normal(g, (S, H * gqa, D)), "bf16"), "bf16")
        want = K.decode_attention(cache.desc, q, sl, 2048, SCALE)
        got = K.decode_attention_static(cache.desc, q, sl, 2048, SCALE)
        torch.cuda.synchronize()
        assert cache.device_status() == 0
        assert torch.equal(got, want), "call %d" % call


def test_static_workspace_after_a_larger_call():
    # A large call (more sequences and splits, so its partials and item
    # counter sit at other offsets of the array) followed by smaller ones: the
    # smaller calls must not read anything the larger one left.
    g = np.random.default_rng(2025)
    H, gqa = 8, 4
    big, sl_big = _cache(g, [8000, 5000, 3000, 7000, 6000, 1, 4096, 8192], H, 8192)
    q_big = dev(W.finish(W.normal(g, (8, H * gqa, D)), "bf16"), "bf16")
    got_big = K.decode_attention_static(big.desc, q_big, sl_big, 8192, SCALE)
    want_big = K.decode_attention(big.desc, q_big, sl_big, 8192, SCALE)
    small, sl_small = _cache(g, [300, 17], H, 512)
    q_small = dev(W.finish(W.normal(g, (2, H * gqa, D)), "bf16"), "bf16")
    got_small = K.decode_attention_static(small.desc, q_small, sl_small, 512, SCALE)
    want_small = K.decode_attention(small.desc, q_small, sl_small, 512, SCALE)
    torch.cuda.synchronize()
    assert big.device_status() == 0 and small.device_status() == 0
    assert torch.equal(got_big, want_big)
    assert torch.equal(got_small, want_small)


def test_static_workspace_empty_context():
    # max_seq_len = 0: nothing is attended and the output is all zeros, even
    # though the array still holds the previous calls' partials.
    g = np.random.default_rng(2026)
    H, gqa = 8, 4
    cache, _ = _cache(g, [64, 64], H, 128)
    q = dev(W.finish(W.normal(g, (2, H * gqa, D)), "bf16"), "bf16")
    zero = lens_tensor([0, 0])
    out = K.decode_attention_static(cache.desc, q, zero, 0, SCALE)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0


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
