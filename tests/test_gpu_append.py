"""Quantize-append parity: packed codes and fp16 scale/zero from the CUDA
kernel must equal the oracle's bit for bit."""
import numpy as np
import pytest
import torch

import bit_kv_cache_21_b200 as K
import workloads as W
from gpu_common import (D, append, assign_pages, expected_tokens, gather_tokens, lens_tensor)

pytestmark = pytest.mark.gpu


def _history(seed, lens, H, dtype, outliers=True):
    g = np.random.default_rng(seed)
    ch = W.outlier_channels(g)
    ks = [W.finish(W.keys(g, (t, H, D), ch) if outliers else W.normal(g, (t, H, D)), dtype) for t in lens]
    vs = [W.finish(W.normal(g, (t, H, D)), dtype) for t in lens]
    return ks, vs


def _check_all(cache, ks, vs, lens, heads=None, signs=None):
    s = cache.spec
    for q, T in enumerate(lens):
        for h in (heads if heads is not None else range(s.num_kv_heads)):
            todo = [("k", ks[q], s.hadamard_block_k, s.group_k, s.bits_k, signs)]
            if s.with_v:
                todo.append(("v", vs[q], 0, s.group_v, s.bits_v, None))
            for which, hist, hb, G, bits, sg in todo:
                c, z = gather_tokens(cache, which, q, h, T)
                ec, ez = expected_tokens(hist, h, hb, G, bits, signs=sg)
                assert np.array_equal(c, ec), (which, q, h)
                assert np.array_equal(z, ez), (which, q, h)


def test_append_tiny_fp32():
    w = W.TINY
    ks, vs, _ = W.kv_history(w, [w.context])
    spec = K.CacheSpec(1, 1, bits_k=4, bits_v=4, group_k=32, group_v=32, hadamard_block_k=128,
                       capacity_tokens=256)
    cache = K.KVCache(spec)
    lens = lens_tensor([0])
    append(cache, ks, vs, lens, dtype="fp32")
    torch.cuda.synchronize()
    assert lens.tolist() == [256]
    assert cache.device_status() == 0
    _check_all(cache, ks, vs, [256])


@pytest.mark.parametrize("bits,G,hb,dtype", [
    (4, 128, 128, "bf16"), (4, 64, 0, "bf16"), (2, 32, 128, "bf16"), (2, 16, 64, "fp16"),
    (4, 16, 32, "fp32"), (2, 128, 0, "bf16"), (4, 32, 2, "bf16"), (2, 64, 16, "fp16")])
def test_append_variants_ragged(bits, G, hb, dtype):
    lens = [37, 130, 1, 64, 0]
    H = 3
    ks, vs = _history(bits * 100 + G + hb, lens, H, dtype)
    spec = K.CacheSpec(len(lens), H, bits_k=bits, bits_v=bits, group_k=G, group_v=G,
                       hadamard_block_k=hb, capacity_tokens=192)
    cache = K.KVCache(spec)
    sl = lens_tensor([0] * len(lens))
    append(cache, ks, vs, sl, dtype=dtype)
    torch.cuda.synchronize()
    assert sl.tolist() == lens
    _check_all(cache, ks, vs, lens)


def test_incremental_append_equals_bulk():
    lens = [200, 77]
    H = 2
    ks, vs = _history(5, lens, H, "bf16")
    spec = K.CacheSpec(2, H, bits_k=4, bits_v=2, group_k=128, group_v=32, hadamard_block_k=128,
                       capacity_tokens=256)
    bulk = K.KVCache(spec)
    append(bulk, ks, vs, lens_tensor([0, 0]))
    inc = K.KVCache(spec)
    sl = lens_tensor([0, 0])
    g = np.random.default_rng(1)
    pos = [0, 0]
    while pos[0] < lens[0] or pos[1] < lens[1]:
        n = [min(int(g.integers(0, 9)), lens[q] - pos[q]) for q in range(2)]
        append(inc, [ks[q][pos[q]:pos[q] + n[q]] for q in range(2)],
               [vs[q][pos[q]:pos[q] + n[q]] for q in range(2)], sl)
        pos = [pos[q] + n[q] for q in range(2)]
    torch.cuda.synchronize()
    assert sl.tolist() == lens
    for a, b in ((bulk.k_codes, inc.k_codes), (bulk.v_codes, inc.v_codes), (bulk.k_sz, inc.k_sz),
                 (bulk.v_sz, inc.v_sz)):
        assert torch.equal(a, b)


def test_paged_equals_contiguous_and_oracle():
    lens = [100, 16, 33, 250]
    H = 2
    ks, vs = _history(9, lens, H, "bf16")
    base = dict(bits_k=4, bits_v=4, group_k=128, group_v=128, hadamard_block_k=128)
    cont = K.KVCache(K.CacheSpec(4, H, capacity_tokens=256, **base))
    append(cont, ks, vs, lens_tensor([0] * 4))
    for ps in (16, 64, 128):
        paged = K.KVCache(K.CacheSpec(4, H, paged=True, page_size=ps, max_pages_per_seq=256 // ps + 1,
                                      num_pages=4 * (256 // ps + 1), **base))
        assign_pages(paged, lens, seed=ps)
        # append in two chunks to cross page boundaries mid-call
        half = [t // 2 for t in lens]
        sl = lens_tensor([0] * 4)
        append(paged, [k[:h] for k, h in zip(ks, half)], [v[:h] for v, h in zip(vs, half)], sl)
        append(paged, [k[h:] for k, h in zip(ks, half)], [v[h:] for v, h in zip(vs, half)], sl)
        torch.cuda.synchronize()
        assert paged.device_status() == 0
        for q, T in enumerate(lens):
            for h in range(H):
                for which in ("k", "v"):
                    a = gather_tokens(paged, which, q, h, T)
                    b = gather_tokens(cont, which, q, h, T)
                    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
        _check_all(paged, ks, vs, lens, heads=[1])


def test_capacity_overflow_sets_status_and_skips():
    H = 1
    ks, vs = _history(3, [70, 10], H, "bf16")
    spec = K.CacheSpec(2, H, bits_k=4, bits_v=4, group_k=128, group_v=128, capacity_tokens=64)
    cache = K.KVCache(spec)
    sl = lens_tensor([0, 0])
    append(cache, ks, vs, sl)
    torch.cuda.synchronize()
    assert cache.device_status() & K.DEV_CAPACITY
    # sequence 1 is intact and sequence 0 holds its first 64 tokens
    c, z = gather_tokens(cache, "k", 1, 0, 10)
    ec, ez = expected_tokens(ks[1], 0, 0, 128, 4)
    assert np.array_equal(c, ec) and np.array_equal(z, ez)
    assert not cache.codes_view("k")[1, 0, 10:].any()
    c0, _ = gather_tokens(cache, "k", 0, 0, 64)
    assert np.array_equal(c0, expected_tokens(ks[0][:64], 0, 0, 128, 4)[0])


def test_paged_missing_page_sets_status():
    H = 2
    ks, vs = _history(4, [40], H, "bf16")
    cache = K.KVCache(K.CacheSpec(1, H, paged=True, page_size=16, max_pages_per_seq=2, num_pages=4))
    cache.block_table.copy_(torch.tensor([[2, 0]], dtype=torch.int32))
    sl = lens_tensor([0])
    append(cache, ks, vs, sl)
    torch.cuda.synchronize()
    assert cache.device_status() & K.DEV_CAPACITY
    c, _ = gather_tokens(cache, "k", 0, 1, 32)
    assert np.array_equal(c, expected_tokens(ks[0][:32], 1, 0, 128, 4)[0])


def test_empty_append_is_noop():
    cache = K.KVCache(K.CacheSpec(2, 2, capacity_tokens=64))
    sl = lens_tensor([5, 7])
    append(cache, [np.zeros((0, 2, D), np.float32)] * 2, [np.zeros((0, 2, D), np.float32)] * 2, sl)
    torch.cuda.synchronize()
    assert sl.tolist() == [5, 7]
    assert not cache.k_codes.any()


def test_x_cache_k_only():
    # quantized layer inputs X viewed as hidden/128 heads, no values
    g = np.random.default_rng(2)
    x = W.finish(W.normal(g, (96, 8, D)), "bf16")
    cache = K.KVCache(K.CacheSpec(1, 8, bits_k=4, group_k=128, capacity_tokens=128, with_v=False))
    sl = lens_tensor([0])
    append(cache, [x], None, sl)
    torch.cuda.synchronize()
    _check_all(cache, [x], None, [96])


def test_llama8b_prefill_full_size_sampled():
    w = W.LLAMA8B_LAYER
    lens = [w.context] * w.batch
    ks, vs, _ = W.kv_history(w, lens)
    spec = K.CacheSpec(w.batch, w.n_kv_heads, bits_k=4, bits_v=4, group_k=128, group_v=128,
                       hadamard_block_k=128, capacity_tokens=w.context + 128)
    cache = K.KVCache(spec)
    sl = lens_tensor([0] * w.batch)
    append(cache, ks, vs, sl)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    for q in (0, 9, 15):
        for h in (0, 5):
            for which, hist, hb in (("k", ks[q], 128), ("v", vs[q], 0)):
                c, z = gather_tokens(cache, which, q, h, w.context)
                ec, ez = expected_tokens(hist, h, hb, 128, 4)
                assert np.array_equal(c, ec) and np.array_equal(z, ez)


@pytest.mark.parametrize("bits,G,hb,paged", [(4, 128, 128, False), (2, 32, 64, False), (4, 64, 32, True)])
def test_append_randomized_hadamard(bits, G, hb, paged):
    # QuaRot's randomized Hadamard: keys take H diag(signs) / sqrt(hb); codes
    # and scale/zero stay bit-exact with the oracle.
    lens = [150, 33, 1, 64]
    H = 2
    ks, vs = _history(700 + bits + G + hb, lens, H, "bf16")
    signs = W.hadamard_signs(17)
    sg = torch.from_numpy(signs).cuda()
    if paged:
        spec = K.CacheSpec(len(lens), H, bits_k=bits, bits_v=bits, group_k=G, group_v=G,
                           hadamard_block_k=hb, paged=True, page_size=16, max_pages_per_seq=16,
                           num_pages=64, hadamard_signs=sg)
        cache = K.KVCache(spec)
        assign_pages(cache, lens)
    else:
        spec = K.CacheSpec(len(lens), H, bits_k=bits, bits_v=bits, group_k=G, group_v=G,
                           hadamard_block_k=hb, capacity_tokens=192, hadamard_signs=sg)
        cache = K.KVCache(spec)
    sl = lens_tensor([0] * len(lens))
    append(cache, ks, vs, sl)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    _check_all(cache, ks, vs, lens, signs=signs)
