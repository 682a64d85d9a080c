"""Hybrid symmetric/asymmetric groups (InnerQ, Abstract, "(i) hybrid
quantization"): the append and window-flush kernels pick, per group, the grid
the oracle picks, bit for bit, and decode attention over such a cache matches
the oracle's float64 attention."""
import numpy as np
import pytest
import torch

import bit_kv_cache_21_b200 as K
import oracle
import workloads as W
from gpu_common import (D, SCALE, append, assert_close, assign_pages, dev, expected_tokens, gather_tokens,
                        lens_tensor, oracle_decode_tokens)

pytestmark = pytest.mark.gpu


def _mixed(g, shape, df, scale):
    # half the token rows heavy-tailed (Student t), half sparse values on a
    # coarse grid (multiples of 1/3, half of them exact zeros): the symmetric
    # grid, with its exact zero level, wins some groups of the second kind
    cont = g.standard_t(df, shape)
    grid = np.round(g.standard_normal(shape) * 3) / 3 * (g.random(shape) < 0.5)
    pick = (g.random(shape[:-1]) < 0.5)[..., None]
    return (np.where(pick, grid, cont) * scale).astype(np.float32)


def _heavy(g, T, H, dtype, df=2, scale=1.0):
    # channels 0..3 of the keys carry x20 outliers as usual
    out = np.where(np.arange(D) < 4, 20, 1).astype(np.float32)
    k = W.finish(_mixed(g, (T, H, D), df, scale) * out, dtype)
    v = W.finish(_mixed(g, (T, H, D), df, scale), dtype)
    return k, v


@pytest.mark.parametrize("bits,G,hb,paged,dtype", [(2, 32, 0, False, "bf16"), (4, 128, 128, False, "bf16"),
                                                   (2, 16, 64, True, "fp32"), (4, 64, 0, True, "fp16"),
                                                   (4, 32, 32, False, "fp32")])
def test_append_hybrid_bit_exact(bits, G, hb, paged, dtype):
    lens = [300, 17, 1, 128]
    H = 2
    g = np.random.default_rng(900 + bits + G + hb)
    hist = [_heavy(g, t, H, dtype) for t in lens]
    ks, vs = [h[0] for h in hist], [h[1] for h in hist]
    if paged:
        spec = K.CacheSpec(len(lens), H, bits_k=bits, bits_v=bits, group_k=G, group_v=G, hadamard_block_k=hb,
                           paged=True, page_size=16, max_pages_per_seq=24, num_pages=96, hybrid=True)
        cache = K.KVCache(spec)
        assign_pages(cache, lens)
    else:
        spec = K.CacheSpec(len(lens), H, bits_k=bits, bits_v=bits, group_k=G, group_v=G, hadamard_block_k=hb,
                           capacity_tokens=320, hybrid=True)
        cache = K.KVCache(spec)
    sl = lens_tensor([0] * len(lens))
    append(cache, ks, vs, sl, dtype=dtype)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    n_groups = n_sym = 0
    for q, T in enumerate(lens):
        for h in range(H):
            for which, hist_x, rot in (("k", ks[q], hb), ("v", vs[q], 0)):
                c, z = gather_tokens(cache, which, q, h, T)
                ec, ez = expected_tokens(hist_x, h, rot, G, bits, hybrid=True)
                assert np.array_equal(c, ec), (which, q, h)
                assert np.array_equal(z, ez), (which, q, h)
                _, za = expected_tokens(hist_x, h, rot, G, bits)
                n_groups += za.shape[0] * za.shape[1]
                n_sym += int(np.sum(np.any(za != ez, axis=-1)))
    assert 0 < n_sym < n_groups  # both grids occur


@pytest.mark.parametrize("bits,G,hb,gqa", [(4, 128, 128, 4), (2, 32, 0, 2), (2, 16, 64, 1)])
def test_decode_over_hybrid_cache(bits, G, hb, gqa):
    lens = [700, 256, 3]
    H = 2
    g = np.random.default_rng(950 + bits + gqa)
    hist = [_heavy(g, t, H, "bf16", df=4, scale=0.7) for t in lens]
    ks, vs = [h[0] for h in hist], [h[1] for h in hist]
    spec = K.CacheSpec(len(lens), H, bits_k=bits, bits_v=bits, group_k=G, group_v=G, hadamard_block_k=hb,
                       capacity_tokens=704, hybrid=True)
    cache = K.KVCache(spec)
    sl = lens_tensor([0] * len(lens))
    append(cache, ks, vs, sl)
    qs = W.finish(W.normal(g, (len(lens), gqa * H, D)), "bf16")
    out = K.decode_attention(cache.desc, dev(qs, "bf16"), sl, 704, SCALE).cpu().numpy()
    assert cache.device_status() == 0
    for s in range(len(lens)):
        assert_close(out[s], oracle_decode_tokens(ks[s], vs[s], qs[s], spec), "seq %d" % s)


@pytest.mark.parametrize("bits,per_channel_k,per_channel_v", [(2, True, False), (4, False, True), (2, True, True)])
def test_window_flush_hybrid(bits, per_channel_k, per_channel_v):
    from test_gpu_kivi import _check_state, _oracle_decode
    H, Hq, S, R = 2, 8, 2, 128
    total = [517, 129]
    g = np.random.default_rng(970 + bits + 2 * per_channel_k + per_channel_v)
    hist = [_heavy(g, t, H, "bf16", df=4, scale=0.7) for t in total]
    ks, vs = [h[0] for h in hist], [h[1] for h in hist]
    spec = K.CacheSpec(S, H, bits_k=bits, bits_v=bits, group_k=R if per_channel_k else 32,
                       group_v=R if per_channel_v else 32, per_channel_k=per_channel_k,
                       per_channel_v=per_channel_v, residual_len=R, capacity_tokens=640, hybrid=True)
    cache = K.KVCache(spec)
    sl = lens_tensor([0] * S)
    half = [t // 2 for t in total]
    append(cache, [ks[s][:half[s]] for s in range(S)], [vs[s][:half[s]] for s in range(S)], sl)
    for s_ in range(3):  # a few one-token steps across a flush
        append(cache, [ks[s][half[s] + s_:half[s] + s_ + 1] for s in range(S)],
               [vs[s][half[s] + s_:half[s] + s_ + 1] for s in range(S)], sl)
    append(cache, [ks[s][half[s] + 3:] for s in range(S)], [vs[s][half[s] + 3:] for s in range(S)], sl)
    torch.cuda.synchronize()
    assert sl.tolist() == total and cache.device_status() == 0
    for s in range(S):
        for h in range(H):
            _check_state(cache, ks[s], vs[s], total[s], s, h)
    qs = W.finish(W.normal(g, (S, Hq, D)), "bf16")
    out = K.decode_attention(cache.desc, dev(qs, "bf16"), sl, 640, SCALE).cpu().numpy()
    for s in range(S):
        assert_close(out[s], _oracle_decode(ks[s], vs[s], qs[s], spec), "seq %d" % s)
