"""Residual-window path (KIVI keys per channel over 128-token blocks, values
per token, most recent tokens in bf16): flush parity with the oracle, bit for
bit, and attention over blocks plus window."""
import numpy as np
import pytest
import torch

import bit_kv_cache_21_b200 as K
import oracle
import workloads as W
from gpu_common import (D, SCALE, append, assert_close, dev, lens_tensor, oracle_decode_kivi)

pytestmark = pytest.mark.gpu


def _spec(S, H, cap, bits=2, G_v=32, R=128, per_channel=True, per_channel_v=False):
    return K.CacheSpec(S, H, bits_k=bits, bits_v=bits, group_k=R if per_channel else 128,
                       group_v=R if per_channel_v else G_v, per_channel_k=per_channel,
                       per_channel_v=per_channel_v, residual_len=R, capacity_tokens=cap)


def _oracle_tensor(x, Tq, R, bits, G, per_channel, hybrid=False):
    """Codes, scale/zero bit patterns and dequantized rows of x[:Tq] (one head):
    per channel over R-token blocks, or per token in groups of G."""
    if not per_channel:
        c, z = oracle.quantize_tokens(np.ascontiguousarray(x[:Tq]), 0, G, bits, hybrid=hybrid)
        return c, z, (oracle.dequant_tokens(c, z, G, bits) if Tq else np.zeros((0, D)))
    codes = np.zeros((Tq, D * bits // 8), np.uint8)
    sz = np.zeros((Tq // R, D, 2), np.uint16)
    xh = np.zeros((Tq, D))
    for b in range(Tq // R):
        sl = slice(b * R, (b + 1) * R)
        codes[sl], sz[b] = oracle.quantize_channel_block(np.ascontiguousarray(x[sl]), bits, hybrid=hybrid)
        xh[sl] = oracle.dequant_channel_block(codes[sl], sz[b], bits)
    return codes, sz, xh


def _tensors(spec):
    return (("k", spec.group_k, spec.bits_k, spec.per_channel_k),
            ("v", spec.group_v, spec.bits_v, spec.per_channel_v))


def _check_state(cache, k, v, T, s, h):
    sp = cache.spec
    R = sp.residual_len
    Tq = oracle.kivi_split(T, R)
    if sp.per_channel_k and not sp.per_channel_v and not sp.hybrid:  # the oracle's KIVI composition
        want = oracle.quantize_kivi_sequence(np.ascontiguousarray(k[:T, h]), np.ascontiguousarray(v[:T, h]),
                                             R, sp.bits_k, sp.bits_v, sp.group_v)
        assert want["Tq"] == Tq
        assert np.array_equal(cache.codes_view("k")[s, h, :Tq].cpu().numpy(), want["k_codes"])
        assert np.array_equal(cache.sz_view("k")[s, h, :Tq // R].cpu().numpy().view(np.uint16), want["k_sz"])
    for which, G, bits, pc in _tensors(sp):
        x = k if which == "k" else v
        ec, ez, _ = _oracle_tensor(x[:, h], Tq, R, bits, G, pc, sp.hybrid)
        n_sz = Tq // R if pc else Tq
        assert np.array_equal(cache.codes_view(which)[s, h, :Tq].cpu().numpy(), ec), (which, s, h, T)
        assert np.array_equal(cache.sz_view(which)[s, h, :n_sz].cpu().numpy().view(np.uint16), ez), (which, s, h, T)
    S, H = sp.num_seqs, sp.num_kv_heads
    kw = cache.k_res.view(S, H, R, D)[s, h, :T - Tq].float().cpu().numpy()
    vw = cache.v_res.view(S, H, R, D)[s, h, :T - Tq].float().cpu().numpy()
    assert np.array_equal(kw, k[Tq:T, h]) and np.array_equal(vw, v[Tq:T, h])


def _oracle_decode(k, v, q, spec):
    if spec.per_channel_k and not spec.per_channel_v and not spec.hybrid:
        return oracle_decode_kivi(k, v, q, spec)
    H, T = k.shape[1], k.shape[0]
    R = spec.residual_len
    Tq = oracle.kivi_split(T, R)
    kh = np.zeros((H, T, D))
    vh = np.zeros((H, T, D))
    for h in range(H):
        for (which, G, bits, pc), dst, x in zip(_tensors(spec), (kh, vh), (k, v)):
            dst[h, :Tq] = _oracle_tensor(x[:, h], Tq, R, bits, G, pc, spec.hybrid)[2]
            dst[h, Tq:] = x[Tq:, h]
    return oracle.decode_attention_gqa(q, kh, vh, SCALE)


@pytest.mark.parametrize("bits,G_v,per_channel,per_channel_v",
                         [(2, 32, True, False), (4, 128, True, False), (2, 16, True, False),
                          (4, 32, False, False), (4, 0, False, True), (2, 0, False, True),
                          (2, 0, True, True), (4, 0, True, True)])
def test_window_flush_and_attention(bits, G_v, per_channel, per_channel_v):
    H, Hq, S = 2, 8, 3
    total = [702, 141, 130]
    g = np.random.default_rng(bits + G_v)
    ch = W.outlier_channels(g)
    ks = [W.finish(W.keys(g, (t, H, D), ch), "bf16") for t in total]
    vs = [W.finish(W.normal(g, (t, H, D)), "bf16") for t in total]
    cache = K.KVCache(_spec(S, H, 768, bits, G_v, per_channel=per_channel, per_channel_v=per_channel_v))
    sl = lens_tensor([0] * S)
    # bulk chunk, then single tokens across flush boundaries, then another chunk
    plan = [[300, 5, 127]] + [[1, 1, 1]] * 3 + [[0, 130, 0]] + [[1, 1, 0]] * 2 + [[397, 1, 0]]
    pos = [0] * S
    qs = W.finish(W.normal(g, (S, Hq, D)), "bf16")
    for step in plan:
        append(cache, [ks[s][pos[s]:pos[s] + step[s]] for s in range(S)],
               [vs[s][pos[s]:pos[s] + step[s]] for s in range(S)], sl)
        pos = [pos[s] + step[s] for s in range(S)]
        torch.cuda.synchronize()
        assert sl.tolist() == pos
        for s in range(S):
            _check_state(cache, ks[s], vs[s], pos[s], s, 1)
    assert cache.device_status() == 0
    out = K.decode_attention(cache.desc, dev(qs, "bf16"), sl, 768, SCALE).cpu().numpy()
    for s in range(S):
        assert_close(out[s], _oracle_decode(ks[s][:pos[s]], vs[s][:pos[s]], qs[s], cache.spec),
                     "seq %d" % s)


@pytest.mark.parametrize("per_channel_v", [False, True])
def test_window_64_channel_blocks(per_channel_v):
    # residual window and per-channel blocks of 64 tokens: a tile spans four
    # blocks of key (and value) scales, one per warp
    H, Hq, S = 2, 8, 2
    total = [517, 64]
    g = np.random.default_rng(64 + per_channel_v)
    ch = W.outlier_channels(g)
    ks = [W.finish(W.keys(g, (t, H, D), ch), "bf16") for t in total]
    vs = [W.finish(W.normal(g, (t, H, D)), "bf16") for t in total]
    cache = K.KVCache(_spec(S, H, 576, 2, 32, R=64, per_channel_v=per_channel_v))
    sl = lens_tensor([0] * S)
    append(cache, ks, vs, sl)
    torch.cuda.synchronize()
    for s in range(S):
        _check_state(cache, ks[s], vs[s], total[s], s, 1)
    qs = W.finish(W.normal(g, (S, Hq, D)), "bf16")
    out = K.decode_attention(cache.desc, dev(qs, "bf16"), sl, 576, SCALE).cpu().numpy()
    assert cache.device_status() == 0
    for s in range(S):
        assert_close(out[s], _oracle_decode(ks[s], vs[s], qs[s], cache.spec), "seq %d" % s)


def test_token_by_token_equals_bulk():
    H = 1
    g = np.random.default_rng(12)
    k = W.finish(W.normal(g, (400, H, D)), "bf16")
    v = W.finish(W.normal(g, (400, H, D)), "bf16")
    bulk = K.KVCache(_spec(1, H, 512))
    append(bulk, [k], [v], lens_tensor([0]))
    inc = K.KVCache(_spec(1, H, 512))
    sl = lens_tensor([0])
    for t in range(400):
        append(inc, [k[t:t + 1]], [v[t:t + 1]], sl)
    torch.cuda.synchronize()
    for a, b in ((bulk.k_codes, inc.k_codes), (bulk.v_codes, inc.v_codes), (bulk.k_sz, inc.k_sz),
                 (bulk.v_sz, inc.v_sz)):
        assert torch.equal(a, b)
    # window slots past the live tokens may hold stale rows; compare the live ones
    live = 400 - oracle.kivi_split(400, 128)
    for a, b in ((bulk.k_res, inc.k_res), (bulk.v_res, inc.v_res)):
        assert torch.equal(a.view(128, D)[:live], b.view(128, D)[:live])


def test_long_int2_full_size():
    w = W.LONG_INT2
    ks, vs, _ = W.kv_history(w, [w.context])
    cache = K.KVCache(_spec(1, w.n_kv_heads, w.context))
    sl = lens_tensor([0])
    append(cache, ks, vs, sl)
    q = W.queries(w, 1)
    out = K.decode_attention(cache.desc, dev(q, "bf16"), sl, w.context, SCALE).cpu().numpy()
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    assert sl.tolist() == [w.context]
    for h in (0, 7):
        _check_state(cache, ks[0], vs[0], w.context, 0, h)
    assert_close(out[0], oracle_decode_kivi(ks[0], vs[0], q[0], cache.spec), "long int2")


@pytest.mark.parametrize("gqa,R,bits,G_k", [(1, 256, 4, 32), (2, 128, 2, 64), (4, 64, 4, 128),
                                            (2, 256, 2, 128)])
def test_values_grouped_along_tokens(gqa, R, bits, G_k):
    # InnerQ layout: keys grouped along channels (per token), values along
    # tokens (per channel over the window's R-token blocks)
    H, S = 2, 3
    Hq = gqa * H
    total = [3 * R + 37, R + 1, 5]
    cap = 4 * R
    g = np.random.default_rng(R + gqa)
    ch = W.outlier_channels(g)
    ks = [W.finish(W.keys(g, (t, H, D), ch), "bf16") for t in total]
    vs = [W.finish(W.normal(g, (t, H, D)), "bf16") for t in total]
    spec = K.CacheSpec(S, H, bits_k=bits, bits_v=bits, group_k=G_k, group_v=R, per_channel_v=True,
                       residual_len=R, capacity_tokens=cap)
    cache = K.KVCache(spec)
    sl = lens_tensor([0] * S)
    half = [t // 2 for t in total]
    append(cache, [ks[s][:half[s]] for s in range(S)], [vs[s][:half[s]] for s in range(S)], sl)
    append(cache, [ks[s][half[s]:] for s in range(S)], [vs[s][half[s]:] for s in range(S)], sl)
    torch.cuda.synchronize()
    assert sl.tolist() == total
    for s in range(S):
        for h in range(H):
            _check_state(cache, ks[s], vs[s], total[s], s, h)
    qs = W.finish(W.normal(g, (S, Hq, D)), "bf16")
    out = K.decode_attention(cache.desc, dev(qs, "bf16"), sl, cap, SCALE).cpu().numpy()
    assert cache.device_status() == 0
    for s in range(S):
        assert_close(out[s], _oracle_decode(ks[s], vs[s], qs[s], spec), "seq %d" % s)


def test_values_grouped_along_tokens_long():
    # 32K-token INT4 cache of the llama8b layer shape (8 KV heads, GQA 4),
    # keys per token in 128-channel groups, values per channel in 128-token
    # blocks: several splits per sequence, every tile full
    H, Hq, S, T = 8, 32, 2, 32768
    g = np.random.default_rng(77)
    ch = W.outlier_channels(g)
    ks = [W.finish(W.keys(g, (T, H, D), ch), "bf16") for _ in range(S)]
    vs = [W.finish(W.normal(g, (T, H, D)), "bf16") for _ in range(S)]
    spec = K.CacheSpec(S, H, bits_k=4, bits_v=4, group_k=128, group_v=128, per_channel_v=True,
                       residual_len=128, capacity_tokens=T)
    cache = K.KVCache(spec)
    sl = lens_tensor([0] * S)
    append(cache, ks, vs, sl)
    qs = W.finish(W.normal(g, (S, Hq, D)), "bf16")
    out = K.decode_attention(cache.desc, dev(qs, "bf16"), sl, T, SCALE).cpu().numpy()
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    for h in (0, 5):
        _check_state(cache, ks[1], vs[1], T, 1, h)
    for s in range(S):
        assert_close(out[s], _oracle_decode(ks[s], vs[s], qs[s], spec), "seq %d" % s)
