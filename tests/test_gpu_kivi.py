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


def _spec(S, H, cap, bits=2, G_v=32, R=128, per_channel=True):
    return K.CacheSpec(S, H, bits_k=bits, bits_v=bits, group_k=R if per_channel else 128,
                       group_v=G_v, per_channel_k=per_channel, residual_len=R, capacity_tokens=cap)


def _check_state(cache, k, v, T, s, h):
    sp = cache.spec
    R = sp.residual_len
    if not sp.per_channel_k:
        return _check_state_token_keys(cache, k, v, T, s, h)
    want = oracle.quantize_kivi_sequence(np.ascontiguousarray(k[:T, h]), np.ascontiguousarray(v[:T, h]),
                                         R, sp.bits_k, sp.bits_v, sp.group_v)
    Tq = want["Tq"]
    assert Tq == oracle.kivi_split(T, R)
    kc = cache.codes_view("k")[s, h, :Tq].cpu().numpy()
    ksz = cache.sz_view("k")[s, h, :Tq // R].cpu().numpy().view(np.uint16)
    vc = cache.codes_view("v")[s, h, :Tq].cpu().numpy()
    vsz = cache.sz_view("v")[s, h, :Tq].cpu().numpy().view(np.uint16)
    assert np.array_equal(kc, want["k_codes"]), (s, h, T)
    assert np.array_equal(ksz, want["k_sz"]), (s, h, T)
    assert np.array_equal(vc, want["v_codes"]), (s, h, T)
    assert np.array_equal(vsz, want["v_sz"]), (s, h, T)
    S, H = sp.num_seqs, sp.num_kv_heads
    kw = cache.k_res.view(S, H, R, D)[s, h, :T - Tq].float().cpu().numpy()
    vw = cache.v_res.view(S, H, R, D)[s, h, :T - Tq].float().cpu().numpy()
    assert np.array_equal(kw, want["k_win"]) and np.array_equal(vw, want["v_win"])


def _check_state_token_keys(cache, k, v, T, s, h):
    # residual window with token-wise key groups: blocks quantized per token
    sp = cache.spec
    R = sp.residual_len
    Tq = oracle.kivi_split(T, R)
    for which, x, G, bits in (("k", k, sp.group_k, sp.bits_k), ("v", v, sp.group_v, sp.bits_v)):
        ec, ez = oracle.quantize_tokens(np.ascontiguousarray(x[:Tq, h]), 0, G, bits)
        assert np.array_equal(cache.codes_view(which)[s, h, :Tq].cpu().numpy(), ec)
        assert np.array_equal(cache.sz_view(which)[s, h, :Tq].cpu().numpy().view(np.uint16), ez)
    S, H = sp.num_seqs, sp.num_kv_heads
    kw = cache.k_res.view(S, H, R, D)[s, h, :T - Tq].float().cpu().numpy()
    assert np.array_equal(kw, k[Tq:T, h])


def _oracle_decode(k, v, q, spec):
    if spec.per_channel_k:
        return oracle_decode_kivi(k, v, q, spec)
    H, T = k.shape[1], k.shape[0]
    R = spec.residual_len
    Tq = oracle.kivi_split(T, R)
    kh = np.zeros((H, T, D))
    vh = np.zeros((H, T, D))
    for h in range(H):
        for dst, x, G, bits in ((kh, k, spec.group_k, spec.bits_k), (vh, v, spec.group_v, spec.bits_v)):
            c, z = oracle.quantize_tokens(np.ascontiguousarray(x[:Tq, h]), 0, G, bits)
            dst[h, :Tq] = oracle.dequant_tokens(c, z, G, bits) if Tq else 0
            dst[h, Tq:] = x[Tq:, h]
    return oracle.decode_attention_gqa(q, kh, vh, SCALE)


@pytest.mark.parametrize("bits,G_v,per_channel", [(2, 32, True), (4, 128, True), (2, 16, True),
                                                   (4, 32, False)])
def test_window_flush_and_attention(bits, G_v, per_channel):
    H, Hq, S = 2, 8, 3
    total = [702, 141, 130]
    g = np.random.default_rng(bits + G_v)
    ch = W.outlier_channels(g)
    ks = [W.finish(W.keys(g, (t, H, D), ch), "bf16") for t in total]
    vs = [W.finish(W.normal(g, (t, H, D)), "bf16") for t in total]
    cache = K.KVCache(_spec(S, H, 768, bits, G_v, per_channel=per_channel))
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


def test_window_64_channel_blocks():
    # residual window and per-channel key blocks of 64 tokens: every block of
    # key scales is its own tile
    H, Hq, S = 2, 8, 2
    total = [517, 64]
    g = np.random.default_rng(64)
    ch = W.outlier_channels(g)
    ks = [W.finish(W.keys(g, (t, H, D), ch), "bf16") for t in total]
    vs = [W.finish(W.normal(g, (t, H, D)), "bf16") for t in total]
    cache = K.KVCache(_spec(S, H, 576, 2, 32, R=64))
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
