"""Attention-sink window (InnerQ Abstract: high-precision windows for recent
tokens and attention-sink tokens): a sequence's first sink_len tokens are kept
as bf16 rows, the rest are quantized as usual, and decode attention reads both.
Sink rows must equal the input rounded to bf16 bit for bit, the quantized rows
the oracle's codes, and the attention output the oracle's float64 attention."""
import numpy as np
import pytest
import torch

import bit_kv_cache_21_b200 as K
import oracle
import workloads as W
from gpu_common import (D, SCALE, append, assert_close, assign_pages, dev, expected_tokens,
                        gather_tokens, lens_tensor)

pytestmark = pytest.mark.gpu


def _history(seed, lens, H, dtype="bf16"):
    g = np.random.default_rng(seed)
    ch = W.outlier_channels(g)
    ks = [W.finish(W.keys(g, (t, H, D), ch), dtype) for t in lens]
    vs = [W.finish(W.normal(g, (t, H, D)), dtype) for t in lens]
    return ks, vs


def _check_append(cache, ks, vs, lens, signs=None):
    s = cache.spec
    sk, sv = K.sink_view(cache, "k").cpu(), K.sink_view(cache, "v").cpu()
    for q, T in enumerate(lens):
        n_sink = min(T, s.sink_len)
        for h in range(s.num_kv_heads):
            for which, hist, sink in (("k", ks[q], sk), ("v", vs[q], sv)):
                want = oracle.f32_to_bf16_bits(np.asarray(hist[:n_sink, h], np.float32))
                got = sink[q, h, :n_sink].view(torch.int16).numpy().view(np.uint16)
                assert np.array_equal(got, want), (which, q, h)
            if T > s.sink_len:
                for which, hist, hb, G, bits, sg in (("k", ks[q], s.hadamard_block_k, s.group_k, s.bits_k, signs),
                                                     ("v", vs[q], 0, s.group_v, s.bits_v, None)):
                    c, z = gather_tokens(cache, which, q, h, T)
                    ec, ez = expected_tokens(hist[s.sink_len:], h, hb, G, bits, signs=sg)
                    assert np.array_equal(c[s.sink_len:], ec), (which, q, h)
                    assert np.array_equal(z[s.sink_len:], ez), (which, q, h)


def _bf16_f64(x):
    """The values kept for sink tokens: the input rounded to bf16 (oracle rounding)."""
    b = oracle.f32_to_bf16_bits(np.asarray(x, np.float32)).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def _expected(kh, vh, q, spec, signs=None):
    """Oracle decode output of one sequence with sinks."""
    T, H = kh.shape[0], kh.shape[1]
    n_sink = min(T, spec.sink_len)
    ks = np.stack([_bf16_f64(kh[:n_sink, h]) for h in range(H)])
    vs = np.stack([_bf16_f64(vh[:n_sink, h]) for h in range(H)])
    kq = np.zeros((H, T - n_sink, D))
    vq = np.zeros((H, T - n_sink, D))
    if T > n_sink:
        for h in range(H):
            kc, ksz = oracle.quantize_tokens(np.ascontiguousarray(kh[n_sink:, h]), spec.hadamard_block_k,
                                             spec.group_k, spec.bits_k, signs=signs)
            vc, vsz = oracle.quantize_tokens(np.ascontiguousarray(vh[n_sink:, h]), 0, spec.group_v, spec.bits_v)
            kq[h] = oracle.dequant_tokens(kc, ksz, spec.group_k, spec.bits_k)
            vq[h] = oracle.dequant_tokens(vc, vsz, spec.group_v, spec.bits_v)
    return oracle.decode_attention_gqa_sinks(q, kq, vq, ks, vs, SCALE, rotate_q_block=spec.hadamard_block_k,
                                             signs=signs)


@pytest.mark.parametrize("sink_len,paged,dtype", [(4, False, "bf16"), (64, False, "fp32"), (16, True, "bf16")])
def test_sink_append_bulk_and_incremental(sink_len, paged, dtype):
    lens = [3, sink_len, sink_len + 1, 200]
    H = 2
    ks, vs = _history(sink_len + 5, lens, H, dtype)
    kw = dict(bits_k=4, bits_v=4, group_k=128, group_v=128, hadamard_block_k=128, sink_len=sink_len)
    if paged:
        spec = K.CacheSpec(len(lens), H, paged=True, page_size=16, max_pages_per_seq=16, num_pages=64, **kw)
    else:
        spec = K.CacheSpec(len(lens), H, capacity_tokens=256, **kw)
    for incremental in (False, True):
        cache = K.KVCache(spec)
        if paged:
            assign_pages(cache, lens)
        sl = lens_tensor([0] * len(lens))
        if not incremental:
            append(cache, ks, vs, sl, dtype=dtype)
        else:  # one token per sequence and step, crossing the sink boundary
            for t in range(max(lens)):
                live = [i for i, T in enumerate(lens) if t < T]
                kk = [ks[i][t:t + 1] if i in live else ks[i][:0] for i in range(len(lens))]
                vv = [vs[i][t:t + 1] if i in live else vs[i][:0] for i in range(len(lens))]
                append(cache, kk, vv, sl, dtype=dtype)
        torch.cuda.synchronize()
        assert sl.tolist() == lens and cache.device_status() == 0
        _check_append(cache, ks, vs, lens)


@pytest.mark.parametrize("sink_len,paged,gqa,signed", [(4, False, 4, False), (64, False, 2, True),
                                                        (16, True, 4, False), (1, False, 1, False)])
def test_sink_decode(sink_len, paged, gqa, signed):
    lens = [2, sink_len, sink_len + 1, 700, 1100]
    H = 2
    Hq = H * gqa
    ks, vs = _history(100 + sink_len + gqa, lens, H)
    signs = W.hadamard_signs(9) if signed else None
    kw = dict(bits_k=4, bits_v=4, group_k=128, group_v=128, hadamard_block_k=128, sink_len=sink_len,
              hadamard_signs=torch.from_numpy(signs).cuda() if signed else None)
    if paged:
        spec = K.CacheSpec(len(lens), H, paged=True, page_size=16, max_pages_per_seq=80, num_pages=256, **kw)
    else:
        spec = K.CacheSpec(len(lens), H, capacity_tokens=1152, **kw)
    cache = K.KVCache(spec)
    if paged:
        assign_pages(cache, lens)
    sl = lens_tensor([0] * len(lens))
    append(cache, ks, vs, sl)
    g = np.random.default_rng(7)
    q = W.finish(W.normal(g, (len(lens), Hq, D)), "bf16")
    out = K.decode_attention(cache.desc, dev(q, "bf16"), sl, 1152, SCALE).cpu().numpy()
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    for s_, T in enumerate(lens):
        assert_close(out[s_], _expected(ks[s_], vs[s_], q[s_], spec, signs), "seq %d" % s_)
