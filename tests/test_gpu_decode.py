"""Decode-attention parity: the split-K kernel over the packed cache against
the oracle's float64 attention over its own dequantized cache."""
import math

import numpy as np
import pytest
import torch

import bit_kv_cache_21_b200 as K
import workloads as W
from gpu_common import (D, SCALE, append, assert_close, assign_pages, dev, lens_tensor,
                        oracle_decode_tokens)

pytestmark = pytest.mark.gpu


def _hist(seed, lens, H, dtype):
    g = np.random.default_rng(seed)
    ch = W.outlier_channels(g)
    ks = [W.finish(W.keys(g, (t, H, D), ch), dtype) for t in lens]
    vs = [W.finish(W.normal(g, (t, H, D)), dtype) for t in lens]
    return ks, vs


def _queries(seed, S, Hq, dtype):
    return W.finish(W.normal(np.random.default_rng(seed), (S, Hq, D)), dtype)


def test_decode_tiny():
    w = W.TINY
    ks, vs, _ = W.kv_history(w, [w.context])
    q = W.queries(w, 1)
    spec = K.CacheSpec(1, 1, bits_k=4, bits_v=4, group_k=32, group_v=32, hadamard_block_k=128,
                       capacity_tokens=256)
    cache = K.KVCache(spec)
    sl = lens_tensor([0])
    append(cache, ks, vs, sl, dtype="fp32")
    out = K.decode_attention(cache.desc, dev(q, "fp32"), sl, 256, SCALE)
    torch.cuda.synchronize()
    assert_close(out.cpu().numpy()[0], oracle_decode_tokens(ks[0], vs[0], q[0], spec), "tiny")


@pytest.mark.parametrize("gqa,bits_k,bits_v,G_k,G_v,hb", [
    (4, 4, 4, 128, 128, 128), (4, 2, 2, 32, 32, 0), (2, 4, 2, 64, 16, 64), (1, 2, 4, 16, 128, 128),
    (4, 4, 2, 128, 32, 32), (2, 4, 4, 32, 64, 0)])
def test_decode_variants_ragged(gqa, bits_k, bits_v, G_k, G_v, hb):
    lens = [1, 63, 64, 65, 700, 0, 129]
    H = 2
    Hq = H * gqa
    ks, vs = _hist(gqa * 7 + bits_k + G_k + hb, lens, H, "bf16")
    spec = K.CacheSpec(len(lens), H, bits_k=bits_k, bits_v=bits_v, group_k=G_k, group_v=G_v,
                       hadamard_block_k=hb, capacity_tokens=768)
    cache = K.KVCache(spec)
    sl = lens_tensor([0] * len(lens))
    append(cache, ks, vs, sl)
    q = _queries(11, len(lens), Hq, "bf16")
    out = K.decode_attention(cache.desc, dev(q, "bf16"), sl, 768, SCALE).cpu().numpy()
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    for s, T in enumerate(lens):
        if T == 0:
            assert not np.any(out[s])
            continue
        assert_close(out[s], oracle_decode_tokens(ks[s], vs[s], q[s], spec), "seq %d" % s)


def test_split_count_invariance_and_two_pass_api():
    # The same sequence decoded with different split sizes (the split plan
    # depends on the batch's unit count and max_seq_len) gives the same output.
    H = 2
    ks, vs = _hist(3, [3000], H, "bf16")
    q0 = _queries(4, 1, 8, "bf16")
    spec_a = K.CacheSpec(1, H, hadamard_block_k=128, capacity_tokens=3072)
    a = K.KVCache(spec_a)
    sl_a = lens_tensor([0])
    append(a, ks, vs, sl_a)
    out_a = K.decode_attention(a.desc, dev(q0, "bf16"), sl_a, 3000, SCALE).cpu().numpy()
    S_b = 40
    b = K.KVCache(K.CacheSpec(S_b, H, hadamard_block_k=128, capacity_tokens=8192))
    sl_b = lens_tensor([0] * S_b)
    g = np.random.default_rng(9)
    append(b, ks + [W.finish(W.normal(g, (1, H, D)), "bf16")] * (S_b - 1),
           vs + [W.finish(W.normal(g, (1, H, D)), "bf16")] * (S_b - 1), sl_b)
    qb = np.concatenate([q0, _queries(5, S_b - 1, 8, "bf16")])
    out_b = K.decode_attention(b.desc, dev(qb, "bf16"), sl_b, 8192, SCALE).cpu().numpy()
    # split boundaries change the fp32 summation order and the softmax reference
    assert np.max(np.abs(out_b[0] - out_a[0])) < 1e-4
    # the two passes called separately give the attention call's result
    qd = dev(q0, "bf16")
    ws = torch.empty(K.decode_workspace_size(a.desc, 1, 8, 3000), dtype=torch.uint8, device="cuda")
    out2 = torch.empty((1, 8, D), dtype=torch.float32, device="cuda")
    K.decode_splitk(a.desc, qd, sl_a, 3000, SCALE, ws)
    K.decode_merge(a.desc, 8, sl_a, 3000, out2, ws)
    assert np.array_equal(out2.cpu().numpy(), out_a)
    assert_close(out_a[0], oracle_decode_tokens(ks[0], vs[0], q0[0], spec_a), "seq 0")


def test_seq_longer_than_max_sets_status():
    H = 1
    ks, vs = _hist(5, [300], H, "bf16")
    spec = K.CacheSpec(1, H, capacity_tokens=512)
    cache = K.KVCache(spec)
    sl = lens_tensor([0])
    append(cache, ks, vs, sl)
    q = _queries(6, 1, 4, "bf16")
    out = K.decode_attention(cache.desc, dev(q, "bf16"), sl, 256, SCALE).cpu().numpy()
    torch.cuda.synchronize()
    assert cache.device_status() & K.DEV_SEQLEN
    assert_close(out[0], oracle_decode_tokens(ks[0][:256], vs[0][:256], q[0], spec), "truncated")


def test_paged_mix_shrunk():
    # 12 sequences, lognormal lengths, 3 append a 70-token chunk, the rest 1 token
    g = np.random.default_rng(44)
    pre = np.clip(np.rint(g.lognormal(np.log(300), 1.0, 12)), 20, 2000).astype(int)
    new = np.array([70, 70, 70] + [1] * 9)
    final = pre + new
    H, Hq = 2, 8
    ks, vs = _hist(45, final, H, "bf16")
    spec = K.CacheSpec(12, H, hadamard_block_k=128, paged=True, page_size=16,
                       max_pages_per_seq=2100 // 16 + 1, num_pages=int(sum(final // 16 + 1)) + 8)
    cache = K.KVCache(spec)
    assign_pages(cache, final, seed=3)
    sl = lens_tensor([0] * 12)
    append(cache, [k[:p] for k, p in zip(ks, pre)], [v[:p] for v, p in zip(vs, pre)], sl)
    append(cache, [k[p:] for k, p in zip(ks, pre)], [v[p:] for v, p in zip(vs, pre)], sl)
    q = _queries(46, 12, Hq, "bf16")
    out = K.decode_attention(cache.desc, dev(q, "bf16"), sl, int(final.max()), SCALE).cpu().numpy()
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    for s in range(12):
        assert_close(out[s], oracle_decode_tokens(ks[s], vs[s], q[s], spec), "seq %d" % s)


def test_llama8b_decode_steps_full_size():
    """The benchmark's workload: 16 sequences x 8 KV heads, prefill 8192, then
    decode steps that each append one token and attend to everything."""
    w = W.LLAMA8B_LAYER
    steps = 4
    lens = [w.context + steps] * w.batch
    ks, vs, _ = W.kv_history(w, lens)
    spec = K.CacheSpec(w.batch, w.n_kv_heads, hadamard_block_k=128,
                       capacity_tokens=w.context + w.decode_steps + 64)
    cache = K.KVCache(spec)
    sl = lens_tensor([0] * w.batch)
    append(cache, [k[:w.context] for k in ks], [v[:w.context] for v in vs], sl)
    for step in range(steps):
        t = w.context + step
        append(cache, [k[t:t + 1] for k in ks], [v[t:t + 1] for v in vs], sl)
        q = W.queries(w, w.batch, seed_offset=step)
        out = K.decode_attention(cache.desc, dev(q, "bf16"), sl, spec.capacity_tokens, SCALE)
        if step in (0, steps - 1):
            o = out.cpu().numpy()
            for s in ((0, 15) if step == 0 else (7,)):
                assert_close(o[s], oracle_decode_tokens(ks[s][:t + 1], vs[s][:t + 1], q[s], spec),
                             "step %d seq %d" % (step, s))
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    assert sl.tolist() == lens


def test_paged_mix_full_size_sampled():
    w = W.PAGED_MIX
    pre = W.paged_lengths(w.seed)
    new = np.array([512] * 8 + [1] * 56)
    final = pre + new
    ks, vs, _ = W.kv_history(w, final)
    ps = w.page_size
    spec = K.CacheSpec(64, w.n_kv_heads, hadamard_block_k=128, paged=True, page_size=ps,
                       max_pages_per_seq=int(final.max()) // ps + 1,
                       num_pages=int(sum(final // ps + 1)))
    cache = K.KVCache(spec)
    assign_pages(cache, final, seed=w.seed)
    sl = lens_tensor([0] * 64)
    append(cache, [k[:p] for k, p in zip(ks, pre)], [v[:p] for v, p in zip(vs, pre)], sl)
    append(cache, [k[p:] for k, p in zip(ks, pre)], [v[p:] for v, p in zip(vs, pre)], sl)
    q = W.queries(w, 64)
    out = K.decode_attention(cache.desc, dev(q, "bf16"), sl, int(final.max()), SCALE).cpu().numpy()
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    longest = int(np.argmax(final))
    for s in sorted({0, 8, 63, longest}):
        assert_close(out[s], oracle_decode_tokens(ks[s], vs[s], q[s], spec), "seq %d" % s)
    assert math.isfinite(float(out.sum()))


@pytest.mark.parametrize("hb,gqa", [(128, 4), (64, 2)])
def test_decode_randomized_hadamard(hb, gqa):
    # Keys and queries both take H diag(signs) / sqrt(hb), so the scores are
    # those of the unrotated vectors; the output matches the oracle's float64
    # attention over its own dequantized cache.
    lens = [257, 70, 1]
    H = 2
    Hq = H * gqa
    ks, vs = _hist(900 + hb, lens, H, "bf16")
    signs = W.hadamard_signs(23)
    spec = K.CacheSpec(len(lens), H, bits_k=4, bits_v=4, group_k=128, group_v=128,
                       hadamard_block_k=hb, capacity_tokens=384,
                       hadamard_signs=torch.from_numpy(signs).cuda())
    cache = K.KVCache(spec)
    sl = lens_tensor([0] * len(lens))
    append(cache, ks, vs, sl)
    q = _queries(31, len(lens), Hq, "bf16")
    out = K.decode_attention(cache.desc, dev(q, "bf16"), sl, 384, SCALE).cpu().numpy()
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    for s_, T in enumerate(lens):
        assert_close(out[s_], oracle_decode_tokens(ks[s_], vs[s_], q[s_], spec, signs=signs), "seq %d" % s_)


@pytest.mark.parametrize("packed", [False, True])
def test_decode_step_graph_replays_the_eager_step(packed):
    # the CUDA-graph step (uploads, append, decode, download) gives the eager
    # calls' results bit for bit, step after step, and advances the lengths;
    # packed: k, v and q back to back in one pinned buffer, uploaded by one copy
    import workloads as W
    S, H, Hq, T0, steps = 3, 2, 8, 300, 4
    g = np.random.default_rng(77)
    ch = W.outlier_channels(g)
    hist_k = W.finish(W.keys(g, (S, T0 + steps, H, D), ch), "bf16")
    hist_v = W.finish(W.normal(g, (S, T0 + steps, H, D)), "bf16")
    qs = W.finish(W.normal(g, (steps, S, Hq, D)), "bf16")
    caches, lens = [], []
    for _ in range(2):
        c = K.KVCache(K.CacheSpec(S, H, bits_k=4, bits_v=4, group_k=128, group_v=128, hadamard_block_k=128,
                                  capacity_tokens=384))
        sl = lens_tensor([0] * S)
        append(c, [hist_k[s, :T0] for s in range(S)], [hist_v[s, :T0] for s in range(S)], sl)
        caches.append(c)
        lens.append(sl)
    cu_one = torch.arange(0, S + 1, dtype=torch.int32, device="cuda")
    if packed:
        buf = torch.empty(2 * (2 * S * H * D + S * Hq * D), dtype=torch.uint8).pin_memory()
        n_kv = 2 * S * H * D
        hk = buf[:n_kv].view(torch.bfloat16).view(S, H, D)
        hv = buf[n_kv:2 * n_kv].view(torch.bfloat16).view(S, H, D)
        hq = buf[2 * n_kv:].view(torch.bfloat16).view(S, Hq, D)
    else:
        hk = torch.empty((S, H, D), dtype=torch.bfloat16).pin_memory()
        hv = torch.empty_like(hk).pin_memory()
        hq = torch.empty((S, Hq, D), dtype=torch.bfloat16).pin_memory()
    step = K.DecodeStep(caches[1].desc, lens[1], cu_one, 384, SCALE, hk, hv, hq)
    assert (step.h_all is not None) == packed
    for i in range(steps):
        kk = torch.from_numpy(hist_k[:, T0 + i]).to(torch.bfloat16)
        vv = torch.from_numpy(hist_v[:, T0 + i]).to(torch.bfloat16)
        qq = torch.from_numpy(qs[i]).to(torch.bfloat16)
        K.quantize_append(caches[0].desc, kk.cuda(), vv.cuda(), cu_one, lens[0])
        want = K.decode_attention(caches[0].desc, qq.cuda(), lens[0], 384, SCALE).cpu()
        hk.copy_(kk)
        hv.copy_(vv)
        hq.copy_(qq)
        step.run()
        torch.cuda.synchronize()
        assert torch.equal(step.out_host, want), i
        assert lens[1].tolist() == [T0 + i + 1] * S
    assert torch.equal(caches[0].k_codes, caches[1].k_codes) and torch.equal(caches[0].v_sz, caches[1].v_sz)
    assert caches[1].device_status() == 0
