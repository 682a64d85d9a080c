"""Token-range sharded decode, its kernels on one GPU: R "ranks" are R caches
holding consecutive token ranges of the same sequences (as R GPUs would);
each runs the split-K pass and the partial merge into its part of one buffer,
and the cross-part merge must give attention over all tokens. The launches
are independent (no kernel waits on another), so emulating the ranks on one
GPU is safe."""
import numpy as np
import pytest
import torch

import bit_kv_cache_21_b200 as K
import oracle
import workloads as W
from bit_kv_cache_21_b200.sharded import decode_attention_sharded, shard_token_range
from gpu_common import D, SCALE, append, assert_close, dev, lens_tensor

pytestmark = pytest.mark.gpu


def _oracle_rank(k, v, spec):
    """Dequantized keys and values [H][T][D] of one rank's cache (its range)."""
    T, H = k.shape[0], k.shape[1]
    R = spec.residual_len
    Tq = oracle.kivi_split(T, R) if R else T
    kh = np.zeros((H, T, D))
    vh = np.zeros((H, T, D))
    for h in range(H):
        for dst, x, G, bits, pc, hb in ((kh, k, spec.group_k, spec.bits_k, spec.per_channel_k,
                                         spec.hadamard_block_k),
                                        (vh, v, spec.group_v, spec.bits_v, spec.per_channel_v, 0)):
            xs = np.ascontiguousarray(x[:Tq, h])
            if pc:
                for b in range(Tq // R):
                    c, z = oracle.quantize_channel_block(xs[b * R:(b + 1) * R], bits)
                    dst[h, b * R:(b + 1) * R] = oracle.dequant_channel_block(c, z, bits)
            elif Tq:
                c, z = oracle.quantize_tokens(xs, hb, G, bits)
                dst[h, :Tq] = oracle.dequant_tokens(c, z, G, bits)
            dst[h, Tq:] = x[Tq:, h]
    return kh, vh


@pytest.mark.parametrize("case", ["int4_rotated", "kivi_int2_window", "innerq_window"])
@pytest.mark.parametrize("world", [2, 3])
def test_sharded_ranks_merge_to_full_attention(case, world):
    H, gqa = 2, 4
    Hq = H * gqa
    lens = [3000, 700, 90]
    kw = {"int4_rotated": dict(bits_k=4, bits_v=4, group_k=128, group_v=128, hadamard_block_k=128),
          "kivi_int2_window": dict(bits_k=2, bits_v=2, group_k=128, group_v=32, per_channel_k=True,
                                   residual_len=128),
          "innerq_window": dict(bits_k=4, bits_v=4, group_k=32, group_v=128, per_channel_v=True,
                                residual_len=128)}[case]
    g = np.random.default_rng(world * 10 + len(case))
    ch = W.outlier_channels(g)
    ks = [W.finish(W.keys(g, (t, H, D), ch), "bf16") for t in lens]
    vs = [W.finish(W.normal(g, (t, H, D)), "bf16") for t in lens]
    qs = W.finish(W.normal(g, (len(lens), Hq, D)), "bf16")
    q = dev(qs, "bf16")
    S = len(lens)
    parts = K.partial_buffer(S, Hq, q.device, n_part=world)
    ranges = [[shard_token_range(t, world, r, 256) for t in lens] for r in range(world)]
    per_rank_oracle = []
    for r in range(world):
        loc = [hi - lo for lo, hi in ranges[r]]
        cap = max(256, -(-max(loc) // 256) * 256)
        cache = K.KVCache(K.CacheSpec(S, H, capacity_tokens=cap, **kw))
        sl = lens_tensor([0] * S)
        append(cache, [ks[s][lo:hi] for s, (lo, hi) in enumerate(ranges[r])],
               [vs[s][lo:hi] for s, (lo, hi) in enumerate(ranges[r])], sl)
        ws = torch.empty(K.decode_workspace_size(cache.desc, S, Hq, cap), dtype=torch.uint8, device=q.device)
        o_part, ml = K.partial_views(parts[r], S, Hq)
        K.decode_splitk(cache.desc, q, sl, cap, SCALE, ws)
        K.decode_merge_partial(cache.desc, Hq, sl, cap, o_part, ml, ws)
        torch.cuda.synchronize()
        assert cache.device_status() == 0
        per_rank_oracle.append([_oracle_rank(ks[s][lo:hi], vs[s][lo:hi], cache.spec)
                                for s, (lo, hi) in enumerate(ranges[r])])
        # this rank's partial alone: o / l is attention over its range, and
        # an empty range gives (-inf, 0) and zeros
        o_np, ml_np = o_part.cpu().numpy(), ml.cpu().numpy()
        for s, (lo, hi) in enumerate(ranges[r]):
            if hi == lo:
                assert np.all(np.isneginf(ml_np[s, :, 0])) and np.all(ml_np[s, :, 1] == 0)
                assert np.all(o_np[s] == 0)
                continue
            kh, vh = per_rank_oracle[r][s]
            want = oracle.decode_attention_gqa(qs[s], kh, vh, SCALE, rotate_q_block=cache.spec.hadamard_block_k)
            assert_close(o_np[s] / ml_np[s, :, 1:2], want, "rank %d seq %d partial" % (r, s))
    out = K.merge_partials(parts, S, Hq).cpu().numpy()
    for s in range(S):
        kh = np.concatenate([per_rank_oracle[r][s][0] for r in range(world)], axis=1)
        vh = np.concatenate([per_rank_oracle[r][s][1] for r in range(world)], axis=1)
        want = oracle.decode_attention_gqa(qs[s], kh, vh, SCALE, rotate_q_block=kw.get("hadamard_block_k", 0))
        assert_close(out[s], want, "seq %d" % s)


def test_sharded_entry_on_one_process_equals_decode():
    # without a process group the sharded entry is split-K, partial merge and
    # a one-part merge: the same output as the plain decode
    H, Hq, S = 2, 8, 2
    g = np.random.default_rng(3)
    lens = [1500, 40]
    ks = [W.finish(W.normal(g, (t, H, D)), "bf16") for t in lens]
    vs = [W.finish(W.normal(g, (t, H, D)), "bf16") for t in lens]
    cache = K.KVCache(K.CacheSpec(S, H, capacity_tokens=1536))
    sl = lens_tensor([0] * S)
    append(cache, ks, vs, sl)
    q = dev(W.finish(W.normal(g, (S, Hq, D)), "bf16"), "bf16")
    a = decode_attention_sharded(cache.desc, q, sl, 1536, SCALE).cpu().numpy()
    b = K.decode_attention(cache.desc, q, sl, 1536, SCALE).cpu().numpy()
    assert np.allclose(a, b, rtol=1e-6, atol=1e-6)
