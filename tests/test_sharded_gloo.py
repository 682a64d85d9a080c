"""Host side of the token-range sharded decode, on CPU: two gloo ranks each
hold one range of every sequence, compute their partial (here with the
oracle, standing in for the GPU kernels), exchange them with the package's
all-gather, and merge. The result must equal attention over all tokens, also
when one rank holds nothing of a sequence."""
import datetime
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from bit_kv_cache_21_b200 import partial_buffer, partial_views
from bit_kv_cache_21_b200.sharded import gather_partials, shard_token_range

D, HQ, SCALE = 128, 4, 1.0 / np.sqrt(128)
LENS = [1000, 100, 513]   # the second sequence lives on rank 0 alone


def _data(seed=5):
    g = np.random.default_rng(seed)
    ks = [g.standard_normal((t, D)) for t in LENS]
    vs = [g.standard_normal((t, D)) for t in LENS]
    q = g.standard_normal((len(LENS), HQ, D))
    return ks, vs, q


def _rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ks, vs, q = _data()
        S = len(LENS)
        buf = partial_buffer(S, HQ, "cpu")
        o_view, ml_view = partial_views(buf[0], S, HQ)
        for s in range(S):
            lo, hi = shard_token_range(LENS[s], world, rank, align=256)
            o, m, l = oracle.attention_partial(q[s], ks[s][lo:hi], vs[s][lo:hi], SCALE)
            o_view[s] = torch.from_numpy(o)
            ml_view[s, :, 0] = torch.from_numpy(m)
            ml_view[s, :, 1] = torch.from_numpy(l)
        parts = gather_partials(buf)
        assert parts.shape == (world, buf.shape[1])
        got = np.zeros((S, HQ, D))
        for s in range(S):
            per_rank = []
            for r in range(world):
                o_r, ml_r = partial_views(parts[r], S, HQ)
                per_rank.append((o_r[s].double().numpy(), ml_r[s, :, 0].double().numpy(),
                                 ml_r[s, :, 1].double().numpy()))
            got[s] = oracle.merge_partials(per_rank)
        np.save(os.path.join(out_dir, "rank%d.npy" % rank), got)
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def test_shard_token_range_covers_in_block_runs():
    for total, world, align in ((131072, 4, 256), (1000, 3, 256), (100, 2, 256), (0, 2, 128), (5000, 8, 128)):
        ranges = [shard_token_range(total, world, r, align) for r in range(world)]
        assert ranges[0][0] == 0 and max(hi for _, hi in ranges) == total
        for (lo, hi), (lo2, _) in zip(ranges, ranges[1:]):
            assert hi == lo2  # contiguous, in rank order
        for lo, hi in ranges:
            assert lo == hi or (lo % align == 0 and (hi == total or hi % align == 0))


def test_two_rank_exchange_merges_to_full_attention(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    ks, vs, q = _data()
    for r in range(world):
        got = np.load(os.path.join(str(tmp_path), "rank%d.npy" % r))
        for s in range(len(LENS)):
            want = oracle.attention(q[s], ks[s], vs[s], SCALE)
            assert np.allclose(got[s], want, atol=1e-5), (r, s)  # fp32 partial buffers
    # the short sequence sat on rank 0 alone: rank 1's partial for it was empty
    assert shard_token_range(LENS[1], world, 1, 256) == (100, 100)
