"""Decode attention over sequences sharded by token range across processes,
one GPU each (the multi-GPU path for very long sequences).

Every rank keeps a contiguous token range of each sequence in its own cache;
lengths are local to the cache. Softmax attention over the union of the ranges
is the log-sum-exp combination of the per-rank partials, the identity the
split-K merge already uses inside one cache. A step is: split-K and the partial
merge on every rank (libkvq.so), ONE all-gather of the partials (130 floats per
query head per rank, over NCCL between GPUs), then the cross-rank merge
(libkvq.so). Only the all-gather is plumbing; every arithmetic step runs in the
library's kernels.
"""
from __future__ import annotations

from . import _binding as B


def shard_token_range(total: int, world: int, rank: int, align: int = 256):
    """[lo, hi) of a `total`-token sequence held by `rank` of `world`: ranks
    take consecutive runs of whole `align`-token blocks (a multiple of the
    recent window and of the per-channel blocks, so block boundaries stay
    where an unsharded cache has them), the same number each, in rank order;
    the last non-empty rank ends at `total` and so holds the newest tokens.
    Ranks past the end hold nothing (lo == hi)."""
    if total < 0 or world <= 0 or not 0 <= rank < world or align <= 0:
        raise ValueError("bad shard arguments")
    blocks = -(-total // align)
    per = -(-blocks // world) * align
    lo = min(total, rank * per)
    hi = total if rank == world - 1 else min(total, lo + per)
    return lo, hi


def gather_partials(buf, group=None):
    """All-gather one rank's partial buffer [1][n] into [world][n] (rank order)."""
    import torch
    import torch.distributed as dist
    if group is None and not dist.is_initialized():
        return buf
    world = dist.get_world_size(group)
    if world == 1:
        return buf
    out = torch.empty((world, buf.shape[1]), dtype=buf.dtype, device=buf.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, buf, group=group)
    else:
        dist.all_gather(list(out.unbind(0)), buf[0], group=group)
    return out


def decode_attention_sharded(desc: B.CacheDesc, q, seq_lens, max_seq_len: int, softmax_scale: float,
                             group=None, workspace=None, out=None, stream=None):
    """Decode attention of q [S][Hq][128] over the token ranges that all ranks
    of `group` hold for the same S sequences (this rank's in `desc`, its local
    lengths in seq_lens). Every rank calls it and gets the full output."""
    num_seqs, num_q_heads, workspace = B._decode_common(desc, q, seq_lens, max_seq_len, workspace)
    buf = B.partial_buffer(num_seqs, num_q_heads, q.device)
    o_part, ml = B.partial_views(buf[0], num_seqs, num_q_heads)
    B.decode_splitk(desc, q, seq_lens, max_seq_len, softmax_scale, workspace, stream=stream)
    B.decode_merge_partial(desc, num_q_heads, seq_lens, max_seq_len, o_part, ml, workspace, stream=stream)
    parts = gather_partials(buf, group)
    return B.merge_partials(parts, num_seqs, num_q_heads, out=out, stream=stream)
