"""Device buffers of a low-bit KV cache and their kvq_cache_desc.

Memory comes from torch (the caller's allocator); the sizes follow the layouts
that include/kvq.h defines. Nothing here computes on the data.
"""
from __future__ import annotations

import dataclasses

from . import _binding as B

HEAD_DIM = 128


@dataclasses.dataclass
class CacheSpec:
    num_seqs: int
    num_kv_heads: int
    bits_k: int = 4
    bits_v: int = 4
    group_k: int = 128
    group_v: int = 128
    per_channel_k: bool = False
    per_channel_v: bool = False    # values grouped along tokens (group_v == residual_len)
    hadamard_block_k: int = 0
    residual_len: int = 0
    capacity_tokens: int = 0      # contiguous layout
    paged: bool = False
    page_size: int = 16
    max_pages_per_seq: int = 0
    num_pages: int = 0
    with_v: bool = True
    hadamard_signs: object = None  # device float32 [128] of +-1 (randomized Hadamard), or None
    sink_len: int = 0              # attention-sink tokens kept in bf16
    hybrid: bool = False           # per-group symmetric/asymmetric choice


def _row_bytes(bits: int) -> int:
    return HEAD_DIM * 2 if bits == 16 else HEAD_DIM * bits // 8


class KVCache:
    """Owns the device tensors of one cache and the descriptor pointing at them."""

    def __init__(self, spec: CacheSpec, device="cuda"):
        import torch
        self.spec = spec
        s = spec
        u8 = torch.uint8
        if s.paged:
            rows = s.num_pages * s.num_kv_heads * s.page_size
        else:
            rows = s.num_seqs * s.num_kv_heads * s.capacity_tokens
        self.k_codes = torch.zeros(rows * _row_bytes(s.bits_k), dtype=u8, device=device)
        self.v_codes = (torch.zeros(rows * _row_bytes(s.bits_v), dtype=u8, device=device)
                        if s.with_v else None)
        self.k_sz = self.v_sz = None
        if s.bits_k != 16:
            if s.per_channel_k:
                n = s.num_seqs * s.num_kv_heads * (s.capacity_tokens // s.group_k) * HEAD_DIM
            else:
                n = rows * (HEAD_DIM // s.group_k)
            self.k_sz = torch.zeros(n * 4, dtype=u8, device=device)
        if s.with_v and s.bits_v != 16:
            if s.per_channel_v:
                n = s.num_seqs * s.num_kv_heads * (s.capacity_tokens // s.group_v) * HEAD_DIM
            else:
                n = rows * (HEAD_DIM // s.group_v)
            self.v_sz = torch.zeros(n * 4, dtype=u8, device=device)
        self.k_res = self.v_res = None
        if s.residual_len:
            n = s.num_seqs * s.num_kv_heads * s.residual_len * HEAD_DIM
            self.k_res = torch.zeros(n, dtype=torch.bfloat16, device=device)
            self.v_res = torch.zeros(n, dtype=torch.bfloat16, device=device)
        self.k_sink = self.v_sink = None
        if s.sink_len:
            n = s.num_seqs * s.num_kv_heads * s.sink_len * HEAD_DIM
            self.k_sink = torch.zeros(n, dtype=torch.bfloat16, device=device)
            self.v_sink = torch.zeros(n, dtype=torch.bfloat16, device=device)
        self.block_table = None
        if s.paged:
            self.block_table = torch.full((s.num_seqs, s.max_pages_per_seq), -1,
                                          dtype=torch.int32, device=device)
        self.status = torch.zeros(4, dtype=torch.int32, device=device)
        self.desc = self._make_desc()

    def _make_desc(self) -> B.CacheDesc:
        s = self.spec
        p = (lambda t: None if t is None else t.data_ptr())
        return B.CacheDesc(
            num_seqs=s.num_seqs, num_kv_heads=s.num_kv_heads, head_dim=HEAD_DIM,
            bits_k=s.bits_k, bits_v=s.bits_v if s.with_v else 0,
            group_k=s.group_k, group_v=s.group_v,
            axis_k=B.PER_CHANNEL if s.per_channel_k else B.PER_TOKEN,
            axis_v=B.PER_CHANNEL if s.per_channel_v else B.PER_TOKEN,
            hadamard_block_k=s.hadamard_block_k, residual_len=s.residual_len,
            paged=int(s.paged), page_size=s.page_size if s.paged else 0,
            max_pages_per_seq=s.max_pages_per_seq, num_pages=s.num_pages,
            capacity_tokens=s.capacity_tokens, reserved=0,
            k_codes=p(self.k_codes), v_codes=p(self.v_codes), k_sz=p(self.k_sz), v_sz=p(self.v_sz),
            k_res=p(self.k_res), v_res=p(self.v_res), block_table=p(self.block_table),
            status=p(self.status), hadamard_signs=p(s.hadamard_signs),
            k_sink=p(self.k_sink), v_sink=p(self.v_sink), sink_len=s.sink_len,
            hybrid=int(s.hybrid))

    def device_status(self) -> int:
        return int(self.status[0].item())

    def clear_status(self) -> None:
        self.status.zero_()

    # views of the layouts (for tests and inspection)
    def codes_view(self, which: str):
        s = self.spec
        t = self.k_codes if which == "k" else self.v_codes
        bits = s.bits_k if which == "k" else s.bits_v
        if s.paged:
            return t.view(s.num_pages, s.num_kv_heads, s.page_size, _row_bytes(bits))
        return t.view(s.num_seqs, s.num_kv_heads, s.capacity_tokens, _row_bytes(bits))

    def sz_view(self, which: str):
        """uint16 [..., groups, 2] (scale, zero) bit patterns."""
        s = self.spec
        t = self.k_sz if which == "k" else self.v_sz
        G = s.group_k if which == "k" else s.group_v
        import torch
        t16 = t.view(torch.int16)
        if (s.per_channel_k if which == "k" else s.per_channel_v):
            return t16.view(s.num_seqs, s.num_kv_heads, s.capacity_tokens // G, HEAD_DIM, 2)
        if s.paged:
            return t16.view(s.num_pages, s.num_kv_heads, s.page_size, HEAD_DIM // G, 2)
        return t16.view(s.num_seqs, s.num_kv_heads, s.capacity_tokens, HEAD_DIM // G, 2)


def bf16_cache_desc(k, v, status=None) -> B.CacheDesc:
    """Descriptor of an unquantized bf16 cache (bits 16) over k, v
    [S][H][T][128] -- the layout kvq_remat_kv writes -- so that
    kvq_decode_attention reads rematerialized keys and values directly."""
    import torch
    if k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16 or k.shape != v.shape or k.dim() != 4:
        raise ValueError("k, v must be bf16 tensors of one shape [S][H][T][128]")
    if not (k.is_contiguous() and v.is_contiguous()) or k.shape[-1] != HEAD_DIM:
        raise ValueError("k, v must be contiguous with head_dim 128")
    S, H, T, _ = k.shape
    return B.CacheDesc(
        num_seqs=S, num_kv_heads=H, head_dim=HEAD_DIM, bits_k=16, bits_v=16,
        group_k=0, group_v=0, axis_k=B.PER_TOKEN, axis_v=B.PER_TOKEN, hadamard_block_k=0,
        residual_len=0, paged=0, page_size=0, max_pages_per_seq=0, num_pages=0,
        capacity_tokens=T, reserved=0, k_codes=k.data_ptr(), v_codes=v.data_ptr(),
        k_sz=None, v_sz=None, k_res=None, v_res=None, block_table=None,
        status=None if status is None else status.data_ptr())


def sink_view(cache: KVCache, which: str):
    """bf16 [S][H][sink_len][128] view of a cache's attention-sink rows."""
    s = cache.spec
    t = cache.k_sink if which == "k" else cache.v_sink
    return t.view(s.num_seqs, s.num_kv_heads, s.sink_len, HEAD_DIM)
