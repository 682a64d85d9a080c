"""Helpers shared by the GPU parity tests: upload seeded inputs, drive the
C-ABI calls, read the cache back in logical order, and build the oracle's
expected values from the same inputs."""
from __future__ import annotations

import math

import numpy as np
import torch

import bit_kv_cache_21_b200 as K
import oracle

D = 128
SCALE = 1.0 / math.sqrt(D)
ATOL = 2e-3     # max-abs bound on attention outputs
RTOL_L2 = 1e-3  # relative L2 bound on attention outputs


def dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    elif dtype == "fp16":
        t = t.to(torch.float16)
    return t.cuda()


def cu(counts) -> torch.Tensor:
    c = np.concatenate([[0], np.cumsum(np.asarray(counts, np.int64))]).astype(np.int32)
    return torch.from_numpy(c).cuda()


def lens_tensor(lens) -> torch.Tensor:
    return torch.tensor(np.asarray(lens, np.int32), dtype=torch.int32, device="cuda")


def append(cache: K.KVCache, ks, vs, seq_lens: torch.Tensor, dtype="bf16"):
    """Append per-sequence chunks ks[s], vs[s] ([n_s][H][D] float32 values)."""
    counts = [k.shape[0] for k in ks]
    H = cache.spec.num_kv_heads
    kk = np.concatenate(ks) if sum(counts) else np.zeros((0, H, D), np.float32)
    k_new = dev(kk, dtype)
    v_new = None
    if cache.spec.with_v:
        vv = np.concatenate(vs) if sum(counts) else np.zeros((0, H, D), np.float32)
        v_new = dev(vv, dtype)
    K.quantize_append(cache.desc, k_new, v_new, cu(counts), seq_lens)


def assign_pages(cache: K.KVCache, lens_final, seed=0):
    """Give every sequence the pages it needs, from a shuffled free list."""
    s = cache.spec
    need = [(int(t) + s.page_size - 1) // s.page_size for t in lens_final]
    assert sum(need) <= s.num_pages and max(need) <= s.max_pages_per_seq
    free = np.random.default_rng(seed).permutation(s.num_pages)
    bt = np.full((s.num_seqs, s.max_pages_per_seq), -1, np.int32)
    i = 0
    for q, n in enumerate(need):
        bt[q, :n] = free[i:i + n]
        i += n
    cache.block_table.copy_(torch.from_numpy(bt))
    return bt


def gather_tokens(cache: K.KVCache, which: str, seq: int, head: int, T: int):
    """Codes [T][row] and scale/zero [T][groups][2] of one (sequence, head)
    in token order, read from the contiguous or paged layout."""
    s = cache.spec
    codes = cache.codes_view(which)
    sz = cache.sz_view(which)
    if not s.paged:
        c = codes[seq, head, :T]
        z = sz[seq, head, :T]
    else:
        n_pages = (T + s.page_size - 1) // s.page_size
        pages = cache.block_table[seq, :n_pages].long()
        c = codes[pages, head].reshape(-1, codes.shape[-1])[:T]
        z = sz[pages, head].reshape(-1, sz.shape[-2], 2)[:T]
    return c.cpu().numpy(), z.cpu().numpy().view(np.uint16)


def expected_tokens(x_hist: np.ndarray, head: int, hb: int, G: int, bits: int, signs=None, hybrid=False):
    """Oracle codes and scale/zero for one head of a [T][H][D] history."""
    return oracle.quantize_tokens(np.ascontiguousarray(x_hist[:, head, :]), hb, G, bits, signs=signs,
                                  hybrid=hybrid)


def oracle_decode_tokens(k_hist, v_hist, q, spec: K.CacheSpec, scale=SCALE, signs=None):
    """Expected decode output of one sequence from its K/V history
    [T][H][D] and query [Hq][D]: the oracle quantizes, dequantizes and
    attends in float64. `signs`: the randomized Hadamard's signs (numpy)."""
    H = k_hist.shape[1]
    T = k_hist.shape[0]
    kh = np.zeros((H, T, D))
    vh = np.zeros((H, T, D))
    for h in range(H):
        kc, ksz = oracle.quantize_tokens(np.ascontiguousarray(k_hist[:, h]), spec.hadamard_block_k,
                                         spec.group_k, spec.bits_k, signs=signs, hybrid=spec.hybrid)
        vc, vsz = oracle.quantize_tokens(np.ascontiguousarray(v_hist[:, h]), 0, spec.group_v,
                                         spec.bits_v, hybrid=spec.hybrid)
        kh[h] = oracle.dequant_tokens(kc, ksz, spec.group_k, spec.bits_k)
        vh[h] = oracle.dequant_tokens(vc, vsz, spec.group_v, spec.bits_v)
    return oracle.decode_attention_gqa(q, kh, vh, scale, rotate_q_block=spec.hadamard_block_k,
                                       signs=signs)


def oracle_decode_kivi(k_hist, v_hist, q, spec: K.CacheSpec, scale=SCALE):
    H = k_hist.shape[1]
    T = k_hist.shape[0]
    kh = np.zeros((H, T, D))
    vh = np.zeros((H, T, D))
    for h in range(H):
        c = oracle.quantize_kivi_sequence(np.ascontiguousarray(k_hist[:, h]),
                                          np.ascontiguousarray(v_hist[:, h]), spec.residual_len,
                                          spec.bits_k, spec.bits_v, spec.group_v)
        kh[h], vh[h] = oracle.dequant_kivi_sequence(c, spec.residual_len, spec.bits_k,
                                                    spec.bits_v, spec.group_v)
    return oracle.decode_attention_gqa(q, kh, vh, scale)


def assert_close(got: np.ndarray, want: np.ndarray, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    err = np.abs(got - want)
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    assert np.all(np.isfinite(got)), what + ": non-finite output"
    assert err.max() <= ATOL, "%s: max abs err %.3g" % (what, err.max())
    assert rel <= RTOL_L2, "%s: rel L2 err %.3g" % (what, rel)
