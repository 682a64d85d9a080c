"""Seeded synthetic inputs for the five workloads of the low-bit KV-cache path.

This module only draws random numbers and shapes them. It holds none of the
method's arithmetic (no rotation, quantization, attention or GEMM), so both
the CUDA path and the CPU oracle can take their inputs from it.

Recipe (every draw is numpy PCG64 ``default_rng(seed)``, float32, then rounded
to bf16 where the workload is bf16):
  * K ~ N(0, 1) with 4 of the 128 head_dim channels scaled by 20 (outlier
    channels; indices drawn once per workload with ``rng.choice(128, 4,
    replace=False)`` and shared by every head and token).
  * V ~ N(0, 1), Q ~ N(0, 1).
  * paged mix: context lengths lognormal(ln 4096, sigma = 1), rounded and
    clipped to [1024, 32768].
  * XQuant: X ~ N(0, 1), W_k and W_v ~ N(0, 0.02^2).
  * randomized Hadamard (QuaRot): 128 signs, each -1 or +1 with probability
    1/2 (``hadamard_signs``).
These stand in for the pages' Llama-3.1-8B-shaped layers at 4K-128K contexts;
no dataset or trained weights are used.
"""
from __future__ import annotations

import dataclasses

import numpy as np

HEAD_DIM = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int            # sequences
    n_q_heads: int
    n_kv_heads: int
    context: int          # tokens already cached before the decode steps
    dtype: str            # "fp32" or "bf16" input values
    bits_k: int
    bits_v: int
    group_k: int
    group_v: int
    hadamard_k: int       # 0 = no rotation, else block size
    per_channel_k: bool = False
    residual: int = 0
    paged: bool = False
    page_size: int = 16
    decode_steps: int = 1
    seed: int = 0
    hidden: int = 0       # XQuant only


TINY = Workload("tiny", 1, 4, 1, 256, "fp32", 4, 4, 32, 32, 128, seed=1)
LLAMA8B_LAYER = Workload("llama8b_layer", 16, 32, 8, 8192, "bf16", 4, 4, 128, 128, 128,
                         decode_steps=64, seed=2)
LONG_INT2 = Workload("long_int2", 1, 32, 8, 131072, "bf16", 2, 2, 128, 32, 0,
                     per_channel_k=True, residual=128, seed=3)
PAGED_MIX = Workload("paged_mix", 64, 32, 8, 4096, "bf16", 4, 4, 128, 128, 128,
                     paged=True, page_size=16, seed=4)
XQUANT = Workload("xquant", 8, 32, 8, 16384, "bf16", 16, 16, 128, 128, 0,
                  seed=5, hidden=4096)

ALL = {w.name: w for w in (TINY, LLAMA8B_LAYER, LONG_INT2, PAGED_MIX, XQUANT)}


def rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def to_bf16_values(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (input preparation only; the
    library routine is torch's RNE conversion). Returns float32."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns of float32 values that are already bf16."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def outlier_channels(g: np.random.Generator, d: int = HEAD_DIM, n: int = 4) -> np.ndarray:
    return np.sort(g.choice(d, n, replace=False))


def normal(g: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    x = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def keys(g: np.random.Generator, shape, channels: np.ndarray, factor: float = 20.0) -> np.ndarray:
    """N(0,1) keys whose last-axis `channels` are scaled by `factor`."""
    k = normal(g, shape)
    k[..., channels] *= np.float32(factor)
    return k


def to_fp16_values(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest fp16 (input preparation only)."""
    return np.ascontiguousarray(x, dtype=np.float32).astype(np.float16).astype(np.float32)


def finish(x: np.ndarray, dtype: str) -> np.ndarray:
    """Values of the workload's input dtype ("bf16", "fp16" or "fp32") as float32."""
    if dtype == "bf16":
        return to_bf16_values(x)
    if dtype == "fp16":
        return to_fp16_values(x)
    return np.ascontiguousarray(x, np.float32)


def paged_lengths(seed: int, n: int = 64, median: int = 4096, sigma: float = 1.0,
                  lo: int = 1024, hi: int = 32768) -> np.ndarray:
    g = rng(seed)
    x = g.lognormal(mean=np.log(median), sigma=sigma, size=n)
    return np.clip(np.rint(x), lo, hi).astype(np.int64)


def kv_history(w: Workload, lengths, seed_offset: int = 0):
    """Per-sequence K and V histories [T_s][H_kv][D] (float32 values of the
    workload's dtype) plus the outlier channel indices.

    Sequences are drawn one after another from one generator, K then V, so a
    sequence's values do not depend on how the caller batches them."""
    g = rng(w.seed * 1000 + seed_offset)
    ch = outlier_channels(g)
    ks, vs = [], []
    for T in lengths:
        ks.append(finish(keys(g, (int(T), w.n_kv_heads, HEAD_DIM), ch), w.dtype))
        vs.append(finish(normal(g, (int(T), w.n_kv_heads, HEAD_DIM)), w.dtype))
    return ks, vs, ch


def queries(w: Workload, n_seqs: int, seed_offset: int = 0) -> np.ndarray:
    g = rng(w.seed * 1000 + 500 + seed_offset)
    return finish(normal(g, (n_seqs, w.n_q_heads, HEAD_DIM)), w.dtype)


def xquant_inputs(w: Workload, n_tokens: int, seed_offset: int = 0):
    """X [n_tokens][hidden] and W_kv [2*H_kv*D][hidden] (K rows, then V rows),
    both bf16 values as float32."""
    g = rng(w.seed * 1000 + seed_offset)
    x = finish(normal(g, (n_tokens, w.hidden)), "bf16")
    wkv = finish(normal(g, (2 * w.n_kv_heads * HEAD_DIM, w.hidden), std=0.02), "bf16")
    return x, wkv


def hadamard_signs(seed: int, n: int = HEAD_DIM) -> np.ndarray:
    """n random signs (+1.0 / -1.0, float32) for a randomized Hadamard
    rotation; a seeded input of the method, drawn here so both sides share it."""
    rng = np.random.default_rng(seed)
    return np.where(rng.random(n) < 0.5, -1.0, 1.0).astype(np.float32)
