"""Rematerialization parity (XQuant Abstract): K and V rebuilt on the tensor
cores from the quantized layer-input cache X must match the oracle's float64
GEMM + RoPE. The GPU accumulates in fp32 and rounds once to bf16, so every
element must lie within one bf16 step of the oracle's exact value (the
correctly rounded value or its neighbour across a rounding boundary), and such
flips must be rare. Attention over the rematerialized K/V must match the
oracle's attention over its own rematerialized (bf16-rounded) K/V within the
attention bounds."""
import numpy as np
import pytest
import torch

import bit_kv_cache_21_b200 as K
import oracle
import workloads as W
from gpu_common import D, SCALE, append, assert_close, dev, lens_tensor

pytestmark = pytest.mark.gpu

THETA = 500000.0
MAX_FLIP_RATE = 0.02


def _inputs(seed, B, T, hidden, H):
    g = np.random.default_rng(seed)
    xs = [W.finish(W.normal(g, (T, hidden)), "bf16") for _ in range(B)]
    w = W.finish(W.normal(g, (2 * H * D, hidden), std=0.02), "bf16")
    return xs, w


def _x_cache(xs, cap, dtype="bf16"):
    B = len(xs)
    T, hidden = xs[0].shape
    XH = hidden // D
    cache = K.KVCache(K.CacheSpec(B, XH, bits_k=4, group_k=128, capacity_tokens=cap, with_v=False))
    lens = lens_tensor([0] * B)
    append(cache, [x.reshape(T, XH, D) for x in xs], None, lens, dtype=dtype)
    return cache


def _remat(cache, w, H, B, T):
    cos, sin = K.rope_tables(T, D, THETA)
    k_out = torch.empty((B, H, T, D), dtype=torch.bfloat16, device="cuda")
    v_out = torch.empty_like(k_out)
    K.remat_kv(cache.desc, dev(w, "bf16"), H, cos, sin, B, T, k_out, v_out)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    return k_out, v_out


def _oracle_kv(x_rows, w, H, pos):
    """Oracle K, V float64 [n][H][D] for token rows x_rows [n][hidden], and
    the matching sums of |x^_k * w_k| that bound fp32 accumulation error."""
    codes, sz = oracle.quantize_tokens(np.ascontiguousarray(x_rows, np.float32), 0, 128, 4)
    return _oracle_kv_codes(codes, sz, w, H, pos)


def _oracle_kv_codes(codes, sz, w, H, pos):
    w32 = np.ascontiguousarray(w, np.float32)
    k, v = oracle.remat_kv(codes, sz, 128, 4, w32, H, D, np.asarray(pos, np.int64), THETA)
    xh = oracle.dequant_x_bf16(codes, sz, 128, 4)
    mag = oracle.matmul_nt(np.abs(xh), np.abs(w32))          # [n][2HD]
    n = mag.shape[0]
    mk = mag[:, :H * D].reshape(n, H, D)
    mv = mag[:, H * D:].reshape(n, H, D)
    # RoPE mixes channel i with i + 64 (|cos|, |sin| <= 1): both bounds add.
    pair = np.concatenate([mk[..., D // 2:], mk[..., :D // 2]], axis=-1)
    return k, v, mk + pair, mv


def _to_bf16(x64):
    return torch.from_numpy(np.ascontiguousarray(x64, np.float64)).to(torch.bfloat16).double().numpy()


def _check_kv(got, want, mag, hidden, what):
    """Each element within one bf16 step of the exact value plus the fp32
    dot-product error bound gamma_n * sum|x^_k w_k| (n = hidden, gamma_n =
    n * 2^-24): near-zero results of cancelling sums cannot be held to a bf16
    step of their own size. Few elements may differ from the correctly
    rounded bf16 value."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert np.all(np.isfinite(got)), what
    e = np.floor(np.log2(np.maximum(np.abs(want), 2.0 ** -126)))
    step = 2.0 ** (e - 7)
    tol = step + hidden * 2.0 ** -24 * mag
    err = np.abs(got - want)
    bad = err > tol
    assert not bad.any(), "%s: %d elements outside the bound, worst %.3g of it" % (
        what, int(bad.sum()), float((err / tol).max()))
    flips = float(np.mean(got != _to_bf16(want)))
    assert flips <= MAX_FLIP_RATE, "%s: flip rate %.4f" % (what, flips)


def _compare_rows(k_out, v_out, xs, w, H, rows):
    """rows: list of (b, t). Compares every K and V channel of those tokens."""
    x_rows = np.stack([xs[b][t] for b, t in rows])
    pos = [t for _, t in rows]
    ek, ev, mk, mv = _oracle_kv(x_rows, w, H, pos)
    bi = torch.tensor([b for b, _ in rows], device="cuda")
    ti = torch.tensor(pos, device="cuda")
    gk = k_out[bi, :, ti].double().cpu().numpy()   # [n][H][D]
    gv = v_out[bi, :, ti].double().cpu().numpy()
    hidden = x_rows.shape[1]
    _check_kv(gv, ev, mv, hidden, "V")
    _check_kv(gk, ek, mk, hidden, "K")


@pytest.mark.parametrize("B,T,hidden,H,cap", [
    (2, 256, 512, 2, 256),      # 8 tiles, every element compared
    (3, 128, 128, 3, 384),      # one K head per group row, a tile mixing K and V heads, Tc > T
    (1, 384, 1024, 1, 512),     # single KV head: each tile is one K and one V head
])
def test_remat_small_all_elements(B, T, hidden, H, cap):
    xs, w = _inputs(100 + B * 10 + H, B, T, hidden, H)
    cache = _x_cache(xs, cap)
    k_out, v_out = _remat(cache, w, H, B, T)
    _compare_rows(k_out, v_out, xs, w, H, [(b, t) for b in range(B) for t in range(T)])


def test_remat_many_tiles_per_cta_sampled():
    # 2048 tiles over at most 148 CTAs: every CTA walks many tiles, so both
    # accumulators and every pipeline stage wrap many times.
    B, T, hidden, H = 8, 4096, 256, 8
    xs, w = _inputs(7, B, T, hidden, H)
    cache = _x_cache(xs, T)
    k_out, v_out = _remat(cache, w, H, B, T)
    g = np.random.default_rng(8)
    rows = [(int(b), int(t)) for b, t in zip(g.integers(0, B, 384), g.integers(0, T, 384))]
    rows += [(0, 0), (B - 1, T - 1), (3, 127), (3, 128)]
    _compare_rows(k_out, v_out, xs, w, H, rows)


def test_remat_position_zero_and_identity_weights():
    # W = [I; I] slices: V equals the dequantized X channels, K equals RoPE of
    # them, and at position 0 RoPE is the identity.
    B, T, hidden, H = 1, 128, 256, 1
    g = np.random.default_rng(3)
    xs = [W.finish(W.normal(g, (T, hidden)), "bf16")]
    w = np.zeros((2 * H * D, hidden), np.float32)
    w[np.arange(D), np.arange(D)] = 1.0
    w[D + np.arange(D), np.arange(D)] = 1.0
    cache = _x_cache(xs, T)
    k_out, v_out = _remat(cache, w, H, B, T)
    codes, sz = oracle.quantize_tokens(xs[0], 0, 128, 4)
    xhat = oracle.dequant_x_bf16(codes, sz, 128, 4)[:, :D]
    assert np.array_equal(v_out[0, 0].float().cpu().numpy(), xhat)
    assert np.array_equal(k_out[0, 0, 0].float().cpu().numpy(), xhat[0])


def test_remat_dequant_exact_on_awkward_groups():
    # Groups far from zero with a small range, and groups spanning a large
    # range above a tiny (or fp16-subnormal) minimum, where z - 128 s is not
    # exact in fp32: the dequantized X must still equal the oracle's
    # bf16_rn(fp32(q*s + z)) bit for bit (V = X^ through identity weights).
    B, T, hidden, H = 1, 128, 256, 1
    g = np.random.default_rng(4)
    x = W.normal(g, (T, hidden))
    x[0::4] = 1000.0 + 0.01 * x[0::4]
    x[1::4] = -3000.0 + 0.003 * x[1::4]
    x[2::4] = np.abs(x[2::4]) * 500.0
    x[2::4, ::128] = 1e-4
    x[3::4] = np.abs(x[3::4]) * 500.0
    x[3::4, ::128] = -2e-5
    xs = [np.ascontiguousarray(x, np.float32)]
    w = np.zeros((2 * H * D, hidden), np.float32)
    w[D + np.arange(D), np.arange(D)] = 1.0
    cache = _x_cache(xs, T, dtype="fp32")
    _, v_out = _remat(cache, w, H, B, T)
    codes, sz = oracle.quantize_tokens(xs[0], 0, 128, 4)
    xhat = oracle.dequant_x_bf16(codes, sz, 128, 4)[:, :D]
    assert np.array_equal(v_out[0, 0].float().cpu().numpy(), xhat)


def test_attention_over_rematerialized_kv():
    B, T, hidden, H, HQ = 2, 1024, 1024, 8, 32
    xs, w = _inputs(21, B, T, hidden, H)
    cache = _x_cache(xs, T)
    k_out, v_out = _remat(cache, w, H, B, T)
    g = np.random.default_rng(22)
    q = W.finish(W.normal(g, (B, HQ, D)), "bf16")
    lens = [T, 700]
    sl = lens_tensor(lens)
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    desc = K.bf16_cache_desc(k_out, v_out, status)
    out = K.decode_attention(desc, dev(q, "bf16"), sl, T, SCALE).cpu().numpy()
    torch.cuda.synchronize()
    assert int(status[0]) == 0
    for b in range(B):
        n = lens[b]
        ek, ev, _, _ = _oracle_kv(xs[b][:n], w, H, np.arange(n))
        kh = _to_bf16(ek).transpose(1, 0, 2)   # [H][T][D], bf16 values as materialized
        vh = _to_bf16(ev).transpose(1, 0, 2)
        want = oracle.decode_attention_gqa(q[b], kh, vh, SCALE)
        assert_close(out[b], want, "seq %d" % b)


@pytest.mark.parametrize("HQ,q_dtype", [(32, "bf16"), (16, "fp32"), (8, "fp16")])
def test_fused_remat_attention(HQ, q_dtype):
    # K and V rematerialized in tensor memory and attended in the GEMM's
    # epilogue, never stored: the oracle's attention over its own
    # rematerialized, bf16-rounded K/V, and the unfused path's output
    B, T, hidden, H = 2, 1024, 1024, 8
    xs, w = _inputs(31 + HQ, B, T, hidden, H)
    cache = _x_cache(xs, T)
    g = np.random.default_rng(32 + HQ)
    q = W.finish(W.normal(g, (B, HQ, D)), q_dtype)
    cos, sin = K.rope_tables(T, D, THETA)
    wd = dev(w, "bf16")
    qd = dev(q, q_dtype)
    out = K.remat_attention(cache.desc, wd, H, cos, sin, B, T, qd, SCALE).cpu().numpy()
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    k_out, v_out = _remat(cache, w, H, B, T)
    unfused = K.decode_attention(K.bf16_cache_desc(k_out, v_out), qd, lens_tensor([T] * B), T,
                                 SCALE).cpu().numpy()
    for b in range(B):
        ek, ev, _, _ = _oracle_kv(xs[b], w, H, np.arange(T))
        kh = _to_bf16(ek).transpose(1, 0, 2)
        vh = _to_bf16(ev).transpose(1, 0, 2)
        want = oracle.decode_attention_gqa(q[b].astype(np.float64), kh, vh, SCALE)
        assert_close(out[b], want, "fused seq %d" % b)
        assert_close(out[b], unfused[b], "fused vs unfused seq %d" % b)


def test_xquant_full_size_sampled():
    # 8 sequences x 16384 positions, hidden 4096 (32 X heads), 8 KV heads:
    # the full GEMM runs; sampled tokens are compared channel by channel, and
    # the X codes of those tokens must equal the oracle's bit for bit.
    w_ = W.XQUANT
    B, T, hidden, H = w_.batch, w_.context, w_.hidden, w_.n_kv_heads
    XH = hidden // D
    g = np.random.default_rng(w_.seed)
    cache = K.KVCache(K.CacheSpec(B, XH, bits_k=4, group_k=128, capacity_tokens=T, with_v=False))
    lens = lens_tensor([0] * B)
    rows_g = np.random.default_rng(55)
    picks = sorted(set((int(b), int(t)) for b, t in zip(rows_g.integers(0, B, 48),
                                                       rows_g.integers(0, T, 48))))
    picks += [(0, 0), (B - 1, T - 1)]
    sampled = {}
    for b in range(B):
        x = W.finish(W.normal(g, (T, hidden)), "bf16")
        counts = [0] * B
        counts[b] = T
        cu = torch.tensor(np.concatenate([[0], np.cumsum(counts)]).astype(np.int32), device="cuda")
        K.quantize_append(cache.desc, dev(x.reshape(T, XH, D), "bf16"), None, cu, lens)
        for bb, t in picks:
            if bb == b:
                sampled[(bb, t)] = x[t].copy()
        del x
    w = W.finish(W.normal(g, (2 * H * D, hidden), std=0.02), "bf16")
    k_out, v_out = _remat(cache, w, H, B, T)
    rows = sorted(sampled)
    x_rows = np.stack([sampled[r] for r in rows])
    codes, sz = oracle.quantize_tokens(x_rows, 0, 128, 4)
    cv = cache.codes_view("k")
    zv = cache.sz_view("k")
    for i, (b, t) in enumerate(rows):
        got_c = cv[b, :, t].cpu().numpy().reshape(-1)
        got_z = zv[b, :, t].cpu().numpy().view(np.uint16).reshape(-1, 2)
        assert np.array_equal(got_c, codes[i]), (b, t)
        assert np.array_equal(got_z, sz[i]), (b, t)
    ek, ev, mk, mv = _oracle_kv_codes(codes, sz, w, H, [t for _, t in rows])
    bi = torch.tensor([b for b, _ in rows], device="cuda")
    ti = torch.tensor([t for _, t in rows], device="cuda")
    _check_kv(v_out[bi, :, ti].double().cpu().numpy(), ev, mv, hidden, "V")
    _check_kv(k_out[bi, :, ti].double().cpu().numpy(), ek, mk, hidden, "K")
