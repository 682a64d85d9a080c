"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test ties one oracle function to something other than itself: a library
routine, a closed form, an invariant, brute force on tiny inputs, or a value
the pages print. No test retypes the oracle's own formula.
"""
import os

import numpy as np
import pytest
import scipy.linalg
import scipy.special
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# Number encodings: pinned to numpy's and torch's conversions
# ---------------------------------------------------------------------------

def _edge_values():
    g = np.random.default_rng(11)
    spans = [g.standard_normal(2000).astype(np.float32) * np.float32(10.0) ** e
             for e in (-9, -7, -5, -3, 0, 2, 4)]
    edges = np.array([0.0, -0.0, 1.0, -1.0, 65504.0, 65505.0, 65519.99, 65520.0, 70000.0,
                      -65520.0, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -14,
                      2.0 ** -14 - 2.0 ** -24, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11,
                      np.inf, -np.inf], dtype=np.float32)
    return np.concatenate(spans + [edges])


def test_f16_nearest_matches_numpy():
    v = _edge_values()
    got = oracle.f32_to_f16_bits(v, oracle.ROUND_NEAREST)
    want = v.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("mode", [oracle.ROUND_DOWN, oracle.ROUND_UP])
def test_f16_directed_brackets_value(mode):
    v = _edge_values()
    v = v[np.isfinite(v) & (np.abs(v) <= 65504)]
    h = oracle.f32_to_f16_bits(v, mode).view(np.float16)
    hv = h.astype(np.float64)
    x = v.astype(np.float64)
    if mode == oracle.ROUND_DOWN:
        assert np.all(hv <= x)
        nxt = np.nextafter(h, np.float16(np.inf)).astype(np.float64)
        assert np.all((hv == x) | (nxt > x))
    else:
        assert np.all(hv >= x)
        prv = np.nextafter(h, np.float16(-np.inf)).astype(np.float64)
        assert np.all((hv == x) | (prv < x))


def test_bf16_nearest_matches_torch():
    v = _edge_values()
    v = v[np.abs(v) < 1e38]
    got = oracle.f32_to_bf16_bits(v)
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)


# ---------------------------------------------------------------------------
# Rotation: Sylvester Hadamard (scipy), orthogonality, q.k invariance
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 64, 128])
def test_fwht_matrix_is_sylvester_hadamard(n):
    # Rotating the unit vectors gives the columns of c*H_n exactly (the
    # butterflies only add +-1, and the final scale is one multiply).
    rows = oracle.rotate_f32(np.eye(n, dtype=np.float32), n)
    c = np.float32(1.0 / np.sqrt(n))
    H = scipy.linalg.hadamard(n)
    assert np.array_equal(rows.T, (H * c).astype(np.float32))
    assert np.array_equal(H @ H.T, n * np.eye(n, dtype=H.dtype))


@pytest.mark.parametrize("n", [2, 8, 32, 128])
def test_fwht_close_to_dense_transform(n):
    g = np.random.default_rng(n)
    x = (g.standard_normal((500, n)) * 20).astype(np.float32)
    H = scipy.linalg.hadamard(n).astype(np.float64)
    want = x.astype(np.float64) @ H.T / np.sqrt(n)
    got32 = oracle.rotate_f32(x, n).astype(np.float64)
    # log2(n) fp32 roundings of partial sums bounded by sum|x|, plus the scale.
    bound = (np.log2(n) + 2) * 2.0 ** -24 * np.abs(x).astype(np.float64).sum(1, keepdims=True)
    assert np.all(np.abs(got32 - want) <= bound)
    got64 = oracle.rotate_f64(x, n)
    assert np.allclose(got64, want, rtol=0, atol=1e-12 * np.abs(x).sum())


def test_fwht_golden_worked_example():
    with open(os.path.join(GOLDEN, "fwht_h4.txt")) as f:
        lines = [ln for ln in f if ln.strip() and not ln.startswith("#")]
    for ln in lines:
        a, b = ln.split(";")
        x = np.array(a.split(), np.float32)
        y = np.array(b.split(), np.float64)
        assert np.array_equal(oracle.rotate_f32(x, 4).astype(np.float64), y)
        assert np.array_equal(oracle.rotate_f64(x, 4), y)


def test_block_diagonal_rotation_acts_per_block():
    g = np.random.default_rng(3)
    x = g.standard_normal((7, 128)).astype(np.float32)
    full = oracle.rotate_f32(x, 32)
    for b in range(4):
        assert np.array_equal(full[:, 32 * b:32 * (b + 1)], oracle.rotate_f32(x[:, 32 * b:32 * (b + 1)], 32))


@pytest.mark.parametrize("hb", [128, 64, 16])
def test_rotation_preserves_query_key_dot(hb):
    # Dual-QK Abstract: applying the same orthogonal transform to q and k
    # preserves q.k.
    g = np.random.default_rng(hb)
    q = g.standard_normal((64, 128))
    k = g.standard_normal((64, 128)) * np.where(np.arange(128) % 37 == 0, 20, 1)
    dots = np.einsum("nd,nd->n", q, k)
    rq, rk = oracle.rotate_f64(q, hb), oracle.rotate_f64(k, hb)
    assert np.allclose(np.einsum("nd,nd->n", rq, rk), dots, rtol=1e-12, atol=1e-12 * np.abs(q * k).sum(1).max())
    rq32, rk32 = oracle.rotate_f32(q, hb).astype(np.float64), oracle.rotate_f32(k, hb).astype(np.float64)
    scale = (np.abs(q).sum(1) * np.abs(k).sum(1))
    assert np.all(np.abs(np.einsum("nd,nd->n", rq32, rk32) - dots) <= 1e-5 * scale)


# ---------------------------------------------------------------------------
# Quantizer: error bound, special cases, packing layout
# ---------------------------------------------------------------------------

def _groups(g, n, G):
    out = [g.standard_normal((n, G)),
           g.standard_normal((n, G)) * 20 + 7,
           g.uniform(100.0, 100.05, (n, G)),           # tiny range far from 0
           -np.abs(g.standard_normal((n, G))) * 1e-3,  # all negative, small
           g.standard_normal((n, G)) * 1e-6,           # subnormal-range scales
           np.where(g.random((n, G)) < 0.05, 60.0, g.standard_normal((n, G)))]  # spikes
    return np.concatenate(out).astype(np.float32)


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("G", [32, 128])
def test_quantizer_error_bound(bits, G):
    # |x - (q*s + z)| <= s * (1/2 + 2^-17): the rounding of q is at most half a
    # step, plus three fp32 roundings of a quotient of at most 2^bits - 1.
    g = np.random.default_rng(bits * 1000 + G)
    x = _groups(g, 40, G)
    codes, sz = oracle.quantize_tokens(x, 0, G, bits)
    xh = oracle.dequant_tokens(codes, sz, G, bits)
    s = sz[..., 0].view(np.float16).astype(np.float64)        # [n, 1]
    err = np.abs(xh - x.astype(np.float64))
    assert np.all(err <= s * (0.5 + 2.0 ** -17) + 1e-300)
    # z <= min and z + L*s >= max (the grid covers the group)
    z = sz[..., 1].view(np.float16).astype(np.float64)[:, 0]
    L = 2 ** bits - 1
    assert np.all(z <= x.min(1))
    assert np.all(z + L * s[:, 0] >= x.max(1) * (1 - 2.0 ** -22) - 1e-30)


@pytest.mark.parametrize("bits", [2, 4])
def test_quantizer_integer_group_is_exact(bits):
    L = 2 ** bits - 1
    g = np.random.default_rng(5)
    x = g.integers(0, L + 1, 64).astype(np.float32)
    x[0], x[1] = 0, L
    s, z, q = oracle.quantize_group(x, bits)
    assert np.float16(np.uint16(s).view(np.float16)) == 1.0
    assert z == 0
    assert np.array_equal(q, x.astype(np.uint8))


def test_quantizer_constant_group():
    # A constant group whose value is an fp16 number has zero range: s = 0,
    # every code 0 and x_hat = z = x exactly. Otherwise z lies below the
    # value, s > 0, and every element gets the same code.
    for val in (3.25, -7.5, 0.0, 1e-3, -123.456):
        x = np.full(32, val, np.float32)
        s, z, q = oracle.quantize_group(x, 4)
        zf = float(np.uint16(z).view(np.float16))
        sf = float(np.uint16(s).view(np.float16))
        assert zf <= np.float32(val)
        assert np.all(q == q[0])
        if float(np.float16(val)) == float(np.float32(val)):
            assert s == 0 and np.all(q == 0) and zf == float(np.float32(val))
        else:
            assert sf > 0 and abs(q[0] * sf + zf - float(np.float32(val))) <= sf / 2


def test_quantizer_grid_values_reconstruct():
    # Values that lie on an fp16 grid z + k*s with z = min and s exact are
    # reproduced exactly.
    z0, s0 = np.float32(-1.5), np.float32(0.25)
    k = np.array([0, 15, 3, 7, 11, 15, 0, 1], np.float32)
    x = z0 + k * s0
    s, z, q = oracle.quantize_group(x, 4)
    assert float(np.uint16(s).view(np.float16)) == 0.25
    assert float(np.uint16(z).view(np.float16)) == -1.5
    assert np.array_equal(q, k.astype(np.uint8))


def test_packing_layout():
    q4 = np.array([1, 2, 3, 4, 15, 0, 9, 10], np.uint8)
    assert list(oracle.pack_codes(q4, 4)) == [0x21, 0x43, 0x0F, 0xA9]
    q2 = np.array([0, 1, 2, 3, 3, 2, 1, 0], np.uint8)
    assert list(oracle.pack_codes(q2, 2)) == [0b11100100, 0b00011011]
    for bits in (2, 4):
        g = np.random.default_rng(bits)
        q = g.integers(0, 2 ** bits, 128).astype(np.uint8)
        assert np.array_equal(oracle.unpack_codes(oracle.pack_codes(q, bits), 128, bits), q)


def test_token_quantization_uses_rotated_groups():
    # Quantizing with rotation equals rotating (fp32 recipe) and quantizing.
    g = np.random.default_rng(8)
    x = g.standard_normal((9, 128)).astype(np.float32)
    x[:, [3, 50, 77, 120]] *= 20
    c1, s1 = oracle.quantize_tokens(x, 128, 32, 4)
    c2, s2 = oracle.quantize_tokens(oracle.rotate_f32(x, 128), 0, 32, 4)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)
    # each group's scale/zero is that of the group on its own
    for v in range(9):
        xr = oracle.rotate_f32(x[v], 128)
        for gi in range(4):
            s, z, q = oracle.quantize_group(xr[gi * 32:(gi + 1) * 32], 4)
            assert (s, z) == tuple(s1[v, gi])
            assert np.array_equal(oracle.pack_codes(q, 4), c1[v, gi * 16:(gi + 1) * 16])


def test_rotation_reduces_outlier_error():
    # SAW-INT4 Abstract: the rotation recovers accuracy lost by naive INT4 on
    # keys with outlier channels; compare q.k errors with and without it.
    g = np.random.default_rng(21)
    k = g.standard_normal((512, 128)).astype(np.float32)
    k[:, [5, 40, 90, 127]] *= 20
    q = g.standard_normal((512, 128))
    exact = np.einsum("nd,nd->n", q, k)
    c0, s0 = oracle.quantize_tokens(k, 0, 128, 4)
    e0 = np.einsum("nd,nd->n", q, oracle.dequant_tokens(c0, s0, 128, 4)) - exact
    c1, s1 = oracle.quantize_tokens(k, 128, 128, 4)
    e1 = np.einsum("nd,nd->n", oracle.rotate_f64(q, 128), oracle.dequant_tokens(c1, s1, 128, 4)) - exact
    assert np.sqrt(np.mean(e1 ** 2)) < 0.5 * np.sqrt(np.mean(e0 ** 2))


def test_channel_block_groups_are_columns():
    g = np.random.default_rng(9)
    x = g.standard_normal((128, 128)).astype(np.float32) * (1 + np.arange(128, dtype=np.float32))
    codes, sz = oracle.quantize_channel_block(x, 2)
    q = np.stack([oracle.unpack_codes(codes[t], 128, 2) for t in range(128)])
    for d in (0, 1, 63, 127):
        s, z, qc = oracle.quantize_group(np.ascontiguousarray(x[:, d]), 2)
        assert (s, z) == tuple(sz[d])
        assert np.array_equal(q[:, d], qc)
    xh = oracle.dequant_channel_block(codes, sz, 2)
    s = sz[:, 0].view(np.float16).astype(np.float64)
    assert np.all(np.abs(xh - x) <= s[None, :] * (0.5 + 2.0 ** -17))


# ---------------------------------------------------------------------------
# Attention: brute force and closed forms
# ---------------------------------------------------------------------------

def test_attention_brute_force_tiny():
    g = np.random.default_rng(4)
    for T in (1, 2, 5, 8):
        q = g.standard_normal((3, 16))
        k = g.standard_normal((T, 16))
        v = g.standard_normal((T, 16))
        scale = 1 / np.sqrt(16)
        want = scipy.special.softmax(q @ k.T * scale, axis=1) @ v
        assert np.allclose(oracle.attention(q, k, v, scale), want, rtol=1e-13, atol=1e-13)


def test_attention_closed_forms():
    g = np.random.default_rng(6)
    v = g.standard_normal((6, 8))
    q = g.standard_normal((2, 8))
    k = np.tile(g.standard_normal(8), (6, 1))       # equal keys -> mean of V
    assert np.allclose(oracle.attention(q, k, v, 0.3), np.tile(v.mean(0), (2, 1)), atol=1e-14)
    k2 = np.zeros((6, 8))
    k2[4] = 1000 * q[0] / np.linalg.norm(q[0])      # one dominant logit
    out = oracle.attention(q[:1], k2, v, 1.0)
    assert np.allclose(out[0], v[4], atol=1e-12)


def test_gqa_head_mapping_and_query_rotation():
    g = np.random.default_rng(7)
    H_kv, g_sz, T, D = 2, 3, 5, 128
    q = g.standard_normal((H_kv * g_sz, D))
    k = g.standard_normal((H_kv, T, D))
    v = g.standard_normal((H_kv, T, D))
    out = oracle.decode_attention_gqa(q, k, v, 0.1)
    for h in range(H_kv * g_sz):
        want = scipy.special.softmax(k[h // g_sz] @ q[h] * 0.1) @ v[h // g_sz]
        assert np.allclose(out[h], want, atol=1e-13)
    # rotated keys with rotated queries give the unrotated result
    kr = oracle.rotate_f64(k, 128)
    out_r = oracle.decode_attention_gqa(q, kr, v, 0.1, rotate_q_block=128)
    assert np.allclose(out_r, out, atol=1e-12)


# ---------------------------------------------------------------------------
# KIVI window split and byte accounting (Dual-QK Tables 1 and 9)
# ---------------------------------------------------------------------------

def test_kivi_split():
    assert oracle.kivi_split(131072, 128) == 130944
    assert [oracle.kivi_split(t, 4) for t in range(10)] == [0, 0, 0, 0, 0, 4, 4, 4, 4, 8]


def test_kivi_sequence_window_holds_recent_tokens():
    g = np.random.default_rng(10)
    T, D = 300, 128
    k = g.standard_normal((T, D)).astype(np.float32)
    v = g.standard_normal((T, D)).astype(np.float32)
    c = oracle.quantize_kivi_sequence(k, v, 128, 2, 2, 32)
    assert c["Tq"] == 256
    kh, vh = oracle.dequant_kivi_sequence(c, 128, 2, 2, 32)
    assert np.array_equal(kh[256:], k[256:]) and np.array_equal(vh[256:], v[256:])
    cb, sb = oracle.quantize_channel_block(k[128:256], 2)
    assert np.array_equal(c["k_codes"][128:256], cb) and np.array_equal(c["k_sz"][1], sb)


def test_kivi_values_grouped_along_tokens():
    # InnerQ (Abstract): V grouped along the inner dimension of p @ V, the
    # tokens -- one group per (channel, R-token block)
    g = np.random.default_rng(13)
    T, D, R = 300, 128, 64
    k = g.standard_normal((T, D)).astype(np.float32)
    v = (g.standard_normal((T, D)) * (1 + np.arange(D) / 16)).astype(np.float32)
    c = oracle.quantize_kivi_sequence(k, v, R, 4, 4, 0, v_per_channel=True)
    Tq = c["Tq"]
    assert Tq == 256 and c["v_sz"].shape == (Tq // R, D, 2)
    # same data on both sides: values quantize exactly like the per-channel keys
    ck = oracle.quantize_kivi_sequence(v, v, R, 4, 4, 0, v_per_channel=True)
    assert np.array_equal(ck["v_codes"], ck["k_codes"]) and np.array_equal(ck["v_sz"], ck["k_sz"])
    # a group is one channel's R tokens of one block
    q = np.stack([oracle.unpack_codes(c["v_codes"][t], D, 4) for t in range(Tq)])
    for b, d in ((0, 0), (1, 77), (3, 127)):
        s, z, qc = oracle.quantize_group(np.ascontiguousarray(v[b * R:(b + 1) * R, d]), 4)
        assert (s, z) == tuple(c["v_sz"][b, d])
        assert np.array_equal(q[b * R:(b + 1) * R, d], qc)
    kh, vh = oracle.dequant_kivi_sequence(c, R, 4, 4, 0, v_per_channel=True)
    assert np.array_equal(vh[Tq:], v[Tq:])
    s = c["v_sz"][:, :, 0].view(np.float16).astype(np.float64)  # [nb][D]
    assert np.all(np.abs(vh[:Tq] - v[:Tq]).reshape(Tq // R, R, D) <= s[:, None, :] * (0.5 + 2.0 ** -17))
    # the scale and zero of a channel factor out of a block's weighted sum:
    # sum_t p_t vhat_t = s * sum_t p_t q_t + z * sum_t p_t
    pw = g.random(Tq)
    z = c["v_sz"][:, :, 1].view(np.float16).astype(np.float64)
    for b in range(Tq // R):
        sl = slice(b * R, (b + 1) * R)
        want = pw[sl] @ vh[sl]
        got = s[b] * (pw[sl] @ q[sl]) + z[b] * pw[sl].sum()
        assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_effective_bits_match_printed_table():
    with open(os.path.join(GOLDEN, "effective_bits.txt")) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    for table, method, cap, bw, T, sparsity, bits, group, res in rows:
        T, bits, group, res = int(T), int(bits), int(group), int(res)
        sparsity = float(sparsity)
        if bits == 16:
            per = 16.0
        else:
            per = oracle.effective_bits(bits, group, T, residual=res)
        capacity = per                          # K and V stored alike
        bandwidth = ((1 - sparsity) * per + per) / 2
        assert round(capacity, 2) == float(cap), (table, method)
        assert round(bandwidth, 2) == float(bw), (table, method)


def test_packed_bytes_per_token_head():
    assert oracle.packed_bytes_per_token_head(4, 128) == 68
    assert oracle.packed_bytes_per_token_head(4, 32) == 80
    assert oracle.packed_bytes_per_token_head(2, 32) == 48


# ---------------------------------------------------------------------------
# Rematerialization: GEMM (numpy), identity weights, RoPE closed forms
# ---------------------------------------------------------------------------

def test_matmul_matches_numpy():
    g = np.random.default_rng(12)
    a = g.standard_normal((17, 64)).astype(np.float32)
    w = g.standard_normal((24, 64)).astype(np.float32)
    assert np.allclose(oracle.matmul_nt(a, w), a.astype(np.float64) @ w.astype(np.float64).T, rtol=1e-13, atol=1e-12)


def test_rope_closed_forms():
    g = np.random.default_rng(13)
    x = g.standard_normal((6, 2, 128))
    pos = np.array([0, 1, 7, 100, 16383, 5])
    y = oracle.rope(x, pos, 500000.0)
    assert np.array_equal(y[0], x[0])                               # position 0
    n_in = x[..., :64] ** 2 + x[..., 64:] ** 2
    n_out = y[..., :64] ** 2 + y[..., 64:] ** 2
    assert np.allclose(n_in, n_out, rtol=1e-12)                     # pairwise norm
    # complex form: (x_i + j x_{i+64}) * exp(j * p * theta^(-2i/128))
    inv = 500000.0 ** (-np.arange(64) / 64.0)
    zc = (x[..., :64] + 1j * x[..., 64:]) * np.exp(1j * pos[:, None, None] * inv)
    assert np.allclose(y[..., :64], zc.real, atol=1e-9) and np.allclose(y[..., 64:], zc.imag, atol=1e-9)


def test_remat_identity_weights_give_rope_of_x():
    g = np.random.default_rng(14)
    hidden, H, D, M = 256, 1, 128, 9
    x = g.standard_normal((M, hidden)).astype(np.float32)
    codes, sz = oracle.quantize_tokens(x, 0, 128, 4)
    w = np.zeros((2 * H * D, hidden), np.float32)
    w[:D, :D] = np.eye(D)               # K = first 128 channels of x_hat
    w[D:, D:2 * D] = np.eye(D)          # V = next 128 channels
    pos = np.arange(M) * 3
    k, v = oracle.remat_kv(codes, sz, 128, 4, w, H, D, pos, 500000.0)
    xh = oracle.dequant_x_bf16(codes, sz, 128, 4).astype(np.float64)
    assert np.array_equal(v[:, 0], xh[:, D:2 * D])
    assert np.allclose(k, oracle.rope(xh[:, None, :D], pos, 500000.0), atol=0)


def test_dequant_x_is_bf16_near_exact_value():
    g = np.random.default_rng(15)
    x = g.standard_normal((5, 256)).astype(np.float32)
    codes, sz = oracle.quantize_tokens(x, 0, 128, 4)
    xh = oracle.dequant_x_bf16(codes, sz, 128, 4)
    exact = oracle.dequant_tokens(codes, sz, 128, 4)
    # bf16 values (low 16 bits zero) within half a bf16 ulp (2^-8 relative) of q*s+z
    assert np.all((xh.view(np.uint32) & 0xFFFF) == 0)
    assert np.all(np.abs(xh - exact) <= np.abs(exact) * 2.0 ** -8 * (1 + 2.0 ** -15) + 1e-30)


def test_quantizer_permutation_invariance_with_signed_zeros():
    # Scale and zero depend on the group's values only, not on their order;
    # with both signed zeros present at the minimum this needs the zero
    # extreme taken as +0.
    g = np.random.default_rng(16)
    for trial in range(50):
        x = np.abs(g.standard_normal(32)).astype(np.float32)
        x[g.choice(32, 6, replace=False)] = np.where(g.random(6) < 0.5, -0.0, 0.0).astype(np.float32)
        perm = g.permutation(32)
        s1, z1, q1 = oracle.quantize_group(x, 4)
        s2, z2, q2 = oracle.quantize_group(x[perm], 4)
        assert (s1, z1) == (s2, z2)
        assert np.array_equal(q1[perm], q2)


# ---------------------------------------------------------------------------
# Randomized Hadamard (QuaRot): signs first, then the block transform
# ---------------------------------------------------------------------------

RH_D = 128  # head dimension

def test_randomized_hadamard_golden_worked_example():
    with open(os.path.join(GOLDEN, "randomized_hadamard_h4.txt")) as f:
        lines = [l for l in f if l.strip() and not l.startswith("#")]
    assert len(lines) == 2
    for line in lines:
        s, x, y = (np.array([float(t) for t in part.split()]) for part in line.split(";"))
        got = oracle.rotate_f64(oracle.apply_signs(x, s), 4)
        assert np.array_equal(got, y), (got, y)
        got32 = oracle.rotate_f32(oracle.apply_signs(x.astype(np.float32), s), 4)
        assert np.array_equal(got32.astype(np.float64), y)


def test_randomized_hadamard_is_orthogonal_and_keeps_dot_products():
    import workloads as W
    s = W.hadamard_signs(11)
    assert set(np.unique(s)) == {-1.0, 1.0}
    for hb in (32, 64, 128):
        # columns of M = H_blk diag(s) / sqrt(blk), block-diagonal over 128
        M = oracle.rotate_f64(oracle.apply_signs(np.eye(RH_D), s), hb).T
        assert np.allclose(M @ M.T, np.eye(RH_D), atol=1e-12)
        rng = np.random.default_rng(hb)
        q, k = rng.standard_normal(RH_D), rng.standard_normal(RH_D)
        qr = oracle.rotate_f64(oracle.apply_signs(q, s), hb)
        kr = oracle.rotate_f64(oracle.apply_signs(k, s), hb)
        assert abs(qr @ kr - q @ k) <= 1e-12 * (abs(q) @ abs(k))


def test_all_plus_signs_quantize_like_the_plain_rotation():
    import workloads as W
    x = W.finish(W.normal(np.random.default_rng(5), (16, RH_D)), "bf16")
    ones = np.ones(RH_D, np.float32)
    for bits, G in ((4, 128), (2, 32)):
        a = oracle.quantize_tokens(x, 128, G, bits)
        b = oracle.quantize_tokens(x, 128, G, bits, signs=ones)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    s = W.hadamard_signs(3)
    c = oracle.quantize_tokens(x, 128, 128, 4, signs=s)
    assert not np.array_equal(c[0], oracle.quantize_tokens(x, 128, 128, 4)[0])


# ---------------------------------------------------------------------------
# Attention-sink window (InnerQ): sink tokens kept in bf16, the rest quantized
# ---------------------------------------------------------------------------

def test_sink_attention_equals_attention_over_the_concatenated_tokens():
    import workloads as W
    g = np.random.default_rng(41)
    H_kv, H_q, n_sink, T = 2, 8, 4, 37
    q = g.standard_normal((H_q, RH_D))
    ks, vs = g.standard_normal((H_kv, n_sink, RH_D)), g.standard_normal((H_kv, n_sink, RH_D))
    kq, vq = g.standard_normal((H_kv, T - n_sink, RH_D)), g.standard_normal((H_kv, T - n_sink, RH_D))
    scale = 1.0 / np.sqrt(RH_D)
    # no rotation: one textbook softmax over sinks followed by the others
    want = oracle.decode_attention_gqa(q, np.concatenate([ks, kq], 1), np.concatenate([vs, vq], 1), scale)
    got = oracle.decode_attention_gqa_sinks(q, kq, vq, ks, vs, scale)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-14)
    # rotated keys: the rotated query against rotated keys equals the plain
    # query against the keys rotated back (H diag(s) / sqrt(n) is orthogonal)
    s = W.hadamard_signs(2)
    kr = oracle.rotate_f64(oracle.apply_signs(kq, s), 128)
    got = oracle.decode_attention_gqa_sinks(q, kr, vq, ks, vs, scale, rotate_q_block=128, signs=s)
    assert np.allclose(got, want, rtol=1e-10, atol=1e-12)
    # a dominant sink logit returns that sink's value row
    q2 = np.zeros((H_q, RH_D))
    q2[:, 0] = 1.0
    ks2 = ks.copy()
    ks2[:, 1, 0] = 1e4
    got = oracle.decode_attention_gqa_sinks(q2, kq, vq, ks2, vs, 1.0)
    assert np.allclose(got[0], vs[0, 1]) and np.allclose(got[-1], vs[1, 1])


# ---------------------------------------------------------------------------
# Hybrid symmetric/asymmetric choice per group (InnerQ Abstract, "(i)")
# ---------------------------------------------------------------------------

def test_quantizer_rounding_golden():
    # Hand-derived groups that fix each rounding step of the recipe: ties to
    # even, multiplication by fp32(1/s) rather than division, z rounded down,
    # s rounded up (a slip at any step changes the stored bits or codes).
    with open(os.path.join(GOLDEN, "quantizer_rounding.txt")) as f:
        lines = [l for l in f if l.strip() and not l.startswith("#")]
    assert len(lines) == 5
    for line in lines:
        bits, xh, sz, q, _slip = (part.split() for part in line.split(";"))
        x = np.array([int(t, 16) for t in xh], np.uint32).view(np.float32)
        s, z, codes = oracle.quantize_group(x, int(bits[0]))
        assert (s, z) == (int(sz[0], 16), int(sz[1], 16)), line
        assert codes.tolist() == [int(t) for t in q], line


def test_hybrid_golden_worked_examples():
    with open(os.path.join(GOLDEN, "hybrid_sym_asym.txt")) as f:
        lines = [l for l in f if l.strip() and not l.startswith("#")]
    assert len(lines) == 5
    for line in lines:
        bits, x, sz, q = (part.split() for part in line.split(";"))
        s, z, codes = oracle.quantize_group_hybrid(np.array([float(t) for t in x], np.float32), int(bits[0]))
        assert (s, z) == (int(sz[0], 16), int(sz[1], 16)), line
        assert codes.tolist() == [int(t) for t in q], line


def _sym_candidate(x, bits):
    # the symmetric grid written out independently: s = fp16_ru(max|x| / Qp),
    # z = -C s, q = clamp(rint(x / s), -Qp, Qp) + C
    C = 1 << (bits - 1)
    Qp = C - 1
    m = np.float32(max(abs(float(x.min())), abs(float(x.max()))))
    s_bits = int(oracle.f32_to_f16_bits(np.array([m / np.float32(Qp)], np.float32), oracle.ROUND_UP)[0])
    s = float(oracle.f16_bits_to_f64(np.array([s_bits], np.uint16))[0])
    if s == 0.0:
        return s_bits, None, np.full(x.size, C, np.uint8)
    r = np.float32(1.0) / np.float32(s)
    q = np.clip(np.rint(x.astype(np.float32) * r), -Qp, Qp) + C
    z_bits = int(oracle.f32_to_f16_bits(np.array([-C * s], np.float32))[0])
    return s_bits, z_bits, q.astype(np.uint8)


def _max_err(x, s_bits, z_bits, q):
    s, z = oracle.f16_bits_to_f64(np.array([s_bits, z_bits], np.uint16))
    return float(np.max(np.abs(x.astype(np.float64) - (q * s + z))))


def test_hybrid_takes_one_candidate_and_the_better_one():
    g = np.random.default_rng(31)
    picked_sym = 0
    for trial in range(600):
        n = (16, 32, 64, 128)[trial % 4]
        bits = (2, 4)[(trial // 4) % 2]
        if trial % 3 == 0:
            x = g.standard_normal(n)
        elif trial % 3 == 1:
            x = g.standard_t(2, n)
        else:  # sparse values on a coarse grid: the symmetric grid's exact zero level pays
            x = np.round(g.standard_normal(n) * 3) / 3 * (g.random(n) < 0.5)
        x = x.astype(np.float32)
        s, z, q = oracle.quantize_group_hybrid(x, bits)
        sa, za, qa = oracle.quantize_group(x, bits)
        ss, zs, qs = _sym_candidate(x, bits)
        if (s, z) == (sa, za) and np.array_equal(q, qa):
            if zs is not None:  # kept the asymmetric one: not worse (float64, fp32 decision slack)
                assert _max_err(x, sa, za, qa) <= _max_err(x, ss, zs, qs) * (1 + 1e-6) + 1e-12
        else:
            picked_sym += 1
            assert (s, z) == (ss, zs) and np.array_equal(q, qs)
            assert _max_err(x, ss, zs, qs) <= _max_err(x, sa, za, qa) * (1 + 1e-6) + 1e-12
            # the symmetric grid has an exact zero level
            sf, zf = oracle.f16_bits_to_f64(np.array([s, z], np.uint16))
            assert np.all((q * sf + zf)[x == 0] == 0)
    assert 20 < picked_sym < 580  # both candidates occur on these heavy-tailed groups


def test_hybrid_applies_per_group_in_token_and_channel_layouts():
    g = np.random.default_rng(32)
    x = g.standard_t(2, (3, 128)).astype(np.float32)
    for G, bits in ((16, 2), (32, 4), (128, 2)):
        codes, sz = oracle.quantize_tokens(x, 0, G, bits, hybrid=True)
        for v in range(3):
            q = oracle.unpack_codes(codes[v], 128, bits)
            for grp in range(128 // G):
                s, z, qg = oracle.quantize_group_hybrid(x[v, grp * G:(grp + 1) * G], bits)
                assert (s, z) == tuple(sz[v, grp]) and np.array_equal(q[grp * G:(grp + 1) * G], qg)
    blk = g.standard_t(2, (64, 128)).astype(np.float32)
    codes, sz = oracle.quantize_channel_block(blk, 2, hybrid=True)
    q = np.stack([oracle.unpack_codes(codes[t], 128, 2) for t in range(64)])
    for d in (0, 5, 127):
        s, z, qg = oracle.quantize_group_hybrid(np.ascontiguousarray(blk[:, d]), 2)
        assert (s, z) == tuple(sz[d]) and np.array_equal(q[:, d], qg)


# ---------------------------------------------------------------------------
# Partials of disjoint token ranges (the sharded decode's merge)
# ---------------------------------------------------------------------------

def test_partials_of_any_token_split_merge_to_attention():
    g = np.random.default_rng(41)
    q = g.standard_normal((4, 16))
    k = g.standard_normal((37, 16)) * 3
    v = g.standard_normal((37, 16))
    want = scipy.special.softmax(q @ k.T * 0.25, axis=1) @ v
    for cuts in ([0, 37], [0, 1, 37], [0, 10, 10, 37], [0, 5, 20, 36, 37]):
        parts = [oracle.attention_partial(q, k[a:b], v[a:b], 0.25) for a, b in zip(cuts[:-1], cuts[1:])]
        assert np.allclose(oracle.merge_partials(parts), want, atol=1e-13)
    # one range: o / l is the attention, and m is the largest log2-unit score
    o, m, l = oracle.attention_partial(q, k, v, 0.25)
    assert np.allclose(o / l[:, None], want, atol=1e-13)
    assert np.allclose(m, (q @ k.T).max(axis=1) * 0.25 / np.log(2), atol=1e-12)
    # every range empty -> zeros
    e = oracle.attention_partial(q, k[:0], v[:0], 0.25)
    assert np.array_equal(oracle.merge_partials([e, e]), np.zeros((4, 16)))
