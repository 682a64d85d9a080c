"""CPU oracle for the low-bit KV-cache hot path (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package. It shares no code with the CUDA library: the
arithmetic lives in ``oracle.c`` (plain C, float64 accumulation, the fp32
quantizer recipe reproduced operation by operation) and this module only
marshals numpy arrays into it and composes its steps in the order the method
states them.

Sources, by page title and section:
  * "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM
    Serving", Abstract -- token-wise INT4 quantization after a block-diagonal
    Hadamard rotation; fused attention over the quantized paged cache.
  * "InnerQ: Hardware-Aware Tuning-Free Quantization of KV Cache for Large
    Language Models", Abstract -- group-wise quantization; a high-precision
    window of recent tokens.
  * "XQuant: Breaking the Memory Wall for LLM Inference with KV Cache
    Rematerialization", Abstract -- cache quantized X, recompute K and V.
  * "Dual-QK: Sharp Queries and Flat Keys for Prunable 2-bit KV Caches",
    Abstract (queries take the keys' orthogonal transform) and Tables 1 and 9
    (effective bits per KV element at a 128K context).
  * KIVI (listed among the references of the SAW-INT4 and InnerQ pages) --
    keys quantized per channel over blocks of tokens, values per token, with a
    full-precision residual of the most recent tokens.

Parity status: every function here is pinned by a test in
``tests/test_oracle_*.py`` except where noted "parity unpinned".
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

ROUND_NEAREST, ROUND_DOWN, ROUND_UP = 0, 1, 2

_lib = None


def lib():
    """Load (building first if needed) liboracle.so."""
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = ctypes.CDLL(path)
        _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_I = ctypes.c_int
_L = ctypes.c_int64
_D = ctypes.c_double


def _declare(l):
    sig = {
        "oracle_f32_to_f16": (ctypes.c_uint16, [ctypes.c_float, _I]),
        "oracle_f32_to_f16_array": (None, [_P, _L, _I, _P]),
        "oracle_f16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
        "oracle_f32_to_bf16_rn": (ctypes.c_uint16, [ctypes.c_float]),
        "oracle_f32_to_bf16_rn_array": (None, [_P, _L, _P]),
        "oracle_bf16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
        "oracle_fwht_f32": (None, [_P, _I]),
        "oracle_rotate_blocks_f32": (None, [_P, _L, _I, _I]),
        "oracle_fwht_f64": (None, [_P, _I]),
        "oracle_rotate_blocks_f64": (None, [_P, _L, _I, _I]),
        "oracle_quantize_group": (None, [_P, _I, _I, _I, _P, _P, _P, _I]),
        "oracle_quantize_group_hybrid": (None, [_P, _I, _I, _I, _P, _P, _P, _I]),
        "oracle_pack_codes": (None, [_P, _I, _I, _P]),
        "oracle_unpack_codes": (None, [_P, _I, _I, _P]),
        "oracle_quantize_tokens": (None, [_P, _L, _I, _I, _I, _I, _I, _P, _P]),
        "oracle_quantize_channel_block": (None, [_P, _I, _I, _I, _I, _P, _P]),
        "oracle_dequant_tokens": (None, [_P, _P, _L, _I, _I, _I, _P]),
        "oracle_dequant_channel_block": (None, [_P, _P, _I, _I, _I, _P]),
        "oracle_attention": (None, [_P, _I, _P, _P, _L, _I, _D, _P]),
        "oracle_dequant_x_bf16": (None, [_P, _P, _L, _I, _I, _I, _P]),
        "oracle_matmul_nt": (None, [_P, _P, _L, _I, _I, _P]),
        "oracle_rope": (None, [_P, _P, _L, _I, _I, _D]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(l, name)
        fn.restype = res
        fn.argtypes = args


def _c(a, dtype):
    """Contiguous array of the given dtype (copy only if needed)."""
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# Number encodings
# --------------------------------------------------------------------------

def f32_to_f16_bits(v, mode=ROUND_NEAREST):
    """fp32 values -> fp16 bit patterns, rounding mode 0 nearest-even,
    1 toward -inf, 2 toward +inf."""
    a = _c(v, np.float32)
    out = np.empty(a.shape, dtype=np.uint16)
    lib().oracle_f32_to_f16_array(_ptr(a), a.size, mode, _ptr(out))
    return out


def f16_bits_to_f64(h):
    """fp16 bit patterns -> float64 values (exact)."""
    h = _c(h, np.uint16)
    out = np.empty(h.shape, np.float64)
    flat = out.reshape(-1)
    for i, x in enumerate(h.reshape(-1)):
        flat[i] = lib().oracle_f16_to_f32(int(x))
    return out


def f32_to_bf16_bits(v):
    a = _c(v, np.float32)
    out = np.empty(a.shape, dtype=np.uint16)
    lib().oracle_f32_to_bf16_rn_array(_ptr(a), a.size, _ptr(out))
    return out


# --------------------------------------------------------------------------
# Rotation (SAW-INT4 Abstract: block-diagonal Hadamard; Dual-QK Abstract:
# the same orthogonal transform on queries)
# --------------------------------------------------------------------------

def rotate_f32(x, hb):
    """Block-diagonal normalized Hadamard rotation of the last axis in the
    fp32 recipe (ascending butterfly stages, then one multiply by
    fp32(1/sqrt(hb))). Returns a new float32 array."""
    a = _c(x, np.float32).copy()
    D = a.shape[-1]
    lib().oracle_rotate_blocks_f32(_ptr(a), a.size // D, D, hb)
    return a


def rotate_f64(x, hb):
    """The same rotation carried out in float64."""
    a = _c(x, np.float64).copy()
    D = a.shape[-1]
    lib().oracle_rotate_blocks_f64(_ptr(a), a.size // D, D, hb)
    return a


# --------------------------------------------------------------------------
# Quantization
# --------------------------------------------------------------------------

def quantize_group(x, bits):
    """One asymmetric min/max group: returns (s_bits, z_bits, codes)."""
    a = _c(x, np.float32)
    s = np.zeros(1, np.uint16)
    z = np.zeros(1, np.uint16)
    q = np.zeros(a.size, np.uint8)
    lib().oracle_quantize_group(_ptr(a), a.size, 1, bits, _ptr(s), _ptr(z),
                                _ptr(q), 1)
    return int(s[0]), int(z[0]), q


def quantize_group_hybrid(x, bits):
    """One group with InnerQ's hybrid choice (Abstract, "(i) hybrid
    quantization"): the asymmetric min/max candidate or a symmetric one with
    an exact zero level, whichever reconstructs the group with the smaller
    largest absolute error, ties to the asymmetric one (the criterion is this
    library's reading; oracle.c states it). Returns (s_bits, z_bits, codes)."""
    a = _c(x, np.float32)
    s = np.zeros(1, np.uint16)
    z = np.zeros(1, np.uint16)
    q = np.zeros(a.size, np.uint8)
    lib().oracle_quantize_group_hybrid(_ptr(a), a.size, 1, bits, _ptr(s), _ptr(z),
                                       _ptr(q), 1)
    return int(s[0]), int(z[0]), q


def pack_codes(q, bits):
    q = _c(q, np.uint8)
    out = np.zeros(q.size * bits // 8, np.uint8)
    lib().oracle_pack_codes(_ptr(q), q.size, bits, _ptr(out))
    return out


def unpack_codes(packed, n, bits):
    p = _c(packed, np.uint8)
    out = np.zeros(n, np.uint8)
    lib().oracle_unpack_codes(_ptr(p), n, bits, _ptr(out))
    return out


def apply_signs(x, signs):
    """diag(signs) x along the last axis: the random sign flip that QuaRot
    puts before the Hadamard ("QuaRot: Outlier-Free 4-Bit Inference in Rotated
    LLMs", randomized Hadamard). With signs of +-1 the product is exact in any
    precision. Returns x itself when signs is None."""
    if signs is None:
        return x
    x = np.asarray(x)
    return x * np.asarray(signs, x.dtype)


def quantize_tokens(x, hb, G, bits, signs=None, hybrid=False):
    """Token-wise group quantization (SAW-INT4 Abstract "token-wise INT4";
    InnerQ Abstract groups along the inner dimension of q.k).

    x: float32 [..., D] (bf16 or fp32 values). Each vector is multiplied by
    the random signs (if given), rotated (hb > 0) and split into D/G groups of
    G consecutive elements. hybrid: each group takes the symmetric or the
    asymmetric candidate (quantize_group_hybrid).
    Returns codes uint8 [..., D*bits/8] and sz uint16 [..., D/G, 2] holding
    the fp16 bit patterns (scale, zero)."""
    a = _c(apply_signs(_c(x, np.float32), signs), np.float32)
    D = a.shape[-1]
    n = a.size // D
    codes = np.zeros(a.shape[:-1] + (D * bits // 8,), np.uint8)
    sz = np.zeros(a.shape[:-1] + (D // G, 2), np.uint16)
    lib().oracle_quantize_tokens(_ptr(a), n, D, hb, G, bits, int(hybrid), _ptr(codes), _ptr(sz))
    return codes, sz


def quantize_channel_block(x, bits, hybrid=False):
    """Channel-wise quantization of one block of R tokens (KIVI keys): each
    channel's R values are one group. x: float32 [R][D].
    Returns codes uint8 [R][D*bits/8] and sz uint16 [D][2]."""
    a = _c(x, np.float32)
    R, D = a.shape
    codes = np.zeros((R, D * bits // 8), np.uint8)
    sz = np.zeros((D, 2), np.uint16)
    lib().oracle_quantize_channel_block(_ptr(a), R, D, bits, int(hybrid), _ptr(codes), _ptr(sz))
    return codes, sz


def dequant_tokens(codes, sz, G, bits):
    """x_hat = q*s + z in float64 for token-wise groups."""
    c = _c(codes, np.uint8)
    s = _c(sz, np.uint16)
    D = c.shape[-1] * 8 // bits
    n = c.size // c.shape[-1]
    out = np.zeros(c.shape[:-1] + (D,), np.float64)
    lib().oracle_dequant_tokens(_ptr(c), _ptr(s), n, D, G, bits, _ptr(out))
    return out


def dequant_channel_block(codes, sz, bits):
    c = _c(codes, np.uint8)
    s = _c(sz, np.uint16)
    R = c.shape[0]
    D = c.shape[1] * 8 // bits
    out = np.zeros((R, D), np.float64)
    lib().oracle_dequant_channel_block(_ptr(c), _ptr(s), R, D, bits, _ptr(out))
    return out


# --------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------

def attention(q, k, v, scale):
    """Exact softmax attention in float64 for n_q query rows over T keys:
    q [n_q][D], k [T][D], v [T][D] -> [n_q][D]."""
    qa = _c(q, np.float64)
    ka = _c(k, np.float64)
    va = _c(v, np.float64)
    n_q, D = qa.shape
    T = ka.shape[0]
    out = np.zeros((n_q, D), np.float64)
    lib().oracle_attention(_ptr(qa), n_q, _ptr(ka), _ptr(va), T, D, float(scale), _ptr(out))
    return out


def decode_attention_gqa(q, khat, vhat, scale, rotate_q_block=0, signs=None):
    """Decode attention of one sequence with grouped-query heads.

    q: [H_q][D] (bf16/fp32 values); khat, vhat: [H_kv][T][D] float64, the
    dequantized cache as attended. Query head h reads KV head
    h // (H_q // H_kv). When the cache keys were rotated with block size
    rotate_q_block, the query is rotated by the same transform first (Dual-QK
    Abstract), in float64, random signs included."""
    q = apply_signs(np.asarray(q, np.float64), signs)
    H_q, D = q.shape
    H_kv = khat.shape[0]
    g = H_q // H_kv
    qr = rotate_f64(q, rotate_q_block) if rotate_q_block else q
    out = np.zeros((H_q, D), np.float64)
    for h in range(H_kv):
        out[h * g:(h + 1) * g] = attention(qr[h * g:(h + 1) * g], khat[h], vhat[h], scale)
    return out


def decode_attention_gqa_sinks(q, khat, vhat, k_sink, v_sink, scale, rotate_q_block=0, signs=None):
    """Decode attention of one sequence whose first tokens are attention sinks
    kept in high precision (InnerQ Abstract: high-precision windows for
    recent tokens and attention-sink tokens).

    q: [H_q][D]; k_sink, v_sink: [H_kv][n_sink][D] float64, the sink tokens as
    kept (bf16 values, never rotated); khat, vhat: [H_kv][T - n_sink][D]
    float64, the dequantized later tokens, keys in the rotated domain. Sink
    scores take the query as given; the other scores take the query rotated
    like the keys (randomized with `signs`). One max-shifted softmax over all
    T tokens, in float64."""
    q = np.asarray(q, np.float64)
    H_q, D = q.shape
    H_kv = khat.shape[0]
    g = H_q // H_kv
    qr = rotate_f64(apply_signs(q, signs), rotate_q_block) if rotate_q_block else q
    out = np.zeros((H_q, D), np.float64)
    for h in range(H_q):
        kv = h // g
        s = np.concatenate([k_sink[kv] @ q[h], khat[kv] @ qr[h]]) * scale
        e = np.exp(s - s.max())
        vals = np.concatenate([v_sink[kv], vhat[kv]])
        out[h] = (e @ vals) / e.sum()
    return out


# --------------------------------------------------------------------------
# Cache composition for one sequence (the method's steps in order)
# --------------------------------------------------------------------------

def attention_partial(q, k, v, scale):
    """Unnormalized softmax attention of query rows q [n][D] over one range of
    tokens k, v [T][D], in float64 and log2 units: x_t = log2(e) * scale *
    q . k_t, m = max_t x_t, l = sum_t 2^(x_t - m), o = sum_t 2^(x_t - m) v_t.
    No tokens: m = -inf, l = 0, o = 0. Returns (o [n][D], m [n], l [n])."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    n, D = q.shape
    if k.shape[0] == 0:
        return np.zeros((n, D)), np.full(n, -np.inf), np.zeros(n)
    x = (q @ k.T) * (scale * np.log2(np.e))
    m = x.max(axis=1)
    p = np.exp2(x - m[:, None])
    return p @ v, m, p.sum(axis=1)


def merge_partials(parts):
    """Attention output from partials (o, m, l) of disjoint token ranges
    (attention_partial's form): sum_r 2^(m_r - M) o_r / sum_r 2^(m_r - M) l_r,
    M = max_r m_r; zeros where every range is empty."""
    M = np.max(np.stack([m for _, m, _ in parts]), axis=0)
    o = np.zeros_like(parts[0][0])
    l = np.zeros_like(parts[0][2])
    for o_r, m_r, l_r in parts:
        live = ~np.isneginf(m_r)  # an empty range weighs 0
        e = np.zeros_like(l_r)
        e[live] = np.exp2(m_r[live] - M[live])
        o = o + e[:, None] * o_r
        l = l + e * l_r
    with np.errstate(invalid="ignore", divide="ignore"):
        return np.where(l[:, None] > 0, o / np.where(l > 0, l, 1.0)[:, None], 0.0)


def kivi_split(T, R):
    """Number of quantized tokens when the most recent tokens stay in a
    full-precision window of capacity R that is flushed as one block only
    when a new token arrives and it is full: R * floor((T - 1) / R)."""
    if T <= 0:
        return 0
    return R * ((T - 1) // R)


def quantize_kivi_sequence(k, v, R, bits_k, bits_v, G_v, v_per_channel=False):
    """KIVI-style cache of one (sequence, KV head): k, v float32 [T][D].

    Keys in [0, Tq) are quantized per channel over aligned blocks of R tokens
    (KIVI Abstract). Values are quantized per token in groups of G_v, or, with
    v_per_channel, per channel over the same R-token blocks: InnerQ (Abstract)
    groups each cache matrix along the inner dimension of its product with the
    attention vector, and for p @ V that dimension is the tokens. Tokens in
    [Tq, T) stay as they are (the bf16 window). Returns dict with codes/sz and
    the window; v_sz is [Tq/R][D][2] when v_per_channel, else [Tq][D/G_v][2]."""
    T, D = k.shape
    Tq = kivi_split(T, R)
    nb = Tq // R

    def channel_blocks(x, bits):
        codes = np.zeros((Tq, D * bits // 8), np.uint8)
        sz = np.zeros((nb, D, 2), np.uint16)
        for b in range(nb):
            codes[b * R:(b + 1) * R], sz[b] = quantize_channel_block(x[b * R:(b + 1) * R], bits)
        return codes, sz

    kc, ksz = channel_blocks(k, bits_k)
    if v_per_channel:
        vc, vsz = channel_blocks(v, bits_v)
    else:
        vc, vsz = quantize_tokens(v[:Tq], 0, G_v, bits_v)
    return {"Tq": Tq, "k_codes": kc, "k_sz": ksz, "v_codes": vc, "v_sz": vsz,
            "k_win": np.asarray(k[Tq:], np.float64), "v_win": np.asarray(v[Tq:], np.float64)}


def dequant_kivi_sequence(c, R, bits_k, bits_v, G_v, v_per_channel=False):
    """Dequantized [T][D] float64 keys and values of quantize_kivi_sequence."""
    Tq = c["Tq"]
    nb = Tq // R
    D = c["k_win"].shape[1] if c["k_win"].size else c["k_codes"].shape[1] * 8 // bits_k
    kh = np.zeros((Tq, D))
    vh = np.zeros((Tq, D))
    for b in range(nb):
        kh[b * R:(b + 1) * R] = dequant_channel_block(c["k_codes"][b * R:(b + 1) * R], c["k_sz"][b], bits_k)
        if v_per_channel:
            vh[b * R:(b + 1) * R] = dequant_channel_block(c["v_codes"][b * R:(b + 1) * R], c["v_sz"][b], bits_v)
    if not v_per_channel and Tq:
        vh = dequant_tokens(c["v_codes"], c["v_sz"], G_v, bits_v)
    return np.concatenate([kh, c["k_win"]]), np.concatenate([vh, c["v_win"]])


# --------------------------------------------------------------------------
# Rematerialization (XQuant Abstract)
# --------------------------------------------------------------------------

def dequant_x_bf16(codes, sz, G, bits):
    """bf16 GEMM operand from token-wise quantized X: bf16_rn(fp32(q*s+z)),
    returned as float32 values. codes [M][hidden*bits/8], sz [M][hidden/G][2]."""
    c = _c(codes, np.uint8)
    s = _c(sz, np.uint16)
    M = c.shape[0]
    hidden = c.shape[1] * 8 // bits
    out = np.zeros((M, hidden), np.float32)
    lib().oracle_dequant_x_bf16(_ptr(c), _ptr(s), M, hidden, G, bits, _ptr(out))
    return out


def matmul_nt(a, w):
    """a [M][K] float32 times w [N][K] float32 transposed, in float64."""
    aa = _c(a, np.float32)
    ww = _c(w, np.float32)
    M, K = aa.shape
    N = ww.shape[0]
    out = np.zeros((M, N), np.float64)
    lib().oracle_matmul_nt(_ptr(aa), _ptr(ww), M, N, K, _ptr(out))
    return out


def rope(x, pos, theta):
    """Rotate-half RoPE of x [M][H][D] float64 at positions pos [M]."""
    a = _c(x, np.float64).copy()
    p = _c(pos, np.int64)
    M, H, D = a.shape
    lib().oracle_rope(_ptr(a), _ptr(p), M, H, D, float(theta))
    return a


def remat_kv(x_codes, x_sz, G, bits, w_kv, n_kv_heads, head_dim, pos, theta):
    """Rematerialized keys and values for the tokens of x_codes:
    [K V] = x_hat . w_kv^T (float64), RoPE on K. w_kv: [2*H*D][hidden] float32
    (K rows first, then V rows). Returns (k, v) float64 [M][H][D]."""
    xh = dequant_x_bf16(x_codes, x_sz, G, bits)
    kv = matmul_nt(xh, w_kv)
    M = kv.shape[0]
    HD = n_kv_heads * head_dim
    k = kv[:, :HD].reshape(M, n_kv_heads, head_dim)
    v = kv[:, HD:].reshape(M, n_kv_heads, head_dim)
    return rope(k, pos, theta), v


# --------------------------------------------------------------------------
# Byte accounting (Dual-QK Tables 1 and 9: effective bits per KV element)
# --------------------------------------------------------------------------

def effective_bits(bits, group, T, residual=0, sz_bits=32, residual_bits=16):
    """Average stored bits per cached element of one tensor (K or V) at
    context T: quantized tokens cost bits + sz_bits/group (an fp16 scale and
    an fp16 zero per group), the most recent `residual` tokens cost
    residual_bits."""
    r = min(residual, T)
    return ((T - r) * (bits + sz_bits / group) + r * residual_bits) / T


def packed_bytes_per_token_head(bits, group, head_dim=128):
    """Bytes of one quantized (token, head) vector: codes plus fp16 s and z
    per group."""
    return head_dim * bits // 8 + (head_dim // group) * 4


__all__ = [n for n in dir() if not n.startswith("_")]
