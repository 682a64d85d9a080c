// kvq_append.cu -- fused rotate + quantize + pack + append (sm_100a).
//
// SAW-INT4 ("SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for
// Real-World LLM Serving", Abstract): token-wise INT4 quantization after a
// block-diagonal Hadamard rotation, done by one fused kernel that writes
// straight into a paged KV layout. InnerQ (Abstract): groups along the inner
// dimension and a high-precision window of recent tokens. KIVI (listed in the
// references of both pages): keys per channel over blocks of tokens.
//
// Work mapping: four lanes own one (token, head) vector of 128 channels, 32
// consecutive channels each, so a warp handles 8 vectors. The rotation's
// butterfly stages of half-width 1..16 stay inside a lane, the stages 32 and
// 64 are one shuffle each; a group of 32 is one lane, a group of 128 is a
// two-level shuffle min/max. Each lane packs its 32 codes into one 16-byte
// (INT4) or 8-byte (INT2) store.
//
// Quantizer, bit-exact with the CPU oracle (every op is an IEEE-754
// single-rounding intrinsic, so nothing is contracted into an FMA):
//   z = fp16_rd(min), s = fp16_ru(fp32(fp32(max - z) / L)),
//   q = clamp(rint(fp32(fp32(x - z) * fp32(1/s))), 0, L), all q = 0 if s == 0.
#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

struct AppendTensor {
    uint8_t *codes;
    __half2 *sz;
    const void *src;   // [N][H][D]
    int bits;          // 2 or 4
    int group;         // 16, 32, 64 or 128
    int hb;            // rotation block, 0 = none
    float hscale;      // fp32(1/sqrt(hb))
    const float *signs;  // [128] +-1 applied before the rotation, or null
};

struct AppendParams {
    AppendTensor t[2];
    int H;
    const int32_t *cu_new;
    const int32_t *seq_lens;
    int num_seqs;
    int total_tokens;
    int paged, page_size, max_pages, num_pages, cap;
    const int32_t *block_table;
    int32_t *status;
    uint16_t *sink[2];  // bf16 [S][H][sink_len][D] for keys and values, or null
    int sink_len;
};

// ---- lane-level building blocks -------------------------------------------

// Load the 32 channels [32*part, 32*part + 32) of vector `vec` as fp32.
template <int DT>
__device__ __forceinline__ void load32(const void *src, int64_t vec, int part, float x[32]) {
    if constexpr (DT == KVQ_FP32) {
        const float4 *p = reinterpret_cast<const float4 *>(
            static_cast<const float *>(src) + vec * kHeadDim + part * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float4 f = __ldcs(p + i);
            x[4 * i] = f.x; x[4 * i + 1] = f.y; x[4 * i + 2] = f.z; x[4 * i + 3] = f.w;
        }
    } else {
        const uint4 *p = reinterpret_cast<const uint4 *>(
            static_cast<const uint16_t *>(src) + vec * kHeadDim + part * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint4 u = __ldcs(p + i);
            uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if constexpr (DT == KVQ_BF16) {
                    x[8 * i + 2 * j] = bf16_bits_to_float(w[j] & 0xFFFFu);
                    x[8 * i + 2 * j + 1] = bf16_bits_to_float(w[j] >> 16);
                } else {
                    x[8 * i + 2 * j] = __half2float(__ushort_as_half((unsigned short)(w[j] & 0xFFFFu)));
                    x[8 * i + 2 * j + 1] = __half2float(__ushort_as_half((unsigned short)(w[j] >> 16)));
                }
            }
        }
    }
}

// ---- packed f32x2 arithmetic: two independent round-to-nearest fp32 ops ----
__device__ __forceinline__ unsigned long long f2u(float a, float b) {
    return (static_cast<unsigned long long>(__float_as_uint(b)) << 32) | __float_as_uint(a);
}
__device__ __forceinline__ float lo_f(unsigned long long v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi_f(unsigned long long v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }
__device__ __forceinline__ unsigned long long add2(unsigned long long a, unsigned long long b) {
    unsigned long long r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ unsigned long long sub2(unsigned long long a, unsigned long long b) {
    unsigned long long r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b) {
    unsigned long long r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b,
                                                   unsigned long long c) {
    unsigned long long r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// Normalized Sylvester Walsh-Hadamard transform of each hb-block, the four
// lanes of a vector holding 32 channels each. Stage half-widths ascend
// 1, 2, ..., hb/2; butterfly (a, b) -> (a + b, a - b) with a the lower index;
// finally one multiply by c = fp32(1/sqrt(hb)). Stages of half-width >= 2 run
// on channel pairs (j, j+1) with packed f32x2 adds; the cross-lane stages
// compute o + s*x with s = +-1 in one packed fma, which rounds like the add
// or subtract it stands for.
__device__ __forceinline__ void fwht_lane(float x[32], int hb, int part, float c) {
    if (hb > 1) {
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
            const float a = x[j], b = x[j + 1];
            x[j] = __fadd_rn(a, b);
            x[j + 1] = __fsub_rn(a, b);
        }
    }
    unsigned long long v[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) v[k] = f2u(x[2 * k], x[2 * k + 1]);
#pragma unroll
    for (int h = 2; h < 32; h <<= 1) {  // pair index half-width h / 2
        if (h < hb) {
            const int hp = h / 2;
#pragma unroll
            for (int i = 0; i < 16; i += 2 * hp) {
#pragma unroll
                for (int k = i; k < i + hp; ++k) {
                    const unsigned long long a = v[k], b = v[k + hp];
                    v[k] = add2(a, b);
                    v[k + hp] = sub2(a, b);
                }
            }
        }
    }
#pragma unroll
    for (int m = 1; m <= 2; m <<= 1) {  // half-widths 32 and 64: partner lane part ^ m
        if (32 * m < hb) {
            const float sg = (part & m) ? -1.0f : 1.0f;  // upper: o - x, lower: x + o
            const unsigned long long sg2 = f2u(sg, sg);
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float o0 = __shfl_xor_sync(0xffffffffu, lo_f(v[k]), m);
                const float o1 = __shfl_xor_sync(0xffffffffu, hi_f(v[k]), m);
                v[k] = fma2(sg2, v[k], f2u(o0, o1));
            }
        }
    }
    const unsigned long long c2 = f2u(c, c);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        v[k] = mul2(v[k], c2);
        x[2 * k] = lo_f(v[k]);
        x[2 * k + 1] = hi_f(v[k]);
    }
}

struct QParams {
    __half2 sz;   // {scale, zero}
    float sf;     // scale as fp32
    float zf;     // zero as fp32
    float r;      // fp32(1/scale), 0 when scale == 0
};

__device__ __forceinline__ QParams qparams(float mn, float mx, int L) {
    mn = __fadd_rn(mn, 0.0f);  // a zero extreme counts as +0
    mx = __fadd_rn(mx, 0.0f);
    const __half z = __float2half_rd(mn);
    const float zf = __half2float(z);
    const float range = __fsub_rn(mx, zf);
    const float step = __fdiv_rn(range, static_cast<float>(L));
    const __half s = __float2half_ru(step);
    const float sf = __half2float(s);
    QParams p;
    p.sz = __halves2half2(s, z);
    p.sf = sf;
    p.zf = zf;
    p.r = (sf == 0.0f) ? 0.0f : __frcp_rn(sf);
    return p;
}

__device__ __forceinline__ uint32_t qcode(float x, const QParams &p, float Lf) {
    // r == 0 exactly when s == 0; then every code is 0.
    const float t = __fmul_rn(__fsub_rn(x, p.zf), p.r);
    const float q = fminf(fmaxf(rintf(t), 0.0f), Lf);
    return static_cast<uint32_t>(q);
}

// ---- hybrid symmetric/asymmetric choice (InnerQ, Abstract, "(i)") ---------
// The symmetric candidate: Qp = 2^(bits-1) - 1, C = 2^(bits-1),
// s = fp16_ru(fp32(max|x| / Qp)), z = -C s (exact in fp32; the candidate is
// dropped when |z| exceeds the largest fp16), q = clamp(rint(x / s), -Qp, Qp) + C
// with x / s taken as fp32(x * fp32(1/s)). It has an exact zero level. A group
// takes it when its largest reconstruction error is smaller than the
// asymmetric one's: |e| with fp32 e = x - fma(q, s, z), the maximum over the
// group (exact, so the lanes may visit the elements in any order).
struct SymParams {
    __half2 sz;
    float sf, zf, r;
    bool ok;
};

__device__ __forceinline__ SymParams sym_params(float mn, float mx, int bits) {
    const int C = 1 << (bits - 1);
    mn = __fadd_rn(mn, 0.0f);
    mx = __fadd_rn(mx, 0.0f);
    const float m = fmaxf(fabsf(mn), fabsf(mx));
    const __half s = __float2half_ru(__fdiv_rn(m, static_cast<float>(C - 1)));
    SymParams p;
    p.sf = __half2float(s);
    p.zf = -static_cast<float>(C) * p.sf;
    p.ok = fabsf(p.zf) <= 65504.0f;
    p.sz = __halves2half2(s, __float2half_rn(p.zf));
    p.r = (p.sf == 0.0f) ? 0.0f : __frcp_rn(p.sf);
    return p;
}

__device__ __forceinline__ uint32_t sym_code(float x, const SymParams &p, int bits) {
    const float C = static_cast<float>(1 << (bits - 1));
    const float t = fminf(fmaxf(rintf(__fmul_rn(x, p.r)), 1.0f - C), C - 1.0f);
    return static_cast<uint32_t>(__fadd_rn(t, C));
}

// Largest reconstruction error so far, with the element x of code q.
__device__ __forceinline__ float max_err(float x, uint32_t q, float s, float z, float m) {
    return fmaxf(m, fabsf(__fsub_rn(x, __fmaf_rn(static_cast<float>(q), s, z))));
}

// Codes of n consecutive elements (n even) of one group:
// q = clamp(rint_even(fp32(fp32(x - z) * r)), 0, L). Every value reaching the
// rounding lies in [0, L (1 + 3 2^-24)] (z <= x <= max, s >= (max - z) / L up
// to one rounding, r = fp32(1/s)), so the upper clamp never binds; the lower
// one also maps NaN to 0. Adding 2^23 rounds to the nearest integer, ties to
// even, and leaves the code in the low bits of the float: q[j] holds 0x4B00000q.
// r == 0 exactly when s == 0; then every code is 0.
__device__ __forceinline__ void qcodes(const float *x, int n, const QParams &p, uint32_t *q) {
    const unsigned long long z2 = f2u(p.zf, p.zf), r2 = f2u(p.r, p.r);
    const unsigned long long magic = f2u(8388608.0f, 8388608.0f);
#pragma unroll
    for (int j = 0; j < n; j += 2) {
        const unsigned long long t = mul2(sub2(f2u(x[j], x[j + 1]), z2), r2);
        const unsigned long long y = add2(f2u(fmaxf(lo_f(t), 0.0f), fmaxf(hi_f(t), 0.0f)), magic);
        q[j] = static_cast<uint32_t>(y);
        q[j + 1] = static_cast<uint32_t>(y >> 32);
    }
}

// Quantize the lane's 32 channels in groups of G (the group spans G/32 lanes
// when G > 32) and pack them. Returns the scale/zero pairs of the groups that
// start in this lane (n_sz of them) and the packed words (4 for INT4, 2 for
// INT2).
template <int BITS, bool HYB = false>
__device__ __forceinline__ void quant_pack_lane(const float x[32], int G, uint32_t words[4],
                                                __half2 sz[2], int &n_sz, int part) {
    constexpr int L = (1 << BITS) - 1;
    uint32_t q[32];  // 0x4B00000q
    // hybrid: replace the asymmetric codes of elements [j0, j0 + n) by the
    // symmetric ones when the group's largest error `es` is below `ea`
    auto choose = [&](int j0, int n, const SymParams &ps, float ea, float es, __half2 &out_sz) {
        if (ps.ok && es < ea) {
#pragma unroll
            for (int j = j0; j < j0 + n; ++j) q[j] = 0x4B000000u | sym_code(x[j], ps, BITS);
            out_sz = ps.sz;
        }
    };
    auto run_errs = [&](int j0, int n, const QParams &p, const SymParams &ps, float &ea, float &es) {
        ea = 0.0f;
        es = 0.0f;
#pragma unroll
        for (int j = j0; j < j0 + n; ++j) {
            ea = max_err(x[j], q[j] - 0x4B000000u, p.sf, p.zf, ea);
            es = max_err(x[j], sym_code(x[j], ps, BITS), ps.sf, ps.zf, es);
        }
    };
    if (G >= 32) {
        float mn = x[0], mx = x[0];
#pragma unroll
        for (int j = 1; j < 32; ++j) { mn = fminf(mn, x[j]); mx = fmaxf(mx, x[j]); }
        for (int m = 1; m < G / 32; m <<= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, m));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
        }
        const QParams p = qparams(mn, mx, L);
        qcodes(x, 32, p, q);
        sz[0] = p.sz;
        if constexpr (HYB) {
            const SymParams ps = sym_params(mn, mx, BITS);
            float ea, es;
            run_errs(0, 32, p, ps, ea, es);
            // the group's largest errors over its lanes
            for (int m = 1; m < G / 32; m <<= 1) {
                ea = fmaxf(ea, __shfl_xor_sync(0xffffffffu, ea, m));
                es = fmaxf(es, __shfl_xor_sync(0xffffffffu, es, m));
            }
            choose(0, 32, ps, ea, es, sz[0]);
        }
        n_sz = ((part * 32) % G == 0) ? 1 : 0;
    } else {  // G == 16: two groups in the lane
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            float mn = x[16 * g], mx = x[16 * g];
#pragma unroll
            for (int j = 1; j < 16; ++j) { mn = fminf(mn, x[16 * g + j]); mx = fmaxf(mx, x[16 * g + j]); }
            const QParams p = qparams(mn, mx, L);
            qcodes(x + 16 * g, 16, p, q + 16 * g);
            sz[g] = p.sz;
            if constexpr (HYB) {
                const SymParams ps = sym_params(mn, mx, BITS);
                float ea, es;
                run_errs(16 * g, 16, p, ps, ea, es);
                choose(16 * g, 16, ps, ea, es, sz[g]);
            }
        }
        n_sz = 2;
    }
    if constexpr (BITS == 4) {
        // word w: byte k = q[8w+2k] | q[8w+2k+1] << 4. Gather the even and the
        // odd codes' low bytes with byte permutes, then E + 16 O.
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const uint32_t *c = q + 8 * w;
            const uint32_t e = __byte_perm(__byte_perm(c[0], c[2], 0x0040), __byte_perm(c[4], c[6], 0x0040), 0x5410);
            const uint32_t o = __byte_perm(__byte_perm(c[1], c[3], 0x0040), __byte_perm(c[5], c[7], 0x0040), 0x5410);
            words[w] = e + (o << 4);
        }
    } else {
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            uint32_t v = 0;
#pragma unroll
            for (int j = 0; j < 16; ++j) v |= (q[16 * w + j] & 3u) << (2 * j);
            words[w] = v;
        }
    }
}

// Store the lane's packed words and scale/zero pairs into cache row `row`.
template <int BITS>
__device__ __forceinline__ void store_lane(uint8_t *codes, __half2 *sz, int64_t row, int G,
                                           int part, const uint32_t words[4], const __half2 s[2],
                                           int n_sz) {
    constexpr int kRowBytes = kHeadDim * BITS / 8;
    uint8_t *dst = codes + row * kRowBytes + part * (32 * BITS / 8);
    if constexpr (BITS == 4)
        *reinterpret_cast<uint4 *>(dst) = make_uint4(words[0], words[1], words[2], words[3]);
    else
        *reinterpret_cast<uint2 *>(dst) = make_uint2(words[0], words[1]);
    const int ng = kHeadDim / G;
    __half2 *srow = sz + row * ng;
    if (G >= 32) {
        if (n_sz) srow[(part * 32) / G] = s[0];
    } else {
        srow[part * 2] = s[0];
        srow[part * 2 + 1] = s[1];
    }
}

__device__ __forceinline__ int find_seq(const int32_t *cu, int n, int tok) {
    int lo = 0, hi = n;  // last s in [0, n) with cu[s] <= tok
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(cu + mid) <= tok) lo = mid; else hi = mid;
    }
    return lo;
}

__device__ __forceinline__ bool dest_row(const AppendParams &p, int s, int pos, int h,
                                         int64_t &row) {
    if (!p.paged) {
        if (pos < 0 || pos >= p.cap) return false;
        row = (static_cast<int64_t>(s) * p.H + h) * p.cap + pos;
        return true;
    }
    const int pi = pos / p.page_size;
    if (pos < 0 || pi >= p.max_pages) return false;
    const int page = __ldg(p.block_table + static_cast<int64_t>(s) * p.max_pages + pi);
    if (page < 0 || page >= p.num_pages) return false;
    row = (static_cast<int64_t>(page) * p.H + h) * p.page_size + (pos & (p.page_size - 1));
    return true;
}

// ---- kernel: per-token append ----------------------------------------------
// grid.x: blocks of 64 vectors; grid.y: 0 = keys, 1 = values.
template <int DT, bool HYB>
__global__ void __launch_bounds__(256) append_tokens_kernel(const AppendParams p) {
    pdl_launch_dependents();  // the length advance may be scheduled; it waits for us
    const AppendTensor &T = p.t[blockIdx.y];
    const int lane = threadIdx.x & 31;
    const int part = lane & 3;
    const int64_t n_vec = static_cast<int64_t>(p.total_tokens) * p.H;
    const int64_t vec = (static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5)) * 8 + (lane >> 2);
    const bool active = vec < n_vec;
    const int64_t v = active ? vec : n_vec - 1;  // idle lanes still join the shuffles

    float x[32];
    load32<DT>(T.src, v, part, x);
    if (T.signs != nullptr) {  // randomized Hadamard: diag(signs) first (exact)
        const float4 *sg = reinterpret_cast<const float4 *>(T.signs + part * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 f = __ldg(sg + i);
            x[4 * i] *= f.x; x[4 * i + 1] *= f.y; x[4 * i + 2] *= f.z; x[4 * i + 3] *= f.w;
        }
    }
    if (T.hb > 0) fwht_lane(x, T.hb, part, T.hscale);

    uint32_t words[4];
    __half2 s[2];
    int n_sz = 0;
    if (T.bits == 4) quant_pack_lane<4, HYB>(x, T.group, words, s, n_sz, part);
    else quant_pack_lane<2, HYB>(x, T.group, words, s, n_sz, part);
    if (!active) return;

    const int tok = static_cast<int>(v / p.H);
    const int h = static_cast<int>(v - static_cast<int64_t>(tok) * p.H);
    const int seq = find_seq(p.cu_new, p.num_seqs, tok);
    const int pos = __ldg(p.seq_lens + seq) + (tok - __ldg(p.cu_new + seq));
    if (pos >= 0 && pos < p.sink_len) {
        // attention-sink token: kept as the input rounded to bf16, not quantized
        float raw[32];
        load32<DT>(T.src, v, part, raw);
        uint32_t w[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(raw[2 * j], raw[2 * j + 1]);
            w[j] = *reinterpret_cast<const uint32_t *>(&b2);
        }
        uint4 *dst = reinterpret_cast<uint4 *>(
            p.sink[blockIdx.y] + ((static_cast<int64_t>(seq) * p.H + h) * p.sink_len + pos) * kHeadDim + part * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        return;
    }
    int64_t row;
    if (!dest_row(p, seq, pos, h, row)) {
        if (part == 0) status_or(p.status, KVQ_DEV_CAPACITY);
        return;
    }
    if (T.bits == 4) store_lane<4>(T.codes, T.sz, row, T.group, part, words, s, n_sz);
    else store_lane<2>(T.codes, T.sz, row, T.group, part, words, s, n_sz);
}

// ---- residual window: flush full blocks, then write the window ------------

struct WindowParams {
    const uint16_t *k_new, *v_new;  // bf16 [N][H][D]
    uint16_t *k_res, *v_res;        // bf16 [S][H][R][D]
    uint8_t *k_codes, *v_codes;
    __half2 *k_sz, *v_sz;
    int bits_k, bits_v, group_k, group_v;
    int k_per_channel, v_per_channel;
    int hybrid;
    int R, H, cap;
    const int32_t *cu_new;
    const int32_t *seq_lens;  // lengths before this append
    int num_seqs, total_tokens;
    int32_t *status;
};

// Quantize one block of R staged bf16 rows [R][128] per channel (each
// channel's R values one group; KIVI keys, InnerQ values) into `codes`
// (R rows packed along channels) and `sz` ([128] half2). With `hybrid`, each
// group takes the symmetric candidate when its largest error is smaller.
// Called by the whole CTA; `qk` is [R][128] bytes of scratch.
__device__ void flush_channel_block(const uint16_t *src, uint8_t *qk, int R, int bits, int hybrid,
                                    uint8_t *codes, __half2 *sz) {
    const int L = (1 << bits) - 1;
    const float Lf = static_cast<float>(L);
    for (int d = threadIdx.x; d < kHeadDim; d += blockDim.x) {
        float mn = bf16_bits_to_float(src[d]), mx = mn;
        for (int t = 1; t < R; ++t) {
            const float v = bf16_bits_to_float(src[t * kHeadDim + d]);
            mn = fminf(mn, v);
            mx = fmaxf(mx, v);
        }
        const QParams qp = qparams(mn, mx, L);
        bool use_sym = false;
        SymParams ps{};
        if (hybrid) {
            ps = sym_params(mn, mx, bits);
            float ea = 0.0f, es = 0.0f;
            for (int t = 0; t < R; ++t) {
                const float v = bf16_bits_to_float(src[t * kHeadDim + d]);
                ea = max_err(v, qcode(v, qp, Lf), qp.sf, qp.zf, ea);
                es = max_err(v, sym_code(v, ps, bits), ps.sf, ps.zf, es);
            }
            use_sym = ps.ok && es < ea;
        }
        for (int t = 0; t < R; ++t) {
            const float v = bf16_bits_to_float(src[t * kHeadDim + d]);
            qk[t * kHeadDim + d] = static_cast<uint8_t>(use_sym ? sym_code(v, ps, bits) : qcode(v, qp, Lf));
        }
        sz[d] = use_sym ? ps.sz : qp.sz;
    }
    __syncthreads();
    // Pack along channels: one 32-bit word holds 32/bits channels.
    const int per_word = 32 / bits;
    const int words_per_row = kHeadDim / per_word;
    for (int i = threadIdx.x; i < R * words_per_row; i += blockDim.x) {
        const int t = i / words_per_row, w = i - t * words_per_row;
        uint32_t v = 0;
        for (int j = 0; j < per_word; ++j)
            v |= static_cast<uint32_t>(qk[t * kHeadDim + w * per_word + j]) << (bits * j);
        reinterpret_cast<uint32_t *>(codes + static_cast<size_t>(t) * (kHeadDim * bits / 8))[w] = v;
    }
    __syncthreads();  // qk is free for the next tensor
}

// One CTA per (flushed block slot, head, sequence). The block's R tokens come
// from the old window (positions below the old length) and from the new
// tokens; each tensor is quantized per channel or per token.
__global__ void __launch_bounds__(256) window_flush_kernel(const WindowParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int seq = blockIdx.z, h = blockIdx.y;
    const int R = p.R;
    const int T0 = __ldg(p.seq_lens + seq);
    const int c0 = __ldg(p.cu_new + seq);
    const int n = __ldg(p.cu_new + seq + 1) - c0;
    const int T1 = T0 + n;
    const int Tq0 = quantized_len(T0, R), Tq1 = quantized_len(T1, R);
    const int b = Tq0 / R + static_cast<int>(blockIdx.x);
    if (b * R >= Tq1) return;
    if (b * R + R > p.cap) {
        if (threadIdx.x == 0) status_or(p.status, KVQ_DEV_CAPACITY);
        return;
    }
    uint16_t *kb = reinterpret_cast<uint16_t *>(smem);                 // [R][128] bf16
    uint16_t *vb = kb + static_cast<size_t>(R) * kHeadDim;             // [R][128] bf16
    uint8_t *qk = reinterpret_cast<uint8_t *>(vb + static_cast<size_t>(R) * kHeadDim);  // [R][128]
    const int64_t sh = static_cast<int64_t>(seq) * p.H + h;

    // Stage the block: 16 chunks of 16 bytes per token row, K and V.
    for (int i = threadIdx.x; i < R * 16; i += blockDim.x) {
        const int t = i >> 4, c = i & 15;
        const int pos = b * R + t;
        const uint4 *ks, *vs;
        if (pos < T0) {
            const int64_t slot = sh * R + (pos - Tq0);
            ks = reinterpret_cast<const uint4 *>(p.k_res + slot * kHeadDim);
            vs = reinterpret_cast<const uint4 *>(p.v_res + slot * kHeadDim);
        } else {
            const int64_t r = static_cast<int64_t>(c0 + pos - T0) * p.H + h;
            ks = reinterpret_cast<const uint4 *>(p.k_new + r * kHeadDim);
            vs = reinterpret_cast<const uint4 *>(p.v_new + r * kHeadDim);
        }
        reinterpret_cast<uint4 *>(kb)[i] = ks[c];
        reinterpret_cast<uint4 *>(vb)[i] = vs[c];
    }
    __syncthreads();

    const int lane = threadIdx.x & 31, part = lane & 3;
    const int64_t row0 = sh * p.cap + static_cast<int64_t>(b) * R;

    // Per-channel tensors (keys; values grouped along tokens).
    if (p.k_per_channel) flush_channel_block(kb, qk, R, p.bits_k, p.hybrid, p.k_codes + row0 * (kHeadDim * p.bits_k / 8),
                                             p.k_sz + (sh * (p.cap / R) + b) * kHeadDim);
    if (p.v_per_channel) flush_channel_block(vb, qk, R, p.bits_v, p.hybrid, p.v_codes + row0 * (kHeadDim * p.bits_v / 8),
                                             p.v_sz + (sh * (p.cap / R) + b) * kHeadDim);
    // Per-token tensors: 8 vectors per warp, 64 per pass.
    for (int tsel = 0; tsel < 2; ++tsel) {
        if (tsel ? p.v_per_channel : p.k_per_channel) continue;
        const uint16_t *src = tsel ? vb : kb;
        const int bits = tsel ? p.bits_v : p.bits_k;
        const int G = tsel ? p.group_v : p.group_k;
        uint8_t *codes = tsel ? p.v_codes : p.k_codes;
        __half2 *sz = tsel ? p.v_sz : p.k_sz;
        for (int t0 = 0; t0 < R; t0 += 64) {
            const int t = t0 + (threadIdx.x >> 2);
            float x[32];
            const uint16_t *rowp = src + static_cast<size_t>(t) * kHeadDim + part * 32;
#pragma unroll
            for (int j = 0; j < 32; ++j) x[j] = bf16_bits_to_float(rowp[j]);
            uint32_t words[4];
            __half2 s[2];
            int n_sz = 0;
            if (bits == 4) {
                if (p.hybrid) quant_pack_lane<4, true>(x, G, words, s, n_sz, part);
                else quant_pack_lane<4, false>(x, G, words, s, n_sz, part);
                store_lane<4>(codes, sz, row0 + t, G, part, words, s, n_sz);
            } else {
                if (p.hybrid) quant_pack_lane<2, true>(x, G, words, s, n_sz, part);
                else quant_pack_lane<2, false>(x, G, words, s, n_sz, part);
                store_lane<2>(codes, sz, row0 + t, G, part, words, s, n_sz);
            }
        }
    }
}

// Copy the new tokens that stay in the window into their slots. One thread
// per 16-byte chunk of a (token, head) row; K and V.
__global__ void __launch_bounds__(256) window_write_kernel(const WindowParams p) {
    pdl_launch_dependents();  // the length advance may be scheduled; it waits for us
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t n_chunks = static_cast<int64_t>(p.total_tokens) * p.H * 16;
    if (i >= n_chunks) return;
    const int64_t vrow = i >> 4;
    const int c = static_cast<int>(i & 15);
    const int tok = static_cast<int>(vrow / p.H);
    const int h = static_cast<int>(vrow - static_cast<int64_t>(tok) * p.H);
    const int seq = find_seq(p.cu_new, p.num_seqs, tok);
    const int T0 = __ldg(p.seq_lens + seq);
    const int c0 = __ldg(p.cu_new + seq);
    const int T1 = T0 + (__ldg(p.cu_new + seq + 1) - c0);
    const int pos = T0 + (tok - c0);
    const int Tq1 = quantized_len(T1, p.R);
    if (pos < Tq1) return;
    const int64_t slot = (static_cast<int64_t>(seq) * p.H + h) * p.R + (pos - Tq1);
    reinterpret_cast<uint4 *>(p.k_res + slot * kHeadDim)[c] =
        reinterpret_cast<const uint4 *>(p.k_new + vrow * kHeadDim)[c];
    reinterpret_cast<uint4 *>(p.v_res + slot * kHeadDim)[c] =
        reinterpret_cast<const uint4 *>(p.v_new + vrow * kHeadDim)[c];
}

// Launched as a programmatic dependent of the append kernel: scheduled early,
// it waits for that grid (which reads the old lengths) to complete.
__global__ void advance_lens_kernel(const int32_t *cu_new, int32_t *seq_lens, int num_seqs) {
    pdl_wait_prior_grid();
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s < num_seqs) seq_lens[s] += cu_new[s + 1] - cu_new[s];
}

}  // namespace

// ---------------------------------------------------------------------------
// Host launcher (arguments already validated by kvq_api.cu)
// ---------------------------------------------------------------------------
kvq_status launch_append(const kvq_cache_desc &d, const void *k_new, const void *v_new,
                         kvq_dtype dtype, const int32_t *cu_new, int32_t *seq_lens,
                         int num_seqs, int total_new, cudaStream_t stream) {
    if (total_new == 0) return KVQ_OK;
    const bool has_v = v_new != nullptr;
    if (d.residual_len > 0) {
        WindowParams w{};
        w.k_new = static_cast<const uint16_t *>(k_new);
        w.v_new = static_cast<const uint16_t *>(v_new);
        w.k_res = static_cast<uint16_t *>(d.k_res);
        w.v_res = static_cast<uint16_t *>(d.v_res);
        w.k_codes = static_cast<uint8_t *>(d.k_codes);
        w.v_codes = static_cast<uint8_t *>(d.v_codes);
        w.k_sz = static_cast<__half2 *>(d.k_sz);
        w.v_sz = static_cast<__half2 *>(d.v_sz);
        w.bits_k = d.bits_k; w.bits_v = d.bits_v;
        w.group_k = d.group_k; w.group_v = d.group_v;
        w.k_per_channel = d.axis_k == KVQ_PER_CHANNEL;
        w.v_per_channel = d.axis_v == KVQ_PER_CHANNEL;
        w.hybrid = d.hybrid;
        w.R = d.residual_len; w.H = d.num_kv_heads; w.cap = d.capacity_tokens;
        w.cu_new = cu_new; w.seq_lens = seq_lens;
        w.num_seqs = num_seqs; w.total_tokens = total_new;
        w.status = d.status;
        const int max_blocks = (total_new + w.R - 1) / w.R;
        const size_t smem = static_cast<size_t>(w.R) * kHeadDim * (2 + 2 + 1);
        if (smem > 48 * 1024 &&
            cudaFuncSetAttribute(window_flush_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess)
            return KVQ_ERR_CUDA;
        window_flush_kernel<<<dim3(max_blocks, w.H, num_seqs), 256, smem, stream>>>(w);
        if (cudaGetLastError() != cudaSuccess) return KVQ_ERR_CUDA;
        const int64_t chunks = static_cast<int64_t>(total_new) * w.H * 16;
        window_write_kernel<<<static_cast<unsigned>((chunks + 255) / 256), 256, 0, stream>>>(w);
        if (cudaGetLastError() != cudaSuccess) return KVQ_ERR_CUDA;
    } else {
        AppendParams p{};
        p.t[0] = {static_cast<uint8_t *>(d.k_codes), static_cast<__half2 *>(d.k_sz), k_new,
                  d.bits_k, d.group_k, d.hadamard_block_k, hadamard_scale(d.hadamard_block_k),
                  d.hadamard_block_k > 0 ? d.hadamard_signs : nullptr};
        p.t[1] = {static_cast<uint8_t *>(d.v_codes), static_cast<__half2 *>(d.v_sz), v_new,
                  d.bits_v, d.group_v, 0, 0.0f, nullptr};
        p.H = d.num_kv_heads;
        p.cu_new = cu_new; p.seq_lens = seq_lens;
        p.num_seqs = num_seqs; p.total_tokens = total_new;
        p.paged = d.paged; p.page_size = d.page_size; p.max_pages = d.max_pages_per_seq;
        p.num_pages = d.num_pages; p.cap = d.capacity_tokens;
        p.block_table = d.block_table; p.status = d.status;
        p.sink[0] = static_cast<uint16_t *>(d.k_sink);
        p.sink[1] = static_cast<uint16_t *>(d.v_sink);
        p.sink_len = d.sink_len;
        const int64_t n_vec = static_cast<int64_t>(total_new) * d.num_kv_heads;
        const dim3 grid(static_cast<unsigned>((n_vec + 63) / 64), has_v ? 2 : 1);
        switch (dtype) {
            case KVQ_BF16:
                if (d.hybrid) append_tokens_kernel<KVQ_BF16, true><<<grid, 256, 0, stream>>>(p);
                else append_tokens_kernel<KVQ_BF16, false><<<grid, 256, 0, stream>>>(p);
                break;
            case KVQ_FP16:
                if (d.hybrid) append_tokens_kernel<KVQ_FP16, true><<<grid, 256, 0, stream>>>(p);
                else append_tokens_kernel<KVQ_FP16, false><<<grid, 256, 0, stream>>>(p);
                break;
            default:
                if (d.hybrid) append_tokens_kernel<KVQ_FP32, true><<<grid, 256, 0, stream>>>(p);
                else append_tokens_kernel<KVQ_FP32, false><<<grid, 256, 0, stream>>>(p);
                break;
        }
        if (cudaGetLastError() != cudaSuccess) return KVQ_ERR_CUDA;
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((num_seqs + 127) / 128);
    cfg.blockDim = dim3(128);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, advance_lens_kernel, cu_new, seq_lens, num_seqs) != cudaSuccess)
        return KVQ_ERR_CUDA;
    return KVQ_OK;
}

}  // namespace kvq
