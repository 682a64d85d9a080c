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
#include <algorithm>

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

// ---- kernel: per-token append, two lanes per (token, head) vector --------
// A warp takes batches of 16 consecutive input vectors (one contiguous run of
// the [N][H][128] input), staged into shared memory by cp.async; each warp
// keeps kAppendStages batch buffers, so the copies of its next batches run
// under this batch's arithmetic. Lanes 2t and 2t+1 own vector t of the batch, channels
// [0, 64) and [64, 128): the rotation's stages of half-width 1..32 stay in
// the lane and the stage 64 is one exchange with the partner; groups of up
// to 64 lie in one lane and a group of 128 takes one exchange of extremes.
// The steps and their rounding are those of the lane-group path (fwht_lane,
// qparams, qcodes), so both give the oracle's bits.
constexpr int kAppendWarps = 4;
constexpr int kAppendBlocksPerSm = 3;
constexpr int kAppendStages = 2;  // batches per warp: one in use, one in flight

template <int DT>
struct StagedRows {
    static constexpr int half_bytes = (DT == KVQ_FP32) ? 256 : 128;  // one lane's 64 channels
    static constexpr int in_bytes = 2 * half_bytes;                   // one input row
    // staged row: [half 0][16-byte pad][half 1][16-byte pad], so the eight
    // lanes of a shared-memory phase read eight distinct bank groups
    static constexpr int half_stride = half_bytes + 16;
    static constexpr int stride = 2 * half_stride;
    static constexpr int batch = 16 * stride;  // one warp's buffer
};

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Copies of batch b (vectors [16b, 16b + 16) below n_vec) into buf: 16-byte
// chunks, consecutive lanes on consecutive chunks of the run. Lane l copies
// chunks l + 32 i; their places in the padded buffer are `dst_lane` (the
// lane's first) plus i rows of 32 / CPR each.
template <int DT>
__device__ __forceinline__ void stage_batch(const void *src, int64_t b, int64_t n_vec, uint8_t *buf,
                                            int dst_lane, int lane) {
    using SR = StagedRows<DT>;
    constexpr int CPR = SR::in_bytes / 16;  // chunks per row
    constexpr int ROWS_PER_STEP = 32 / CPR;
    const int64_t v0 = b * 16;
    const int64_t left = n_vec - v0;
    const uint8_t *g = static_cast<const uint8_t *>(src) + v0 * SR::in_bytes + lane * 16;
    uint8_t *d = buf + dst_lane;
    if (left >= 16) {
#pragma unroll
        for (int i = 0; i < CPR / 2; ++i) cp_async16(d + i * ROWS_PER_STEP * SR::stride, g + i * 512);
    } else {
        const int n_chunks = static_cast<int>(left) * CPR;
#pragma unroll
        for (int i = 0; i < CPR / 2; ++i)
            if (lane + 32 * i < n_chunks) cp_async16(d + i * ROWS_PER_STEP * SR::stride, g + i * 512);
    }
}

// Offset of lane l's first chunk in the padded batch buffer.
template <int DT>
__device__ __forceinline__ int stage_offset(int lane) {
    using SR = StagedRows<DT>;
    constexpr int CPR = SR::in_bytes / 16;
    constexpr int CPH = SR::half_bytes / 16;
    const int row = lane / CPR, col = lane % CPR;
    const int hh = col >= CPH ? 1 : 0;
    return row * SR::stride + hh * SR::half_stride + (col - hh * CPH) * 16;
}

// The lane's staged half row as 32 channel pairs {2k, 2k + 1} in fp32.
template <int DT>
__device__ __forceinline__ void read_half(const uint8_t *hrow, float2 v[32]) {
    if constexpr (DT == KVQ_FP32) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint4 u = *reinterpret_cast<const uint4 *>(hrow + 16 * i);
            v[2 * i] = make_float2(__uint_as_float(u.x), __uint_as_float(u.y));
            v[2 * i + 1] = make_float2(__uint_as_float(u.z), __uint_as_float(u.w));
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint4 u = *reinterpret_cast<const uint4 *>(hrow + 16 * i);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if constexpr (DT == KVQ_BF16) {
                    v[4 * i + j] = make_float2(bf16_bits_to_float(w[j] & 0xFFFFu), bf16_bits_to_float(w[j] >> 16));
                } else {
                    v[4 * i + j] = make_float2(__half2float(__ushort_as_half((unsigned short)(w[j] & 0xFFFFu))),
                                               __half2float(__ushort_as_half((unsigned short)(w[j] >> 16))));
                }
            }
        }
    }
}

// f32x2 register pairs: a float2 is one 64-bit register pair, so these are
// moves the compiler drops.
__device__ __forceinline__ unsigned long long u64_of(float2 a) {
    return *reinterpret_cast<unsigned long long *>(&a);
}
__device__ __forceinline__ float2 f2_of(unsigned long long u) { return *reinterpret_cast<float2 *>(&u); }

// Normalized Sylvester Walsh-Hadamard transform of each HB-block of the 128
// channels, the lane holding 64 of them (`half` says which): half-widths 1, 2,
// ..., HB/2 in ascending order, butterfly (a, b) -> (a + b, a - b) with a the
// lower index, each op rounded to fp32; then one multiply by
// c = fp32(1/sqrt(HB)). The half-width 64 stage pairs the lane with its
// partner (lane ^ 1): o + s x with s = +-1 in one fma rounds like the add or
// subtract it stands for.
template <int HB>
__device__ __forceinline__ void fwht_half(float2 v[32], int half, float c) {
    if constexpr (HB > 1) {
#pragma unroll
        for (int k = 0; k < 32; ++k) v[k] = make_float2(__fadd_rn(v[k].x, v[k].y), __fsub_rn(v[k].x, v[k].y));
    }
#pragma unroll
    for (int st = 0; st < 5; ++st) {  // pair half-width hp = 2^st: channel half-width 2 hp
        const int hp = 1 << st;
        if (2 * hp < HB) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {  // butterfly j: pairs k and k + hp
                const int k = (j / hp) * 2 * hp + (j % hp);
                const unsigned long long a = u64_of(v[k]), b = u64_of(v[k + hp]);
                v[k] = f2_of(add2(a, b));
                v[k + hp] = f2_of(sub2(a, b));
            }
        }
    }
    if constexpr (HB == 128) {
        const float sg = half ? -1.0f : 1.0f;  // upper: o - x, lower: x + o
        const unsigned long long sg2 = f2u(sg, sg);
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            const float o0 = __shfl_xor_sync(0xffffffffu, v[k].x, 1);
            const float o1 = __shfl_xor_sync(0xffffffffu, v[k].y, 1);
            v[k] = f2_of(fma2(sg2, u64_of(v[k]), f2u(o0, o1)));
        }
    }
    const unsigned long long c2 = f2u(c, c);
#pragma unroll
    for (int k = 0; k < 32; ++k) v[k] = f2_of(mul2(u64_of(v[k]), c2));
}

__device__ __forceinline__ void fwht_half_any(float2 v[32], int hb, int half, float c) {
    switch (hb) {
        case 2: fwht_half<2>(v, half, c); break;
        case 4: fwht_half<4>(v, half, c); break;
        case 8: fwht_half<8>(v, half, c); break;
        case 16: fwht_half<16>(v, half, c); break;
        case 32: fwht_half<32>(v, half, c); break;
        case 64: fwht_half<64>(v, half, c); break;
        default: fwht_half<128>(v, half, c); break;
    }
}

// Quantize the lane's 64 channels in groups of G (16, 32, 64; or 128, shared
// with the partner lane) and pack them: words[0 .. 64 * BITS / 32), and in
// szb[b] the (scale, zero) pair of the group of 16-channel block b.
// Extremes are taken per 16-channel block and combined within each group;
// the group's parameters are computed once, at its first block. HYB: each
// group takes the symmetric grid when its largest error is smaller (two
// passes: errors, then codes).
template <int BITS, bool HYB>
__device__ __forceinline__ void quant_pack_half(const float2 v[32], int G, uint32_t words[8], __half2 szb[4]) {
    constexpr int L = (1 << BITS) - 1;
    const int bpg = G >> 4;  // 16-channel blocks per group
    float mn[4], mx[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        float lo = fminf(v[8 * b].x, v[8 * b].y), hi = fmaxf(v[8 * b].x, v[8 * b].y);
#pragma unroll
        for (int k = 8 * b + 1; k < 8 * b + 8; ++k) {
            lo = fminf(lo, fminf(v[k].x, v[k].y));
            hi = fmaxf(hi, fmaxf(v[k].x, v[k].y));
        }
        mn[b] = lo;
        mx[b] = hi;
    }
#pragma unroll
    for (int step = 1; step < 4; step <<= 1) {  // every block gets its group's extremes
        if (step < bpg) {
#pragma unroll
            for (int b = 0; b < 4; ++b)
                if ((b & step) == 0) {
                    const float lo = fminf(mn[b], mn[b | step]), hi = fmaxf(mx[b], mx[b | step]);
                    mn[b] = lo; mn[b | step] = lo;
                    mx[b] = hi; mx[b | step] = hi;
                }
        }
    }
    if (G == 128) {  // the group spans both lanes of the vector
        const float lo = fminf(mn[0], __shfl_xor_sync(0xffffffffu, mn[0], 1));
        const float hi = fmaxf(mx[0], __shfl_xor_sync(0xffffffffu, mx[0], 1));
#pragma unroll
        for (int b = 0; b < 4; ++b) { mn[b] = lo; mx[b] = hi; }
    }
    const int lbpg = bpg < 4 ? bpg : 4;  // blocks per group within the lane
    float zf[4], rf[4], sf[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        if (b == 0 || (b & (lbpg - 1)) == 0) {
            const QParams p = qparams(mn[b], mx[b], L);
            zf[b] = p.zf; rf[b] = p.r; sf[b] = p.sf;
            szb[b] = p.sz;
        } else {
            zf[b] = zf[b - 1]; rf[b] = rf[b - 1]; sf[b] = sf[b - 1];
            szb[b] = szb[b - 1];
        }
    }
    bool sym[4] = {false, false, false, false};
    SymParams ps[4];
    if constexpr (HYB) {
        float ea[4], es[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            if (b == 0 || (b & (lbpg - 1)) == 0) ps[b] = sym_params(mn[b], mx[b], BITS);
            else ps[b] = ps[b - 1];
            QParams pa;
            pa.zf = zf[b]; pa.r = rf[b];
            float a = 0.0f, e = 0.0f;
#pragma unroll
            for (int k = 8 * b; k < 8 * b + 8; ++k) {
                a = max_err(v[k].x, qcode(v[k].x, pa, static_cast<float>(L)), sf[b], zf[b], a);
                a = max_err(v[k].y, qcode(v[k].y, pa, static_cast<float>(L)), sf[b], zf[b], a);
                e = max_err(v[k].x, sym_code(v[k].x, ps[b], BITS), ps[b].sf, ps[b].zf, e);
                e = max_err(v[k].y, sym_code(v[k].y, ps[b], BITS), ps[b].sf, ps[b].zf, e);
            }
            ea[b] = a;
            es[b] = e;
        }
#pragma unroll
        for (int step = 1; step < 4; step <<= 1) {
            if (step < bpg) {
#pragma unroll
                for (int b = 0; b < 4; ++b)
                    if ((b & step) == 0) {
                        const float a = fmaxf(ea[b], ea[b | step]), e = fmaxf(es[b], es[b | step]);
                        ea[b] = a; ea[b | step] = a;
                        es[b] = e; es[b | step] = e;
                    }
            }
        }
        if (G == 128) {
            const float a = fmaxf(ea[0], __shfl_xor_sync(0xffffffffu, ea[0], 1));
            const float e = fmaxf(es[0], __shfl_xor_sync(0xffffffffu, es[0], 1));
#pragma unroll
            for (int b = 0; b < 4; ++b) { ea[b] = a; es[b] = e; }
        }
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            sym[b] = ps[b].ok && es[b] < ea[b];
            if (sym[b]) szb[b] = ps[b].sz;
        }
    }
    // codes, packed: INT4 byte i = q[2i] | q[2i+1] << 4; INT2 byte i holds
    // q[4i + j] in bits 2j..2j+1
    const unsigned long long magic = f2u(8388608.0f, 8388608.0f);
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        uint32_t q[16];
        if (HYB && sym[b]) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                q[2 * k] = sym_code(v[8 * b + k].x, ps[b], BITS);
                q[2 * k + 1] = sym_code(v[8 * b + k].y, ps[b], BITS);
            }
        } else {
            // q = rint_even(fp32(fp32(x - z) * r)) through the 2^23 trick; the
            // lower clamp maps NaN to 0 (the upper one never binds)
            const unsigned long long z2 = f2u(zf[b], zf[b]), r2 = f2u(rf[b], rf[b]);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float2 t = f2_of(mul2(sub2(u64_of(v[8 * b + k]), z2), r2));
                const float2 y = f2_of(add2(u64_of(make_float2(fmaxf(t.x, 0.0f), fmaxf(t.y, 0.0f))), magic));
                q[2 * k] = __float_as_uint(y.x);
                q[2 * k + 1] = __float_as_uint(y.y);
            }
        }
        if constexpr (BITS == 4) {
#pragma unroll
            for (int w = 0; w < 2; ++w) {
                const uint32_t *c = q + 8 * w;
                const uint32_t e = __byte_perm(__byte_perm(c[0], c[2], 0x0040), __byte_perm(c[4], c[6], 0x0040), 0x5410);
                const uint32_t o = __byte_perm(__byte_perm(c[1], c[3], 0x0040), __byte_perm(c[5], c[7], 0x0040), 0x5410);
                words[2 * b + w] = e + (o << 4);
            }
        } else {
            uint32_t wv = 0;
#pragma unroll
            for (int j = 0; j < 16; ++j) wv |= (q[j] & 3u) << (2 * j);
            words[b] = wv;
        }
    }
}

template <int DT, bool HYB>
__global__ void __launch_bounds__(kAppendWarps * 32, kAppendBlocksPerSm) append_rows_kernel(const AppendParams p) {
    pdl_launch_dependents();  // the length advance may be scheduled; it waits for us
    using SR = StagedRows<DT>;
    extern __shared__ __align__(16) uint8_t smem[];
    const AppendTensor &T = p.t[blockIdx.y];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int half = lane & 1;
    uint8_t *bufs = smem + warp * kAppendStages * SR::batch;
    const int64_t n_vec = static_cast<int64_t>(p.total_tokens) * p.H;
    const int64_t n_batches = (n_vec + 15) / 16;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kAppendWarps;
    int64_t b = static_cast<int64_t>(blockIdx.x) * kAppendWarps + warp;
    if (b >= n_batches) return;
    const int dst_lane = stage_offset<DT>(lane);
    // the first kAppendStages - 1 batches in flight (a commit per slot, empty
    // groups past the end, so the wait count below is always the same)
#pragma unroll
    for (int j = 0; j < kAppendStages - 1; ++j) {
        if (b + j * stride < n_batches)
            stage_batch<DT>(T.src, b + j * stride, n_vec, bufs + j * SR::batch, dst_lane, lane);
        cp_async_commit();
    }
    for (int i = 0; b < n_batches; ++i, b += stride) {
        const uint8_t *cur = bufs + (i % kAppendStages) * SR::batch;
        const int64_t ahead = b + (kAppendStages - 1) * stride;
        if (ahead < n_batches)
            stage_batch<DT>(T.src, ahead, n_vec, bufs + ((i + kAppendStages - 1) % kAppendStages) * SR::batch,
                            dst_lane, lane);
        cp_async_commit();
        cp_async_wait<kAppendStages - 1>();
        __syncwarp();
        // idle lanes of a short last batch work on a copy of the batch's
        // first vector (both lanes of a pair stay together for the exchanges)
        const int64_t vraw = b * 16 + (lane >> 1);
        const bool active = vraw < n_vec;
        const int t = active ? (lane >> 1) : 0;
        const int64_t vec = b * 16 + t;
        float2 v[32];
        read_half<DT>(cur + t * SR::stride + half * SR::half_stride, v);
        __syncwarp();  // every lane has read its row: the buffer may be refilled
        const uint32_t vec32 = static_cast<uint32_t>(vec);  // n_vec < 2^31 (host check)
        const int tok = static_cast<int>(vec32 / static_cast<uint32_t>(p.H));
        const int h = static_cast<int>(vec32 - static_cast<uint32_t>(tok) * static_cast<uint32_t>(p.H));
        const int seq = find_seq(p.cu_new, p.num_seqs, tok);
        const int pos = __ldg(p.seq_lens + seq) + (tok - __ldg(p.cu_new + seq));
        const bool sink = pos >= 0 && pos < p.sink_len;  // the same for both lanes of a pair
        if (sink) {
            // attention-sink token: kept as the input rounded to bf16, not quantized
            if (active) {
                uint4 *dst = reinterpret_cast<uint4 *>(
                    p.sink[blockIdx.y] + ((static_cast<int64_t>(seq) * p.H + h) * p.sink_len + pos) * kHeadDim +
                    half * 64);
#pragma unroll
                for (int i4 = 0; i4 < 8; ++i4) {
                    uint32_t w[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[4 * i4 + j].x, v[4 * i4 + j].y);
                        w[j] = *reinterpret_cast<const uint32_t *>(&b2);
                    }
                    dst[i4] = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            continue;
        }
        if (T.signs != nullptr) {  // randomized Hadamard: diag(signs) first (exact)
            const float2 *sg = reinterpret_cast<const float2 *>(T.signs) + half * 32;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const float2 s2 = __ldg(sg + k);
                v[k].x *= s2.x;
                v[k].y *= s2.y;
            }
        }
        if (T.hb > 0) fwht_half_any(v, T.hb, half, T.hscale);
        uint32_t words[8];
        __half2 szb[4];
        if (T.bits == 4) quant_pack_half<4, HYB>(v, T.group, words, szb);
        else quant_pack_half<2, HYB>(v, T.group, words, szb);
        if (!active) continue;
        int64_t drow;
        if (!dest_row(p, seq, pos, h, drow)) {
            if (half == 0) status_or(p.status, KVQ_DEV_CAPACITY);
            continue;
        }
        if (T.bits == 4) {
            uint4 *dst = reinterpret_cast<uint4 *>(T.codes + drow * 64 + half * 32);
            dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
            dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
        } else {
            *reinterpret_cast<uint4 *>(T.codes + drow * 32 + half * 16) =
                make_uint4(words[0], words[1], words[2], words[3]);
        }
        // the pairs of the groups that start in this lane: group (64 half + 16 b) / G
        const int ng = kHeadDim / T.group;
        __half2 *srow = T.sz + drow * ng;
        const int bpg = T.group >> 4;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int blk = 4 * half + b;  // 16-channel block of the row
            if ((blk & (bpg - 1)) == 0) srow[blk / bpg] = szb[b];
        }
    }
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

template <int DT, bool HYB>
kvq_status launch_rows(dim3 grid, const AppendParams &p, cudaStream_t stream) {
    const size_t smem = static_cast<size_t>(kAppendWarps) * kAppendStages * StagedRows<DT>::batch;
    auto kern = append_rows_kernel<DT, HYB>;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
        return KVQ_ERR_CUDA;
    kern<<<grid, kAppendWarps * 32, smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
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
        if (n_vec >= (int64_t(1) << 31)) return KVQ_ERR_UNSUPPORTED;  // vector indices are 32-bit
        const int64_t n_batches = (n_vec + 15) / 16;
        int sms = 148, dev = 0;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int64_t blocks = std::min<int64_t>((n_batches + kAppendWarps - 1) / kAppendWarps,
                                                 static_cast<int64_t>(kAppendBlocksPerSm) * std::max(sms, 1));
        const dim3 grid(static_cast<unsigned>(blocks), has_v ? 2 : 1);
        kvq_status st = KVQ_OK;
        switch (dtype) {
            case KVQ_BF16:
                st = d.hybrid ? launch_rows<KVQ_BF16, true>(grid, p, stream) : launch_rows<KVQ_BF16, false>(grid, p, stream);
                break;
            case KVQ_FP16:
                st = d.hybrid ? launch_rows<KVQ_FP16, true>(grid, p, stream) : launch_rows<KVQ_FP16, false>(grid, p, stream);
                break;
            default:
                st = d.hybrid ? launch_rows<KVQ_FP32, true>(grid, p, stream) : launch_rows<KVQ_FP32, false>(grid, p, stream);
                break;
        }
        if (st != KVQ_OK) return st;
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
