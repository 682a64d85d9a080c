// kvq_decode.cu -- split-K grouped-query decode attention over the packed
// cache (sm_100a), and the log-sum-exp merge of the splits.
//
// SAW-INT4 (Abstract): attention runs fused over the quantized paged cache.
// InnerQ (Abstract): with groups along the inner dimension of q.k the scale
// and zero factor out of the dot product,
//     q . k^ = s * sum_i q_i c_i + z * sum_i q_i,
// and for values  sum_t p_t v^_t = sum_t (p_t s_t) c_t + sum_t p_t z_t,
// so no dequantized element is ever formed. Dual-QK (Abstract): queries take
// the keys' orthogonal transform, so q~ . k~ = q . k.
//
// Work items are (sequence, KV head, split of `chunk` tokens). The kernel is
// persistent: each CTA (4 consumer warps + 1 producer warp) runs until a
// global item counter is exhausted. The producer's elected lane claims items
// and streams every item's tiles (K codes, K scale/zero, V codes, V scale/zero;
// bf16 rows for the recent-token window; the item's query rows with its first
// tile) into a shared-memory ring with 1-D bulk copies (TMA engine, mbarrier
// complete_tx), resolving page tables per page. Each stage carries a small
// header, so the consumers follow the stream without further coordination and
// the ring never drains between items.
//
// Inner loop. The path is bound by the FP32 FMA pipe, not by the tensor
// cores: every cached element meets GQA query heads, one multiply-add each.
// So the loop spends as few issue slots as possible besides those:
//   * multiply-adds are packed f32x2 FMAs (two lanes of work per issue);
//   * codes become floats 0.5 + X/256 with ONE byte permute per code, from
//     byte planes kept below 128; the query is transformed once per item so
//     that its dot product with these floats is the one with the codes, and
//     the value sums are untangled once per item;
//   * each consumer warp owns a quarter of every tile with its own
//     online-softmax state, so tiles need no cross-warp synchronisation;
//   * scores: 8 lanes per token, 16 channels per lane, all GQA heads at once,
//     a select-free reduce-scatter over the 8 lanes (heads held in a per-lane
//     permuted order) leaves one head's score per lane pair;
//   * values: 16 lanes cover the 128 channels (8 each) for all GQA heads; the
//     two half-warps take alternate tokens;
//   * common group sizes are compile-time constants.
// The four warps' states are merged once per item; the merge kernel combines
// the splits.
#include <algorithm>

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

constexpr int kTile = 128;         // tokens per quantized tile
constexpr int kWinTile = 16;       // tokens per bf16 window tile (quantized caches)
constexpr int kConsumerWarps = 4;
constexpr int kTokensPerWarp = kTile / kConsumerWarps;  // of a quantized tile
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr float kLog2e = 1.4426950408889634f;
#ifndef KVQ_DECODE_MIN_BLOCKS
#define KVQ_DECODE_MIN_BLOCKS 2  // resident CTAs per SM the register budget targets
#endif

enum KMode { K_TOKEN = 0, K_CHANNEL = 1, K_BF16 = 2 };
enum VMode { V_TOKEN = 0, V_BF16 = 2 };

// Stage header flags.
constexpr int kFirst = 1, kLast = 2, kWindow = 4, kDone = 8;

struct TileHdr {
    int seq, kvh, split, t0;
    int n, flags, pad0, pad1;
};

struct DecodeParams {
    const uint8_t *k_codes, *v_codes;  // packed codes, or bf16 rows (bits 16)
    const __half2 *k_sz, *v_sz;
    const uint16_t *k_res, *v_res;
    const int32_t *block_table;
    const int32_t *seq_lens;
    const void *q;
    float *o_part;  // [S][Hq][n_split][D]
    float2 *ml;     // [S][Hq][n_split]
    int *counter;   // item counter, zeroed before the launch
    int32_t *status;
    int S, H, Hq;
    int gk_log2, gv_log2;  // log2 of the group sizes (token-wise groups)
    int hb;
    float hscale;   // fp32(1/sqrt(hb))
    float qscale;   // softmax_scale * log2(e)
    int R;
    int paged, page_size, max_pages, num_pages, cap;
    int chunk, n_split, max_seq_len;
    int q_dtype, q_bytes;  // element type and bytes of q
    // shared-memory stage layout (bytes)
    int stage_bytes, off_ksz, off_vc, off_vsz, off_q, off_hdr;
    int bf_tile, bf_off_v;  // bf16 tiles: tokens per tile, offset of the V rows
    int wsm_floats;         // per-warp value-weight scratch: tokens x value groups x GQA x 2
    int64_t timeout_ns;
    int skip_tile;
};

template <int KM, int KBITS>
struct KRow {
    static constexpr int bytes = (KM == K_BF16) ? kHeadDim * 2 : kHeadDim * KBITS / 8;
};
template <int VM, int VBITS>
struct VRow {
    static constexpr int bytes = (VM == V_BF16) ? kHeadDim * 2 : kHeadDim * VBITS / 8;
};

// ---- packed f32x2 arithmetic (sm_100) --------------------------------------
__device__ __forceinline__ unsigned long long as_u64(float2 v) {
    return *reinterpret_cast<unsigned long long *>(&v);
}
__device__ __forceinline__ float2 as_f2(unsigned long long v) {
    return *reinterpret_cast<float2 *>(&v);
}
// d = a * b + d, two lanes
__device__ __forceinline__ void ffma2(float2 &d, float2 a, float2 b) {
    unsigned long long r = as_u64(d);
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(r) : "l"(as_u64(a)), "l"(as_u64(b)));
    d = as_f2(r);
}

// ---- shared-memory loads ----------------------------------------------------
// Plain typed loads: the compiler sees their dependence on the stores and on
// the mbarrier waits (asm with a memory clobber) and keeps them in order; the
// pointers all derive from the kernel's shared array.
__device__ __forceinline__ uint32_t lds32(const void *p) { return *static_cast<const uint32_t *>(p); }
__device__ __forceinline__ uint32_t lds16(const void *p) { return *static_cast<const uint16_t *>(p); }
__device__ __forceinline__ uint2 lds64(const void *p) { return *static_cast<const uint2 *>(p); }
__device__ __forceinline__ uint4 lds128(const void *p) { return *static_cast<const uint4 *>(p); }
__device__ __forceinline__ float2 half2_lds(const void *p) {
    const uint32_t u = lds32(p);
    return __half22float2(*reinterpret_cast<const __half2 *>(&u));
}

// ---- code -> float ----------------------------------------------------------
// A byte value X < 128 placed into bits 16..22 of 0.5 gives the float
// 0.5 + X/256 exactly (bit 23, the exponent's low bit, stays 0). One PRMT.
// Every encoded byte below is < 128: INT4 codes are split into their low and
// high nibble planes; INT2 codes use the planes
//   X0 = c0, X1 = c0 + 4c1, X2 = c0 + 4c1 + 16c2, X3 = c1 + 4c2 + 16c3
// (three masks and one shift of the packed word), all < 64. The floats are
// linear in the codes; the query is transformed once per item so that its dot
// product with them is the dot product with the codes (query_coeffs), and the
// value accumulators are untangled once per item (value_channels).
__device__ __forceinline__ float byte_f(uint32_t b, int k) {
    return __uint_as_float(__byte_perm(b, 0x3F000000u, 0x7054u | (static_cast<uint32_t>(k) << 8)));
}

// 16 key channels [16*part, 16*part + 16) as 8 float pairs.
//   INT4 byte k (channels lo, hi): {f(lo), f(hi)}
//   INT2 byte k (channels c0..c3): {f(X0), f(X1)}, {f(X2), f(X3)}
//   bf16: the channel values themselves.
template <int KM, int KBITS>
__device__ __forceinline__ void key_pairs(const uint8_t *row, int part, float2 f[8]) {
    if constexpr (KM == K_BF16) {
        const uint4 a = lds128(row + part * 32), b = lds128(row + part * 32 + 16);
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) f[j] = make_float2(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xFFFF0000u));
    } else if constexpr (KBITS == 4) {
        const uint2 w = lds64(row + part * 8);
        const uint32_t a0 = w.x & 0x0F0F0F0Fu, b0 = (w.x >> 4) & 0x0F0F0F0Fu;
        const uint32_t a1 = w.y & 0x0F0F0F0Fu, b1 = (w.y >> 4) & 0x0F0F0F0Fu;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            f[k] = make_float2(byte_f(a0, k), byte_f(b0, k));
            f[4 + k] = make_float2(byte_f(a1, k), byte_f(b1, k));
        }
    } else {
        const uint32_t w = lds32(row + part * 4);
        const uint32_t x0 = w & 0x03030303u, x1 = w & 0x0F0F0F0Fu, x2 = w & 0x3F3F3F3Fu;
        const uint32_t x3 = (w >> 2) & 0x3F3F3F3Fu;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            f[2 * k] = make_float2(byte_f(x0, k), byte_f(x1, k));
            f[2 * k + 1] = make_float2(byte_f(x2, k), byte_f(x3, k));
        }
    }
}

// 8 value channels [8*slice, 8*slice + 8) as 4 float pairs, same encoding.
template <int VM, int VBITS>
__device__ __forceinline__ void value_pairs(const uint8_t *row, int slice, float2 f[4]) {
    if constexpr (VM == V_BF16) {
        const uint4 a = lds128(row + slice * 16);
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) f[j] = make_float2(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xFFFF0000u));
    } else if constexpr (VBITS == 4) {
        const uint32_t w = lds32(row + slice * 4);
        const uint32_t a = w & 0x0F0F0F0Fu, b = (w >> 4) & 0x0F0F0F0Fu;
#pragma unroll
        for (int k = 0; k < 4; ++k) f[k] = make_float2(byte_f(a, k), byte_f(b, k));
    } else {
        const uint32_t w = lds16(row + slice * 2);
        const uint32_t x0 = w & 0x0303u, x1 = w & 0x0F0Fu, x2 = w & 0x3F3Fu, x3 = (w >> 2) & 0x3F3Fu;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            f[2 * k] = make_float2(byte_f(x0, k), byte_f(x1, k));
            f[2 * k + 1] = make_float2(byte_f(x2, k), byte_f(x3, k));
        }
    }
}

// Query coefficients for 16 channels x[0..15] of one head, in the pair
// layout of key_pairs and times 256, such that
//   sum_j qk[j] . f[j] = 128 * first + sum_i x_i c_i,
// `first` being the sum of the (unscaled) coefficients.
template <int KM, int KBITS>
__device__ __forceinline__ void query_coeffs(const float x[16], float2 qk[8], float &first) {
    first = 0.0f;
    if constexpr (KM == K_BF16) {
#pragma unroll
        for (int j = 0; j < 8; ++j) qk[j] = make_float2(x[2 * j], x[2 * j + 1]);
    } else if constexpr (KBITS == 4) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            qk[j] = make_float2(256.0f * x[2 * j], 256.0f * x[2 * j + 1]);
            first += x[2 * j] + x[2 * j + 1];
        }
    } else {
        // a0 X0 + a1 X1 + a2 X2 + a3 X3 = q0 c0 + q1 c1 + q2 c2 + q3 c3
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float q0 = x[4 * k], q1 = x[4 * k + 1], q2 = x[4 * k + 2], q3 = x[4 * k + 3];
            const float a3 = q3 * 0.0625f;
            const float a2 = (q2 - 4.0f * a3) * 0.0625f;
            const float a1 = (q1 - 4.0f * a2 - a3) * 0.25f;
            const float a0 = q0 - a1 - a2;
            qk[2 * k] = make_float2(256.0f * a0, 256.0f * a1);
            qk[2 * k + 1] = make_float2(256.0f * a2, 256.0f * a3);
            first += (a0 + a1) + (a2 + a3);
        }
    }
}

// Untangle one slice's value accumulators into its 8 channel sums
// sum_t w_t c_t (without the zero-point term); W = sum_t w_t of its group.
template <int VM, int VBITS>
__device__ __forceinline__ void value_channels(const float2 o[4], float W, float out[8]) {
    if constexpr (VM == V_BF16) {
#pragma unroll
        for (int c = 0; c < 4; ++c) { out[2 * c] = o[c].x; out[2 * c + 1] = o[c].y; }
    } else if constexpr (VBITS == 4) {
        // acc = sum w (0.5 + c/256)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            out[2 * c] = fmaf(256.0f, o[c].x, -128.0f * W);
            out[2 * c + 1] = fmaf(256.0f, o[c].y, -128.0f * W);
        }
    } else {
        // acc_i = sum w (0.5 + X_i/256) with the X planes of value_pairs
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            const float2 a = o[2 * b], c = o[2 * b + 1];
            out[4 * b] = fmaf(256.0f, a.x, -128.0f * W);
            out[4 * b + 1] = 64.0f * (a.y - a.x);
            out[4 * b + 2] = 16.0f * (c.x - a.y);
            out[4 * b + 3] = fmaf(16.0f, c.y, -8.0f * W) - 4.0f * (c.x - a.x);
        }
    }
}

template <int GQA>
__device__ __forceinline__ void load_sums(const float *p, float v[GQA]) {
    if constexpr (GQA == 4) {
        const uint4 u = lds128(p);
        v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y);
        v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
    } else {
#pragma unroll
        for (int g = 0; g < GQA; ++g) v[g] = p[g];
    }
}

template <int GQA>
struct LaneMap {
    static constexpr int kPerHead = 8 / GQA;  // lanes of a token per head
    static constexpr int kOwnShift = (GQA == 4) ? 1 : (GQA == 2 ? 2 : 3);
};

// Group-size geometry: compile-time when GK/GV > 0, else from the params.
template <int GK, int GV, int GQA>
struct Geo {
    int gk_log2, gv_log2;
    __device__ __forceinline__ int ngk() const { return GK ? kHeadDim / GK : kHeadDim >> gk_log2; }
    __device__ __forceinline__ int nvg() const { return GV ? kHeadDim / GV : kHeadDim >> gv_log2; }
    __device__ __forceinline__ int kgroup(int part) const { return GK ? (part * 16) / GK : (part * 16) >> gk_log2; }
    __device__ __forceinline__ int vgroup(int slice) const { return GV ? (slice * 8) / GV : (slice * 8) >> gv_log2; }
    __device__ __forceinline__ bool k_whole() const { return GK ? GK == kHeadDim : gk_log2 == 7; }
    // value-group slots per owner lane
    static constexpr int kVSlots =
        GV ? ((kHeadDim / GV + LaneMap<GQA>::kPerHead - 1) / LaneMap<GQA>::kPerHead) : 4;
};

// Per-warp decode state of the current item.
template <int GQA, int VSLOTS>
struct WarpState {
    float m_own;           // running max (log2 domain) used for this lane's head
    float l_own;           // running sum of the weights of this lane's tokens (own head)
    float wsum[VSLOTS];    // value groups owned by this lane: sum of p*s (own head)
    float zsum[VSLOTS];    //                                   sum of p*z
    float2 o[GQA][4];      // value accumulators: 8 channels (4 pairs) x GQA heads
};

// Scores are kept in log2 units; a new tile maximum only moves the reference
// when it exceeds the old one by more than this (weights then stay <= 2^8).
constexpr float kRescaleSlack = 8.0f;

// Per-lane query data for the key pass. Per-lane sums the inner loop needs
// once per pass live in shared memory (qsum, [8 parts][3][GQA] floats, head
// order as in qk): [0] sum of q, [1] sum of the code-byte coefficients,
// [2] channel-wise groups: sum q z - 128 * coefficient sum of q s.
template <int GQA>
struct QueryRegs {
    float2 qk[GQA][8];     // coefficients, head order permuted for the reduce-scatter
    float qa_own, qe_own;  // groups of 128: whole-head sums of the lane's own head
};

// One tile: rows at kc / ks / vc / vs (shared memory), `n` valid tokens, TPW
// tokens per warp (warp w owns tile tokens [w*TPW, w*TPW + TPW)). FULL: all
// 4*TPW tokens are valid, so no token needs masking.
template <int GQA, int KM, int VM, int KBITS, int VBITS, int TPW, int GK, int GV, int VSLOTS, bool FULL>
__device__ __forceinline__ void process_tile(const uint8_t *kc, const uint8_t *ks,
                                             const uint8_t *vc, const uint8_t *vs, int n,
                                             const Geo<GK, GV, GQA> geo, const QueryRegs<GQA> &Q,
                                             const float *qsum, WarpState<GQA, VSLOTS> &st,
                                             float *wsm, int warp, int lane) {
    constexpr int KROW = KRow<KM, KBITS>::bytes;
    constexpr int VROW = VRow<VM, VBITS>::bytes;
    constexpr int PASSES = TPW / 4;
    constexpr int kPerHead = LaneMap<GQA>::kPerHead;
    constexpr int kOwnShift = LaneMap<GQA>::kOwnShift;
    const int i = lane >> 3, part = lane & 7;
    const int h_own = part >> kOwnShift;
    const int r_own = part & (kPerHead - 1);  // rank of this lane among its head's lanes
    const int n_vg = (VM == V_BF16) ? 1 : geo.nvg();
    const int ngk = (KM == K_TOKEN) ? geo.ngk() : 0;
    const bool post_scale = (KM == K_TOKEN) && geo.k_whole();
    const int t_warp = warp * TPW;

    // ---- scores ----
    float sc[PASSES];
#pragma unroll
    for (int pass = 0; pass < PASSES; ++pass) {
        const int tt = t_warp + pass * 4 + i;
        const int tr = (FULL || tt < n) ? tt : 0;  // masked tokens read row 0 (always staged)
        float2 f[8];
        key_pairs<KM, KBITS>(kc + tr * KROW, part, f);
        float acc[GQA];
#pragma unroll
        for (int g = 0; g < GQA; ++g) {
            float2 a = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int j = 0; j < 8; ++j) ffma2(a, Q.qk[g][j], f[j]);
            acc[g] = a.x + a.y;
        }
        float2 szf = make_float2(0.0f, 0.0f);
        if constexpr (KM == K_TOKEN) {
            szf = half2_lds(ks + (tr * ngk + (post_scale ? 0 : geo.kgroup(part))) * 4);
            if (!post_scale) {
                float qa[GQA], qe[GQA];
                load_sums<GQA>(qsum + (part * 3 + 0) * GQA, qa);
                load_sums<GQA>(qsum + (part * 3 + 1) * GQA, qe);
#pragma unroll
                for (int g = 0; g < GQA; ++g)
                    acc[g] = fmaf(szf.x, fmaf(-128.0f, qe[g], acc[g]), szf.y * qa[g]);
            }
        } else if constexpr (KM == K_CHANNEL) {
            float qc[GQA];
            load_sums<GQA>(qsum + (part * 3 + 2) * GQA, qc);
#pragma unroll
            for (int g = 0; g < GQA; ++g) acc[g] += qc[g];
        }
        float val;
        if constexpr (GQA == 4) {
            // heads are held in the order g ^ (2*b2 + b1), so no selects
            const float ka = acc[0] + __shfl_xor_sync(0xffffffffu, acc[2], 4);
            const float kb = acc[1] + __shfl_xor_sync(0xffffffffu, acc[3], 4);
            val = ka + __shfl_xor_sync(0xffffffffu, kb, 2);
            val += __shfl_xor_sync(0xffffffffu, val, 1);
        } else {
#pragma unroll
            for (int g = 0; g < GQA; ++g) {
#pragma unroll
                for (int m = 1; m < 8; m <<= 1) acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], m);
            }
            val = acc[0];
#pragma unroll
            for (int g = 1; g < GQA; ++g)
                if (h_own == g) val = acc[g];
        }
        if constexpr (KM == K_TOKEN) {
            if (post_scale) val = fmaf(szf.x, fmaf(-128.0f, Q.qe_own, val), szf.y * Q.qa_own);
        }
        sc[pass] = (FULL || tt < n) ? val : -INFINITY;
    }

    // ---- online softmax (per warp, per head), lazy rescaling ----
    float mx = sc[0];
#pragma unroll
    for (int pass = 1; pass < PASSES; ++pass) mx = fmaxf(mx, sc[pass]);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    float alpha = 1.0f;
    if (mx > st.m_own + kRescaleSlack) {   // also true the first time (m_own = -inf)
        alpha = fast_exp2(st.m_own - mx);  // 0 when m_own = -inf
        st.m_own = mx;
    }
    // reference 0 while no token of this warp has been seen (all sc = -inf)
    const float mref = (st.m_own == -INFINITY) ? 0.0f : st.m_own;
    float p[PASSES];
#pragma unroll
    for (int k = 0; k < PASSES; ++k) p[k] = fast_exp2(sc[k] - mref);  // 0 for masked
    float psum = p[0];
#pragma unroll
    for (int k = 1; k < PASSES; ++k) psum += p[k];
    st.l_own = fmaf(st.l_own, alpha, psum);
#pragma unroll
    for (int c = 0; c < VSLOTS; ++c) {
        st.wsum[c] *= alpha;
        st.zsum[c] *= alpha;
    }
    // Value weights w = p * s per (token, value group), stored as a pair; the
    // lanes of a head split the groups between them.
#pragma unroll
    for (int pass = 0; pass < PASSES; ++pass) {
        const int j = pass * 4 + i;  // warp-local token index
        const int tt = t_warp + j;
        const int tr = (FULL || tt < n) ? tt : 0;
        float2 *wrow = reinterpret_cast<float2 *>(wsm) + j * n_vg * GQA;
        if constexpr (VM == V_BF16) {
            if (r_own == 0) wrow[h_own] = make_float2(p[pass], p[pass]);
        } else {
#pragma unroll
            for (int c = 0; c < VSLOTS; ++c) {
                const int gv = r_own + c * kPerHead;
                if (gv < n_vg) {
                    const float2 szf = half2_lds(vs + (tr * n_vg + gv) * 4);
                    const float w = p[pass] * szf.x;
                    st.wsum[c] += w;
                    st.zsum[c] = fmaf(p[pass], szf.y, st.zsum[c]);
                    wrow[gv * GQA + h_own] = make_float2(w, w);
                }
            }
        }
    }
    float alpha_g[GQA];
    bool rescale = false;
#pragma unroll
    for (int g = 0; g < GQA; ++g) {
        alpha_g[g] = __shfl_sync(0xffffffffu, alpha, g << kOwnShift);
        rescale |= alpha_g[g] != 1.0f;
    }
    __syncwarp();

    // ---- values ----
    const int slice = lane & 15, parity = lane >> 4;
    if (rescale) {
#pragma unroll
        for (int g = 0; g < GQA; ++g)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                st.o[g][c].x *= alpha_g[g];
                st.o[g][c].y *= alpha_g[g];
            }
    }
    const int gv_lane = (VM == V_BF16) ? 0 : geo.vgroup(slice);
#pragma unroll
    for (int k = 0; k < TPW / 2; ++k) {
        const int j = 2 * k + parity;
        const int tt = t_warp + j;
        if (VM == V_BF16 && !FULL && tt >= n) continue;  // stale bf16 rows may be NaN
        float2 f[4];
        value_pairs<VM, VBITS>(vc + tt * VROW, slice, f);
        const float2 *wrow = reinterpret_cast<const float2 *>(wsm) + (j * n_vg + gv_lane) * GQA;
        float2 w[GQA];
        if constexpr (GQA >= 2) {
#pragma unroll
            for (int g = 0; g < GQA; g += 2) {
                const uint4 u = lds128(wrow + g);
                w[g] = make_float2(__uint_as_float(u.x), __uint_as_float(u.y));
                w[g + 1] = make_float2(__uint_as_float(u.z), __uint_as_float(u.w));
            }
        } else {
            const uint2 u = lds64(wrow);
            w[0] = make_float2(__uint_as_float(u.x), __uint_as_float(u.y));
        }
#pragma unroll
        for (int g = 0; g < GQA; ++g)
#pragma unroll
            for (int c = 0; c < 4; ++c) ffma2(st.o[g][c], w[g], f[c]);
    }
    __syncwarp();
}

// Decode an item index into (sequence, KV head, split): items are numbered
// sequence-major, pref[s] = first item of sequence s.
__device__ __forceinline__ void item_coords(const int *pref, int S, int H, int item, int &seq,
                                            int &kvh, int &split) {
    int lo = 0, hi = S;  // last s with pref[s] <= item
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (pref[mid] <= item) lo = mid; else hi = mid;
    }
    seq = lo;
    const int r = item - pref[lo];
    split = r / H;
    kvh = r - split * H;
}

template <int GQA, int KM, int VM, int KBITS, int VBITS, int NS, int GK, int GV>
__global__ void __launch_bounds__(kThreads, KVQ_DECODE_MIN_BLOCKS) decode_splitk_kernel(const DecodeParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    using G = Geo<GK, GV, GQA>;
    constexpr int VSLOTS = G::kVSlots;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const G geo{p.gk_log2, p.gv_log2};

    uint8_t *stages = smem;
    uint8_t *tail = smem + static_cast<size_t>(NS) * p.stage_bytes;
    float *qs = reinterpret_cast<float *>(tail);                    // [GQA][128]
    // value weights per warp: [token of the warp][value group][GQA][2]
    float *wsm_all = qs + GQA * kHeadDim;
    float *red = wsm_all + kConsumerWarps * p.wsm_floats;            // [4][GQA][130]
    float *qsum_all = red + kConsumerWarps * GQA * 130;              // [4][8][3][GQA]
    float *qhead = qsum_all + kConsumerWarps * 8 * 3 * GQA;          // [2][GQA]
    uint64_t *full = reinterpret_cast<uint64_t *>(qhead + 2 * GQA + 2);
    uint64_t *empty = full + NS;
    int *abort_word = reinterpret_cast<int *>(empty + NS);
    volatile int *abort_flag = abort_word;
    int *pref = abort_word + 4;  // [S + 1]

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // A dependent launch (the merge pass) may be scheduled from now on; it
    // waits for this grid's completion before reading anything.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == kConsumerWarps) {
        // ------------------------- producer -------------------------
        // Item prefix over sequences: sequence s has H * ceil(T_s / chunk) items.
        int carry = 0;
        for (int base = 0; base < p.S; base += 32) {
            const int s = base + lane;
            int cnt = 0;
            if (s < p.S) {
                int T = __ldg(p.seq_lens + s);
                if (T > p.max_seq_len) {
                    if (blockIdx.x == 0) status_or(p.status, KVQ_DEV_SEQLEN);
                    T = p.max_seq_len;
                }
                cnt = T > 0 ? p.H * ((T + p.chunk - 1) / p.chunk) : 0;
            }
            int incl = cnt;
#pragma unroll
            for (int m = 1; m < 32; m <<= 1) {
                const int o = __shfl_up_sync(0xffffffffu, incl, m);
                if (lane >= m) incl += o;
            }
            if (s < p.S) pref[s] = carry + incl - cnt;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) pref[p.S] = carry;
        __syncwarp();
        if (lane != 0) return;
        const int n_items = carry;

        constexpr int KROW = KRow<KM, KBITS>::bytes;
        constexpr int VROW = VRow<VM, VBITS>::bytes;
        const int ngk = (KM == K_TOKEN) ? geo.ngk() : 0;
        const int ngv = (VM == V_TOKEN) ? geo.nvg() : 0;
        int it = 0;  // tile counter of this CTA (stage it % NS, round it / NS)
        bool stop = false;
        // Quantized tiles never straddle a block of per-channel key scales.
        const int qtile = (KM == K_CHANNEL) ? min(kTile, p.R) : kTile;
        while (!stop) {
            const int item = atomicAdd(p.counter, 1);
            int seq = 0, kvh = 0, split = 0;
            int t_begin = 0, t_end = 0, Tq = 0, q_end = 0, n_qt = 0, w_begin = 0, n_wt = 0;
            if (item < n_items) {
                item_coords(pref, p.S, p.H, item, seq, kvh, split);
                const int T = min(__ldg(p.seq_lens + seq), p.max_seq_len);
                t_begin = split * p.chunk;
                t_end = min(T, t_begin + p.chunk);
                Tq = quantized_len(T, p.R);
                q_end = min(t_end, Tq);
                n_qt = q_end > t_begin ? (q_end - t_begin + qtile - 1) / qtile : 0;
                w_begin = max(t_begin, Tq);
                n_wt = t_end > w_begin ? (t_end - w_begin + p.bf_tile - 1) / p.bf_tile : 0;
            }
            const int n_tiles = (item < n_items) ? n_qt + n_wt : 1;  // 1 = the done marker
            const int64_t sh = static_cast<int64_t>(seq) * p.H + kvh;
            for (int ti = 0; ti < n_tiles; ++ti, ++it) {
                const int s = it % NS, r = it / NS;
                if (r > 0 &&
                    !mbar_wait_bounded(&empty[s], (r - 1) & 1, p.timeout_ns, p.status, abort_flag)) {
                    stop = true;
                    break;
                }
                uint8_t *st = stages + static_cast<size_t>(s) * p.stage_bytes;
                uint64_t *bar = &full[s];
                TileHdr *hdr = reinterpret_cast<TileHdr *>(st + p.off_hdr);
                if (item >= n_items) {  // no work left: tell the consumers
                    hdr->flags = kDone;
                    mbar_arrive(bar);
                    stop = true;
                    ++it;
                    break;
                }
                if (it == p.skip_tile) continue;  // test hook: never arrive
                const bool window = ti >= n_qt;
                const int t0 = window ? w_begin + (ti - n_qt) * p.bf_tile : t_begin + ti * qtile;
                const int n = window ? min(p.bf_tile, t_end - t0) : min(qtile, q_end - t0);
                hdr->seq = seq;
                hdr->kvh = kvh;
                hdr->split = split;
                hdr->t0 = t0;
                hdr->n = n;
                hdr->flags = (ti == 0 ? kFirst : 0) | (ti == n_tiles - 1 ? kLast : 0) | (window ? kWindow : 0);
                const uint32_t qb = (ti == 0) ? GQA * kHeadDim * p.q_bytes : 0;
                const uint8_t *qsrc = static_cast<const uint8_t *>(p.q) +
                                      ((static_cast<int64_t>(seq) * p.Hq + kvh * GQA) * kHeadDim) * p.q_bytes;
                if (window) {
                    const uint32_t bytes = n * kHeadDim * 2;
                    const int64_t slot = sh * p.R + (t0 - Tq);
                    mbar_arrive_expect_tx(bar, 2 * bytes + qb);
                    bulk_g2s(st, p.k_res + slot * kHeadDim, bytes, bar);
                    bulk_g2s(st + p.bf_off_v, p.v_res + slot * kHeadDim, bytes, bar);
                } else if (!p.paged) {
                    const int64_t row = sh * p.cap + t0;
                    const uint32_t kb = n * KROW, vb = n * VROW;
                    const uint32_t kzb = (KM == K_TOKEN) ? ((n * ngk * 4 + 15) & ~15)
                                                         : (KM == K_CHANNEL ? kHeadDim * 4 : 0);
                    const uint32_t vzb = (VM == V_TOKEN) ? ((n * ngv * 4 + 15) & ~15) : 0;
                    mbar_arrive_expect_tx(bar, kb + vb + kzb + vzb + qb);
                    bulk_g2s(st, p.k_codes + row * KROW, kb, bar);
                    bulk_g2s(st + p.off_vc, p.v_codes + row * VROW, vb, bar);
                    if (KM == K_TOKEN) bulk_g2s(st + p.off_ksz, p.k_sz + row * ngk, kzb, bar);
                    if (KM == K_CHANNEL)
                        bulk_g2s(st + p.off_ksz, p.k_sz + (sh * (p.cap / p.R) + t0 / p.R) * kHeadDim, kzb, bar);
                    if (VM == V_TOKEN) bulk_g2s(st + p.off_vsz, p.v_sz + row * ngv, vzb, bar);
                } else {
                    // Paged (token-wise groups only): one copy of each part per page.
                    const int ps = p.page_size;
                    const int span = ps < kTile ? ps : kTile;  // tokens per copy
                    const uint32_t per_copy = span * (KROW + VROW + 4 * ngk + 4 * ngv);
                    const int32_t *bt = p.block_table + static_cast<int64_t>(seq) * p.max_pages;
                    uint32_t bytes = qb;
                    for (int tp = t0; tp < t0 + n; tp += span) {
                        const int pi = tp / ps;
                        const int page = (pi < p.max_pages) ? __ldg(bt + pi) : -1;
                        if (page >= 0 && page < p.num_pages) bytes += per_copy;
                        else status_or(p.status, KVQ_DEV_CAPACITY);
                    }
                    mbar_arrive_expect_tx(bar, bytes);
                    for (int tp = t0; tp < t0 + n; tp += span) {
                        const int pi = tp / ps;
                        const int page = (pi < p.max_pages) ? __ldg(bt + pi) : -1;
                        if (page < 0 || page >= p.num_pages) continue;
                        const int64_t prow = (static_cast<int64_t>(page) * p.H + kvh) * ps + (tp % ps);
                        const uint32_t dt = tp - t0;
                        bulk_g2s(st + dt * KROW, p.k_codes + prow * KROW, span * KROW, bar);
                        bulk_g2s(st + p.off_ksz + dt * ngk * 4, p.k_sz + prow * ngk, span * ngk * 4, bar);
                        bulk_g2s(st + p.off_vc + dt * VROW, p.v_codes + prow * VROW, span * VROW, bar);
                        bulk_g2s(st + p.off_vsz + dt * ngv * 4, p.v_sz + prow * ngv, span * ngv * 4, bar);
                    }
                }
                if (qb) bulk_g2s(st + p.off_q, qsrc, qb, bar);
            }
        }
        // Drain: wait for the copies of the last stages issued so none lands
        // after the CTA has gone.
        for (int j = max(0, it - NS); j < it; ++j) {
            if (j == p.skip_tile) continue;
            const int s = j % NS, r = j / NS;
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(&full[s], r & 1)) {
                if (static_cast<int64_t>(global_timer_ns() - t0) > p.timeout_ns) {
                    status_or(p.status, KVQ_DEV_TIMEOUT);
                    break;
                }
            }
        }
        return;
    }

    // --------------------------- consumers ---------------------------
    const int part = lane & 7;
    constexpr int kOwnShift = LaneMap<GQA>::kOwnShift;
    // head held in register slot g (reduce-scatter order for GQA 4)
    const int perm = (GQA == 4) ? (((part >> 2) & 1) << 1 | ((part >> 1) & 1)) : 0;
    QueryRegs<GQA> Q;
    float *qsum = qsum_all + warp * 8 * 3 * GQA;
    float *wsm = wsm_all + warp * p.wsm_floats;

    // mode: 0 = token-wise codes, 1 = channel-wise codes (per-channel scales
    // folded in from `chan_sz`), 2 = bf16 keys.
    auto load_query = [&](int mode, const uint8_t *chan_sz) {
        __syncwarp();  // this warp is done reading the previous sums
#pragma unroll
        for (int g = 0; g < GQA; ++g) {
            const int h = g ^ perm;
            float x[16];
            float qa = 0.0f, qz = 0.0f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float v = qs[h * kHeadDim + part * 16 + j];
                qa += v;
                if (mode == 1) {
                    const float2 sz = half2_lds(chan_sz + (part * 16 + j) * 4);
                    x[j] = v * sz.x;
                    qz = fmaf(v, sz.y, qz);
                } else {
                    x[j] = v;
                }
            }
            float first;
            if (mode == 2) query_coeffs<K_BF16, 16>(x, Q.qk[g], first);
            else query_coeffs<KM == K_BF16 ? K_TOKEN : KM, KBITS == 16 ? 4 : KBITS>(x, Q.qk[g], first);
            if ((lane >> 3) == 0) {
                qsum[(part * 3 + 0) * GQA + g] = qa;
                qsum[(part * 3 + 1) * GQA + g] = first;
                qsum[(part * 3 + 2) * GQA + g] = (mode == 1) ? fmaf(-128.0f, first, qz) : 0.0f;
            }
        }
        // whole-head sums of the lane's own head (written by the item prologue)
        Q.qa_own = qhead[part >> kOwnShift];
        Q.qe_own = qhead[GQA + (part >> kOwnShift)];
        __syncwarp();
    };

    WarpState<GQA, VSLOTS> st;
    bool folded = false;
    // Turn the value accumulators of quantized tiles into plain channel sums
    // (adding the zero-point terms), once: before the first bf16 window tile
    // or at the end of the item. Half-warp 1 adds no group terms, so the
    // halves still sum.
    auto fold_values = [&]() {
        constexpr int kPH = LaneMap<GQA>::kPerHead;
        float wsum[VSLOTS], zsum[VSLOTS];
#pragma unroll
        for (int c = 0; c < VSLOTS; ++c) {
            wsum[c] = st.wsum[c];
            wsum[c] += __shfl_xor_sync(0xffffffffu, wsum[c], 8);
            wsum[c] += __shfl_xor_sync(0xffffffffu, wsum[c], 16);
            zsum[c] = st.zsum[c];
            zsum[c] += __shfl_xor_sync(0xffffffffu, zsum[c], 8);
            zsum[c] += __shfl_xor_sync(0xffffffffu, zsum[c], 16);
            st.wsum[c] = 0.0f;
            st.zsum[c] = 0.0f;
        }
        const int gv_lane = geo.vgroup(lane & 15);
        const bool first_half = lane < 16;
#pragma unroll
        for (int g = 0; g < GQA; ++g) {
            // group gv of head g: lane (g << kOwnShift) + gv % kPH, slot gv / kPH
            float Wg = 0.0f, Zg = 0.0f;
#pragma unroll
            for (int c = 0; c < VSLOTS; ++c) {
#pragma unroll
                for (int r = 0; r < kPH; ++r) {
                    const float wv = __shfl_sync(0xffffffffu, wsum[c], (g << kOwnShift) + r);
                    const float zv = __shfl_sync(0xffffffffu, zsum[c], (g << kOwnShift) + r);
                    if (gv_lane == r + c * kPH) { Wg = wv; Zg = zv; }
                }
            }
            if (!first_half) { Wg = 0.0f; Zg = 0.0f; }
            float ch[8];
            value_channels<VM, VBITS>(st.o[g], Wg, ch);
#pragma unroll
            for (int c = 0; c < 4; ++c) st.o[g][c] = make_float2(ch[2 * c] + Zg, ch[2 * c + 1] + Zg);
        }
        folded = true;
    };

    int cur_block = -1;
    for (int it = 0;; ++it) {
        const int s = it % NS, r = it / NS;
        if (!mbar_wait_bounded(&full[s], r & 1, p.timeout_ns, p.status, abort_flag)) break;
        const uint8_t *sb = stages + static_cast<size_t>(s) * p.stage_bytes;
        const TileHdr hdr = *reinterpret_cast<const TileHdr *>(sb + p.off_hdr);
        if (hdr.flags & kDone) break;

        if (hdr.flags & kFirst) {
            // ---- item prologue: the query rows arrived with this tile ----
            if (warp < GQA) {
                const uint8_t *qrow = sb + p.off_q + warp * kHeadDim * p.q_bytes;
                float x[4];
                if (p.q_dtype == KVQ_FP32) {
                    const uint4 v = lds128(qrow + 16 * lane);
                    x[0] = __uint_as_float(v.x); x[1] = __uint_as_float(v.y);
                    x[2] = __uint_as_float(v.z); x[3] = __uint_as_float(v.w);
                } else {
                    const uint2 v = lds64(qrow + 8 * lane);
                    const uint32_t w[2] = {v.x, v.y};
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        if (p.q_dtype == KVQ_BF16) {
                            x[2 * j] = bf16_bits_to_float(w[j] & 0xFFFFu);
                            x[2 * j + 1] = bf16_bits_to_float(w[j] >> 16);
                        } else {
                            x[2 * j] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[j] & 0xFFFFu)));
                            x[2 * j + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[j] >> 16)));
                        }
                    }
                }
                if (p.hb > 0) {
                    if (p.hb > 1) { float a = x[0], b = x[1]; x[0] = a + b; x[1] = a - b;
                                    a = x[2]; b = x[3]; x[2] = a + b; x[3] = a - b; }
                    if (p.hb > 2) { float a = x[0], b = x[2]; x[0] = a + b; x[2] = a - b;
                                    a = x[1]; b = x[3]; x[1] = a + b; x[3] = a - b; }
                    for (int m = 1; m < 32 && 4 * m < p.hb; m <<= 1) {
                        const bool upper = (lane & m) != 0;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float o = __shfl_xor_sync(0xffffffffu, x[j], m);
                            x[j] = upper ? o - x[j] : x[j] + o;
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) x[j] *= p.hscale;
                }
                float sa = 0.0f, se = 0.0f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    x[j] *= p.qscale;
                    qs[warp * kHeadDim + 4 * lane + j] = x[j];
                    sa += x[j];
                    // sum of the code-byte coefficients: all q (INT4), q0 + q3/16 (INT2)
                    se += (KBITS != 2) ? x[j] : (j == 0 ? x[j] : (j == 3 ? 0.0625f * x[j] : 0.0f));
                }
#pragma unroll
                for (int m = 1; m < 32; m <<= 1) {
                    sa += __shfl_xor_sync(0xffffffffu, sa, m);
                    se += __shfl_xor_sync(0xffffffffu, se, m);
                }
                if (lane == 0) {
                    qhead[warp] = sa;
                    qhead[GQA + warp] = se;
                }
            }
            named_sync(1, kConsumers);
            cur_block = -1;
            if constexpr (KM != K_CHANNEL) load_query(KM == K_BF16 ? 2 : 0, nullptr);
            st.m_own = -INFINITY;
            st.l_own = 0.0f;
#pragma unroll
            for (int c = 0; c < VSLOTS; ++c) { st.wsum[c] = 0.0f; st.zsum[c] = 0.0f; }
#pragma unroll
            for (int g = 0; g < GQA; ++g)
#pragma unroll
                for (int c = 0; c < 4; ++c) st.o[g][c] = make_float2(0.0f, 0.0f);
            folded = false;
        }

        if (!(hdr.flags & kWindow)) {
            if constexpr (KM == K_CHANNEL) {
                const int blk = hdr.t0 / p.R;
                if (blk != cur_block) {  // fold this block's channel scales into q
                    cur_block = blk;
                    load_query(1, sb + p.off_ksz);
                }
            }
            if (hdr.n == kTile)
                process_tile<GQA, KM, VM, KBITS, VBITS, kTokensPerWarp, GK, GV, VSLOTS, true>(
                    sb, sb + p.off_ksz, sb + p.off_vc, sb + p.off_vsz, hdr.n, geo, Q, qsum, st, wsm,
                    warp, lane);
            else
                process_tile<GQA, KM, VM, KBITS, VBITS, kTokensPerWarp, GK, GV, VSLOTS, false>(
                    sb, sb + p.off_ksz, sb + p.off_vc, sb + p.off_vsz, hdr.n, geo, Q, qsum, st, wsm,
                    warp, lane);
        } else if constexpr (KM != K_BF16) {
            if (!folded) {  // first window tile of the item
                load_query(2, nullptr);
                if (VM == V_TOKEN) fold_values();
                folded = true;
            }
            process_tile<GQA, K_BF16, V_BF16, 16, 16, kWinTile / kConsumerWarps, GK, GV, VSLOTS, false>(
                sb, nullptr, sb + p.bf_off_v, nullptr, hdr.n, geo, Q, qsum, st, wsm, warp, lane);
        }

        if (hdr.flags & kLast) {
            // ---- item epilogue: merge the four warps, write the partial ----
            if (VM == V_TOKEN && !folded) fold_values();
            float l_own = st.l_own;
            l_own += __shfl_xor_sync(0xffffffffu, l_own, 8);
            l_own += __shfl_xor_sync(0xffffffffu, l_own, 16);
            const int slice = lane & 15;
#pragma unroll
            for (int g = 0; g < GQA; ++g) {
                const float mg = __shfl_sync(0xffffffffu, st.m_own, g << kOwnShift);
                const float lg = __shfl_sync(0xffffffffu, l_own, g << kOwnShift);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float2 v = st.o[g][c];
                    v.x += __shfl_xor_sync(0xffffffffu, v.x, 16);
                    v.y += __shfl_xor_sync(0xffffffffu, v.y, 16);
                    if (lane < 16) {
                        red[(warp * GQA + g) * 130 + 8 * slice + 2 * c] = v.x;
                        red[(warp * GQA + g) * 130 + 8 * slice + 2 * c + 1] = v.y;
                    }
                }
                if (lane == 0) {
                    red[(warp * GQA + g) * 130 + 128] = mg;
                    red[(warp * GQA + g) * 130 + 129] = lg;
                }
            }
            named_sync(1, kConsumers);
            for (int idx = tid; idx < GQA * kHeadDim; idx += kConsumers) {
                const int g = idx / kHeadDim, d = idx - g * kHeadDim;
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, red[(w * GQA + g) * 130 + 128]);
                float o = 0.0f, l = 0.0f;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) {
                    const float mw = red[(w * GQA + g) * 130 + 128];
                    const float e = (mw == -INFINITY) ? 0.0f : fast_exp2(mw - M);
                    o = fmaf(e, red[(w * GQA + g) * 130 + d], o);
                    l = fmaf(e, red[(w * GQA + g) * 130 + 129], l);
                }
                const int hq = hdr.kvh * GQA + g;
                const int64_t pi = (static_cast<int64_t>(hdr.seq) * p.Hq + hq) * p.n_split + hdr.split;
                p.o_part[pi * kHeadDim + d] = o;
                if (d == 0) p.ml[pi] = make_float2(M, l);
            }
        }
        if (lane == 0) mbar_arrive(&empty[s]);
    }
}

// One CTA of 128 threads per (query head, sequence): combine the splits.
// Launched as a programmatic dependent of the split-K pass: its CTAs may start
// while that pass drains and wait here until its partials are complete.
__global__ void __launch_bounds__(128) decode_merge_kernel(const float *o_part, const float2 *ml,
                                                           const int32_t *seq_lens, float *out,
                                                           int Hq, int n_split, int chunk,
                                                           int max_seq_len) {
    __shared__ float s_max;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int hq = blockIdx.x, seq = blockIdx.y, d = threadIdx.x;
    const int T = min(__ldg(seq_lens + seq), max_seq_len);
    const int nv = T > 0 ? (T + chunk - 1) / chunk : 0;
    const int64_t base = (static_cast<int64_t>(seq) * Hq + hq) * n_split;
    if (d < 32) {  // maximum over the splits, one warp
        float m = -INFINITY;
        for (int j = d; j < nv; j += 32) m = fmaxf(m, ml[base + j].x);
#pragma unroll
        for (int k = 16; k > 0; k >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, k));
        if (d == 0) s_max = m;
    }
    __syncthreads();
    const float M = s_max;
    float o = 0.0f, l = 0.0f;
    const float *op = o_part + base * kHeadDim + d;
#pragma unroll 4
    for (int j = 0; j < nv; ++j) {
        const float2 v = ml[base + j];
        const float e = (v.x == -INFINITY) ? 0.0f : fast_exp2(v.x - M);
        o = fmaf(e, op[static_cast<int64_t>(j) * kHeadDim], o);
        l = fmaf(e, v.y, l);
    }
    out[(static_cast<int64_t>(seq) * Hq + hq) * kHeadDim + d] = (l > 0.0f) ? o / l : 0.0f;
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
struct StageLayout {
    int bytes, off_ksz, off_vc, off_vsz, off_q, off_hdr, bf_tile, bf_off_v;
};

inline int round16(int x) { return (x + 15) & ~15; }

// Stage: tile data, then the query rows of a first tile (GQA x 128 x q_bytes,
// at most 2 KB), then a 32-byte header.
StageLayout stage_layout(const kvq_cache_desc &d, int gqa, int q_bytes) {
    StageLayout L{};
    int data;
    if (d.bits_k == 16) {  // every tile is bf16 rows: K at 0, V after it
        L.bf_tile = kTile;
        L.bf_off_v = kTile * 256;
        L.off_vc = L.bf_off_v;
        data = 2 * kTile * 256;
    } else {
        const int krow = 128 * d.bits_k / 8;
        const int vrow = 128 * d.bits_v / 8;
        const int ksz = (d.axis_k == KVQ_PER_CHANNEL) ? 128 * 4 : kTile * (128 / d.group_k) * 4;
        const int vsz = kTile * (128 / d.group_v) * 4;
        L.off_ksz = round16(kTile * krow);
        L.off_vc = L.off_ksz + round16(ksz);
        L.off_vsz = L.off_vc + round16(kTile * vrow);
        data = L.off_vsz + round16(vsz);
        L.bf_tile = kWinTile;
        L.bf_off_v = kWinTile * 256;
        if (d.residual_len > 0) data = std::max(data, 2 * kWinTile * 256);
    }
    L.off_q = round16(data);
    L.off_hdr = L.off_q + round16(gqa * kHeadDim * q_bytes);
    L.bytes = (L.off_hdr + static_cast<int>(sizeof(TileHdr)) + 127) & ~127;
    return L;
}

template <int GQA>
size_t tail_bytes(int NS, int S, int wsm_floats) {
    return sizeof(float) * (GQA * kHeadDim + kConsumerWarps * wsm_floats +
                            kConsumerWarps * GQA * 130 + kConsumerWarps * 8 * 3 * GQA + 2 * GQA + 2) +
           sizeof(uint64_t) * 2 * NS + 16 + sizeof(int) * (S + 1);
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

template <int GQA, int KM, int VM, int KBITS, int VBITS, int GK, int GV>
kvq_status launch_variant(const DecodeParams &p, int max_items, cudaStream_t stream) {
    constexpr int NS = (KM == K_BF16) ? 3 : 4;
    const size_t smem = static_cast<size_t>(NS) * p.stage_bytes + tail_bytes<GQA>(NS, p.S, p.wsm_floats);
    auto kern = decode_splitk_kernel<GQA, KM, VM, KBITS, VBITS, NS, GK, GV>;
    if (smem > 227 * 1024) return KVQ_ERR_UNSUPPORTED;  // too many sequences for one launch
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return KVQ_ERR_CUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem) != cudaSuccess ||
        per_sm <= 0)
        per_sm = 1;
    const int grid = std::max(1, std::min(max_items, per_sm * sm_count()));
    if (cudaMemsetAsync(p.counter, 0, sizeof(int), stream) != cudaSuccess) return KVQ_ERR_CUDA;
    kern<<<grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

// Compile-time group sizes for the common shapes, runtime ones otherwise.
template <int GQA, int KM, int VM, int KBITS, int VBITS>
kvq_status launch_groups(const kvq_cache_desc &d, const DecodeParams &p, int max_items,
                         cudaStream_t stream) {
    if constexpr (GQA == 4 && VM == V_TOKEN) {
        const int gk = (KM == K_TOKEN) ? d.group_k : 0;
        if (KM == K_TOKEN && gk == 128 && d.group_v == 128)
            return launch_variant<GQA, KM, VM, KBITS, VBITS, 128, 128>(p, max_items, stream);
        if (KM == K_TOKEN && gk == 32 && d.group_v == 32)
            return launch_variant<GQA, KM, VM, KBITS, VBITS, 32, 32>(p, max_items, stream);
        if (KM == K_CHANNEL && d.group_v == 32)
            return launch_variant<GQA, KM, VM, KBITS, VBITS, 0, 32>(p, max_items, stream);
    }
    return launch_variant<GQA, KM, VM, KBITS, VBITS, 0, 0>(p, max_items, stream);
}

template <int GQA>
kvq_status dispatch_modes(const kvq_cache_desc &d, const DecodeParams &p, int max_items,
                          cudaStream_t stream) {
    if (d.bits_k == 16 && d.bits_v == 16)
        return launch_variant<GQA, K_BF16, V_BF16, 16, 16, 0, 0>(p, max_items, stream);
    if (d.axis_k == KVQ_PER_CHANNEL) {
        if (d.bits_k == 2 && d.bits_v == 2) return launch_groups<GQA, K_CHANNEL, V_TOKEN, 2, 2>(d, p, max_items, stream);
        if (d.bits_k == 4 && d.bits_v == 4) return launch_groups<GQA, K_CHANNEL, V_TOKEN, 4, 4>(d, p, max_items, stream);
        if (d.bits_k == 2 && d.bits_v == 4) return launch_groups<GQA, K_CHANNEL, V_TOKEN, 2, 4>(d, p, max_items, stream);
        if (d.bits_k == 4 && d.bits_v == 2) return launch_groups<GQA, K_CHANNEL, V_TOKEN, 4, 2>(d, p, max_items, stream);
        return KVQ_ERR_UNSUPPORTED;
    }
    if (d.bits_k == 4 && d.bits_v == 4) return launch_groups<GQA, K_TOKEN, V_TOKEN, 4, 4>(d, p, max_items, stream);
    if (d.bits_k == 2 && d.bits_v == 2) return launch_groups<GQA, K_TOKEN, V_TOKEN, 2, 2>(d, p, max_items, stream);
    if (d.bits_k == 4 && d.bits_v == 2) return launch_groups<GQA, K_TOKEN, V_TOKEN, 4, 2>(d, p, max_items, stream);
    if (d.bits_k == 2 && d.bits_v == 4) return launch_groups<GQA, K_TOKEN, V_TOKEN, 2, 4>(d, p, max_items, stream);
    return KVQ_ERR_UNSUPPORTED;
}

int log2i(int x) {
    int r = 0;
    while ((1 << r) < x) ++r;
    return r;
}

}  // namespace

bool plan_decode(const kvq_cache_desc &d, int num_seqs, int num_q_heads, int max_seq_len,
                 DecodePlan *plan) {
    if (num_seqs <= 0 || num_q_heads <= 0 || max_seq_len < 0 || d.num_kv_heads <= 0) return false;
    // About six items per resident CTA (2 per SM) when every sequence is at
    // max_seq_len; chunks of 256..4096 tokens, a multiple of the tile.
    const int64_t units = static_cast<int64_t>(num_seqs) * d.num_kv_heads;
    const int64_t target_items = 6 * 2 * 148;
    int64_t chunk = (units * std::max(1, max_seq_len) + target_items - 1) / target_items;
    chunk = ((chunk + kTile - 1) / kTile) * kTile;
    chunk = std::min<int64_t>(std::max<int64_t>(chunk, 256), 4096);
    plan->chunk = static_cast<int>(chunk);
    plan->n_split = static_cast<int>(std::max<int64_t>(1, (max_seq_len + chunk - 1) / chunk));
    const size_t rows = static_cast<size_t>(num_seqs) * num_q_heads * plan->n_split;
    plan->ws_part = rows * kHeadDim * sizeof(float);
    plan->ws_ml = rows * sizeof(float2);
    plan->ws_total = plan->ws_part + plan->ws_ml + 16;  // + the item counter
    return true;
}

kvq_status launch_decode_splitk(const kvq_cache_desc &d, const DecodePlan &plan, const void *q,
                                kvq_dtype q_dtype, int num_q_heads, const int32_t *seq_lens,
                                int num_seqs, int max_seq_len, float softmax_scale,
                                void *workspace, cudaStream_t stream) {
    if (max_seq_len == 0) return KVQ_OK;
    DecodeParams p{};
    p.k_codes = static_cast<const uint8_t *>(d.k_codes);
    p.v_codes = static_cast<const uint8_t *>(d.v_codes);
    p.k_sz = static_cast<const __half2 *>(d.k_sz);
    p.v_sz = static_cast<const __half2 *>(d.v_sz);
    p.k_res = static_cast<const uint16_t *>(d.k_res);
    p.v_res = static_cast<const uint16_t *>(d.v_res);
    p.block_table = d.block_table;
    p.seq_lens = seq_lens;
    p.q = q;
    p.o_part = static_cast<float *>(workspace);
    p.ml = reinterpret_cast<float2 *>(static_cast<uint8_t *>(workspace) + plan.ws_part);
    p.counter = reinterpret_cast<int *>(static_cast<uint8_t *>(workspace) + plan.ws_part + plan.ws_ml);
    p.status = d.status;
    p.S = num_seqs;
    p.H = d.num_kv_heads;
    p.Hq = num_q_heads;
    p.gk_log2 = log2i(std::max(1, d.group_k));
    p.gv_log2 = log2i(std::max(1, d.group_v));
    p.hb = d.hadamard_block_k;
    p.hscale = hadamard_scale(d.hadamard_block_k);
    p.qscale = softmax_scale * kLog2e;
    p.R = d.residual_len;
    p.paged = d.paged;
    p.page_size = d.page_size;
    p.max_pages = d.max_pages_per_seq;
    p.num_pages = d.num_pages;
    p.cap = d.capacity_tokens;
    p.chunk = plan.chunk;
    p.n_split = plan.n_split;
    p.max_seq_len = max_seq_len;
    p.q_dtype = q_dtype;
    p.q_bytes = (q_dtype == KVQ_FP32) ? 4 : 2;
    const int gqa = num_q_heads / d.num_kv_heads;
    const StageLayout L = stage_layout(d, gqa, p.q_bytes);
    p.stage_bytes = L.bytes;
    p.off_ksz = L.off_ksz;
    p.off_vc = L.off_vc;
    p.off_vsz = L.off_vsz;
    p.off_q = L.off_q;
    p.off_hdr = L.off_hdr;
    p.bf_tile = L.bf_tile;
    p.bf_off_v = L.bf_off_v;
    // value groups per token: 1 for bf16 values (and for the bf16 window tiles)
    const int n_vg = (d.bits_v == 16) ? 1 : kHeadDim / d.group_v;
    p.wsm_floats = kTokensPerWarp * n_vg * gqa * 2;
    p.timeout_ns = debug_hooks().wait_timeout_ns;
    p.skip_tile = debug_hooks().skip_tile;
    const int64_t max_items64 = static_cast<int64_t>(num_seqs) * d.num_kv_heads * plan.n_split;
    const int max_items = static_cast<int>(std::min<int64_t>(max_items64, 1 << 30));
    switch (gqa) {
        case 1: return dispatch_modes<1>(d, p, max_items, stream);
        case 2: return dispatch_modes<2>(d, p, max_items, stream);
        case 4: return dispatch_modes<4>(d, p, max_items, stream);
        default: return KVQ_ERR_UNSUPPORTED;
    }
}

kvq_status launch_decode_merge(const kvq_cache_desc &d, const DecodePlan &plan, int num_q_heads,
                               const int32_t *seq_lens, int num_seqs, int max_seq_len,
                               float *out, const void *workspace, cudaStream_t stream) {
    (void)d;
    const float *o_part = static_cast<const float *>(workspace);
    const float2 *ml =
        reinterpret_cast<const float2 *>(static_cast<const uint8_t *>(workspace) + plan.ws_part);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(num_q_heads, num_seqs);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int n_split = plan.n_split, chunk = plan.chunk;
    return cudaLaunchKernelEx(&cfg, decode_merge_kernel, o_part, ml, seq_lens, out, num_q_heads,
                              n_split, chunk, max_seq_len) == cudaSuccess
               ? KVQ_OK
               : KVQ_ERR_CUDA;
}

}  // namespace kvq
