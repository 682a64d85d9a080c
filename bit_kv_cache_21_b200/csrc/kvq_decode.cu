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
// CTA = one (split, KV head, sequence): 4 consumer warps and 1 producer warp.
// The producer's elected lane stages each tile (K codes, K scale/zero, V
// codes, V scale/zero; or bf16 rows of the recent-token window) into a
// shared-memory ring with 1-D bulk copies (TMA engine, mbarrier complete_tx),
// resolving page-table indirection per page.
//
// Inner loop. The path is bound by the FP32 FMA pipe, not by the tensor
// cores: every cached element meets GQA query heads, one multiply-add each.
// So the loop is built to spend as few issue slots as possible besides those
// multiply-adds:
//   * multiply-adds are packed f32x2 FMAs (two lanes of work per issue);
//   * a 4-bit or 2-bit code c becomes the float 0.5 + c/256 with ONE byte
//     permute (the code lands in mantissa bits 16..19 of 0.5); the constant
//     0.5 is folded into the per-group zero-point terms, exactly;
//   * each consumer warp owns a quarter of every tile with its own
//     online-softmax state, so tiles need no cross-warp synchronisation;
//   * scores: 8 lanes per token, 16 channels per lane, all GQA heads at once,
//     a reduce-scatter over the 8 lanes leaves one head's score per lane pair;
//   * values: 16 lanes cover the 128 channels (8 each) for all GQA heads; the
//     two half-warps take alternate tokens.
// The four warps' states are merged once per split; the merge kernel combines
// the splits.
#include <algorithm>

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

constexpr int kTile = 64;          // tokens per quantized tile
constexpr int kWinTile = 16;       // tokens per bf16 window tile (quantized caches)
constexpr int kConsumerWarps = 4;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr float kLog2e = 1.4426950408889634f;

enum KMode { K_TOKEN = 0, K_CHANNEL = 1, K_BF16 = 2 };
enum VMode { V_TOKEN = 0, V_BF16 = 2 };

struct DecodeParams {
    const uint8_t *k_codes, *v_codes;  // packed codes, or bf16 rows (bits 16)
    const __half2 *k_sz, *v_sz;
    const uint16_t *k_res, *v_res;
    const int32_t *block_table;
    const int32_t *seq_lens;
    const void *q;
    float *o_part;  // [S][Hq][n_split][D]
    float2 *ml;     // [S][Hq][n_split]
    int32_t *status;
    int H, Hq;
    int group_k, group_v;
    int hb;
    float hscale;   // fp32(1/sqrt(hb))
    float qscale;   // softmax_scale * log2(e)
    int R;
    int paged, page_size, max_pages, num_pages, cap;
    int chunk, n_split, max_seq_len;
    int q_dtype;
    // shared-memory stage layout (bytes)
    int stage_bytes, off_ksz, off_vc, off_vsz;
    int bf_tile, bf_off_v;  // bf16 tiles: tokens per tile, offset of the V rows
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
__device__ __forceinline__ uint32_t lds32(const void *p) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_addr(p)));
    return v;
}
__device__ __forceinline__ uint32_t lds16(const void *p) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(smem_addr(p)));
    return v;
}
__device__ __forceinline__ uint2 lds64(const void *p) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(smem_addr(p)));
    return v;
}
__device__ __forceinline__ uint4 lds128(const void *p) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_addr(p)));
    return v;
}
__device__ __forceinline__ float2 half2_lds(const void *p) {
    const uint32_t u = lds32(p);
    return __half22float2(*reinterpret_cast<const __half2 *>(&u));
}

// ---- code -> float ----------------------------------------------------------
// Byte k of `b` holds a code in its low bits; the result is the float
// 0.5 + code/256 (the byte becomes mantissa bits 16..23 of 0.5). One PRMT.
__device__ __forceinline__ float code_f(uint32_t b, int k) {
    return __uint_as_float(__byte_perm(b, 0x3F000000u, 0x7054u | (static_cast<uint32_t>(k) << 8)));
}

// 16 key channels [16*part, 16*part + 16) as 8 (even, odd) pairs.
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
            f[k] = make_float2(code_f(a0, k), code_f(b0, k));
            f[4 + k] = make_float2(code_f(a1, k), code_f(b1, k));
        }
    } else {
        const uint32_t w = lds32(row + part * 4);
        const uint32_t a = w & 0x03030303u, b = (w >> 2) & 0x03030303u;
        const uint32_t c = (w >> 4) & 0x03030303u, d = (w >> 6) & 0x03030303u;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            f[2 * k] = make_float2(code_f(a, k), code_f(b, k));
            f[2 * k + 1] = make_float2(code_f(c, k), code_f(d, k));
        }
    }
}

// 8 value channels [8*slice, 8*slice + 8) as 4 pairs.
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
        for (int k = 0; k < 4; ++k) f[k] = make_float2(code_f(a, k), code_f(b, k));
    } else {
        const uint32_t w = lds16(row + slice * 2);
        const uint32_t a = w & 0x0303u, b = (w >> 2) & 0x0303u;
        const uint32_t c = (w >> 4) & 0x0303u, d = (w >> 6) & 0x0303u;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            f[2 * k] = make_float2(code_f(a, k), code_f(b, k));
            f[2 * k + 1] = make_float2(code_f(c, k), code_f(d, k));
        }
    }
}

// Per-warp decode state.
template <int GQA>
struct WarpState {
    float m_own;      // running max (log2 domain) of this lane's head
    float l_own;      // running sum of the weights of this lane's tokens (own head)
    float corr[4];    // value-group correction terms owned by this lane (own head)
    float2 o[GQA][4]; // value accumulators: 8 channels (4 pairs) x GQA heads
};

template <int GQA>
struct LaneMap {
    static constexpr int kPerHead = 8 / GQA;                 // lanes of a token per head
    static constexpr int kOwnShift = (GQA == 4) ? 1 : (GQA == 2 ? 2 : 3);
};

// One tile: rows at kc / ks / vc / vs (shared memory), `n` valid tokens, TPW
// tokens per warp (warp w owns tile tokens [w*TPW, w*TPW + TPW)).
template <int GQA, int KM, int VM, int KBITS, int VBITS, int TPW>
__device__ __forceinline__ void process_tile(const uint8_t *kc, const uint8_t *ks,
                                             const uint8_t *vc, const uint8_t *vs, int n,
                                             int group_k, int group_v, const float2 (&qk)[GQA][8],
                                             const float (&qc)[GQA], WarpState<GQA> &st,
                                             float *wsm, int warp, int lane) {
    constexpr int KROW = KRow<KM, KBITS>::bytes;
    constexpr int VROW = VRow<VM, VBITS>::bytes;
    constexpr int PASSES = TPW / 4;
    constexpr int kPerHead = LaneMap<GQA>::kPerHead;
    constexpr int kOwnShift = LaneMap<GQA>::kOwnShift;
    const int i = lane >> 3, part = lane & 7;
    const int h_own = part >> kOwnShift;
    const int r_own = part & (kPerHead - 1);  // rank of this lane among its head's lanes
    const int n_vg = (VM == V_BF16) ? 1 : kHeadDim / group_v;
    const int ngk = (KM == K_TOKEN) ? kHeadDim / group_k : 0;
    const int t_warp = warp * TPW;

    // ---- scores ----
    float sc[PASSES];
#pragma unroll
    for (int pass = 0; pass < PASSES; ++pass) {
        const int tt = t_warp + pass * 4 + i;
        float2 f[8];
        key_pairs<KM, KBITS>(kc + tt * KROW, part, f);
        float acc[GQA];
#pragma unroll
        for (int g = 0; g < GQA; ++g) {
            float2 a = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int j = 0; j < 8; ++j) ffma2(a, qk[g][j], f[j]);
            acc[g] = a.x + a.y;
        }
        if constexpr (KM == K_TOKEN) {
            const float2 szf = half2_lds(ks + (tt * ngk + (part * 16) / group_k) * 4);
            const float zc = fmaf(-128.0f, szf.x, szf.y);  // z - 128 s
#pragma unroll
            for (int g = 0; g < GQA; ++g) acc[g] = fmaf(szf.x, acc[g], zc * qc[g]);
        } else if constexpr (KM == K_CHANNEL) {
#pragma unroll
            for (int g = 0; g < GQA; ++g) acc[g] += qc[g];
        }
        float val;
        if constexpr (GQA == 4) {
            const bool b2 = (part & 4) != 0, b1 = (part & 2) != 0;
            const float s0 = b2 ? acc[0] : acc[2], s1 = b2 ? acc[1] : acc[3];
            const float r0 = __shfl_xor_sync(0xffffffffu, s0, 4);
            const float r1 = __shfl_xor_sync(0xffffffffu, s1, 4);
            const float ka = (b2 ? acc[2] : acc[0]) + r0;
            const float kb = (b2 ? acc[3] : acc[1]) + r1;
            const float r2 = __shfl_xor_sync(0xffffffffu, b1 ? ka : kb, 2);
            val = (b1 ? kb : ka) + r2;
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
        sc[pass] = tt < n ? val : -INFINITY;
    }

    // ---- online softmax (per warp, per head) ----
    float mx = sc[0];
#pragma unroll
    for (int pass = 1; pass < PASSES; ++pass) mx = fmaxf(mx, sc[pass]);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    const float m_new = fmaxf(st.m_own, mx);
    float alpha, p[PASSES];
    if (m_new == -INFINITY) {
        alpha = 1.0f;
#pragma unroll
        for (int k = 0; k < PASSES; ++k) p[k] = 0.0f;
    } else {
        alpha = fast_exp2(st.m_own - m_new);
#pragma unroll
        for (int k = 0; k < PASSES; ++k) p[k] = fast_exp2(sc[k] - m_new);
    }
    st.m_own = m_new;
    float psum = p[0];
#pragma unroll
    for (int k = 1; k < PASSES; ++k) psum += p[k];
    st.l_own = fmaf(st.l_own, alpha, psum);
    // Value weights: w = 256 * p * s per (token, value group), duplicated as a
    // pair; the owner lanes of a head split the groups between them.
#pragma unroll
    for (int c = 0; c < 4; ++c) st.corr[c] *= alpha;
#pragma unroll
    for (int pass = 0; pass < PASSES; ++pass) {
        const int j = pass * 4 + i;  // warp-local token index
        const int tt = t_warp + j;
        float2 *wrow = reinterpret_cast<float2 *>(wsm) + j * n_vg * GQA;
        if constexpr (VM == V_BF16) {
            if (r_own == 0) wrow[h_own] = make_float2(p[pass], p[pass]);
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int gv = r_own + c * kPerHead;
                if (gv < n_vg) {
                    const float2 szf = half2_lds(vs + (tt * n_vg + gv) * 4);
                    const float w = 256.0f * p[pass] * szf.x;
                    st.corr[c] = fmaf(p[pass], fmaf(-128.0f, szf.x, szf.y), st.corr[c]);
                    wrow[gv * GQA + h_own] = make_float2(w, w);
                }
            }
        }
    }
    float alpha_g[GQA];
#pragma unroll
    for (int g = 0; g < GQA; ++g) alpha_g[g] = __shfl_sync(0xffffffffu, alpha, g << kOwnShift);
    __syncwarp();

    // ---- values ----
    const int slice = lane & 15, parity = lane >> 4;
    bool rescale = false;
#pragma unroll
    for (int g = 0; g < GQA; ++g) rescale |= alpha_g[g] != 1.0f;
    if (rescale) {
#pragma unroll
        for (int g = 0; g < GQA; ++g)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                st.o[g][c].x *= alpha_g[g];
                st.o[g][c].y *= alpha_g[g];
            }
    }
    const int gv_lane = (VM == V_BF16) ? 0 : (8 * slice) / group_v;
#pragma unroll
    for (int k = 0; k < TPW / 2; ++k) {
        const int j = 2 * k + parity;
        const int tt = t_warp + j;
        if (VM == V_BF16 && tt >= n) continue;  // stale bf16 rows may be NaN
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

template <int GQA, int KM, int VM, int KBITS, int VBITS, int NS>
__global__ void __launch_bounds__(kThreads, 2) decode_splitk_kernel(const DecodeParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int split = blockIdx.x, kvh = blockIdx.y, seq = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    int T = __ldg(p.seq_lens + seq);
    if (T > p.max_seq_len) {
        if (tid == 0 && split == 0 && kvh == 0) status_or(p.status, KVQ_DEV_SEQLEN);
        T = p.max_seq_len;
    }
    const int t_begin = split * p.chunk;
    if (t_begin >= T) return;
    const int t_end = min(T, t_begin + p.chunk);
    const int Tq = quantized_len(T, p.R);
    const int q_end = min(t_end, Tq);                // quantized tokens [t_begin, q_end)
    const int n_qt = q_end > t_begin ? (q_end - t_begin + kTile - 1) / kTile : 0;
    const int w_begin = max(t_begin, Tq);            // bf16 window tokens [w_begin, t_end)
    const int n_wt = t_end > w_begin ? (t_end - w_begin + p.bf_tile - 1) / p.bf_tile : 0;
    const int n_tiles = n_qt + n_wt;

    uint8_t *stages = smem;
    uint8_t *tail = smem + static_cast<size_t>(NS) * p.stage_bytes;
    float *qs = reinterpret_cast<float *>(tail);
    float *wsm_all = qs + GQA * kHeadDim;
    float *red = wsm_all + kConsumerWarps * 16 * 8 * GQA * 2;
    uint64_t *full = reinterpret_cast<uint64_t *>(red + kConsumerWarps * GQA * 130);
    uint64_t *empty = full + NS;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + NS);

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    const int64_t sh = static_cast<int64_t>(seq) * p.H + kvh;

    if (warp == kConsumerWarps) {
        // ------------------------- producer -------------------------
        if (lane != 0) return;
        constexpr int KROW = KRow<KM, KBITS>::bytes;
        constexpr int VROW = VRow<VM, VBITS>::bytes;
        const int ngk = (KM == K_TOKEN) ? kHeadDim / p.group_k : 0;
        const int ngv = (VM == V_TOKEN) ? kHeadDim / p.group_v : 0;
        int issued = 0;
        for (int it = 0; it < n_tiles; ++it) {
            const int s = it % NS, r = it / NS;
            if (r > 0 &&
                !mbar_wait_bounded(&empty[s], (r - 1) & 1, p.timeout_ns, p.status, abort_flag))
                break;
            issued = it + 1;
            if (it == p.skip_tile) continue;  // test hook: never arrive
            uint8_t *st = stages + static_cast<size_t>(s) * p.stage_bytes;
            // Collect the copies, sum their bytes, arm the barrier, then issue.
            const uint8_t *src[16];
            uint32_t off[16], len[16];
            int nc = 0;
            if (it >= n_qt) {  // bf16 window rows
                const int t0 = w_begin + (it - n_qt) * p.bf_tile;
                const int n = min(p.bf_tile, t_end - t0);
                const int64_t slot = sh * p.R + (t0 - Tq);
                src[nc] = reinterpret_cast<const uint8_t *>(p.k_res + slot * kHeadDim);
                off[nc] = 0; len[nc++] = n * kHeadDim * 2;
                src[nc] = reinterpret_cast<const uint8_t *>(p.v_res + slot * kHeadDim);
                off[nc] = p.bf_off_v; len[nc++] = n * kHeadDim * 2;
            } else if (!p.paged) {
                const int t0 = t_begin + it * kTile;
                const int n = min(kTile, q_end - t0);
                const int64_t row = sh * p.cap + t0;
                src[nc] = p.k_codes + row * KROW; off[nc] = 0; len[nc++] = n * KROW;
                if (KM == K_TOKEN) {
                    src[nc] = reinterpret_cast<const uint8_t *>(p.k_sz + row * ngk);
                    off[nc] = p.off_ksz; len[nc++] = (n * ngk * 4 + 15) & ~15;
                } else if (KM == K_CHANNEL) {
                    src[nc] = reinterpret_cast<const uint8_t *>(
                        p.k_sz + (sh * (p.cap / p.R) + t0 / p.R) * kHeadDim);
                    off[nc] = p.off_ksz; len[nc++] = kHeadDim * 4;
                }
                src[nc] = p.v_codes + row * VROW; off[nc] = p.off_vc; len[nc++] = n * VROW;
                if (VM == V_TOKEN) {
                    src[nc] = reinterpret_cast<const uint8_t *>(p.v_sz + row * ngv);
                    off[nc] = p.off_vsz; len[nc++] = (n * ngv * 4 + 15) & ~15;
                }
            } else {
                const int t0 = t_begin + it * kTile;
                const int n = min(kTile, q_end - t0);
                const int ps = p.page_size;
                const int span = ps < kTile ? ps : kTile;  // tokens per copy
                for (int tp = t0; tp < t0 + n; tp += span) {
                    const int pi = tp / ps;
                    const int page = (pi < p.max_pages)
                                         ? __ldg(p.block_table + static_cast<int64_t>(seq) * p.max_pages + pi)
                                         : -1;
                    if (page < 0 || page >= p.num_pages) {
                        status_or(p.status, KVQ_DEV_CAPACITY);
                        continue;
                    }
                    const int64_t row = (static_cast<int64_t>(page) * p.H + kvh) * ps + (tp % ps);
                    const uint32_t dt = tp - t0;
                    src[nc] = p.k_codes + row * KROW; off[nc] = dt * KROW; len[nc++] = span * KROW;
                    src[nc] = reinterpret_cast<const uint8_t *>(p.k_sz + row * ngk);
                    off[nc] = p.off_ksz + dt * ngk * 4; len[nc++] = span * ngk * 4;
                    src[nc] = p.v_codes + row * VROW; off[nc] = p.off_vc + dt * VROW; len[nc++] = span * VROW;
                    src[nc] = reinterpret_cast<const uint8_t *>(p.v_sz + row * ngv);
                    off[nc] = p.off_vsz + dt * ngv * 4; len[nc++] = span * ngv * 4;
                }
            }
            uint32_t bytes = 0;
            for (int c = 0; c < nc; ++c) bytes += len[c];
            mbar_arrive_expect_tx(&full[s], bytes);
            for (int c = 0; c < nc; ++c) bulk_g2s(st + off[c], src[c], len[c], &full[s]);
        }
        // Drain: wait for the copies of the last stages issued so none lands
        // after the CTA has gone.
        for (int it = max(0, issued - NS); it < issued; ++it) {
            if (it == p.skip_tile) continue;
            const int s = it % NS, r = it / NS;
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
    // Query: warp g < GQA loads head kvh*GQA + g, 4 channels per lane, and
    // rotates it like the keys; then scales by softmax_scale * log2(e).
    if (warp < GQA) {
        const int hq = kvh * GQA + warp;
        const int64_t base = (static_cast<int64_t>(seq) * p.Hq + hq) * kHeadDim + 4 * lane;
        float x[4];
        if (p.q_dtype == KVQ_FP32) {
            const float4 v = *reinterpret_cast<const float4 *>(static_cast<const float *>(p.q) + base);
            x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
        } else {
            const uint2 v = *reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(p.q) + base);
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
#pragma unroll
        for (int j = 0; j < 4; ++j) qs[warp * kHeadDim + 4 * lane + j] = x[j] * p.qscale;
    }
    named_sync(1, kConsumers);

    const int part = lane & 7;
    // Query registers in the layout of the key mode (see the header comment):
    // token-wise codes: 256 q, with qc = sum of the lane's q (zero-point term);
    // channel-wise codes: set per block below; bf16 keys: q itself.
    float2 qk[GQA][8];
    float qc[GQA];
    auto load_plain_q = [&](float scale_q) {
#pragma unroll
        for (int g = 0; g < GQA; ++g) {
            float s = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float a = qs[g * kHeadDim + part * 16 + 2 * j];
                const float b = qs[g * kHeadDim + part * 16 + 2 * j + 1];
                qk[g][j] = make_float2(a * scale_q, b * scale_q);
                s += a + b;
            }
            qc[g] = s;
        }
    };
    load_plain_q(KM == K_TOKEN ? 256.0f : 1.0f);

    WarpState<GQA> st;
    st.m_own = -INFINITY;
    st.l_own = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) st.corr[c] = 0.0f;
#pragma unroll
    for (int g = 0; g < GQA; ++g)
#pragma unroll
        for (int c = 0; c < 4; ++c) st.o[g][c] = make_float2(0.0f, 0.0f);
    float *wsm = wsm_all + warp * 16 * 8 * GQA * 2;

    int cur_block = -1;
    for (int it = 0; it < n_tiles; ++it) {
        const int s = it % NS, r = it / NS;
        if (!mbar_wait_bounded(&full[s], r & 1, p.timeout_ns, p.status, abort_flag)) break;
        const uint8_t *sb = stages + static_cast<size_t>(s) * p.stage_bytes;
        if (it < n_qt) {
            const int t0 = t_begin + it * kTile;
            const int n = min(kTile, q_end - t0);
            if constexpr (KM == K_CHANNEL) {
                const int blk = t0 / p.R;
                if (blk != cur_block) {  // fold this block's channel scales into q
                    cur_block = blk;
#pragma unroll
                    for (int g = 0; g < GQA; ++g) {
                        float c = 0.0f;
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int ch = part * 16 + 2 * j;
                            const float2 s0 = half2_lds(sb + p.off_ksz + ch * 4);
                            const float2 s1 = half2_lds(sb + p.off_ksz + (ch + 1) * 4);
                            const float qa = qs[g * kHeadDim + ch], qb = qs[g * kHeadDim + ch + 1];
                            qk[g][j] = make_float2(256.0f * qa * s0.x, 256.0f * qb * s1.x);
                            c = fmaf(qa, fmaf(-128.0f, s0.x, s0.y), c);
                            c = fmaf(qb, fmaf(-128.0f, s1.x, s1.y), c);
                        }
                        qc[g] = c;
                    }
                }
            }
            process_tile<GQA, KM, VM, KBITS, VBITS, kTile / kConsumerWarps>(
                sb, sb + p.off_ksz, sb + p.off_vc, sb + p.off_vsz, n, p.group_k, p.group_v, qk, qc,
                st, wsm, warp, lane);
        } else {
            if (it == n_qt && KM != K_BF16) {
                load_plain_q(1.0f);
#pragma unroll
                for (int g = 0; g < GQA; ++g) qc[g] = 0.0f;
            }
            const int t0 = w_begin + (it - n_qt) * p.bf_tile;
            const int n = min(p.bf_tile, t_end - t0);
            if constexpr (KM == K_BF16) {
                process_tile<GQA, K_BF16, V_BF16, 16, 16, kTile / kConsumerWarps>(
                    sb, nullptr, sb + p.bf_off_v, nullptr, n, 128, 128, qk, qc, st, wsm, warp, lane);
            } else {
                process_tile<GQA, K_BF16, V_BF16, 16, 16, kWinTile / kConsumerWarps>(
                    sb, nullptr, sb + p.bf_off_v, nullptr, n, 128, 128, qk, qc, st, wsm, warp, lane);
            }
        }
        if (lane == 0) mbar_arrive(&empty[s]);
    }
    const bool aborted = *abort_flag != 0;

    // ---- merge the four warps ----
    constexpr int kPerHead = LaneMap<GQA>::kPerHead;
    constexpr int kOwnShift = LaneMap<GQA>::kOwnShift;
    float l_own = st.l_own;
    l_own += __shfl_xor_sync(0xffffffffu, l_own, 8);
    l_own += __shfl_xor_sync(0xffffffffu, l_own, 16);
    float corr[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        corr[c] = st.corr[c];
        corr[c] += __shfl_xor_sync(0xffffffffu, corr[c], 8);
        corr[c] += __shfl_xor_sync(0xffffffffu, corr[c], 16);
    }
    const int slice = lane & 15;
    const int gv_lane = (VM == V_BF16) ? 0 : (8 * slice) / p.group_v;
#pragma unroll
    for (int g = 0; g < GQA; ++g) {
        // group gv of head g lives in lane (g << kOwnShift) + gv % kPerHead, slot gv / kPerHead
        float zg = 0.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int r = 0; r < kPerHead; ++r) {
                const float z = __shfl_sync(0xffffffffu, corr[c], (g << kOwnShift) + r);
                if (VM == V_TOKEN && gv_lane == r + c * kPerHead) zg = z;
            }
        }
        const float mg = __shfl_sync(0xffffffffu, st.m_own, g << kOwnShift);
        const float lg = __shfl_sync(0xffffffffu, l_own, g << kOwnShift);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float2 v = st.o[g][c];
            v.x += __shfl_xor_sync(0xffffffffu, v.x, 16);
            v.y += __shfl_xor_sync(0xffffffffu, v.y, 16);
            if (lane < 16) {
                red[(warp * GQA + g) * 130 + 8 * slice + 2 * c] = v.x + zg;
                red[(warp * GQA + g) * 130 + 8 * slice + 2 * c + 1] = v.y + zg;
            }
        }
        if (lane == 0) {
            red[(warp * GQA + g) * 130 + 128] = mg;
            red[(warp * GQA + g) * 130 + 129] = lg;
        }
    }
    named_sync(1, kConsumers);
    if (aborted) return;
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
        const int hq = kvh * GQA + g;
        const int64_t pi = (static_cast<int64_t>(seq) * p.Hq + hq) * p.n_split + split;
        p.o_part[pi * kHeadDim + d] = o;
        if (d == 0) p.ml[pi] = make_float2(M, l);
    }
}

// One CTA of 128 threads per (query head, sequence): combine the splits.
__global__ void __launch_bounds__(128) decode_merge_kernel(const float *o_part, const float2 *ml,
                                                           const int32_t *seq_lens, float *out,
                                                           int Hq, int n_split, int chunk,
                                                           int max_seq_len) {
    const int hq = blockIdx.x, seq = blockIdx.y, d = threadIdx.x;
    const int T = min(__ldg(seq_lens + seq), max_seq_len);
    const int nv = T > 0 ? (T + chunk - 1) / chunk : 0;
    const int64_t base = (static_cast<int64_t>(seq) * Hq + hq) * n_split;
    float M = -INFINITY;
    for (int j = 0; j < nv; ++j) M = fmaxf(M, ml[base + j].x);
    float o = 0.0f, l = 0.0f;
    for (int j = 0; j < nv; ++j) {
        const float2 v = ml[base + j];
        const float e = (v.x == -INFINITY) ? 0.0f : fast_exp2(v.x - M);
        o = fmaf(e, o_part[(base + j) * kHeadDim + d], o);
        l = fmaf(e, v.y, l);
    }
    out[(static_cast<int64_t>(seq) * Hq + hq) * kHeadDim + d] = (l > 0.0f) ? o / l : 0.0f;
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
struct StageLayout {
    int bytes, off_ksz, off_vc, off_vsz, bf_tile, bf_off_v;
};

inline int round16(int x) { return (x + 15) & ~15; }

StageLayout stage_layout(const kvq_cache_desc &d) {
    StageLayout L{};
    if (d.bits_k == 16) {  // every tile is bf16 rows: K at 0, V after it
        L.bf_tile = kTile;
        L.bf_off_v = kTile * 256;
        L.off_vc = L.bf_off_v;
        L.bytes = 2 * kTile * 256;
        return L;
    }
    const int krow = 128 * d.bits_k / 8;
    const int vrow = 128 * d.bits_v / 8;
    const int ksz = (d.axis_k == KVQ_PER_CHANNEL) ? 128 * 4 : kTile * (128 / d.group_k) * 4;
    const int vsz = kTile * (128 / d.group_v) * 4;
    L.off_ksz = round16(kTile * krow);
    L.off_vc = L.off_ksz + round16(ksz);
    L.off_vsz = L.off_vc + round16(kTile * vrow);
    L.bytes = L.off_vsz + round16(vsz);
    L.bf_tile = kWinTile;
    L.bf_off_v = kWinTile * 256;
    if (d.residual_len > 0) L.bytes = std::max(L.bytes, 2 * kWinTile * 256);
    L.bytes = (L.bytes + 127) & ~127;
    return L;
}

template <int GQA>
size_t tail_bytes(int NS) {
    return sizeof(float) * (GQA * kHeadDim + kConsumerWarps * 16 * 8 * GQA * 2 + kConsumerWarps * GQA * 130) +
           sizeof(uint64_t) * 2 * NS + 16;
}

template <int GQA, int KM, int VM, int KBITS, int VBITS>
kvq_status launch_variant(const DecodeParams &p, dim3 grid, cudaStream_t stream) {
    constexpr int NS = (KM == K_BF16) ? 3 : 4;
    const size_t smem = static_cast<size_t>(NS) * p.stage_bytes + tail_bytes<GQA>(NS);
    auto kern = decode_splitk_kernel<GQA, KM, VM, KBITS, VBITS, NS>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return KVQ_ERR_CUDA;
    kern<<<grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

template <int GQA>
kvq_status dispatch_modes(const kvq_cache_desc &d, const DecodeParams &p, dim3 grid,
                          cudaStream_t stream) {
    if (d.bits_k == 16 && d.bits_v == 16)
        return launch_variant<GQA, K_BF16, V_BF16, 16, 16>(p, grid, stream);
    if (d.axis_k == KVQ_PER_CHANNEL) {
        if (d.bits_k == 2 && d.bits_v == 2) return launch_variant<GQA, K_CHANNEL, V_TOKEN, 2, 2>(p, grid, stream);
        if (d.bits_k == 4 && d.bits_v == 4) return launch_variant<GQA, K_CHANNEL, V_TOKEN, 4, 4>(p, grid, stream);
        if (d.bits_k == 2 && d.bits_v == 4) return launch_variant<GQA, K_CHANNEL, V_TOKEN, 2, 4>(p, grid, stream);
        if (d.bits_k == 4 && d.bits_v == 2) return launch_variant<GQA, K_CHANNEL, V_TOKEN, 4, 2>(p, grid, stream);
        return KVQ_ERR_UNSUPPORTED;
    }
    if (d.bits_k == 4 && d.bits_v == 4) return launch_variant<GQA, K_TOKEN, V_TOKEN, 4, 4>(p, grid, stream);
    if (d.bits_k == 2 && d.bits_v == 2) return launch_variant<GQA, K_TOKEN, V_TOKEN, 2, 2>(p, grid, stream);
    if (d.bits_k == 4 && d.bits_v == 2) return launch_variant<GQA, K_TOKEN, V_TOKEN, 4, 2>(p, grid, stream);
    if (d.bits_k == 2 && d.bits_v == 4) return launch_variant<GQA, K_TOKEN, V_TOKEN, 2, 4>(p, grid, stream);
    return KVQ_ERR_UNSUPPORTED;
}

}  // namespace

bool plan_decode(const kvq_cache_desc &d, int num_seqs, int num_q_heads, int max_seq_len,
                 DecodePlan *plan) {
    if (num_seqs <= 0 || num_q_heads <= 0 || max_seq_len < 0 || d.num_kv_heads <= 0) return false;
    const int64_t units = static_cast<int64_t>(num_seqs) * d.num_kv_heads;
    const int64_t want_ctas = 8 * 148;
    const int64_t splits = std::max<int64_t>(1, (want_ctas + units - 1) / units);
    int64_t chunk = (std::max(1, max_seq_len) + splits - 1) / splits;
    chunk = ((chunk + kTile - 1) / kTile) * kTile;
    chunk = std::max<int64_t>(chunk, 256);
    plan->chunk = static_cast<int>(chunk);
    plan->n_split = static_cast<int>(std::max<int64_t>(1, (max_seq_len + chunk - 1) / chunk));
    const size_t rows = static_cast<size_t>(num_seqs) * num_q_heads * plan->n_split;
    plan->ws_part = rows * kHeadDim * sizeof(float);
    plan->ws_ml = rows * sizeof(float2);
    plan->ws_total = plan->ws_part + plan->ws_ml;
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
    p.status = d.status;
    p.H = d.num_kv_heads;
    p.Hq = num_q_heads;
    p.group_k = d.group_k;
    p.group_v = d.group_v;
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
    const StageLayout L = stage_layout(d);
    p.stage_bytes = L.bytes;
    p.off_ksz = L.off_ksz;
    p.off_vc = L.off_vc;
    p.off_vsz = L.off_vsz;
    p.bf_tile = L.bf_tile;
    p.bf_off_v = L.bf_off_v;
    p.timeout_ns = debug_hooks().wait_timeout_ns;
    p.skip_tile = debug_hooks().skip_tile;
    const dim3 grid(plan.n_split, d.num_kv_heads, num_seqs);
    switch (num_q_heads / d.num_kv_heads) {
        case 1: return dispatch_modes<1>(d, p, grid, stream);
        case 2: return dispatch_modes<2>(d, p, grid, stream);
        case 4: return dispatch_modes<4>(d, p, grid, stream);
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
    decode_merge_kernel<<<dim3(num_q_heads, num_seqs), 128, 0, stream>>>(
        o_part, ml, seq_lens, out, num_q_heads, plan.n_split, plan.chunk, max_seq_len);
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // namespace kvq
