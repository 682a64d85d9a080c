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
// The producer's elected lane stages each 64-token tile (K codes, K scale/zero,
// V codes, V scale/zero) into a shared-memory ring with 1-D bulk copies (TMA
// engine, mbarrier complete_tx); page-table indirection is resolved per page.
// Each consumer warp owns 16 of a tile's 64 tokens with its own online-softmax
// state, so tiles need no cross-warp synchronisation:
//   scores: 8 lanes per token, 16 channels per lane, all GQA heads at once;
//           a reduce-scatter over the 8 lanes leaves one head's score per lane
//           pair;
//   values: 16 lanes cover the 128 channels (8 each) for all GQA heads, the
//           two half-warps take alternate tokens.
// The four warps' states are merged once per split; the merge kernel combines
// the splits.
#include <algorithm>

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

constexpr int kTile = 64;
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

__device__ __forceinline__ float load_q_elem(const void *q, int64_t idx, int dt) {
    if (dt == KVQ_FP32) return static_cast<const float *>(q)[idx];
    const uint16_t b = static_cast<const uint16_t *>(q)[idx];
    if (dt == KVQ_BF16) return bf16_bits_to_float(b);
    return __half2float(__ushort_as_half(b));
}

// Codes of 16 channels -> floats (exact small integers).
template <int BITS>
__device__ __forceinline__ void k_codes16(const uint8_t *row, int part, float c[16]) {
    if constexpr (BITS == 4) {
        const uint2 w = *reinterpret_cast<const uint2 *>(row + part * 8);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            c[j] = small_uint_to_float((w.x >> (4 * j)) & 0xFu);
            c[8 + j] = small_uint_to_float((w.y >> (4 * j)) & 0xFu);
        }
    } else {
        const uint32_t w = *reinterpret_cast<const uint32_t *>(row + part * 4);
#pragma unroll
        for (int j = 0; j < 16; ++j) c[j] = small_uint_to_float((w >> (2 * j)) & 0x3u);
    }
}

__device__ __forceinline__ void bf16_16(const uint8_t *row, int part, float c[16]) {
    const uint4 *p = reinterpret_cast<const uint4 *>(row + part * 32);
    const uint4 a = p[0], b = p[1];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        c[2 * j] = __uint_as_float(w[j] << 16);
        c[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
}

// Eight value channels [8*slice, 8*slice + 8) of one token row.
template <int VM, int VBITS>
__device__ __forceinline__ void v_vals8(const uint8_t *row, int slice, float c[8]) {
    if constexpr (VM == V_BF16) {
        const uint4 a = *reinterpret_cast<const uint4 *>(row + slice * 16);
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            c[2 * j] = __uint_as_float(w[j] << 16);
            c[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
    } else if constexpr (VBITS == 4) {
        const uint32_t w = *reinterpret_cast<const uint32_t *>(row + slice * 4);
#pragma unroll
        for (int j = 0; j < 8; ++j) c[j] = small_uint_to_float((w >> (4 * j)) & 0xFu);
    } else {
        const uint32_t w = *reinterpret_cast<const uint16_t *>(row + slice * 2);
#pragma unroll
        for (int j = 0; j < 8; ++j) c[j] = small_uint_to_float((w >> (2 * j)) & 0x3u);
    }
}

// Per-warp decode state.
template <int GQA>
struct WarpState {
    float m_own;     // running max (log2 domain) of this lane's head
    float l_own;     // running sum of this lane's tokens' weights (own head)
    float zs[8];     // running sum of p * zero per value group (own head)
    float o[GQA][8]; // value accumulators: 8 channels x GQA heads
};

// One tile of up to 64 tokens: rows at kc / ks / vc / vs (generic pointers,
// shared or global memory), `n` valid tokens. qk/qc hold the lane's query
// (already scaled) in the layout the key mode needs.
template <int GQA, int KM, int VM, int KBITS, int VBITS>
__device__ __forceinline__ void process_tile(const uint8_t *kc, const __half2 *ks,
                                             const uint8_t *vc, const __half2 *vs, int n,
                                             int group_k, int group_v, const float (&qk)[GQA][16],
                                             const float (&qc)[GQA], WarpState<GQA> &st,
                                             float *wsm, int warp, int lane) {
    constexpr int KROW = KRow<KM, KBITS>::bytes;
    constexpr int VROW = VRow<VM, VBITS>::bytes;
    const int i = lane >> 3, part = lane & 7;
    const int n_vg = (VM == V_BF16) ? 1 : kHeadDim / group_v;
    const int ngk = (KM == K_TOKEN) ? kHeadDim / group_k : 0;
    constexpr int kOwnShift = (GQA == 4) ? 1 : (GQA == 2 ? 2 : 3);
    const int h_own = part >> kOwnShift;

    // ---- scores ----
    float sc[4];
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
        const int tt = pass * 16 + warp * 4 + i;
        const int tr = tt < n ? tt : 0;  // masked tokens read row 0 (always staged)
        float c[16];
        const uint8_t *row = kc + static_cast<size_t>(tr) * KROW;
        if constexpr (KM == K_BF16) bf16_16(row, part, c);
        else k_codes16<KBITS>(row, part, c);
        float acc[GQA];
#pragma unroll
        for (int g = 0; g < GQA; ++g) {
            float a = 0.0f;
#pragma unroll
            for (int j = 0; j < 16; ++j) a = fmaf(qk[g][j], c[j], a);
            acc[g] = a;
        }
        if constexpr (KM == K_TOKEN) {
            const float2 szf = __half22float2(ks[tr * ngk + (part * 16) / group_k]);
#pragma unroll
            for (int g = 0; g < GQA; ++g) acc[g] = fmaf(szf.x, acc[g], szf.y * qc[g]);
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
    float mx = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    const float m_new = fmaxf(st.m_own, mx);
    float alpha, p[4];
    if (m_new == -INFINITY) {
        alpha = 1.0f;
#pragma unroll
        for (int k = 0; k < 4; ++k) p[k] = 0.0f;
    } else {
        alpha = fast_exp2(st.m_own - m_new);
#pragma unroll
        for (int k = 0; k < 4; ++k) p[k] = fast_exp2(sc[k] - m_new);
    }
    st.m_own = m_new;
    st.l_own = st.l_own * alpha + (p[0] + p[1]) + (p[2] + p[3]);
    const bool writer = (part & ((8 / GQA) - 1)) == 0;
#pragma unroll
    for (int gv = 0; gv < 8; ++gv) st.zs[gv] *= alpha;
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
        const int j = pass * 4 + i;  // warp-local token index
        const int tt = pass * 16 + warp * 4 + i;
        const int tr = tt < n ? tt : 0;
        float *wrow = wsm + (j * n_vg) * GQA;
        if constexpr (VM == V_BF16) {
            if (writer) wrow[h_own] = p[pass];
        } else {
            for (int gv = 0; gv < n_vg; ++gv) {
                const float2 szf = __half22float2(vs[tr * n_vg + gv]);
                st.zs[gv] = fmaf(p[pass], szf.y, st.zs[gv]);
                if (writer) wrow[gv * GQA + h_own] = p[pass] * szf.x;
            }
        }
    }
    // alpha of every head, from the lane pair that owns it (token slot 0)
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
            for (int c = 0; c < 8; ++c) st.o[g][c] *= alpha_g[g];
    }
    const int gv_lane = (VM == V_BF16) ? 0 : (8 * slice) / group_v;
#pragma unroll 2
    for (int k = 0; k < 8; ++k) {
        const int j = 2 * k + parity;
        const int tt = (j >> 2) * 16 + warp * 4 + (j & 3);
        if (tt >= n) continue;
        float c[8];
        v_vals8<VM, VBITS>(vc + static_cast<size_t>(tt) * VROW, slice, c);
        const float *wrow = wsm + (j * n_vg + gv_lane) * GQA;
        float w[GQA];
        if constexpr (GQA == 4) {
            const float4 w4 = *reinterpret_cast<const float4 *>(wrow);
            w[0] = w4.x; w[1] = w4.y; w[2] = w4.z; w[3] = w4.w;
        } else {
#pragma unroll
            for (int g = 0; g < GQA; ++g) w[g] = wrow[g];
        }
#pragma unroll
        for (int g = 0; g < GQA; ++g)
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) st.o[g][cc] = fmaf(w[g], c[cc], st.o[g][cc]);
    }
    __syncwarp();
}

struct SmemLayout {
    // after the NS stages:
    float *qs;      // [GQA][128]
    float *wsm;     // [4 warps][16 tokens][8 groups][GQA]
    float *red;     // [4 warps][GQA][130]
    uint64_t *full, *empty;
    int *abort_flag;
};

template <int GQA, int KM, int VM, int KBITS, int VBITS, int NS>
__global__ void __launch_bounds__(kThreads) decode_splitk_kernel(const DecodeParams p) {
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
    const int n_tiles = q_end > t_begin ? (q_end - t_begin + kTile - 1) / kTile : 0;
    const int w_begin = max(t_begin, Tq);            // window tokens [w_begin, t_end)

    uint8_t *stages = smem;
    uint8_t *tail = smem + static_cast<size_t>(NS) * p.stage_bytes;
    float *qs = reinterpret_cast<float *>(tail);
    float *wsm_all = qs + GQA * kHeadDim;
    float *red = wsm_all + kConsumerWarps * 16 * 8 * GQA;
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
            const int t0 = t_begin + it * kTile;
            const int n = min(kTile, q_end - t0);
            uint8_t *st = stages + static_cast<size_t>(s) * p.stage_bytes;
            // Collect the copies, sum their bytes, arm the barrier, then issue.
            const uint8_t *src[4 * 8];
            uint32_t off[4 * 8], len[4 * 8];
            int nc = 0;
            if (!p.paged) {
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
            uint64_t t0 = global_timer_ns();
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
    // rotates it like the keys.
    if (warp < GQA) {
        const int hq = kvh * GQA + warp;
        const int64_t base = (static_cast<int64_t>(seq) * p.Hq + hq) * kHeadDim + 4 * lane;
        float x[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) x[j] = load_q_elem(p.q, base + j, p.q_dtype);
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
    float qk[GQA][16];
    float qc[GQA];
#pragma unroll
    for (int g = 0; g < GQA; ++g) {
        float s = 0.0f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            qk[g][j] = qs[g * kHeadDim + part * 16 + j];
            s += qk[g][j];
        }
        qc[g] = (KM == K_TOKEN) ? s : 0.0f;
    }

    WarpState<GQA> st;
    st.m_own = -INFINITY;
    st.l_own = 0.0f;
#pragma unroll
    for (int gv = 0; gv < 8; ++gv) st.zs[gv] = 0.0f;
#pragma unroll
    for (int g = 0; g < GQA; ++g)
#pragma unroll
        for (int c = 0; c < 8; ++c) st.o[g][c] = 0.0f;
    float *wsm = wsm_all + warp * 16 * 8 * GQA;

    int cur_block = -1;
    for (int it = 0; it < n_tiles; ++it) {
        const int s = it % NS, r = it / NS;
        if (!mbar_wait_bounded(&full[s], r & 1, p.timeout_ns, p.status, abort_flag)) break;
        const uint8_t *st_base = stages + static_cast<size_t>(s) * p.stage_bytes;
        const int t0 = t_begin + it * kTile;
        const int n = min(kTile, q_end - t0);
        if constexpr (KM == K_CHANNEL) {
            const int blk = t0 / p.R;
            if (blk != cur_block) {  // fold this block's channel scales into q
                cur_block = blk;
                const __half2 *ksz = reinterpret_cast<const __half2 *>(st_base + p.off_ksz);
#pragma unroll
                for (int g = 0; g < GQA; ++g) {
                    float c = 0.0f;
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float2 szf = __half22float2(ksz[part * 16 + j]);
                        const float qv = qs[g * kHeadDim + part * 16 + j];
                        qk[g][j] = qv * szf.x;
                        c = fmaf(qv, szf.y, c);
                    }
                    qc[g] = c;
                }
            }
        }
        process_tile<GQA, KM, VM, KBITS, VBITS>(
            st_base, reinterpret_cast<const __half2 *>(st_base + p.off_ksz), st_base + p.off_vc,
            reinterpret_cast<const __half2 *>(st_base + p.off_vsz), n, p.group_k, p.group_v, qk, qc,
            st, wsm, warp, lane);
        if (lane == 0) mbar_arrive(&empty[s]);
    }

    const bool aborted = *abort_flag != 0;
    // bf16 window tokens [w_begin, t_end), read straight from global memory.
    if (!aborted && w_begin < t_end) {
#pragma unroll
        for (int g = 0; g < GQA; ++g) {
            float s = 0.0f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                qk[g][j] = qs[g * kHeadDim + part * 16 + j];
                s += qk[g][j];
            }
            qc[g] = 0.0f;
            (void)s;
        }
        const int Tq_base = Tq;
        for (int t0 = w_begin; t0 < t_end; t0 += kTile) {
            const int n = min(kTile, t_end - t0);
            const int64_t slot = sh * p.R + (t0 - Tq_base);
            const uint8_t *kw = reinterpret_cast<const uint8_t *>(p.k_res + slot * kHeadDim);
            const uint8_t *vw = reinterpret_cast<const uint8_t *>(p.v_res + slot * kHeadDim);
            process_tile<GQA, K_BF16, V_BF16, 16, 16>(kw, nullptr, vw, nullptr, n, 128, 128, qk, qc,
                                                       st, wsm, warp, lane);
        }
    }

    // ---- merge the four warps ----
    constexpr int kOwnShift = (GQA == 4) ? 1 : (GQA == 2 ? 2 : 3);
    const int i_tok = lane >> 3;
    (void)i_tok;
    float l_own = st.l_own;
    l_own += __shfl_xor_sync(0xffffffffu, l_own, 8);
    l_own += __shfl_xor_sync(0xffffffffu, l_own, 16);
    float zs[8];
#pragma unroll
    for (int gv = 0; gv < 8; ++gv) {
        zs[gv] = st.zs[gv];
        zs[gv] += __shfl_xor_sync(0xffffffffu, zs[gv], 8);
        zs[gv] += __shfl_xor_sync(0xffffffffu, zs[gv], 16);
    }
    const int slice = lane & 15;
    const int gv_lane = (VM == V_BF16) ? 0 : (8 * slice) / p.group_v;
#pragma unroll
    for (int g = 0; g < GQA; ++g) {
        const int src = g << kOwnShift;
        float zg = 0.0f;
#pragma unroll
        for (int gv = 0; gv < 8; ++gv) {
            const float z = __shfl_sync(0xffffffffu, zs[gv], src);
            if (gv == gv_lane) zg = z;
        }
        const float mg = __shfl_sync(0xffffffffu, st.m_own, src);
        const float lg = __shfl_sync(0xffffffffu, l_own, src);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            float v = st.o[g][c] + __shfl_xor_sync(0xffffffffu, st.o[g][c], 16);
            if (VM == V_TOKEN) v += zg;
            if (lane < 16) red[(warp * GQA + g) * 130 + 8 * slice + c] = v;
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
    int bytes, off_ksz, off_vc, off_vsz;
};

inline int round16(int x) { return (x + 15) & ~15; }

StageLayout stage_layout(const kvq_cache_desc &d) {
    const int krow = d.bits_k == 16 ? 256 : 128 * d.bits_k / 8;
    const int vrow = d.bits_v == 16 ? 256 : 128 * d.bits_v / 8;
    int ksz = 0, vsz = 0;
    if (d.bits_k != 16) ksz = (d.axis_k == KVQ_PER_CHANNEL) ? 128 * 4 : kTile * (128 / d.group_k) * 4;
    if (d.bits_v != 16) vsz = kTile * (128 / d.group_v) * 4;
    StageLayout L;
    L.off_ksz = round16(kTile * krow);
    L.off_vc = L.off_ksz + round16(ksz);
    L.off_vsz = L.off_vc + round16(kTile * vrow);
    L.bytes = (L.off_vsz + round16(vsz) + 127) & ~127;
    return L;
}

template <int GQA>
size_t tail_bytes(int NS) {
    return sizeof(float) * (GQA * kHeadDim + kConsumerWarps * 16 * 8 * GQA + kConsumerWarps * GQA * 130) +
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
