// kvq_decode_kernel.cuh -- the split-K decode kernel template and its launcher,
// shared by the translation units that instantiate its variants (one per
// family: plain, residual window, values per channel, attention sinks).
//
//
// SAW-INT4 (Abstract): attention runs fused over the quantized paged cache.
// InnerQ (Abstract): with groups along the inner dimension of q.k the scale
// and zero factor out of the dot product,
//     q . k^ = s * sum_i q_i c_i + z * sum_i q_i,
// and for values  sum_t p_t v^_t = sum_t (p_t s_t) c_t + sum_t p_t z_t,
// so no dequantized element is ever formed. Dual-QK (Abstract): queries take
// the keys' orthogonal transform, so q~ . k~ = q . k.
//
// Work items are (sequence, KV head, split): a split is a token range, the
// same for every sequence (the host's plan: equal chunks of whole tiles).
// Items are numbered split-major, so the sequences' last, partial splits are
// claimed last and fill the launch's tail. The kernel is persistent: each CTA
// (4 consumer warps, 1 producer warp, 1 helper warp) takes item blockIdx.x
// first and then claims items from a global counter until none are left. The
// producer warp claims items and streams every item's tiles (K codes, K scale/zero, V codes, V
// scale/zero; bf16 rows for the recent-token window) into a shared-memory ring
// with 1-D bulk copies (TMA engine, mbarrier complete_tx); its lanes issue the
// copies of a tile in parallel, one page per lane for paged caches. Each stage
// carries a small header, so the consumers follow the stream without further
// coordination and the ring never drains between items. The helper warp
// rotates each item's query rows and builds its key coefficients one item
// ahead, and merges the four consumer warps' states into the split's partial
// once they have deposited them, so the consumers never wait for each other.
//
// Every cached element meets GQA query heads, one multiply-add each, on the
// CUDA cores (each cached element meets only GQA = 4 query rows, too thin a
// contraction for the tensor cores). The consumers are bound by instruction
// issue: besides the packed f32x2 multiply-adds (16 warp instructions per
// token and KV head at INT4, GQA 4) they convert codes, load coefficients and
// run the softmax. So they spend as few issue slots as possible besides the
// multiply-adds:
//   * keys: one lane per token. A lane walks its token's code row in 16-byte
//     chunks and multiplies each code with the GQA heads' query coefficients,
//     which every lane reads with the same broadcast shared-memory load. No
//     cross-lane reduction; softmax statistics come out per lane. The chunk
//     order is XOR-rotated per lane so the 8 lanes of a shared-memory phase
//     hit 8 distinct bank groups (their rows are 16-64 bytes apart); the
//     coefficients are stored with a 16-byte pad per chunk for the same
//     reason.
//   * codes become floats 0.5 + X/256 with ONE byte permute per code, from
//     byte planes kept below 128; the query coefficients are transformed once
//     per item so that their dot product with these floats is the one with the
//     codes, and the value sums are untangled once per item;
//   * multiply-adds are packed f32x2 FMAs;
//   * softmax: each warp keeps a reference maximum per head that moves only
//     when a score exceeds it by more than 8 (log2 units); a warp vote decides
//     whether a tile needs the max reduction at all;
//   * values: 16 lanes cover the 128 channels (8 each) for all GQA heads; the
//     two half-warps take alternate tokens; the weights p*s come from the key
//     lanes through shared memory, already duplicated into f32x2 pairs.
// The four warps' states are merged once per item by the helper warp; the
// merge kernel combines the splits.
#pragma once

#include <algorithm>
#include <mutex>

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace dec {

constexpr int kTileQ = 256;        // tokens per quantized tile (64 per warp, 2 per lane)
constexpr int kTileB = 128;        // tokens per tile of a bf16 cache (32 per warp)
constexpr int kWinTile = 64;       // tokens per bf16 window or sink tile (quantized caches)
constexpr int kMaxStages = 4;      // shared-memory ring depth, chosen on the host
constexpr int kMaxDevices = 64;    // launch settings cached per device
constexpr int kConsumerWarps = 4;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kProducerWarp = kConsumerWarps;      // streams the tiles
constexpr int kHelperWarp = kConsumerWarps + 1;    // query rows, coefficients, item merges
constexpr int kThreads = kConsumers + 64;
constexpr int kItemSlots = 2;      // items in flight per CTA (query rows and coefficients)
constexpr int kDepStride = 132;    // floats per (warp, head) deposit: o[128], (m, l), pad
constexpr int kMaxGroups = 8;      // kHeadDim / smallest token-wise group (16)
constexpr float kLog2e = 1.4426950408889634f;

enum KMode { K_TOKEN = 0, K_CHANNEL = 1, K_BF16 = 2 };
// V_CHANNEL: values grouped along tokens, one (scale, zero) per channel and
// R-token block (InnerQ's inner-dimension grouping for p @ V).
enum VMode { V_TOKEN = 0, V_CHANNEL = 1, V_BF16 = 2 };

// Tail of an item's tile stream, fixed per instantiation: nothing, the bf16
// recent-token window, or the bf16 attention-sink rows (both in kWinTile-token
// bf16 tiles). Variants without a tail carry no code for it.
enum TailMode { kTailNone = 0, kTailWindow = 1, kTailSink = 2 };

// Stage header flags. kWindow marks bf16 tiles; kSink those of the sink window.
constexpr int kFirst = 1, kLast = 2, kWindow = 4, kDone = 8, kSink = 16;

struct TileHdr {
    int t0, n, flags, start;  // tokens [start, n) of the tile are attended
    int item, pad[3];         // the CTA's item ordinal (its slot: item % kItemSlots)
};

// Coordinates of an item, posted by the producer for the helper warp.
struct ItemInfo {
    int seq, kvh, split, done;
};

struct DecodeParams {
    const uint8_t *k_codes, *v_codes;  // packed codes, or bf16 rows (bits 16)
    const __half2 *k_sz, *v_sz;
    const uint16_t *k_res, *v_res;
    const int32_t *block_table;
    const int32_t *seq_lens;
    const void *q;
    const float *signs;  // [128] +-1 applied to the query before its rotation, or null
    const uint16_t *k_sink, *v_sink;  // bf16 [S][H][sink_len][D], or null
    int sink_len;                      // sink tokens (read in window-sized bf16 tiles)
    float *o_part;  // [S][Hq][n_split][D]
    float2 *ml;     // [S][Hq][n_split]
    int *counter;   // item counter, zeroed before the launch
    int32_t *status;
    int S, H, Hq;
    int gk, gv;     // token-wise group sizes (K: 128 for per-channel keys)
    int hb;
    float hscale;   // fp32(1/sqrt(hb))
    float qscale;   // softmax_scale * log2(e)
    int R;
    int r_shift;    // log2(R) (R is 64, 128 or 256 when non-zero)
    int paged, page_size, max_pages, num_pages, cap;
    int n_split, max_seq_len;  // partials per query head; longest sequence attended
    SplitBounds sp;            // token ranges of the splits
    int ns;                // ring depth (stages), <= kMaxStages
    int q_dtype, q_bytes;  // element type and bytes of q
    // shared-memory stage layout (bytes)
    int stage_bytes, off_ksz, off_vc, off_vsz, off_hdr;
    int bf_tile, bf_off_v;  // bf16 tiles: tokens per tile, offset of the V rows
    // per-warp scratch (floats): value weights (also the lanes' W/Z partials
    // when they are summed), then the warp's W/Z totals
    int warp_floats, off_tot;
    int n_sets;            // per-channel keys: coefficient sets (2 x blocks per tile)
    int slot_floats;       // floats per item slot
    // byte offsets after the stage ring: item slots, per-channel sets, the
    // warps' deposits, per-warp scratch, barriers and the small words
    int off_slots, off_csets, off_dep, off_scr, off_bar;
    int64_t timeout_ns;
    int skip_tile;
};

// ---- key rows ---------------------------------------------------------------
// A row of KB-bit codes (KB = 16: bf16 values) is read in 16-byte chunks of
// four 32-bit words; a word yields `npw` float pairs.
template <int KB>
struct RowGeo {
    static constexpr int bytes = (KB == 16) ? kHeadDim * 2 : kHeadDim * KB / 8;
    static constexpr int nch = bytes / 16;          // chunks per row
    static constexpr int cpc = kHeadDim / nch;      // channels per chunk
    static constexpr int cpw = cpc / 4;             // channels per word
    static constexpr int npw = (KB == 16) ? 1 : cpw / 2;  // float pairs per word
    static constexpr int cstr = cpc + 4;            // padded coefficient floats per chunk
};

// Chunk order of a lane: step k reads chunk k ^ rot. Rows are 64 (INT4), 32
// (INT2) or 256 (bf16) bytes apart, so without the rotation a phase of 8
// consecutive rows would hit 2, 4 or 1 distinct 16-byte bank groups. With it
// every phase covers all 8. XOR keeps aligned runs of chunks contiguous, so a
// scale group spanning several chunks is still walked in one run.
template <int KB>
__device__ __forceinline__ int chunk_rot(int lane) {
    return KB == 4 ? ((lane >> 1) & 3) : (KB == 2 ? ((lane >> 2) & 1) : (lane & 7));
}

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

// ---- shared-memory access ---------------------------------------------------
// Plain typed loads and stores: the compiler sees their dependence on each
// other and on the mbarrier waits (asm with a memory clobber) and keeps them in
// order; the pointers all derive from the kernel's shared array.
__device__ __forceinline__ uint32_t lds32(const void *p) { return *static_cast<const uint32_t *>(p); }
__device__ __forceinline__ uint32_t lds16(const void *p) { return *static_cast<const uint16_t *>(p); }
__device__ __forceinline__ uint2 lds64(const void *p) { return *static_cast<const uint2 *>(p); }
__device__ __forceinline__ uint4 lds128(const void *p) { return *static_cast<const uint4 *>(p); }
__device__ __forceinline__ float4 ldsf4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
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
// linear in the codes; the query coefficients are transformed once per item so
// that their dot product with them is the dot product with the codes
// (build_head), and the value accumulators are untangled once per item
// (value_channels).
__device__ __forceinline__ float byte_f(uint32_t b, int k) {
    return __uint_as_float(__byte_perm(b, 0x3F000000u, 0x7054u | (static_cast<uint32_t>(k) << 8)));
}

// One 32-bit word of a key row as float pairs, in the order of the coefficient
// layout (natural channel order; INT2 bytes give their four planes):
//   INT4 byte k (channels lo, hi): {f(lo), f(hi)}
//   INT2 byte k (channels c0..c3): {f(X0), f(X1)}, {f(X2), f(X3)}
//   bf16: the two channel values.
template <int KB>
__device__ __forceinline__ void word_pairs(uint32_t w, float2 *f) {
    if constexpr (KB == 16) {
        f[0] = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    } else if constexpr (KB == 4) {
        const uint32_t a = w & 0x0F0F0F0Fu, b = (w >> 4) & 0x0F0F0F0Fu;
#pragma unroll
        for (int k = 0; k < 4; ++k) f[k] = make_float2(byte_f(a, k), byte_f(b, k));
    } else {
        const uint32_t x0 = w & 0x03030303u, x1 = w & 0x0F0F0F0Fu, x2 = w & 0x3F3F3F3Fu;
        const uint32_t x3 = (w >> 2) & 0x3F3F3F3Fu;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            f[2 * k] = make_float2(byte_f(x0, k), byte_f(x1, k));
            f[2 * k + 1] = make_float2(byte_f(x2, k), byte_f(x3, k));
        }
    }
}

// Pairs [jb, jb + 4) of word_pairs (jb = 0 or 4), without converting the rest.
template <int KB>
__device__ __forceinline__ void word_pairs4(uint32_t w, int jb, float2 f[4]) {
    if constexpr (KB == 4) {
        word_pairs<4>(w, f);
    } else {
        // INT2: pairs 2k, 2k+1 come from byte k; this block covers bytes jb/2, jb/2 + 1
        const uint32_t x0 = w & 0x03030303u, x1 = w & 0x0F0F0F0Fu, x2 = w & 0x3F3F3F3Fu;
        const uint32_t x3 = (w >> 2) & 0x3F3F3F3Fu;
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            const int k = jb / 2 + kk;
            f[2 * kk] = make_float2(byte_f(x0, k), byte_f(x1, k));
            f[2 * kk + 1] = make_float2(byte_f(x2, k), byte_f(x3, k));
        }
    }
}

// 8 value channels [8*slice, 8*slice + 8) of two tokens (rows ra, rb) as 8
// float pairs {token a, token b}, same encoding: INT4 channel j; INT2 byte k's
// plane j at 4k + j; bf16 channel j.
template <int VM, int VBITS>
__device__ __forceinline__ void value_pairs(const uint8_t *ra, const uint8_t *rb, int slice, float2 f[8]) {
    if constexpr (VM == V_BF16) {
        const uint4 a = lds128(ra + slice * 16), b = lds128(rb + slice * 16);
        const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            f[2 * j] = make_float2(__uint_as_float(wa[j] << 16), __uint_as_float(wb[j] << 16));
            f[2 * j + 1] = make_float2(__uint_as_float(wa[j] & 0xFFFF0000u), __uint_as_float(wb[j] & 0xFFFF0000u));
        }
    } else if constexpr (VBITS == 4) {
        const uint32_t wa = lds32(ra + slice * 4), wb = lds32(rb + slice * 4);
        const uint32_t la = wa & 0x0F0F0F0Fu, ha = (wa >> 4) & 0x0F0F0F0Fu;
        const uint32_t lb = wb & 0x0F0F0F0Fu, hb = (wb >> 4) & 0x0F0F0F0Fu;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            f[2 * k] = make_float2(byte_f(la, k), byte_f(lb, k));
            f[2 * k + 1] = make_float2(byte_f(ha, k), byte_f(hb, k));
        }
    } else {
        const uint32_t wa = lds16(ra + slice * 2), wb = lds16(rb + slice * 2);
        const uint32_t xa[4] = {wa & 0x0303u, wa & 0x0F0Fu, wa & 0x3F3Fu, (wa >> 2) & 0x3F3Fu};
        const uint32_t xb[4] = {wb & 0x0303u, wb & 0x0F0Fu, wb & 0x3F3Fu, (wb >> 2) & 0x3F3Fu};
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
            for (int j = 0; j < 4; ++j) f[4 * k + j] = make_float2(byte_f(xa[j], k), byte_f(xb[j], k));
    }
}

// Untangle one slice's value sums a[8] (in the encoding of value_pairs) into
// its 8 channel sums sum_t w_t c_t (without the zero-point term);
// W = sum_t w_t of its group.
template <int VM, int VBITS>
__device__ __forceinline__ void value_channels(const float a[8], float W, float out[8]) {
    if constexpr (VM == V_BF16) {
#pragma unroll
        for (int c = 0; c < 8; ++c) out[c] = a[c];
    } else if constexpr (VBITS == 4) {
        // a = sum w (0.5 + c/256)
#pragma unroll
        for (int c = 0; c < 8; ++c) out[c] = fmaf(256.0f, a[c], -128.0f * W);
    } else {
        // a_j = sum w (0.5 + X_j/256) with the X planes of value_pairs
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            const float x0 = a[4 * b], x1 = a[4 * b + 1], x2 = a[4 * b + 2], x3 = a[4 * b + 3];
            out[4 * b] = fmaf(256.0f, x0, -128.0f * W);
            out[4 * b + 1] = 64.0f * (x1 - x0);
            out[4 * b + 2] = 16.0f * (x2 - x1);
            out[4 * b + 3] = fmaf(16.0f, x3, -8.0f * W) - 4.0f * (x2 - x0);
        }
    }
}

// The 4-channel half (channels 4h..4h+3 of a slice) of value_channels: INT4
// channels are independent, and an INT2 byte's planes stay inside one half.
template <int VBITS>
__device__ __forceinline__ void value_channels4(const float a[4], float W, float out[4]) {
    if constexpr (VBITS == 4) {
#pragma unroll
        for (int c = 0; c < 4; ++c) out[c] = fmaf(256.0f, a[c], -128.0f * W);
    } else {
        out[0] = fmaf(256.0f, a[0], -128.0f * W);
        out[1] = 64.0f * (a[1] - a[0]);
        out[2] = 16.0f * (a[2] - a[1]);
        out[3] = fmaf(16.0f, a[3], -8.0f * W) - 4.0f * (a[2] - a[0]);
    }
}

// ---- key coefficients -------------------------------------------------------
// One head's key coefficients, built by one warp from the lane's 4 channels
// x[0..3] (channels 4*lane..4*lane+3 of the rotated query, scaled to log2
// units), in the padded chunk layout of RowGeo<KB> at `cg`, and the per-group
// sums {init, qa} at sums[(group * GQA + g) * 2]:
//   MODE 0 (token-wise groups, KB 4/2): coefficients 256 * a with a the plane
//     coefficients of x; a row's dot product then comes out as
//     128 * first_G + sum_G x c, so the accumulator starts at
//     init = -128 * first_G; qa = sum_G x.
//   MODE 1 (per-channel keys, KB 4/2): x is first multiplied by the block's
//     channel scales `chan_sz`; one group, init = sum x z - 128 * first, so the
//     dot product ends as q.k^.
//   MODE 2 (bf16 keys): coefficients = x, init = 0.
// GKC: compile-time group size (0: runtime gk).
template <int GQA, int KB, int MODE, int GKC>
__device__ __forceinline__ void build_head(const float xin[4], const uint8_t *chan_sz, float *cg,
                                           float *sums, int g, int gk, int lane) {
    using RG = RowGeo<KB>;
    const int i0 = 4 * lane;  // the lane's 4 channels
    const int G = (MODE == 0) ? (GKC ? GKC : gk) : kHeadDim;
    float x[4] = {xin[0], xin[1], xin[2], xin[3]};
    float qa = (x[0] + x[1]) + (x[2] + x[3]);
    float qz = 0.0f;
    if constexpr (MODE == 1) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 sz = half2_lds(chan_sz + (i0 + j) * 4);
            qz = fmaf(x[j], sz.y, qz);
            x[j] *= sz.x;
        }
    }
    float cf[4], first;
    if constexpr (KB == 16) {
#pragma unroll
        for (int j = 0; j < 4; ++j) cf[j] = x[j];
        first = 0.0f;
    } else if constexpr (KB == 4) {
#pragma unroll
        for (int j = 0; j < 4; ++j) cf[j] = 256.0f * x[j];
        first = (x[0] + x[1]) + (x[2] + x[3]);
    } else {
        // a0 X0 + a1 X1 + a2 X2 + a3 X3 = x0 c0 + x1 c1 + x2 c2 + x3 c3
        const float a3 = x[3] * 0.0625f;
        const float a2 = (x[2] - 4.0f * a3) * 0.0625f;
        const float a1 = (x[1] - 4.0f * a2 - a3) * 0.25f;
        const float a0 = x[0] - a1 - a2;
        cf[0] = 256.0f * a0; cf[1] = 256.0f * a1; cf[2] = 256.0f * a2; cf[3] = 256.0f * a3;
        first = (a0 + a1) + (a2 + a3);
    }
    const int c = i0 / RG::cpc, j = i0 - c * RG::cpc;
    *reinterpret_cast<float4 *>(cg + c * RG::cstr + j) = make_float4(cf[0], cf[1], cf[2], cf[3]);
    if constexpr (MODE == 2) {
        if (lane == 0) *reinterpret_cast<float2 *>(sums + g * 2) = make_float2(0.0f, 0.0f);
        return;
    }
    const int lpg = G >> 2;  // lanes per group
    if (GKC || MODE == 1) {
#pragma unroll
        for (int m = 1; m < ((MODE == 0) ? GKC : kHeadDim) / 4; m <<= 1) {
            first += __shfl_xor_sync(0xffffffffu, first, m);
            if (MODE == 0) qa += __shfl_xor_sync(0xffffffffu, qa, m);
            if (MODE == 1) qz += __shfl_xor_sync(0xffffffffu, qz, m);
        }
    } else {
        for (int m = 1; m < lpg; m <<= 1) {
            first += __shfl_xor_sync(0xffffffffu, first, m);
            qa += __shfl_xor_sync(0xffffffffu, qa, m);
        }
    }
    if ((lane & (lpg - 1)) == 0) {
        const int grp = i0 / G;
        const float init = (MODE == 1) ? fmaf(-128.0f, first, qz) : -128.0f * first;
        *reinterpret_cast<float2 *>(sums + (grp * GQA + g) * 2) = make_float2(init, qa);
    }
}

// Folded value sums of V_CHANNEL kernels (absent from the others, whose state
// is then exactly what it was without this mode).
template <int GQA, bool VCH>
struct FoldedSums {
    float of[GQA][4];      // folded value sums of earlier tiles, 4 channels per
                           // lane (half-warp h: channels 4h..4h+3)
};
template <int GQA>
struct FoldedSums<GQA, false> {};

// Per-warp decode state of the current item.
template <int GQA, int NVG, bool VCH>
struct WarpState : FoldedSums<GQA, VCH> {
    float mref[GQA];       // reference maximum per head (log2 units; warp-uniform)
    float thr[GQA];        // mref + slack: scores above it move the reference
    float l[GQA];          // this lane's tokens: sum of the weights p
    float W[GQA][NVG];     //                     sum of p * s per value group (one group)
    float Z[GQA][NVG];     //                     sum of p * z per value group
    float Wv[GQA];         // several value groups: sum of p * s of this lane's group
                           // over the token pairs its half-warp takes (value pass)
    float2 o[GQA][8];      // value accumulators: 8 channels x GQA heads, one
                           // token of a pair in each half (summed at the end)
};

// A new tile maximum moves the reference only when it exceeds the old one by
// more than this (weights then stay <= 2^8).
constexpr float kRescaleSlack = 8.0f;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
    return v;
}

// One tile: rows at kc / ks / vc / vs (shared memory), tokens [start, n) valid, TPW
// tokens per warp (warp w owns tile tokens [w*TPW, w*TPW + TPW)).
//   keys: lane j owns warp tokens j and j + 32 (TPW = 64) or token j (TPW <= 32);
//   values: token pairs (p, p + TPW/2); the half-warps take alternate pairs,
//     16 lanes cover the 128 channels (8 each); the weights of a pair sit
//     side by side, so one f32x2 FMA serves both tokens.
// FULL: all 4*TPW tokens are valid. SNK: the tile may start at `start` > 0
// (sink caches; otherwise start is 0). KMT/KB: key mode and bits of this tile
// (window tiles are bf16). GKC: compile-time key group size (0 = runtime
// gk_rt); GVC likewise for the values (0 = runtime, NVG groups at most).
template <int GQA, int KMT, int VMT, int KB, int VBITS, int TPW, int GKC, int GVC, int NVG, bool FULL,
          bool SNK, bool VCH, bool WV = false>
__device__ __forceinline__ void process_tile(const uint8_t *kc, const uint8_t *ks,
                                             const uint8_t *vc, const uint8_t *vs, int n, int start,
                                             const float *coef, int hstr, int cstr,
                                             const float *sums, int gk_rt, int gv_rt,
                                             WarpState<GQA, NVG, VCH> &st, float *wsm, int warp,
                                             int lane) {
    using RG = RowGeo<KB>;
    constexpr int TPL = (TPW >= 64) ? 2 : 1;  // key tokens per lane
    constexpr int HALF = TPW / 2;             // value pair distance
    constexpr int VROW = (VMT == V_BF16) ? kHeadDim * 2 : kHeadDim * VBITS / 8;
    const int t_warp = warp * TPW;
    int tr[TPL];
    bool valid[TPL];
#pragma unroll
    for (int m = 0; m < TPL; ++m) {
        const int tok = lane + 32 * m;
        valid[m] = FULL || (tok < TPW && t_warp + tok < n && (!SNK || t_warp + tok >= start));
        tr[m] = valid[m] ? t_warp + tok : (SNK ? start : 0);  // masked lanes read a staged, valid row
    }

    // ---- keys: this lane's tokens against every head ----
    const int G = (KMT == K_TOKEN) ? (GKC ? GKC : gk_rt) : kHeadDim;
    const int ngk = kHeadDim / G;
    const int rot = chunk_rot<KB>(lane);
    float sc[TPL][GQA];
    float2 acc[TPL][GQA];
#pragma unroll
    for (int m = 0; m < TPL; ++m)
#pragma unroll
        for (int g = 0; g < GQA; ++g) sc[m][g] = 0.0f;
    auto start_group = [&](int grp) {
#pragma unroll
        for (int g = 0; g < GQA; ++g) {
            const float init = (KMT == K_BF16) ? 0.0f : sums[(grp * GQA + g) * 2];
#pragma unroll
            for (int m = 0; m < TPL; ++m) acc[m][g] = make_float2(init, 0.0f);
        }
    };
    auto end_group = [&](int grp) {
        if constexpr (KMT == K_TOKEN) {
            float qa[GQA];
#pragma unroll
            for (int g = 0; g < GQA; ++g) qa[g] = sums[(grp * GQA + g) * 2 + 1];
#pragma unroll
            for (int m = 0; m < TPL; ++m) {
                const float2 sz = half2_lds(ks + (tr[m] * ngk + grp) * 4);
#pragma unroll
                for (int g = 0; g < GQA; ++g)
                    sc[m][g] = fmaf(sz.x, acc[m][g].x + acc[m][g].y, fmaf(sz.y, qa[g], sc[m][g]));
            }
        } else {
#pragma unroll
            for (int m = 0; m < TPL; ++m)
#pragma unroll
                for (int g = 0; g < GQA; ++g) sc[m][g] = acc[m][g].x + acc[m][g].y;
        }
    };
    const int cpg = G / RG::cpc;  // chunks per group (0: groups inside a chunk)
    const int wpg = G / RG::cpw;  // words per group
    if (KMT == K_BF16) start_group(0);
#pragma unroll
    for (int k = 0; k < RG::nch; ++k) {
        const int c = k ^ rot;
        if (KMT != K_BF16 && cpg > 0 && (k & (cpg - 1)) == 0) start_group(c / cpg);
        uint32_t wv[TPL][4];
#pragma unroll
        for (int m = 0; m < TPL; ++m) {
            const uint4 w4 = lds128(kc + tr[m] * RG::bytes + 16 * c);
            wv[m][0] = w4.x; wv[m][1] = w4.y; wv[m][2] = w4.z; wv[m][3] = w4.w;
        }
        const float *cc = coef + c * cstr;
        if constexpr (KB == 16) {
            // 4 words = 8 channels; coefficients 8 floats per head
            float2 f[TPL][4];
#pragma unroll
            for (int m = 0; m < TPL; ++m)
#pragma unroll
                for (int wi = 0; wi < 4; ++wi) word_pairs<16>(wv[m][wi], &f[m][wi]);
            float4 cv[GQA][2];
#pragma unroll
            for (int g = 0; g < GQA; ++g) {
                cv[g][0] = ldsf4(cc + g * hstr);
                cv[g][1] = ldsf4(cc + g * hstr + 4);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int m = 0; m < TPL; ++m)
#pragma unroll
                    for (int g = 0; g < GQA; ++g) {
                        const float4 v = cv[g][j >> 1];
                        ffma2(acc[m][g], (j & 1) ? make_float2(v.z, v.w) : make_float2(v.x, v.y), f[m][j]);
                    }
        } else {
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
                if (cpg == 0 && (wi & (wpg - 1)) == 0) start_group((c * 4 + wi) / wpg);
                // blocks of 4 pairs: every head's coefficients first, then the
                // multiply-adds interleaved across tokens and heads
#pragma unroll
                for (int jb = 0; jb < RG::npw; jb += 4) {
                    float2 f[TPL][4];
#pragma unroll
                    for (int m = 0; m < TPL; ++m) word_pairs4<KB>(wv[m][wi], jb, f[m]);
                    if constexpr (NVG == 1) {
                        // every head's coefficients first, then the multiply-adds
                        // interleaved across tokens and heads
                        float4 cv[GQA][2];
#pragma unroll
                        for (int g = 0; g < GQA; ++g) {
                            const float *cw = cc + g * hstr + wi * RG::cpw + 2 * jb;
                            cv[g][0] = ldsf4(cw);
                            cv[g][1] = ldsf4(cw + 4);
                        }
#pragma unroll
                        for (int j = 0; j < 4; ++j)
#pragma unroll
                            for (int m = 0; m < TPL; ++m)
#pragma unroll
                                for (int g = 0; g < GQA; ++g) {
                                    const float4 v = cv[g][j >> 1];
                                    ffma2(acc[m][g], (j & 1) ? make_float2(v.z, v.w) : make_float2(v.x, v.y),
                                          f[m][j]);
                                }
                    } else {
                        // head by head (fewer live registers next to the
                        // per-group value sums)
#pragma unroll
                        for (int g = 0; g < GQA; ++g) {
                            const float *cw = cc + g * hstr + wi * RG::cpw + 2 * jb;
                            const float4 c0 = ldsf4(cw), c1 = ldsf4(cw + 4);
#pragma unroll
                            for (int m = 0; m < TPL; ++m) {
                                ffma2(acc[m][g], make_float2(c0.x, c0.y), f[m][0]);
                                ffma2(acc[m][g], make_float2(c0.z, c0.w), f[m][1]);
                                ffma2(acc[m][g], make_float2(c1.x, c1.y), f[m][2]);
                                ffma2(acc[m][g], make_float2(c1.z, c1.w), f[m][3]);
                            }
                        }
                    }
                }
                if (cpg == 0 && ((wi + 1) & (wpg - 1)) == 0) end_group((c * 4 + wi) / wpg);
            }
        }
        if (KMT != K_BF16 && cpg > 0 && ((k + 1) & (cpg - 1)) == 0) end_group(c / cpg);
    }
    if (KMT == K_BF16) end_group(0);
#pragma unroll
    for (int m = 0; m < TPL; ++m)
        if (!valid[m]) {
#pragma unroll
            for (int g = 0; g < GQA; ++g) sc[m][g] = -INFINITY;
        }

    // ---- online softmax (per warp, per head), lazy reference ----
    bool up = false;
#pragma unroll
    for (int m = 0; m < TPL; ++m)
#pragma unroll
        for (int g = 0; g < GQA; ++g) up |= sc[m][g] > st.thr[g];
    if (__any_sync(0xffffffffu, up)) {
#pragma unroll
        for (int g = 0; g < GQA; ++g) {
            float mx = sc[0][g];
#pragma unroll
            for (int m = 1; m < TPL; ++m) mx = fmaxf(mx, sc[m][g]);
            mx = warp_max(mx);
            if (mx > st.thr[g]) {  // also true the first time (thr = -inf)
                const float alpha = (st.mref[g] == -INFINITY) ? 0.0f : fast_exp2(st.mref[g] - mx);
                st.mref[g] = mx;
                st.thr[g] = mx + kRescaleSlack;
                st.l[g] *= alpha;
#pragma unroll
                for (int v = 0; v < NVG; ++v) { st.W[g][v] *= alpha; st.Z[g][v] *= alpha; }
                if constexpr (WV) st.Wv[g] *= alpha;
#pragma unroll
                for (int c = 0; c < 8; ++c) { st.o[g][c].x *= alpha; st.o[g][c].y *= alpha; }
                if constexpr (VCH) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) st.of[g][c] *= alpha;
                }
            }
        }
    }
    float p[TPL][GQA];
#pragma unroll
    for (int g = 0; g < GQA; ++g) {
        // reference 0 while no token of this warp has been seen (all -inf)
        const float mref = (st.mref[g] == -INFINITY) ? 0.0f : st.mref[g];
#pragma unroll
        for (int m = 0; m < TPL; ++m) {
            p[m][g] = fast_exp2(sc[m][g] - mref);  // 0 for masked tokens
            st.l[g] += p[m][g];
        }
    }
    // Value weights w = p * s per (token, value group), at their pair slot.
    const int n_vg = (VMT != V_TOKEN) ? 1 : (GVC ? kHeadDim / GVC : kHeadDim / gv_rt);
    float2 *wsm2 = reinterpret_cast<float2 *>(wsm);
    // pair rows padded by 16 bytes so the lanes' rows start in different bank groups
    const int pstr = n_vg * GQA + 2;
#pragma unroll
    for (int v = 0; v < ((VMT == V_BF16) ? 1 : NVG); ++v) {
        if (v < n_vg) {
            float w[TPL][GQA];
            if constexpr (VMT == V_BF16) {
#pragma unroll
                for (int m = 0; m < TPL; ++m)
#pragma unroll
                    for (int g = 0; g < GQA; ++g) w[m][g] = p[m][g];
            } else if constexpr (VMT == V_CHANNEL) {  // scales come per channel, after the pass
#pragma unroll
                for (int m = 0; m < TPL; ++m)
#pragma unroll
                    for (int g = 0; g < GQA; ++g) {
                        w[m][g] = p[m][g];
                        st.W[g][0] += p[m][g];
                    }
            } else {
#pragma unroll
                for (int m = 0; m < TPL; ++m) {
                    const float2 szf = half2_lds(vs + (tr[m] * n_vg + v) * 4);
#pragma unroll
                    for (int g = 0; g < GQA; ++g) {
                        w[m][g] = p[m][g] * szf.x;
                        if constexpr (!WV) st.W[g][v] += w[m][g];
                        st.Z[g][v] = fmaf(p[m][g], szf.y, st.Z[g][v]);
                    }
                }
            }
            if constexpr (TPL == 2) {  // lane j owns pair j: both halves
#pragma unroll
                for (int g = 0; g < GQA; ++g) wsm2[lane * pstr + v * GQA + g] = make_float2(w[0][g], w[1][g]);
            } else if (lane < TPW) {
                const int slot = lane % HALF, half = lane / HALF;
#pragma unroll
                for (int g = 0; g < GQA; ++g) wsm[(slot * pstr + v * GQA + g) * 2 + half] = w[0][g];
            }
        }
    }
    __syncwarp();

    // ---- values ----
    const int slice = lane & 15, parity = lane >> 4;
    const int gv_lane = (VMT != V_TOKEN) ? 0 : (slice * 8) / (GVC ? GVC : gv_rt);
#pragma unroll 2
    for (int k = 0; k < HALF / 2; ++k) {
        const int pi = 2 * k + parity;
        const int ta = t_warp + pi, tb = ta + HALF;
        float2 f[8];
        value_pairs<VMT, VBITS>(vc + ta * VROW, vc + tb * VROW, slice, f);
        if (VMT == V_BF16 && !FULL) {  // stale bf16 rows may be NaN: drop them
            const bool va = ta < n, vb = tb < n;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                f[c].x = va ? f[c].x : 0.0f;
                f[c].y = vb ? f[c].y : 0.0f;
            }
        }
        const float2 *wrow = wsm2 + pi * pstr + gv_lane * GQA;
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
        // WV (several value groups): the lanes of a group sum its weights here
        // and the key side keeps Z only, which frees GQA x (NVG - 1) registers
        if constexpr (VMT == V_TOKEN && WV) {
#pragma unroll
            for (int g = 0; g < GQA; ++g) st.Wv[g] += w[g].x + w[g].y;
        }
#pragma unroll
        for (int g = 0; g < GQA; ++g)
#pragma unroll
            for (int c = 0; c < 8; ++c) ffma2(st.o[g][c], w[g], f[c]);
    }
    if constexpr (VMT == V_CHANNEL) {
        // The warp's tokens lie in one R-token block (R >= 64, tiles aligned):
        // fold this tile's sums with the block's channel scales, sum_t p_t v_t =
        // s * sum_t p_t c_t + z * sum_t p_t. The halves swap partial sums so
        // half h owns channels 4h..4h+3 of its slice; vs points at the block's
        // [128] (scale, zero) pairs. A warp without valid tokens skips (its
        // block's scales need not be staged).
        if (FULL || t_warp < n) {
            const int half = lane >> 4;
            const uint4 u = lds128(vs + (slice * 8 + 4 * half) * 4);
            const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
            float2 sz[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) sz[j] = __half22float2(*reinterpret_cast<const __half2 *>(&uw[j]));
#pragma unroll
            for (int g = 0; g < GQA; ++g) {
                float Wt = st.W[g][0];
#pragma unroll
                for (int m = 16; m > 0; m >>= 1) Wt += __shfl_xor_sync(0xffffffffu, Wt, m);
                float a[4], ch[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float lo = st.o[g][j].x + st.o[g][j].y;
                    const float hi = st.o[g][4 + j].x + st.o[g][4 + j].y;
                    const float other = __shfl_xor_sync(0xffffffffu, half ? lo : hi, 16);
                    a[j] = (half ? hi : lo) + other;
                }
                value_channels4<VBITS>(a, Wt, ch);
#pragma unroll
                for (int j = 0; j < 4; ++j) st.of[g][j] = fmaf(sz[j].x, ch[j], fmaf(sz[j].y, Wt, st.of[g][j]));
                st.W[g][0] = 0.0f;
#pragma unroll
                for (int c = 0; c < 8; ++c) st.o[g][c] = make_float2(0.0f, 0.0f);
            }
        }
    }
    __syncwarp();
}

// Decode an item index into (sequence, KV head, split). Items are numbered
// split-major: spref[j] is the first item of split j, whose items are the
// (sequence, KV head) units of the sequences with more than j splits
// (nsq[s] > j), in sequence order, KV head fastest. Run by a whole warp.
__device__ __forceinline__ void item_coords(const int *spref, const int *nsq, int n_split, int S, int H,
                                            int item, int &seq, int &kvh, int &split, int lane) {
    int lo = 0, hi = n_split;  // last j with spref[j] <= item
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (spref[mid] <= item) lo = mid; else hi = mid;
    }
    split = lo;
    const int k = item - spref[lo];
    int r = k / H;
    kvh = k - r * H;
    seq = 0;
    // the r-th sequence with more than `split` splits
    for (int base = 0; base < S; base += 32) {
        const unsigned m = __ballot_sync(0xffffffffu, base + lane < S && nsq[base + lane] > split);
        const int c = __popc(m);
        if (r < c) {
            seq = base + __fns(m, 0, r + 1);
            break;
        }
        r -= c;
    }
}

// Expected-transaction bytes for a bulk copy issued by this thread, without an
// arrival (the producer's lane 0 arrives once all lanes have added theirs).
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// Resident CTAs per SM the register budget targets: two, but one for the
// generic variants (runtime key group size, or up to 8 value groups of W/Z per
// lane) and for bf16 caches (whose 128-token stages take 66 KB each).
constexpr int decode_min_blocks(int km, int vm, int gkc, int gvc) {
    return (km == K_BF16 || (km == K_TOKEN && gkc == 0) || (vm == V_TOKEN && gvc == 0)) ? 1 : 2;
}

// Query rows of one item's GQA heads, rotated and scaled to log2 units, into
// qs [GQA][128] (and unrotated into qs_raw for the sink tiles), then the key
// coefficients of every head (token-wise and bf16 keys; per-channel keys
// build theirs per tile from qs). Run by one warp: the heads' loads are issued
// together, then the heads are rotated side by side.
template <int GQA, int KM, int KBF, int GKC, bool SINK>
__device__ __forceinline__ void build_item_query(const DecodeParams &p, const ItemInfo &inf, float *qs,
                                                 float *qs_raw, float *coefs, int lane) {
    using RG = RowGeo<KBF>;
    constexpr int QHSTR = RG::nch * RG::cstr;
    const int64_t row0 = static_cast<int64_t>(inf.seq) * p.Hq + inf.kvh * GQA;
    float x[GQA][4];
    if (p.q_dtype == KVQ_FP32) {
        float4 v[GQA];
#pragma unroll
        for (int g = 0; g < GQA; ++g)
            v[g] = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(p.q) + (row0 + g) * kHeadDim) + lane);
#pragma unroll
        for (int g = 0; g < GQA; ++g) { x[g][0] = v[g].x; x[g][1] = v[g].y; x[g][2] = v[g].z; x[g][3] = v[g].w; }
    } else {
        uint2 v[GQA];
#pragma unroll
        for (int g = 0; g < GQA; ++g)
            v[g] = __ldg(reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(p.q) + (row0 + g) * kHeadDim) + lane);
#pragma unroll
        for (int g = 0; g < GQA; ++g) {
            const uint32_t w[2] = {v[g].x, v[g].y};
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                if (p.q_dtype == KVQ_BF16) {
                    x[g][2 * j] = bf16_bits_to_float(w[j] & 0xFFFFu);
                    x[g][2 * j + 1] = bf16_bits_to_float(w[j] >> 16);
                } else {
                    x[g][2 * j] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[j] & 0xFFFFu)));
                    x[g][2 * j + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[j] >> 16)));
                }
            }
        }
    }
    if (SINK) {
#pragma unroll
        for (int g = 0; g < GQA; ++g)
            *reinterpret_cast<float4 *>(qs_raw + g * kHeadDim + 4 * lane) =
                make_float4(x[g][0] * p.qscale, x[g][1] * p.qscale, x[g][2] * p.qscale, x[g][3] * p.qscale);
    }
    if (p.signs != nullptr) {  // randomized Hadamard: diag(signs) first (exact)
        const float4 sg = __ldg(reinterpret_cast<const float4 *>(p.signs) + lane);
#pragma unroll
        for (int g = 0; g < GQA; ++g) { x[g][0] *= sg.x; x[g][1] *= sg.y; x[g][2] *= sg.z; x[g][3] *= sg.w; }
    }
    if (p.hb > 0) {
#pragma unroll
        for (int g = 0; g < GQA; ++g) {
            if (p.hb > 1) { float a = x[g][0], b = x[g][1]; x[g][0] = a + b; x[g][1] = a - b;
                            a = x[g][2]; b = x[g][3]; x[g][2] = a + b; x[g][3] = a - b; }
            if (p.hb > 2) { float a = x[g][0], b = x[g][2]; x[g][0] = a + b; x[g][2] = a - b;
                            a = x[g][1]; b = x[g][3]; x[g][1] = a + b; x[g][3] = a - b; }
        }
        for (int m = 1; m < 32 && 4 * m < p.hb; m <<= 1) {
            const bool upper = (lane & m) != 0;
#pragma unroll
            for (int g = 0; g < GQA; ++g)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float o = __shfl_xor_sync(0xffffffffu, x[g][j], m);
                    x[g][j] = upper ? o - x[g][j] : x[g][j] + o;
                }
        }
#pragma unroll
        for (int g = 0; g < GQA; ++g)
#pragma unroll
            for (int j = 0; j < 4; ++j) x[g][j] *= p.hscale;
    }
#pragma unroll
    for (int g = 0; g < GQA; ++g) {
#pragma unroll
        for (int j = 0; j < 4; ++j) x[g][j] *= p.qscale;
        *reinterpret_cast<float4 *>(qs + g * kHeadDim + 4 * lane) = make_float4(x[g][0], x[g][1], x[g][2], x[g][3]);
        if constexpr (KM == K_TOKEN)
            build_head<GQA, KBF, 0, GKC>(x[g], nullptr, coefs + g * QHSTR, coefs + GQA * QHSTR, g, p.gk, lane);
        if constexpr (KM == K_BF16)
            build_head<GQA, 16, 2, 0>(x[g], nullptr, coefs + g * QHSTR, coefs + GQA * QHSTR, g, 128, lane);
    }
}

// Warp roles of a CTA: warps 0..3 consume tiles, warp 4 streams them (bulk
// copies into the stage ring), warp 5 prepares every item's query rows and
// coefficients one item ahead and merges the consumers' item states into the
// split's partial. The consumers never wait for each other: an item begins
// when its coefficients are ready and ends with each warp depositing its
// state; per-channel keys alone share per-tile coefficient builds.
//
// Item slots (kItemSlots, used round robin by the CTA's item ordinal n):
//   posted[j]    producer -> helper: the item's coordinates are in info[j]
//   coef_full[j] helper -> consumers: qs / coefficients of slot j are built
//   slot_free[j] helper -> producer: item n merged, slot j may take n + 2
// and, single-buffered, deposited (consumers -> helper: the four states of
// item n are in dep) and merged (helper -> consumers: dep may take n + 1).
template <int GQA, int KM, int VM, int KBITS, int VBITS, int GKC, int GVC, int TL>
__global__ void __launch_bounds__(kThreads, decode_min_blocks(KM, VM, GKC, GVC))
decode_splitk_kernel(const DecodeParams p) {
    constexpr bool SINK = TL == kTailSink;
    constexpr bool WIN = TL == kTailWindow;
    constexpr int NVG = (VM != V_TOKEN) ? 1 : (GVC ? kHeadDim / GVC : kMaxGroups);
    // weight sums of several value groups in the value pass (see process_tile)
    constexpr bool WV = NVG > 1;
    constexpr int KBF = (KM == K_BF16) ? 16 : KBITS;  // key form of quantized tiles
    constexpr int TILE = (KM == K_BF16) ? kTileB : kTileQ;
    constexpr int TPW = TILE / kConsumerWarps;
    using RG = RowGeo<KBF>;
    constexpr int QHSTR = RG::nch * RG::cstr;                 // coefficient floats per head
    constexpr int CBUF = GQA * QHSTR + kMaxGroups * GQA * 2;  // coefficients + group sums
    constexpr int QF = GQA * kHeadDim;                        // floats of one set of query rows
    constexpr int RSTR = kDepStride;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NS = p.ns;

    uint8_t *stages = smem;
    float *slots = reinterpret_cast<float *>(smem + p.off_slots);    // [kItemSlots][slot_floats]
    float *csets = reinterpret_cast<float *>(smem + p.off_csets);    // per-channel keys: [n_sets][CBUF]
    float *dep = reinterpret_cast<float *>(smem + p.off_dep);        // [warps][GQA][RSTR]
    float *scratch_all = reinterpret_cast<float *>(smem + p.off_scr);  // [warps][warp_floats]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.off_bar);
    uint64_t *empty = full + kMaxStages;
    uint64_t *posted = empty + kMaxStages;
    uint64_t *coef_full = posted + kItemSlots;
    uint64_t *slot_free = coef_full + kItemSlots;
    uint64_t *deposited = slot_free + kItemSlots;
    uint64_t *merged = deposited + 1;
    int *abort_word = reinterpret_cast<int *>(merged + 1);
    volatile int *abort_flag = abort_word;
    ItemInfo *info = reinterpret_cast<ItemInfo *>(abort_word + 4);  // [kItemSlots]
    int *spref = reinterpret_cast<int *>(info + kItemSlots);        // [n_split + 1] first item of each split
    int *lens = spref + p.sp.n + 1;                                  // [S] clamped lengths
    int *nsq = lens + p.S;                                           // [S] splits of each sequence

    // The producer's first length load is issued before the set-up barrier.
    const int t_first = (warp == kProducerWarp && lane < p.S) ? __ldg(p.seq_lens + lane) : 0;
    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        for (int j = 0; j < kItemSlots; ++j) {
            mbar_init(&posted[j], 1);
            mbar_init(&coef_full[j], 32);
            mbar_init(&slot_free[j], 32);
        }
        mbar_init(deposited, kConsumers);
        mbar_init(merged, 32);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // A dependent launch (the merge pass) may be scheduled from now on; it
    // waits for this grid's completion before reading anything.
    pdl_launch_dependents();

    if (warp == kHelperWarp) {
        // ------------------------- helper -------------------------
        // Item n's coefficients are built once its coordinates are posted;
        // item n is merged once its four states are deposited. Builds run one
        // item ahead of merges.
        auto build = [&](int j) {
            float *slot = slots + j * p.slot_floats;
            const ItemInfo inf = info[j];
            build_item_query<GQA, KM, KBF, GKC, SINK>(p, inf, slot, slot + QF, slot + (SINK ? 2 : 1) * QF, lane);
            mbar_arrive(&coef_full[j]);
        };
        if (!mbar_wait_bounded(&posted[0], 0, p.timeout_ns, p.status, abort_flag)) return;
        if (info[0].done) return;
        build(0);
        for (int n = 0;; ++n) {
            const int j = n % kItemSlots, j1 = (n + 1) % kItemSlots;
            if (!mbar_wait_bounded(&posted[j1], ((n + 1) / kItemSlots) & 1, p.timeout_ns, p.status, abort_flag))
                return;
            const bool more = !info[j1].done;
            if (more) build(j1);
            if (!mbar_wait_bounded(deposited, n & 1, p.timeout_ns, p.status, abort_flag)) return;
            // merge the warps' states of item n: head g, 4 channels per lane
            const ItemInfo inf = info[j];
#pragma unroll 1
            for (int g = 0; g < GQA; ++g) {
                float2 mlw[kConsumerWarps];
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) {
                    mlw[w] = *reinterpret_cast<const float2 *>(dep + (w * GQA + g) * RSTR + kHeadDim);
                    M = fmaxf(M, mlw[w].x);
                }
                float4 o = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                float l = 0.0f;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) {
                    const float e = (mlw[w].x == -INFINITY) ? 0.0f : fast_exp2(mlw[w].x - M);
                    const float4 ov = ldsf4(dep + (w * GQA + g) * RSTR + 4 * lane);
                    o.x = fmaf(e, ov.x, o.x); o.y = fmaf(e, ov.y, o.y);
                    o.z = fmaf(e, ov.z, o.z); o.w = fmaf(e, ov.w, o.w);
                    l = fmaf(e, mlw[w].y, l);
                }
                const int hq = inf.kvh * GQA + g;
                const int64_t pi = (static_cast<int64_t>(inf.seq) * p.Hq + hq) * p.n_split + inf.split;
                *reinterpret_cast<float4 *>(p.o_part + pi * kHeadDim + 4 * lane) = o;
                if (lane == 0) p.ml[pi] = make_float2(M, l);
            }
            mbar_arrive(merged);
            mbar_arrive(&slot_free[j]);
            if (!more) return;
        }
    }

    if (warp == kProducerWarp) {
        // ------------------------- producer -------------------------
        // CTA b takes item b first (no atomic on the start-up path); later
        // items come from the counter, offset by the grid, one item ahead.
        int next = static_cast<int>(blockIdx.x);
        // Lengths (clamped) and split counts of the sequences. When every
        // sequence has all n_split splits the items are regular (split
        // item / units, unit item % units); otherwise items per split are
        // H x the sequences with more than j splits, and their prefix gives
        // the first item of each split.
        const int n_split = p.sp.n;
        bool full_lane = true;
        for (int s = lane; s < p.S; s += 32) {
            int T_s = (s == lane) ? t_first : __ldg(p.seq_lens + s);
            if (T_s > p.max_seq_len) {
                if (blockIdx.x == 0) status_or(p.status, KVQ_DEV_SEQLEN);
                T_s = p.max_seq_len;
            }
            lens[s] = T_s;
            const int ns = splits_of(p.sp, T_s);
            nsq[s] = ns;
            full_lane = full_lane && ns == n_split;
        }
        const bool regular = __all_sync(0xffffffffu, full_lane);
        const int units = p.S * p.H;
        int n_items = n_split * units;
        if (!regular) {
            for (int j = lane; j <= n_split; j += 32) spref[j] = 0;  // histogram of split counts
            __syncwarp();
            for (int s = lane; s < p.S; s += 32) atomicAdd(&spref[nsq[s]], 1);
            __syncwarp();
            // G_j = #{s : n_s > j} (suffix sums of the histogram), from the top
            int gsum = 0;
            for (int base = ((n_split - 1) / 32) * 32; base >= 0; base -= 32) {
                const int j = base + lane;
                int v = (j < n_split) ? spref[j + 1] : 0;
#pragma unroll
                for (int m = 1; m < 32; m <<= 1) {
                    const int o = __shfl_down_sync(0xffffffffu, v, m);
                    if (lane + m < 32) v += o;
                }
                const int G = v + gsum;
                gsum += __shfl_sync(0xffffffffu, v, 0);
                __syncwarp();
                if (j < n_split) spref[j + 1] = G;  // G_j parked one slot up
                __syncwarp();
            }
            // exclusive prefix of H * G_j: spref[j] = first item of split j
            int carry = 0;
            for (int base = 0; base < n_split; base += 32) {
                const int j = base + lane;
                const int cnt = (j < n_split) ? p.H * spref[j + 1] : 0;
                int incl = cnt;
#pragma unroll
                for (int m = 1; m < 32; m <<= 1) {
                    const int o = __shfl_up_sync(0xffffffffu, incl, m);
                    if (lane >= m) incl += o;
                }
                __syncwarp();
                if (j < n_split) spref[j] = carry + incl - cnt;
                carry += __shfl_sync(0xffffffffu, incl, 31);
                __syncwarp();
            }
            if (lane == 0) spref[n_split] = carry;
            __syncwarp();
            n_items = carry;
        }

        constexpr int KROW = RowGeo<KBF>::bytes;
        constexpr int VROW = (VM == V_BF16) ? kHeadDim * 2 : kHeadDim * VBITS / 8;
        const int ngk = (KM == K_TOKEN) ? kHeadDim / p.gk : 0;
        const int ngv = (VM == V_TOKEN) ? kHeadDim / p.gv : 0;
        int it = 0;  // tile counter of this CTA (stage it % NS, round it / NS)
        int ps = 0, pr = 0;  // it % NS and it / NS, carried
        bool stop = false;
        for (int n_item = 0; !stop; ++n_item) {
            int item = __shfl_sync(0xffffffffu, next, 0);
            if (lane == 0 && item < n_items) next = atomicAdd(p.counter, 1) + static_cast<int>(gridDim.x);
            int seq = 0, kvh = 0, split = 0;
            int t_begin = 0, t_end = 0, Tq = 0, q_end = 0, n_qt = 0, w_begin = 0, n_wt = 0, n_sink = 0, n_st = 0;
            if (item < n_items) {
                if (regular) {
                    split = item / units;
                    const int u = item - split * units;
                    seq = u / p.H;
                    kvh = u - seq * p.H;
                } else {
                    item_coords(spref, nsq, n_split, p.S, p.H, item, seq, kvh, split, lane);
                }
                const int T = lens[seq];
                t_begin = split_begin(p.sp, split);
                t_end = min(T, split_begin(p.sp, split + 1));
                Tq = quantized_len(T, p.R);
                q_end = min(t_end, Tq);
                // sink positions [0, sink_len) are read from the sink rows, in
                // window-sized tiles after the quantized ones (so the value sums
                // are folded first)
                const int q_begin = SINK ? max(t_begin, p.sink_len) : t_begin;
                n_qt = q_end > q_begin ? (q_end - t_begin + TILE - 1) / TILE : 0;
                w_begin = max(t_begin, Tq);
                n_wt = (WIN && t_end > w_begin) ? (t_end - w_begin + p.bf_tile - 1) / p.bf_tile : 0;
                n_sink = (SINK && split == 0 && p.sink_len > 0) ? min(p.sink_len, T) : 0;
                n_st = (n_sink + p.bf_tile - 1) / p.bf_tile;
            }
            // Post the item (or the end marker) in its slot for the helper.
            {
                const int j = n_item % kItemSlots, u = n_item / kItemSlots;
                int ok = 1;
                if (lane == 0 && u > 0)
                    ok = mbar_wait_bounded(&slot_free[j], (u - 1) & 1, p.timeout_ns, p.status, abort_flag);
                if (!__shfl_sync(0xffffffffu, ok, 0)) break;
                if (lane == 0) {
                    info[j] = ItemInfo{seq, kvh, split, item >= n_items ? 1 : 0};
                    mbar_arrive(&posted[j]);
                }
            }
            const int n_tiles = (item < n_items) ? n_qt + n_wt + n_st : 1;  // 1 = the done marker
            const int64_t sh = static_cast<int64_t>(seq) * p.H + kvh;
            for (int ti = 0; ti < n_tiles; ++ti, ++it, (++ps == NS) ? (ps = 0, ++pr) : 0) {
                const int s = ps, r = pr;
                int ok = 1;
                if (lane == 0 && r > 0)
                    ok = mbar_wait_bounded(&empty[s], (r - 1) & 1, p.timeout_ns, p.status, abort_flag);
                if (!__shfl_sync(0xffffffffu, ok, 0)) {
                    stop = true;
                    break;
                }
                uint8_t *st = stages + static_cast<size_t>(s) * p.stage_bytes;
                uint64_t *bar = &full[s];
                TileHdr *hdr = reinterpret_cast<TileHdr *>(st + p.off_hdr);
                if (item >= n_items) {  // no work left: tell the consumers
                    if (lane == 0) {
                        hdr->flags = kDone;
                        mbar_arrive(bar);
                    }
                    stop = true;
                    ++it;
                    break;
                }
                if (it == p.skip_tile) continue;  // test hook: never arrive
                const bool sink = SINK && ti >= n_qt + n_wt;
                const bool window = TL != kTailNone && ti >= n_qt;
                const int t0 = sink ? (ti - n_qt - n_wt) * p.bf_tile
                                    : (window ? w_begin + (ti - n_qt) * p.bf_tile : t_begin + ti * TILE);
                const int n = sink ? min(p.bf_tile, n_sink - t0)
                                   : (window ? min(p.bf_tile, t_end - t0) : min(TILE, q_end - t0));
                if (lane == 0) {
                    hdr->t0 = t0;
                    hdr->n = n;
                    hdr->start = (SINK && !window) ? max(0, p.sink_len - t0) : 0;
                    hdr->flags = (ti == 0 ? kFirst : 0) | (ti == n_tiles - 1 ? kLast : 0) |
                                 (window ? kWindow : 0) | (sink ? kSink : 0);
                    hdr->item = n_item;
                }
                if (sink) {
                    const uint32_t bytes = n * kHeadDim * 2;
                    const int64_t row = sh * p.sink_len + t0;
                    if (lane < 2) {
                        mbar_expect_tx(bar, bytes);
                        if (lane == 0) bulk_g2s(st, p.k_sink + row * kHeadDim, bytes, bar);
                        else bulk_g2s(st + p.bf_off_v, p.v_sink + row * kHeadDim, bytes, bar);
                    }
                } else if (window) {
                    const uint32_t bytes = n * kHeadDim * 2;
                    const int64_t slot = sh * p.R + (t0 - Tq);
                    if (lane < 2) {
                        mbar_expect_tx(bar, bytes);
                        if (lane == 0) bulk_g2s(st, p.k_res + slot * kHeadDim, bytes, bar);
                        else bulk_g2s(st + p.bf_off_v, p.v_res + slot * kHeadDim, bytes, bar);
                    }
                } else if (!p.paged) {
                    // one lane per part: K codes, V codes, K scale/zero, V scale/zero
                    const int64_t row = sh * p.cap + t0;
                    if (lane == 0) {
                        mbar_expect_tx(bar, n * KROW);
                        bulk_g2s(st, p.k_codes + row * KROW, n * KROW, bar);
                    } else if (lane == 1) {
                        mbar_expect_tx(bar, n * VROW);
                        bulk_g2s(st + p.off_vc, p.v_codes + row * VROW, n * VROW, bar);
                    } else if (lane == 2 && KM == K_TOKEN) {
                        const uint32_t b = (n * ngk * 4 + 15) & ~15;
                        mbar_expect_tx(bar, b);
                        bulk_g2s(st + p.off_ksz, p.k_sz + row * ngk, b, bar);
                    } else if (lane == 2 && KM == K_CHANNEL) {
                        // the channel scales of every block the tile touches
                        const int b0 = t0 >> p.r_shift, nb = ((t0 + n - 1) >> p.r_shift) - b0 + 1;
                        mbar_expect_tx(bar, nb * kHeadDim * 4);
                        bulk_g2s(st + p.off_ksz, p.k_sz + (sh * (p.cap / p.R) + b0) * kHeadDim,
                                 nb * kHeadDim * 4, bar);
                    } else if (lane == 3 && VM == V_TOKEN) {
                        const uint32_t b = (n * ngv * 4 + 15) & ~15;
                        mbar_expect_tx(bar, b);
                        bulk_g2s(st + p.off_vsz, p.v_sz + row * ngv, b, bar);
                    } else if (lane == 3 && VM == V_CHANNEL) {
                        const int b0 = t0 >> p.r_shift, nb = ((t0 + n - 1) >> p.r_shift) - b0 + 1;
                        mbar_expect_tx(bar, nb * kHeadDim * 4);
                        bulk_g2s(st + p.off_vsz, p.v_sz + (sh * (p.cap / p.R) + b0) * kHeadDim,
                                 nb * kHeadDim * 4, bar);
                    }
                } else {
                    // Paged (token-wise groups only): one lane per page (or per
                    // tile-sized span of a larger page), four copies each.
                    const int ps = p.page_size;
                    const int span = ps < TILE ? ps : TILE;  // tokens per copy
                    const int tp = t0 + lane * span;
                    if (tp < t0 + n) {
                        const int32_t *bt = p.block_table + static_cast<int64_t>(seq) * p.max_pages;
                        const int pi = tp / ps;
                        const int page = (pi < p.max_pages) ? __ldg(bt + pi) : -1;
                        if (page >= 0 && page < p.num_pages) {
                            const int64_t prow = (static_cast<int64_t>(page) * p.H + kvh) * ps + (tp % ps);
                            const uint32_t dt = tp - t0;
                            mbar_expect_tx(bar, span * (KROW + VROW + 4 * ngk + 4 * ngv));
                            bulk_g2s(st + dt * KROW, p.k_codes + prow * KROW, span * KROW, bar);
                            bulk_g2s(st + p.off_ksz + dt * ngk * 4, p.k_sz + prow * ngk, span * ngk * 4, bar);
                            bulk_g2s(st + p.off_vc + dt * VROW, p.v_codes + prow * VROW, span * VROW, bar);
                            bulk_g2s(st + p.off_vsz + dt * ngv * 4, p.v_sz + prow * ngv, span * ngv * 4, bar);
                        } else {
                            status_or(p.status, KVQ_DEV_CAPACITY);
                        }
                    }
                }
                __syncwarp();  // every lane has added its bytes before the arrival
                if (lane == 0) mbar_arrive(bar);
            }
        }
        // Drain: wait for the copies of the last stages issued so none lands
        // after the CTA has gone.
        if (lane == 0) {
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
        }
        return;
    }

    // --------------------------- consumers ---------------------------
    float *scratch = scratch_all + warp * p.warp_floats;
    float *wsm = scratch;                  // value weights / W-Z partials of the lanes
    float *totals = scratch + p.off_tot;   // W-Z totals of the warp
    const int slice = lane & 15;

    constexpr bool VCH = VM == V_CHANNEL;
    WarpState<GQA, NVG, VCH> st;
    bool folded = false;
    // Turn the value accumulators of quantized tiles into plain channel sums
    // (adding the zero-point terms), once: before the first bf16 window tile
    // or at the end of the item. The lanes' W/Z partials are summed through
    // shared memory (one column per lane). Half-warp 1 adds no group terms, so
    // the halves still sum.
    auto fold_values = [&]() {
        const int n_vg = GVC ? kHeadDim / GVC : kHeadDim / p.gv;
        const int nw = WV ? 0 : GQA * n_vg;
        const int nv = nw + GQA * n_vg;  // values per lane: W (one group) then Z, [g][v]
        const int rs = nv + 1;          // odd row stride: the lanes' rows hit distinct banks
#pragma unroll
        for (int g = 0; g < GQA; ++g)
#pragma unroll
            for (int v = 0; v < NVG; ++v)
                if (v < n_vg) {
                    if constexpr (!WV) wsm[lane * rs + g * n_vg + v] = st.W[g][v];
                    wsm[lane * rs + nw + g * n_vg + v] = st.Z[g][v];
                }
        __syncwarp();
        for (int col = lane; col < nv; col += 32) {
            float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
            for (int r = 0; r < 32; r += 2) {
                a0 += wsm[r * rs + col];
                a1 += wsm[(r + 1) * rs + col];
            }
            totals[col] = a0 + a1;
        }
        __syncwarp();
        const int gv_lane = (slice * 8) / (GVC ? GVC : p.gv);
        const bool first_half = lane < 16;
#pragma unroll
        for (int g = 0; g < GQA; ++g) {
            float Wg;
            if constexpr (WV) {  // the two half-warps took the even and the odd pairs
                const float ws = st.Wv[g] + __shfl_xor_sync(0xffffffffu, st.Wv[g], 16);
                Wg = first_half ? ws : 0.0f;
                st.Wv[g] = 0.0f;
            } else {
                Wg = first_half ? totals[g * n_vg + gv_lane] : 0.0f;
            }
            const float Zg = first_half ? totals[nw + g * n_vg + gv_lane] : 0.0f;
            float a[8], ch[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) a[c] = st.o[g][c].x + st.o[g][c].y;
            value_channels<VM, VBITS>(a, Wg, ch);
#pragma unroll
            for (int c = 0; c < 8; ++c) st.o[g][c] = make_float2(ch[c] + Zg, 0.0f);
#pragma unroll
            for (int v = 0; v < NVG; ++v) { st.W[g][v] = 0.0f; st.Z[g][v] = 0.0f; }
        }
        __syncwarp();
        folded = true;
    };

    int kc_tiles = 0;  // quantized tiles seen (parity of the per-channel coefficient sets)
    // stage s of the ring and the parity of its round, carried from tile to tile
    for (int s = 0, ph = 0;; (++s == NS) ? (s = 0, ph ^= 1) : 0) {
        if (!mbar_wait_bounded(&full[s], ph, p.timeout_ns, p.status, abort_flag)) break;
        const uint8_t *sb = stages + static_cast<size_t>(s) * p.stage_bytes;
        const TileHdr hdr = *reinterpret_cast<const TileHdr *>(sb + p.off_hdr);
        if (hdr.flags & kDone) break;
        const int jslot = hdr.item % kItemSlots;
        const float *qs = slots + jslot * p.slot_floats;
        const float *coefs = qs + (SINK ? 2 : 1) * QF;

        if (hdr.flags & kFirst) {
            // ---- item start: the helper has built this slot's query rows ----
            if (!mbar_wait_bounded(&coef_full[jslot], (hdr.item / kItemSlots) & 1, p.timeout_ns, p.status,
                                   abort_flag))
                break;
#pragma unroll
            for (int g = 0; g < GQA; ++g) {
                st.mref[g] = -INFINITY;
                st.thr[g] = -INFINITY;
                st.l[g] = 0.0f;
#pragma unroll
                for (int v = 0; v < NVG; ++v) { st.W[g][v] = 0.0f; st.Z[g][v] = 0.0f; }
                st.Wv[g] = 0.0f;
#pragma unroll
                for (int c = 0; c < 8; ++c) st.o[g][c] = make_float2(0.0f, 0.0f);
                if constexpr (VCH) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) st.of[g][c] = 0.0f;
                }
            }
            folded = false;
        }

        if (!(hdr.flags & kWindow)) {
            const float *coef = coefs;
            if constexpr (KM == K_CHANNEL) {
                // Fold the channel scales of the tile's blocks into the
                // coefficients: the warps share the (block, head) builds into
                // the sets of this tile's parity (no warp still reads them:
                // all passed the previous tile's barrier), then wait for all.
                const int nbt = TILE >> p.r_shift;  // block sets per tile
                float *sets = csets + (kc_tiles & 1) * nbt * CBUF;
                const int nb = (hdr.n + p.R - 1) >> p.r_shift;
                for (int idx = warp; idx < nb * GQA; idx += kConsumerWarps) {
                    const int b = idx / GQA, g = idx - b * GQA;
                    const float4 xv = ldsf4(qs + g * kHeadDim + 4 * lane);
                    const float x[4] = {xv.x, xv.y, xv.z, xv.w};
                    float *set = sets + b * CBUF;
                    build_head<GQA, KBF, 1, 0>(x, sb + p.off_ksz + b * kHeadDim * 4, set + g * QHSTR,
                                               set + GQA * QHSTR, g, 128, lane);
                }
                named_sync(2, kConsumers);
                ++kc_tiles;
                coef = sets + min((warp * TPW) >> p.r_shift, nbt - 1) * CBUF;
            }
            constexpr int GKC_T = (KM == K_TOKEN) ? GKC : kHeadDim;
            // per-channel values: this warp's block among the tile's staged ones
            const uint8_t *vsz = sb + p.off_vsz;
            if constexpr (VM == V_CHANNEL)
                vsz += (((hdr.t0 + warp * TPW) >> p.r_shift) - (hdr.t0 >> p.r_shift)) * kHeadDim * 4;
            // one code path for full and partial tiles: the masks cost a few
            // instructions per tile, a second unrolled copy costs instruction
            // cache misses
            process_tile<GQA, KM, VM, KBF, VBITS, TPW, GKC_T, GVC, NVG, false, SINK, VM == V_CHANNEL, WV>(
                    sb, sb + p.off_ksz, sb + p.off_vc, vsz, hdr.n, SINK ? hdr.start : 0, coef, QHSTR,
                    RG::cstr, coef + GQA * QHSTR, p.gk, p.gv, st, wsm, warp, lane);
        } else if constexpr (KM != K_BF16 && TL != kTailNone) {
            if (!folded) {  // first window tile of the item
                if (VM == V_TOKEN) fold_values();
                folded = true;
            }
            // bf16 window keys against the query rows (coefficients = q), or
            // sink keys against the unrotated ones (one code path for both)
            const float *qrows = (SINK && (hdr.flags & kSink)) ? qs + QF : qs;
            process_tile<GQA, K_BF16, V_BF16, 16, 16, kWinTile / kConsumerWarps, kHeadDim, 0, NVG, false, false>(
                sb, nullptr, sb + p.bf_off_v, nullptr, hdr.n, 0, qrows, kHeadDim, 8, nullptr, p.gk, p.gv, st,
                wsm, warp, lane);
        }

        if (hdr.flags & kLast) {
            // ---- item end: deposit this warp's state for the helper's merge ----
            if (VM == V_TOKEN && !folded) fold_values();
            if constexpr (VM == V_CHANNEL) {  // the folded sums join the window's
                const bool hi = lane >= 16;
#pragma unroll
                for (int g = 0; g < GQA; ++g)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        st.o[g][j].x += hi ? 0.0f : st.of[g][j];
                        st.o[g][4 + j].x += hi ? st.of[g][j] : 0.0f;
                    }
            }
            if (hdr.item > 0 &&
                !mbar_wait_bounded(merged, (hdr.item - 1) & 1, p.timeout_ns, p.status, abort_flag))
                break;
            float *red = dep + warp * GQA * RSTR;
#pragma unroll
            for (int g = 0; g < GQA; ++g) {
                float lg = st.l[g];
#pragma unroll
                for (int m = 16; m > 0; m >>= 1) lg += __shfl_xor_sync(0xffffffffu, lg, m);
                float v[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float a = st.o[g][c].x + st.o[g][c].y;
                    v[c] = a + __shfl_xor_sync(0xffffffffu, a, 16);
                }
                if (lane < 16) {
                    float *rp = red + g * RSTR + 8 * slice;
                    *reinterpret_cast<float4 *>(rp) = make_float4(v[0], v[1], v[2], v[3]);
                    *reinterpret_cast<float4 *>(rp + 4) = make_float4(v[4], v[5], v[6], v[7]);
                }
                if (lane == 0) *reinterpret_cast<float2 *>(red + g * RSTR + kHeadDim) = make_float2(st.mref[g], lg);
            }
            mbar_arrive(deposited);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
struct StageLayout {
    int bytes, off_ksz, off_vc, off_vsz, off_hdr, bf_tile, bf_off_v;
};

inline int round16(int x) { return (x + 15) & ~15; }

// Stage: tile data, then a 32-byte header.
inline StageLayout stage_layout(const kvq_cache_desc &d) {
    StageLayout L{};
    int data;
    if (d.bits_k == 16) {  // every tile is bf16 rows: K at 0, V after it
        L.bf_tile = kTileB;
        L.bf_off_v = kTileB * 256;
        L.off_vc = L.bf_off_v;
        data = 2 * kTileB * 256;
    } else {
        const int krow = 128 * d.bits_k / 8;
        const int vrow = 128 * d.bits_v / 8;
        const int ksz = (d.axis_k == KVQ_PER_CHANNEL) ? (kTileQ / d.residual_len) * 128 * 4
                                                      : kTileQ * (128 / d.group_k) * 4;
        const int vsz = (d.axis_v == KVQ_PER_CHANNEL) ? (kTileQ / d.residual_len) * 128 * 4
                                                      : kTileQ * (128 / d.group_v) * 4;
        L.off_ksz = round16(kTileQ * krow);
        L.off_vc = L.off_ksz + round16(ksz);
        L.off_vsz = L.off_vc + round16(kTileQ * vrow);
        data = L.off_vsz + round16(vsz);
        L.bf_tile = kWinTile;
        L.bf_off_v = kWinTile * 256;
        if (d.residual_len > 0 || d.sink_len > 0) data = std::max(data, 2 * kWinTile * 256);
    }
    L.off_hdr = round16(data);
    L.bytes = (L.off_hdr + static_cast<int>(sizeof(TileHdr)) + 127) & ~127;
    return L;
}

// Per-warp scratch (floats): the value weights of one tile, which also hold
// the lanes' W/Z partials when they are summed, then the W/Z totals.
struct ScratchLayout {
    int off_tot, floats;
};

inline ScratchLayout scratch_layout(int gqa, int n_vg) {
    ScratchLayout S{};
    S.off_tot = 64 * gqa * n_vg + 128;  // 32 pair rows of (n_vg * gqa + 2) f32x2
    const int used = S.off_tot + 2 * gqa * n_vg;
    S.floats = (used + 3) & ~3;
    return S;
}

inline int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

template <int GQA, int KM, int VM, int KBITS, int VBITS, int GKC, int GVC, int TL = kTailNone>
kvq_status launch_variant(DecodeParams p, int max_items, cudaStream_t stream) {
    constexpr bool SINK = TL == kTailSink;
    constexpr int KBF = (KM == K_BF16) ? 16 : KBITS;
    constexpr int nch = RowGeo<KBF>::nch;
    constexpr int cbuf = GQA * nch * RowGeo<KBF>::cstr + kMaxGroups * GQA * 2;
    const int n_vg = (VM != V_TOKEN) ? 1 : kHeadDim / p.gv;
    const ScratchLayout SL = scratch_layout(GQA, n_vg);
    p.warp_floats = SL.floats;
    p.off_tot = SL.off_tot;
    p.n_sets = (KM == K_CHANNEL) ? 2 * (kTileQ / p.R) : 0;
    // item slots: rotated query rows (+ unrotated for sinks), then the key
    // coefficients (per-channel keys build theirs per tile in the sets)
    p.slot_floats = (SINK ? 2 : 1) * GQA * kHeadDim + (KM == K_CHANNEL ? 0 : cbuf);
    p.slot_floats = (p.slot_floats + 3) & ~3;
    const size_t tail = sizeof(float) * (static_cast<size_t>(kItemSlots) * p.slot_floats +
                                         static_cast<size_t>(p.n_sets) * cbuf +
                                         static_cast<size_t>(kConsumerWarps) * GQA * kDepStride +
                                         kConsumerWarps * static_cast<size_t>(p.warp_floats)) +
                        sizeof(uint64_t) * (2 * kMaxStages + 3 * kItemSlots + 2) + 16 +
                        sizeof(ItemInfo) * kItemSlots + sizeof(int) * (2 * p.S + p.sp.n + 1);
    // Ring depth: as many stages (2..4) as let the targeted CTAs per SM fit.
    const int per_sm_target = decode_min_blocks(KM, VM, GKC, GVC);
    const size_t budget = (232448 - 1024 * per_sm_target) / per_sm_target;
    int ns = static_cast<int>(std::min<size_t>(kMaxStages, (budget > tail ? budget - tail : 0) / p.stage_bytes));
    p.ns = std::max(2, ns);
    p.off_slots = p.ns * p.stage_bytes;
    p.off_csets = p.off_slots + static_cast<int>(sizeof(float)) * kItemSlots * p.slot_floats;
    p.off_dep = p.off_csets + static_cast<int>(sizeof(float)) * p.n_sets * cbuf;
    p.off_scr = p.off_dep + static_cast<int>(sizeof(float)) * kConsumerWarps * GQA * kDepStride;
    p.off_bar = p.off_scr + static_cast<int>(sizeof(float)) * kConsumerWarps * p.warp_floats;
    const size_t smem = static_cast<size_t>(p.off_slots) + tail;
    auto kern = decode_splitk_kernel<GQA, KM, VM, KBITS, VBITS, GKC, GVC, TL>;
    if (smem > 227 * 1024) return KVQ_ERR_UNSUPPORTED;  // too many sequences for one launch
    // The shared-memory opt-in and the occupancy query cost host time on every
    // call; redo them only when this variant's size changes (per device).
    struct Cached {
        size_t smem;
        int per_sm;
    };
    static Cached cache[kMaxDevices];
    static std::mutex lock;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
    int per_sm = 0;
    {
        std::lock_guard<std::mutex> guard(lock);
        if (cache[dev].per_sm > 0 && cache[dev].smem >= smem && cache[dev].smem - smem < 4096) {
            per_sm = cache[dev].per_sm;
        } else {
            const size_t opt_in = std::max(smem, cache[dev].smem);
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(opt_in)) != cudaSuccess)
                return KVQ_ERR_CUDA;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem) != cudaSuccess ||
                per_sm <= 0)
                per_sm = 1;
            cache[dev] = Cached{opt_in, per_sm};
        }
    }
    const int grid = std::max(1, std::min(max_items, per_sm * sm_count()));
    if (cudaMemsetAsync(p.counter, 0, sizeof(int), stream) != cudaSuccess) return KVQ_ERR_CUDA;
    kern<<<grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

// Variant families, each instantiated in its own translation unit.
kvq_status dispatch_plain(const kvq_cache_desc &d, const DecodeParams &p, int gqa, int max_items,
                          cudaStream_t stream);   // kvq_decode_plain.cu: token-wise groups, bf16 caches
kvq_status dispatch_window(const kvq_cache_desc &d, const DecodeParams &p, int gqa, int max_items,
                           cudaStream_t stream);  // kvq_decode_window.cu: recent window, values per token
kvq_status dispatch_innerq(const kvq_cache_desc &d, const DecodeParams &p, int gqa, int max_items,
                           cudaStream_t stream);  // kvq_decode_innerq.cu: recent window, values per channel
kvq_status dispatch_sink(const kvq_cache_desc &d, const DecodeParams &p, int gqa, int max_items,
                         cudaStream_t stream);    // kvq_decode_sink.cu: attention-sink window

}  // namespace dec
}  // namespace kvq
