// kvq_remat.cu -- XQuant-style rematerialization of K and V from a cache of
// quantized layer inputs X ("XQuant: Breaking the Memory Wall for LLM
// Inference with KV Cache Rematerialization", Abstract: cache the layer input
// X in low bit width and recompute K and V from it, trading memory traffic for
// matrix-multiply work), and RoPE tables.
//
// One persistent GEMM on the 5th-generation tensor cores (sm_100a):
//     [K V][m][n] = sum_k x^[m][k] * W[n][k],   x^ = bf16_rn(fp32(q*s + z)),
// RoPE (rotate-half pairs i, i+64) on the K columns, bf16 stores.
//
// Tiles are 128 tokens x 256 output channels (two heads of K or V); one CTA
// per SM walks the tiles. Warp roles:
//   warp 0      W producer: per 64-wide K step, a TMA box of W (256 x 64
//               bf16, 128-byte swizzle) into shared memory. No multicast.
//   warp 2      codes producer: the X codes box (128 tokens x 32 bytes) and
//               the tokens' fp16 scale/zero (512 bytes).
//   warp 1      allocates 512 TMEM columns (one 256-column fp32 accumulator
//               and a ring of A stages); one lane issues tcgen05.mma
//               (kind::f16, A from tensor memory, B from shared memory);
//               tcgen05.commit frees W and A stages and signals the finished
//               accumulator.
//   warps 3-10  dequantize the codes, one token row per thread, in two groups
//               of four warps taking alternate K steps, and store the bf16 A
//               operand into tensor memory with tcgen05.st.
//   warps 11-14 epilogue: tcgen05.ld one accumulator row per thread, RoPE in
//               fp32 on K, round to bf16 into a swizzled shared staging tile,
//               release the accumulator; one thread stores the tile to
//               [B][H][T][128] with TMA while the next tile's main loop runs.
// The fused variant (remat_kernel<true>, kvq_remat_attention) builds each
// tile from one head's K rows and V rows and replaces the stores by decode
// attention of the head's GQA query rows over the tile's 128 tokens, writing
// one (o, m, l) partial per tile; remat_merge_kernel combines the tiles.
// Every mbarrier wait is bounded; on expiry the kernel sets KVQ_DEV_TIMEOUT,
// waits (bounded) for its copies and MMAs in flight, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

constexpr int kBM = 128;                    // tokens per tile (MMA M)
constexpr int kBN = 256;                    // output channels per tile (MMA N)
constexpr int kBK = 64;                     // hidden channels per stage (one 128-byte row)
constexpr int kUmmaK = 16;                  // K of one tcgen05.mma kind::f16
// Pipelines, each recycled by its own consumer:
//   W ring      shared memory, TMA -> MMA, freed by tcgen05.commit
//   codes ring  shared memory, TMA -> dequantizers, freed once they hold the codes
//   A ring      tensor memory, dequantizers (tcgen05.st) -> MMA, freed by tcgen05.commit
// Keeping the A operand in tensor memory takes its writes and the tensor
// core's reads of it off shared-memory bandwidth, which otherwise bounds the
// loop (the W and codes traffic alone use most of it).
constexpr int kWStages = 4;
constexpr int kAStages = 4;
constexpr int kCStages = 6;
constexpr int kBBytes = kBN * kBK * 2;      // 32 KiB of W per stage
constexpr int kCodeBytes = kBM * kBK / 2;   // 4 KiB of INT4 codes
constexpr int kSzBytes = kBM * 4;           // half2 per token
constexpr int kCStageBytes = kCodeBytes + kSzBytes;
constexpr int kOffCRing = kWStages * kBBytes;
constexpr int kOffStage = kOffCRing + kCStages * kCStageBytes;
// Output staging: 2 heads x 2 boxes of 128 rows x 64 bf16 (128-byte swizzle).
constexpr int kBoxBytes = kBM * 64 * 2;
constexpr int kStageOutBytes = 4 * kBoxBytes;
constexpr int kRingBytes = kOffStage + kStageOutBytes;
// Tensor memory: one fp32 accumulator of 256 columns, then the A stages of
// 64 bf16 per row = 32 columns each.
constexpr int kTmemCols = 512;
constexpr int kAccCols = 256;
constexpr int kACols = kBK / 2;
static_assert(kAccCols + kAStages * kACols <= kTmemCols, "tensor memory");
// warps: 0 W producer, 1 MMA issuer (+ TMEM owner), 2 codes producer,
// 3-10 dequantizers (two groups of four taking alternate K steps), 11-14 epilogue
constexpr int kDeqWarp0 = 3;
constexpr int kDeqGroups = 2;
constexpr int kEpiWarp0 = kDeqWarp0 + 4 * kDeqGroups;
constexpr int kThreads = (kEpiWarp0 + 4) * 32;
constexpr int kNumBars = 2 * kWStages + 2 * kAStages + 2 * kCStages + 3;
constexpr int kBarBytes = 512;
constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kRingBytes) + kBarBytes;

static_assert(kBBytes % 1024 == 0 && kOffStage % 1024 == 0, "swizzled tiles need 1024-byte alignment");
static_assert(kOffCRing % 256 == 0 && kCStageBytes % 256 == 0, "TMA destination alignment (32-byte swizzle)");
static_assert(kNumBars * 8 + 8 <= kBarBytes, "barrier area");
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
static_assert(kCStages % kDeqGroups == 0, "a codes slot always goes to the same group");

struct RematParams {
    const __half2 *x_sz;   // [S][XH][Tc] (one group of 128 channels per row)
    // fused attention (remat_kernel<true>): the tile of head h holds its K
    // (accumulator columns 0..127) and V (128..255); per tile a partial
    // (o, m, l) of the GQA query heads over its 128 tokens.
    const void *q;         // [B][Hq][128] of q_dtype
    int q_dtype, gqa;      // gqa = Hq / H (1, 2 or 4)
    float qscale;          // softmax scale * log2(e)
    float *o_part;         // [B][Hq][n_blk][128]
    float2 *ml;            // [B][Hq][n_blk]
    const float *rope_cos; // [T][64]
    const float *rope_sin;
    uint16_t *k_out;       // bf16 [B][H][T][128]
    uint16_t *v_out;
    int XH;                // X viewed as XH heads of 128 channels (hidden / 128)
    int H;                 // KV heads
    int Tc;                // X cache capacity (row stride of a head)
    int T;                 // positions to rematerialize
    int m_tiles;           // batch * T / 128
    int n_tiles;           // 2H * 128 / 256 = H
    int64_t timeout_ns;
    int32_t *status;
};

// ---- tcgen05 / TMA primitives (inline PTX, sm_100a) -----------------------

// Shared-memory matrix descriptor of a K-major tile in the 128-byte swizzle
// (8-row, 1024-byte atoms stacked along M/N): start address, leading-dimension
// offset 1 (unused for swizzled K-major), stride 1024 bytes, version 1,
// layout type 2 = SWIZZLE_128B.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(1u) << 16;
    d |= static_cast<uint64_t>(1024u >> 4) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;
    return d;
}

// Instruction descriptor: D f32, A and B bf16, both K-major, N = 256, M = 128.
constexpr uint32_t kInstrDesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                (static_cast<uint32_t>(kBN >> 3) << 17) |
                                (static_cast<uint32_t>(kBM >> 4) << 24);

__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// One tcgen05.mma kind::f16 (M 128, N 256, K 16, fp32 accumulate into
// d_tmem) with the A operand read from tensor memory (lane = row, 32-bit column
// c = bf16 elements 2c and 2c+1 along K) and B from a shared-memory descriptor.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(kInstrDesc), "r"(accumulate)
        : "memory");
}

// Store 32 consecutive 32-bit columns of this thread's TMEM lane and wait for
// the store to complete.
__device__ __forceinline__ void tmem_st32_wait(uint32_t taddr, const uint32_t v[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
        "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
        "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far has
// completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_addr(bar))
        : "memory");
}

// Two runs of 32 consecutive fp32 columns of this thread's TMEM lane. The
// loads and their wait sit in one asm statement, so no use of the results can
// be scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld32x2(uint32_t taddr_a, uint32_t taddr_b, float a[32],
                                            float b[32]) {
    uint32_t ra[32], rb[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(ra[0]), "=r"(ra[1]), "=r"(ra[2]), "=r"(ra[3]), "=r"(ra[4]), "=r"(ra[5]), "=r"(ra[6]), "=r"(ra[7]), "=r"(ra[8]), "=r"(ra[9]), "=r"(ra[10]), "=r"(ra[11]), "=r"(ra[12]), "=r"(ra[13]), "=r"(ra[14]), "=r"(ra[15]), "=r"(ra[16]), "=r"(ra[17]), "=r"(ra[18]), "=r"(ra[19]), "=r"(ra[20]), "=r"(ra[21]), "=r"(ra[22]), "=r"(ra[23]), "=r"(ra[24]), "=r"(ra[25]), "=r"(ra[26]), "=r"(ra[27]), "=r"(ra[28]), "=r"(ra[29]), "=r"(ra[30]), "=r"(ra[31]),
          "=r"(rb[0]), "=r"(rb[1]), "=r"(rb[2]), "=r"(rb[3]), "=r"(rb[4]), "=r"(rb[5]), "=r"(rb[6]), "=r"(rb[7]), "=r"(rb[8]), "=r"(rb[9]), "=r"(rb[10]), "=r"(rb[11]), "=r"(rb[12]), "=r"(rb[13]), "=r"(rb[14]), "=r"(rb[15]), "=r"(rb[16]), "=r"(rb[17]), "=r"(rb[18]), "=r"(rb[19]), "=r"(rb[20]), "=r"(rb[21]), "=r"(rb[22]), "=r"(rb[23]), "=r"(rb[24]), "=r"(rb[25]), "=r"(rb[26]), "=r"(rb[27]), "=r"(rb[28]), "=r"(rb[29]), "=r"(rb[30]), "=r"(rb[31])
        : "r"(taddr_a), "r"(taddr_b)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        a[i] = __uint_as_float(ra[i]);
        b[i] = __uint_as_float(rb[i]);
    }
}

// 2-D tiled TMA load global -> shared, completing on `bar`. No multicast.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

// 2-D tiled TMA store shared -> global (bulk group of the issuing thread).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, int x, int y, const void *src) {
    asm volatile(
        "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(x), "r"(y), "r"(smem_addr(src))
        : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until the issued bulk stores have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until the issued bulk stores have completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// x rounded to the nearest bf16 (ties to even), as a float.
__device__ __forceinline__ float bf16_round(float x) {
    return __bfloat162float(__float2bfloat16_rn(x));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Byte permute through the intrinsic, so constant operands stay immediates.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) { return __byte_perm(a, b, sel); }

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    unsigned long long r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(r)
        : "l"(*reinterpret_cast<unsigned long long *>(&a)),
          "l"(*reinterpret_cast<unsigned long long *>(&b)),
          "l"(*reinterpret_cast<unsigned long long *>(&c)));
    return *reinterpret_cast<float2 *>(&r);
}

// Rounding error of the fp32 sum a + b (Knuth's TwoSum): zero iff the sum is exact.
__device__ __forceinline__ float two_sum_err(float a, float b) {
    const float s = __fadd_rn(a, b);
    const float bp = __fsub_rn(s, a);
    const float ap = __fsub_rn(s, bp);
    return __fadd_rn(__fsub_rn(a, ap), __fsub_rn(b, bp));
}

// One row's 32 code bytes and its scale/zero word from shared memory. The
// codes box lands with the 32-byte swizzle: 16-byte chunk c of row r sits at
// chunk c ^ ((r >> 2) & 1), so the eight rows of a shared-memory phase (32
// bytes apart) hit eight distinct bank groups.
__device__ __forceinline__ void lds_codes(const uint8_t *codes, int r, const uint8_t *sz, uint4 &c0, uint4 &c1,
                                          uint32_t &szw) {
    const int f = (r >> 2) & 1;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(c0.x), "=r"(c0.y), "=r"(c0.z), "=r"(c0.w)
                 : "r"(smem_addr(codes + 16 * f))
                 : "memory");
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(c1.x), "=r"(c1.y), "=r"(c1.z), "=r"(c1.w)
                 : "r"(smem_addr(codes + 16 * (f ^ 1)))
                 : "memory");
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(szw) : "r"(smem_addr(sz)) : "memory");
}

// Dequantize one token row's 64 INT4 codes (32 bytes, element 2i in the low
// nibble of byte i) into 64 bf16 x^ = bf16_rn(fp32(q*s + z)), packed two per
// word in K order: out[c] = {x^[2c] (low half), x^[2c+1]}, the row's 32
// tensor-memory columns of the A operand.
//
// Fast form: a byte permute puts nibble q in the top mantissa bits of 1.0,
// f = 1 + q/128 exactly, and fma(f, 128 s, z - 128 s) equals q*s + z before
// its single rounding whenever z - 128 s is exact in fp32 (checked per row);
// otherwise the codes go through 2^23 + q - 2^23 and fma(q, s, z).
__device__ __forceinline__ void dequant_row(uint4 c0, uint4 c1, float sc, float zp, uint32_t out[32]) {
    const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    const float s128 = __fmul_rn(sc, 128.0f);
    const float cz = __fsub_rn(zp, s128);
    if (two_sum_err(zp, -s128) == 0.0f) {
        const float2 mul = make_float2(s128, s128), add = make_float2(cz, cz);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint32_t w = words[c];
            const uint32_t lo = (w & 0x0F0F0F0Fu) | 0x80808080u;
            const uint32_t hi = ((w >> 4) & 0x0F0F0F0Fu) | 0x80808080u;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                // bytes {0, 0, 0x80|q, 0x3F}: the float 1 + q/128
                const uint32_t sel = 0x7044u | (static_cast<uint32_t>(i) << 8);
                const float2 f = make_float2(__uint_as_float(prmt(lo, 0x3F000000u, sel)),
                                             __uint_as_float(prmt(hi, 0x3F000000u, sel)));
                const float2 x = ffma2(f, mul, add);
                out[4 * c + i] = pack_bf16x2(x.x, x.y);
            }
        }
    } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint32_t w = words[c];
            const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                // bytes {q, 0, 0, 0x4B}: the float 2^23 + q
                const uint32_t sel = 0x7440u | static_cast<uint32_t>(i);
                const float qe = __fsub_rn(__uint_as_float(prmt(lo, 0x4B000000u, sel)), 8388608.0f);
                const float qo = __fsub_rn(__uint_as_float(prmt(hi, 0x4B000000u, sel)), 8388608.0f);
                out[4 * c + i] = pack_bf16x2(__fmaf_rn(qe, sc, zp), __fmaf_rn(qo, sc, zp));
            }
        }
    }
}

// Tile id -> (batch row block, N tile). N varies fastest so that the CTAs
// running at the same time share X rows in L2.
struct TileCoord {
    int b, t0, n;
};
__device__ __forceinline__ TileCoord tile_coord(const RematParams &p, int tile) {
    TileCoord c;
    const int m = tile / p.n_tiles;
    c.n = tile - m * p.n_tiles;
    const int per_b = p.T / kBM;
    c.b = m / per_b;
    c.t0 = (m - c.b * per_b) * kBM;
    return c;
}

// FUSED: decode attention over the rematerialized tile instead of storing
// it (K and V never reach HBM): W's B tile is head h's 128 K rows then its 128
// V rows (two TMA boxes of tm_w, 64 x 128), and the epilogue scores the tile's
// 128 tokens against the GQA query rows.
template <bool FUSED>
__global__ void __launch_bounds__(kThreads, 1)
    remat_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                 const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 const RematParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *w_ring = smem;
    uint8_t *c_ring = smem + kOffCRing;
    uint8_t *out_stage = smem + kOffStage;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kRingBytes);
    uint64_t *w_full = bars;                       // [kWStages] W landed (tx)
    uint64_t *w_empty = w_full + kWStages;         // [kWStages] MMAs done with W
    uint64_t *a_full = w_empty + kWStages;         // [kAStages] x^ stored (128 threads)
    uint64_t *a_empty = a_full + kAStages;         // [kAStages] MMAs done with x^
    uint64_t *c_full = a_empty + kAStages;         // [kCStages] codes landed (tx)
    uint64_t *c_empty = c_full + kCStages;         // [kCStages] codes taken (128 threads)
    uint64_t *acc_full = c_empty + kCStages;       // accumulator ready
    uint64_t *acc_empty = acc_full + 1;            // accumulator drained (128 threads)
    uint64_t *mma_done = acc_empty + 1;            // every MMA of this CTA finished
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kWStages; ++s) {
            mbar_init(&w_full[s], 1);
            mbar_init(&w_empty[s], 1);
        }
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(&a_full[s], 128);
            mbar_init(&a_empty[s], 1);
        }
        for (int s = 0; s < kCStages; ++s) {
            mbar_init(&c_full[s], 1);
            mbar_init(&c_empty[s], 128);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 128);
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int n_k = 2 * p.XH;  // K steps of 64 hidden channels
    const int n_total = p.m_tiles * p.n_tiles;

    // Wait (bounded) until the copies of a producer's last `depth` ring slots
    // have landed, so none arrives after the CTA has gone.
    auto drain = [&](uint64_t *full, int depth, int issued) {
        for (int j = max(0, issued - depth); j < issued; ++j) {
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(&full[j % depth], (j / depth) & 1)) {
                if (static_cast<int64_t>(global_timer_ns() - t0) > p.timeout_ns) {
                    status_or(p.status, KVQ_DEV_TIMEOUT);
                    break;
                }
            }
        }
    };

    if (warp == 0) {
        // ------------------------------ W producer --------------------------------
        if (lane == 0) {
            int it = 0;
            bool stop = false;
            for (int tile = blockIdx.x; tile < n_total && !stop; tile += gridDim.x) {
                const TileCoord c = tile_coord(p, tile);
                for (int kb = 0; kb < n_k; ++kb, ++it) {
                    const int s = it % kWStages, r = it / kWStages;
                    if (r > 0 && !mbar_wait_bounded(&w_empty[s], (r - 1) & 1, p.timeout_ns, p.status,
                                                    abort_flag)) {
                        stop = true;
                        break;
                    }
                    mbar_arrive_expect_tx(&w_full[s], kBBytes);
                    if constexpr (FUSED) {  // head c.n: its K rows, then its V rows
                        tma_load_2d(w_ring + s * kBBytes, &tm_w, kb * kBK, c.n * kHeadDim, &w_full[s]);
                        tma_load_2d(w_ring + s * kBBytes + kBBytes / 2, &tm_w, kb * kBK,
                                    (p.H + c.n) * kHeadDim, &w_full[s]);
                    } else {
                        tma_load_2d(w_ring + s * kBBytes, &tm_w, kb * kBK, c.n * kBN, &w_full[s]);
                    }
                }
            }
            drain(w_full, kWStages, it);
        }
    } else if (warp == 2) {
        // ---------------------------- codes producer ------------------------------
        if (lane == 0) {
            int it = 0;
            bool stop = false;
            for (int tile = blockIdx.x; tile < n_total && !stop; tile += gridDim.x) {
                const TileCoord c = tile_coord(p, tile);
                for (int kb = 0; kb < n_k; ++kb, ++it) {
                    const int s = it % kCStages, r = it / kCStages;
                    if (r > 0 && !mbar_wait_bounded(&c_empty[s], (r - 1) & 1, p.timeout_ns, p.status,
                                                    abort_flag)) {
                        stop = true;
                        break;
                    }
                    uint8_t *st = c_ring + s * kCStageBytes;
                    const int row = (c.b * p.XH + (kb >> 1)) * p.Tc + c.t0;
                    mbar_arrive_expect_tx(&c_full[s], kCStageBytes);
                    tma_load_2d(st, &tm_x, (kb & 1) * (kBK / 2), row, &c_full[s]);
                    bulk_g2s(st + kCodeBytes, p.x_sz + row, kSzBytes, &c_full[s]);
                }
            }
            drain(c_full, kCStages, it);
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer --------------------------------
        if (lane == 0) {
            int it = 0, lt = 0;
            bool stop = false;
            for (int tile = blockIdx.x; tile < n_total && !stop; tile += gridDim.x, ++lt) {
                // one accumulator: the previous tile's epilogue must have drained it
                if (lt > 0 && !mbar_wait_bounded(acc_empty, (lt - 1) & 1, p.timeout_ns, p.status,
                                                 abort_flag))
                    break;
                tc_fence_after();
                for (int kb = 0; kb < n_k; ++kb, ++it) {
                    const int sw = it % kWStages, rw = it / kWStages;
                    const int sa = it % kAStages, ra = it / kAStages;
                    if (!mbar_wait_bounded(&w_full[sw], rw & 1, p.timeout_ns, p.status, abort_flag) ||
                        !mbar_wait_bounded(&a_full[sa], ra & 1, p.timeout_ns, p.status, abort_flag)) {
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_tmem = tmem_base + kAccCols + sa * kACols;
                    const uint64_t b_desc = sw128_desc(smem_addr(w_ring + sw * kBBytes));
#pragma unroll
                    for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
                        // K step of 16: 8 tensor-memory columns of A; +32 bytes
                        // inside the W swizzle atom = +2 in descriptor units.
                        umma_bf16_ts(tmem_base, a_tmem + kk * (kUmmaK / 2), b_desc + 2 * kk,
                                     (kb | kk) != 0);
                    }
                    umma_commit(&w_empty[sw]);
                    umma_commit(&a_empty[sa]);
                }
                if (!stop) umma_commit(acc_full);
            }
            // Every MMA issued must finish before TMEM is freed.
            umma_commit(mma_done);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(mma_done, 0)) {
                if (static_cast<int64_t>(global_timer_ns() - t0) > p.timeout_ns) {
                    status_or(p.status, KVQ_DEV_TIMEOUT);
                    break;
                }
            }
        }
    } else if (warp < kEpiWarp0) {
        // ------------------------------ dequantizers ------------------------------
        // Group g takes the K steps it with it % kDeqGroups == g; each of its
        // four warps owns the 32 rows (tensor-memory lanes) of its quarter.
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;  // token row of the tile = TMEM lane
        const int group = (warp - kDeqWarp0) >> 2;
        const uint32_t a_lane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + kAccCols;
        int it = 0;
        bool stop = false;
        for (int tile = blockIdx.x; tile < n_total && !stop; tile += gridDim.x) {
            for (int kb = 0; kb < n_k; ++kb, ++it) {
                if (it % kDeqGroups != group) continue;
                const int sc = it % kCStages, rc = it / kCStages;
                // Warp-uniform outcomes: the warp's later steps need all lanes.
                if (!__all_sync(0xffffffffu, mbar_wait_bounded(&c_full[sc], rc & 1, p.timeout_ns,
                                                               p.status, abort_flag))) {
                    stop = true;
                    break;
                }
                const uint8_t *cs = c_ring + sc * kCStageBytes;
                uint4 c0, c1;
                uint32_t szw;
                lds_codes(cs + row * 32, row, cs + kCodeBytes + row * 4, c0, c1, szw);
                const __half2 sz = *reinterpret_cast<const __half2 *>(&szw);
                uint32_t xv[32];
                dequant_row(c0, c1, __low2float(sz), __high2float(sz), xv);
                // Release the codes slot only now. A shared load returns its
                // data asynchronously and an arrive issued right after it does
                // not wait for that data; the arithmetic above consumed the
                // loaded registers, and warps issue in order, so the loads have
                // completed before this arrive can issue.
                mbar_arrive(&c_empty[sc]);
                const int sa = it % kAStages, ra = it / kAStages;
                if (ra > 0 &&
                    !__all_sync(0xffffffffu, mbar_wait_bounded(&a_empty[sa], (ra - 1) & 1,
                                                               p.timeout_ns, p.status, abort_flag))) {
                    stop = true;
                    break;
                }
                tc_fence_after();
                tmem_st32_wait(a_lane + sa * kACols, xv);
                tc_fence_before();
                mbar_arrive(&a_full[sa]);
            }
        }
    } else if constexpr (FUSED) {
        // --------------------------- attention epilogue ---------------------------
        // Thread `row` owns token c.t0 + row (its TMEM lane). K and V are
        // rounded to bf16 as the unfused path stores them; scores, softmax and
        // P V of the tile in fp32; the partial (o, m, l) per query head goes
        // to the workspace for the merge over the tiles.
        const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
        const int row = quarter * 32 + lane;
        float *q_s = reinterpret_cast<float *>(out_stage);              // [4][128] scaled queries
        float *p_s = q_s + 4 * kHeadDim;                                // [128][4] weights
        float *red = p_s + kBM * 4;                                     // [4 warps][4] max, then sums
        uint16_t *v_s = reinterpret_cast<uint16_t *>(red + 32);         // bf16 [128][kVStride]
        constexpr int kVStride = kHeadDim + 8;  // padded rows: 8 consecutive rows hit distinct banks
        const int n_blk = p.T / kBM;
        int lt = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < n_total; tile += gridDim.x, ++lt) {
            ok = ok && __all_sync(0xffffffffu, mbar_wait_bounded(acc_full, lt & 1, p.timeout_ns,
                                                                 p.status, abort_flag));
            tc_fence_after();
            if (!ok) {  // take every barrier of the tile so no epilogue warp is left waiting
                named_sync(1, 128);
                named_sync(1, 128);
                named_sync(1, 128);
                named_sync(1, 128);
                continue;
            }
            const TileCoord c = tile_coord(p, tile);
            const int t = c.t0 + row;
            const int hq0 = c.n * p.gqa;
            const int Hq = p.H * p.gqa;
            // (A) the tile's query rows, scaled, zero for heads past gqa
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int idx = i * kBM + row;  // [g][channel]
                const int g = idx / kHeadDim, ch = idx - g * kHeadDim;
                float v = 0.0f;
                if (g < p.gqa) {
                    const int64_t qi = (static_cast<int64_t>(c.b) * Hq + hq0 + g) * kHeadDim + ch;
                    if (p.q_dtype == KVQ_FP32) v = static_cast<const float *>(p.q)[qi];
                    else if (p.q_dtype == KVQ_BF16) v = bf16_bits_to_float(static_cast<const uint16_t *>(p.q)[qi]);
                    else v = __half2float(static_cast<const __half *>(p.q)[qi]);
                }
                q_s[idx] = v * p.qscale;
            }
            named_sync(1, 128);
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
            // V rows to shared memory as bf16 (first, so the accumulator is
            // released right after the last K load)
#pragma unroll 1
            for (int c32 = 0; c32 < 64; c32 += 32) {
                float a[32], bv[32];
                tmem_ld32x2(tbase + kHeadDim + c32, tbase + kHeadDim + 64 + c32, a, bv);
                uint4 *va = reinterpret_cast<uint4 *>(v_s + row * kVStride + c32);
                uint4 *vb = reinterpret_cast<uint4 *>(v_s + row * kVStride + 64 + c32);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    va[v] = make_uint4(pack_bf16x2(a[8 * v + 0], a[8 * v + 1]), pack_bf16x2(a[8 * v + 2], a[8 * v + 3]),
                                       pack_bf16x2(a[8 * v + 4], a[8 * v + 5]), pack_bf16x2(a[8 * v + 6], a[8 * v + 7]));
                    vb[v] = make_uint4(pack_bf16x2(bv[8 * v + 0], bv[8 * v + 1]), pack_bf16x2(bv[8 * v + 2], bv[8 * v + 3]),
                                       pack_bf16x2(bv[8 * v + 4], bv[8 * v + 5]), pack_bf16x2(bv[8 * v + 6], bv[8 * v + 7]));
                }
            }
            // (B) scores of this token: RoPE on K (pairs i, i + 64), bf16, dot with q
            float sc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 1
            for (int c32 = 0; c32 < 64; c32 += 32) {
                float a[32], bv[32];
                tmem_ld32x2(tbase + c32, tbase + 64 + c32, a, bv);
                if (c32 == 32) {  // the last tensor-memory read: the next tile's MMAs may start
                    tc_fence_before();
                    mbar_arrive(acc_empty);
                }
                const float4 *cs = reinterpret_cast<const float4 *>(p.rope_cos + static_cast<int64_t>(t) * 64 + c32);
                const float4 *sn = reinterpret_cast<const float4 *>(p.rope_sin + static_cast<int64_t>(t) * 64 + c32);
#pragma unroll
                for (int i4 = 0; i4 < 8; ++i4) {
                    const float4 cv = __ldg(cs + i4), sv = __ldg(sn + i4);
                    const float cc[4] = {cv.x, cv.y, cv.z, cv.w};
                    const float ss[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i = i4 * 4 + e;
                        const float x0 = a[i], x1 = bv[i];
                        a[i] = bf16_round(__fmaf_rn(x0, cc[e], -__fmul_rn(x1, ss[e])));
                        bv[i] = bf16_round(__fmaf_rn(x1, cc[e], __fmul_rn(x0, ss[e])));
                    }
                }
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const float *qg = q_s + g * kHeadDim + c32;
                    float acc = sc[g];
#pragma unroll
                    for (int i = 0; i < 32; ++i) acc = fmaf(qg[i], a[i], fmaf(qg[64 + i], bv[i], acc));
                    sc[g] = acc;
                }
            }
            // (C) the tile's maximum and weights per head
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                float m = sc[g];
#pragma unroll
                for (int k = 16; k > 0; k >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, k));
                if (lane == 0) red[quarter * 4 + g] = m;
            }
            named_sync(1, 128);
            float M[4], pw[4];
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                M[g] = fmaxf(fmaxf(red[g], red[4 + g]), fmaxf(red[8 + g], red[12 + g]));
                pw[g] = fast_exp2(sc[g] - M[g]);
            }
            *reinterpret_cast<float4 *>(p_s + row * 4) = make_float4(pw[0], pw[1], pw[2], pw[3]);
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                float l = pw[g];
#pragma unroll
                for (int k = 16; k > 0; k >>= 1) l += __shfl_xor_sync(0xffffffffu, l, k);
                if (lane == 0) red[16 + quarter * 4 + g] = l;
            }
            named_sync(1, 128);
            // (D) thread `row` takes channel `row`: o[g] = sum_t p[t][g] v[t][row]
            float o[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 8
            for (int tt = 0; tt < kBM; ++tt) {
                const float4 pv = *reinterpret_cast<const float4 *>(p_s + tt * 4);
                const float v = bf16_bits_to_float(v_s[tt * kVStride + row]);
                o[0] = fmaf(pv.x, v, o[0]);
                o[1] = fmaf(pv.y, v, o[1]);
                o[2] = fmaf(pv.z, v, o[2]);
                o[3] = fmaf(pv.w, v, o[3]);
            }
            const int blk = c.t0 / kBM;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                if (g >= p.gqa) break;
                const int64_t pi = (static_cast<int64_t>(c.b) * Hq + hq0 + g) * n_blk + blk;
                p.o_part[pi * kHeadDim + row] = o[g];
                if (row == 0) {
                    const float L = (red[16 + g] + red[20 + g]) + (red[24 + g] + red[28 + g]);
                    p.ml[pi] = make_float2(M[g], L);
                }
            }
            named_sync(1, 128);  // q_s, p_s, v_s are free for the next tile
        }
    } else {
        // ------------------------------ epilogue ----------------------------------
        // Drain the accumulator into a swizzled bf16 staging tile (RoPE on K
        // applied on the way), release the accumulator, then one thread
        // stores the tile with four TMA copies while the next tile's main loop
        // runs.
        const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
        const int row = quarter * 32 + lane;
        const bool leader = (warp == kEpiWarp0 && lane == 0);
        const uint32_t swz = row & 7;
        int lt = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < n_total; tile += gridDim.x, ++lt) {
            // Warp-uniform outcome (tcgen05.ld needs the whole warp). After a
            // failed wait the warp skips the work but still takes both named
            // barriers of every tile, so no epilogue warp is left waiting.
            ok = ok && __all_sync(0xffffffffu, mbar_wait_bounded(acc_full, lt & 1, p.timeout_ns,
                                                                 p.status, abort_flag));
            tc_fence_after();
            // The staging tile is free once the previous tile's stores read it.
            if (leader) bulk_wait_read();
            named_sync(1, 128);
            if (!ok) {
                named_sync(1, 128);
                continue;
            }
            const TileCoord c = tile_coord(p, tile);
            const int t = c.t0 + row;
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                const bool is_k = c.n * 2 + half < p.H;  // K heads 0..H-1, then V heads
                const uint32_t col = tbase + half * kHeadDim;
                uint8_t *box0 = out_stage + (half * 2) * kBoxBytes + row * 128;
                uint8_t *box1 = box0 + kBoxBytes;
#pragma unroll 1
                for (int c32 = 0; c32 < 64; c32 += 32) {
                    float a[32], bv[32];
                    tmem_ld32x2(col + c32, col + 64 + c32, a, bv);
                    if (is_k) {
                        const float4 *cs = reinterpret_cast<const float4 *>(p.rope_cos + static_cast<int64_t>(t) * 64 + c32);
                        const float4 *sn = reinterpret_cast<const float4 *>(p.rope_sin + static_cast<int64_t>(t) * 64 + c32);
#pragma unroll
                        for (int i4 = 0; i4 < 8; ++i4) {
                            const float4 cv = __ldg(cs + i4), sv = __ldg(sn + i4);
                            const float cc[4] = {cv.x, cv.y, cv.z, cv.w};
                            const float ss[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int i = i4 * 4 + e;
                                const float x0 = a[i], x1 = bv[i];
                                a[i] = __fmaf_rn(x0, cc[e], -__fmul_rn(x1, ss[e]));
                                bv[i] = __fmaf_rn(x1, cc[e], __fmul_rn(x0, ss[e]));
                            }
                        }
                    }
                    // channels c32 .. c32+31 -> box 0, 64+c32 .. -> box 1; 16-byte
                    // chunk j of a row sits at chunk j ^ (row & 7)
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const uint32_t j = static_cast<uint32_t>(c32 / 8 + v);
                        *reinterpret_cast<uint4 *>(box0 + ((j ^ swz) << 4)) =
                            make_uint4(pack_bf16x2(a[8 * v + 0], a[8 * v + 1]), pack_bf16x2(a[8 * v + 2], a[8 * v + 3]),
                                       pack_bf16x2(a[8 * v + 4], a[8 * v + 5]), pack_bf16x2(a[8 * v + 6], a[8 * v + 7]));
                        *reinterpret_cast<uint4 *>(box1 + ((j ^ swz) << 4)) =
                            make_uint4(pack_bf16x2(bv[8 * v + 0], bv[8 * v + 1]), pack_bf16x2(bv[8 * v + 2], bv[8 * v + 3]),
                                       pack_bf16x2(bv[8 * v + 4], bv[8 * v + 5]), pack_bf16x2(bv[8 * v + 6], bv[8 * v + 7]));
                    }
                }
            }
            // Accumulator read out: the next tile's MMAs may start.
            tc_fence_before();
            mbar_arrive(acc_empty);
            fence_proxy_async_smem();
            named_sync(1, 128);
            if (leader && ok) {
                for (int half = 0; half < 2; ++half) {
                    const int slot = c.n * 2 + half;
                    const bool is_k = slot < p.H;
                    const int h = is_k ? slot : slot - p.H;
                    const int y = (c.b * p.H + h) * p.T + c.t0;
                    const CUtensorMap *map = is_k ? &tm_k : &tm_v;
                    tma_store_2d(map, 0, y, out_stage + (half * 2) * kBoxBytes);
                    tma_store_2d(map, 64, y, out_stage + (half * 2 + 1) * kBoxBytes);
                }
                bulk_commit();
            }
        }
        if (leader) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// One CTA of 512 threads per (query head, sequence): the fused kernel's
// per-tile partials combined into the output, one partial per warp at a time.
__global__ void __launch_bounds__(512) remat_merge_kernel(const float *o_part, const float2 *ml, int n_blk,
                                                          float *out) {
    __shared__ CombineSmemW<16> sm;
    const int64_t row = static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x;
    float M, l;
    float4 o;
    combine_partials_w<16>(o_part, ml, row * n_blk * kHeadDim, kHeadDim, row * n_blk, 1, n_blk, sm, M, o, l);
    if (threadIdx.x < 32)
        reinterpret_cast<float4 *>(out + row * kHeadDim)[threadIdx.x] =
            (l > 0.0f) ? make_float4(o.x / l, o.y / l, o.z / l, o.w / l) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
}

// cos/sin(p * theta^(-2i/D)) in float64, rounded once to fp32.
__global__ void rope_tables_kernel(float *c, float *s, int n_pos, int half, double theta) {
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<int64_t>(n_pos) * half) return;
    const int p = static_cast<int>(idx / half);
    const int i = static_cast<int>(idx - static_cast<int64_t>(p) * half);
    const double inv_freq = pow(theta, -static_cast<double>(i) / static_cast<double>(half));
    const double a = static_cast<double>(p) * inv_freq;
    double sv, cv;
    sincos(a, &sv, &cv);
    c[idx] = static_cast<float>(cv);
    s[idx] = static_cast<float>(sv);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

bool make_map_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner,
                 uint64_t rows, uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows,
                 CUtensorMapSwizzle swz) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

namespace {

// One persistent CTA per SM (at most one per tile).
template <bool FUSED>
kvq_status launch_remat_grid(const CUtensorMap &tm_w, const CUtensorMap &tm_x, const CUtensorMap &tm_k,
                             const CUtensorMap &tm_v, const RematParams &p, cudaStream_t stream) {
    if (cudaFuncSetAttribute(remat_kernel<FUSED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes)) != cudaSuccess)
        return KVQ_ERR_CUDA;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return KVQ_ERR_CUDA;
    const int64_t tiles = static_cast<int64_t>(p.m_tiles) * p.n_tiles;
    if (tiles >= (1LL << 31)) return KVQ_ERR_UNSUPPORTED;
    const int grid = static_cast<int>(std::min<int64_t>(tiles, sms));
    remat_kernel<FUSED><<<grid, kThreads, kSmemBytes, stream>>>(tm_w, tm_x, tm_k, tm_v, p);
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // namespace

kvq_status launch_rope_tables(float *c, float *s, int n_pos, int head_dim, double theta,
                              cudaStream_t stream) {
    const int half = head_dim / 2;
    const int64_t n = static_cast<int64_t>(n_pos) * half;
    rope_tables_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(c, s, n_pos, half,
                                                                                 theta);
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

kvq_status launch_remat(const kvq_cache_desc &x, const void *w_kv, int n_kv_heads,
                        const float *rope_cos, const float *rope_sin, int batch, int ctx_len,
                        void *k_out, void *v_out, cudaStream_t stream) {
    const int XH = x.num_kv_heads;
    const int64_t hidden = static_cast<int64_t>(XH) * kHeadDim;
    const int64_t n_rows = 2LL * n_kv_heads * kHeadDim;
    const int64_t code_rows = static_cast<int64_t>(x.num_seqs) * XH * x.capacity_tokens;
    if (code_rows >= (1LL << 31) || n_rows >= (1LL << 31)) return KVQ_ERR_UNSUPPORTED;
    CUtensorMap tm_w, tm_x;
    if (!make_map_2d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w_kv, hidden, n_rows, hidden * 2,
                     kBK, kBN, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_UINT8, x.k_codes, kHeadDim / 2, code_rows,
                     kHeadDim / 2, kBK / 2, kBM, CU_TENSOR_MAP_SWIZZLE_32B))
        return KVQ_ERR_CUDA;
    // Outputs [B][H][T][128] bf16 as rows of 128 channels, stored in boxes of
    // 128 positions x 64 channels.
    const int64_t out_rows = static_cast<int64_t>(batch) * n_kv_heads * ctx_len;
    if (out_rows >= (1LL << 31)) return KVQ_ERR_UNSUPPORTED;
    CUtensorMap tm_k, tm_v;
    if (!make_map_2d(&tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k_out, kHeadDim, out_rows, kHeadDim * 2,
                     64, kBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, v_out, kHeadDim, out_rows, kHeadDim * 2,
                     64, kBM, CU_TENSOR_MAP_SWIZZLE_128B))
        return KVQ_ERR_CUDA;
    RematParams p{};
    p.x_sz = static_cast<const __half2 *>(x.k_sz);
    p.rope_cos = rope_cos;
    p.rope_sin = rope_sin;
    p.k_out = static_cast<uint16_t *>(k_out);
    p.v_out = static_cast<uint16_t *>(v_out);
    p.XH = XH;
    p.H = n_kv_heads;
    p.Tc = x.capacity_tokens;
    p.T = ctx_len;
    p.m_tiles = batch * (ctx_len / kBM);
    p.n_tiles = n_kv_heads;
    p.timeout_ns = debug_hooks().wait_timeout_ns;
    p.status = x.status;
    return launch_remat_grid<false>(tm_w, tm_x, tm_k, tm_v, p, stream);
}

size_t remat_attention_workspace(int batch, int num_q_heads, int ctx_len) {
    const size_t rows = static_cast<size_t>(batch) * num_q_heads * (ctx_len / kBM);
    return rows * (kHeadDim * sizeof(float) + sizeof(float2));
}

kvq_status launch_remat_attention(const kvq_cache_desc &x, const void *w_kv, int n_kv_heads,
                                  const float *rope_cos, const float *rope_sin, int batch, int ctx_len,
                                  const void *q, kvq_dtype q_dtype, int num_q_heads, float softmax_scale,
                                  float *out, void *workspace, cudaStream_t stream) {
    const int XH = x.num_kv_heads;
    const int64_t hidden = static_cast<int64_t>(XH) * kHeadDim;
    const int64_t n_rows = 2LL * n_kv_heads * kHeadDim;
    const int64_t code_rows = static_cast<int64_t>(x.num_seqs) * XH * x.capacity_tokens;
    if (code_rows >= (1LL << 31) || n_rows >= (1LL << 31)) return KVQ_ERR_UNSUPPORTED;
    // W in boxes of 64 hidden channels x 128 rows: a head's K rows and its V
    // rows make one 256-row B tile.
    CUtensorMap tm_w, tm_x;
    if (!make_map_2d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w_kv, hidden, n_rows, hidden * 2,
                     kBK, kHeadDim, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_UINT8, x.k_codes, kHeadDim / 2, code_rows,
                     kHeadDim / 2, kBK / 2, kBM, CU_TENSOR_MAP_SWIZZLE_32B))
        return KVQ_ERR_CUDA;
    RematParams p{};
    p.x_sz = static_cast<const __half2 *>(x.k_sz);
    p.rope_cos = rope_cos;
    p.rope_sin = rope_sin;
    p.XH = XH;
    p.H = n_kv_heads;
    p.Tc = x.capacity_tokens;
    p.T = ctx_len;
    p.m_tiles = batch * (ctx_len / kBM);
    p.n_tiles = n_kv_heads;
    p.timeout_ns = debug_hooks().wait_timeout_ns;
    p.status = x.status;
    p.q = q;
    p.q_dtype = q_dtype;
    p.gqa = num_q_heads / n_kv_heads;
    p.qscale = softmax_scale * 1.4426950408889634f;
    const int n_blk = ctx_len / kBM;
    const size_t rows = static_cast<size_t>(batch) * num_q_heads * n_blk;
    p.o_part = static_cast<float *>(workspace);
    p.ml = reinterpret_cast<float2 *>(static_cast<uint8_t *>(workspace) + rows * kHeadDim * sizeof(float));
    // the store maps are unused by the fused kernel; any valid map fills the slots
    kvq_status s = launch_remat_grid<true>(tm_w, tm_x, tm_w, tm_w, p, stream);
    if (s != KVQ_OK) return s;
    remat_merge_kernel<<<dim3(num_q_heads, batch), 512, 0, stream>>>(p.o_part, p.ml, n_blk, out);
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // namespace kvq
