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
//   warp 0      TMA producer: per 64-wide K step, the W box (256 x 64 bf16,
//               128-byte swizzle), the X codes box (128 tokens x 32 bytes) and
//               the tokens' fp16 scale/zero (512 bytes), completing on one
//               mbarrier. No multicast.
//   warp 1      allocates 512 TMEM columns (two 256-column fp32
//               accumulators); one lane issues tcgen05.mma (kind::f16, bf16
//               operands, M=128, N=256, K=16) and tcgen05.commit frees each
//               stage and signals a finished accumulator.
//   warps 2-5   dequantize the codes into the A operand (128 x 64 bf16) in the
//               same 128-byte-swizzled K-major layout TMA gives W, one token
//               row per thread, then fence the generic-proxy writes for the
//               tensor core.
//   warps 6-9   epilogue: tcgen05.ld one accumulator row per thread, RoPE in
//               fp32 on K, round to bf16, store [B][H][T][128]. Two accumulators
//               let the epilogue of one tile overlap the main loop of the next.
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
constexpr int kStages = 4;
constexpr int kBBytes = kBN * kBK * 2;      // 32 KiB
constexpr int kABytes = kBM * kBK * 2;      // 16 KiB
constexpr int kCodeBytes = kBM * kBK / 2;   // 4 KiB of INT4 codes
constexpr int kSzBytes = kBM * 4;           // half2 per token
constexpr int kOffA = kBBytes;
constexpr int kOffCodes = kOffA + kABytes;
constexpr int kOffSz = kOffCodes + kCodeBytes;
constexpr int kStageBytes = ((kOffSz + kSzBytes) + 1023) & ~1023;  // 53 KiB
constexpr int kTxBytes = kBBytes + kCodeBytes + kSzBytes;
constexpr int kTmemCols = 512;
constexpr int kAccCols = 256;
constexpr int kThreads = 320;
constexpr int kBarBytes = 256;
constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kStages) * kStageBytes + kBarBytes;

static_assert(kStageBytes % 1024 == 0, "swizzled tiles need 1024-byte alignment");
static_assert(kOffA % 1024 == 0, "A tile alignment");

struct RematParams {
    const __half2 *x_sz;   // [S][XH][Tc] (one group of 128 channels per row)
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

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(kInstrDesc), "r"(accumulate)
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

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
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

__global__ void __launch_bounds__(kThreads, 1)
    remat_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                 const RematParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *stages = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kStages * kStageBytes);
    uint64_t *full_tma = bars;                 // [kStages] TMA bytes landed
    uint64_t *full_a = bars + kStages;         // [kStages] A operand written (4 warps)
    uint64_t *empty = bars + 2 * kStages;      // [kStages] MMAs reading the stage done
    uint64_t *acc_full = bars + 3 * kStages;   // [2] accumulator ready
    uint64_t *acc_empty = acc_full + 2;        // [2] accumulator drained (4 warps)
    uint64_t *mma_done = acc_empty + 2;        // [1] every MMA of this CTA finished
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full_tma[s], 1);
            mbar_init(&full_a[s], 4);
            mbar_init(&empty[s], 1);
        }
        for (int j = 0; j < 2; ++j) {
            mbar_init(&acc_full[j], 1);
            mbar_init(&acc_empty[j], 4);
        }
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

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            int it = 0;
            bool stop = false;
            for (int tile = blockIdx.x; tile < n_total && !stop; tile += gridDim.x) {
                const TileCoord c = tile_coord(p, tile);
                for (int kb = 0; kb < n_k; ++kb, ++it) {
                    const int s = it % kStages, r = it / kStages;
                    if (r > 0 && !mbar_wait_bounded(&empty[s], (r - 1) & 1, p.timeout_ns, p.status,
                                                    abort_flag)) {
                        stop = true;
                        break;
                    }
                    uint8_t *st = stages + s * kStageBytes;
                    const int xh = kb >> 1;
                    const int row = (c.b * p.XH + xh) * p.Tc + c.t0;
                    mbar_arrive_expect_tx(&full_tma[s], kTxBytes);
                    tma_load_2d(st, &tm_w, kb * kBK, c.n * kBN, &full_tma[s]);
                    tma_load_2d(st + kOffCodes, &tm_x, (kb & 1) * (kBK / 2), row, &full_tma[s]);
                    bulk_g2s(st + kOffSz, p.x_sz + row, kSzBytes, &full_tma[s]);
                }
            }
            // Drain: the copies of the last stages must land before exit.
            for (int j = max(0, it - kStages); j < it; ++j) {
                const uint64_t t0 = global_timer_ns();
                while (!mbar_try_wait(&full_tma[j % kStages], (j / kStages) & 1)) {
                    if (static_cast<int64_t>(global_timer_ns() - t0) > p.timeout_ns) {
                        status_or(p.status, KVQ_DEV_TIMEOUT);
                        break;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer --------------------------------
        if (lane == 0) {
            int it = 0, lt = 0;
            bool stop = false;
            for (int tile = blockIdx.x; tile < n_total && !stop; tile += gridDim.x, ++lt) {
                const int j = lt & 1, u = lt >> 1;
                if (u > 0 && !mbar_wait_bounded(&acc_empty[j], (u - 1) & 1, p.timeout_ns, p.status,
                                                abort_flag))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + j * kAccCols;
                for (int kb = 0; kb < n_k; ++kb, ++it) {
                    const int s = it % kStages, r = it / kStages;
                    if (!mbar_wait_bounded(&full_tma[s], r & 1, p.timeout_ns, p.status, abort_flag) ||
                        !mbar_wait_bounded(&full_a[s], r & 1, p.timeout_ns, p.status, abort_flag)) {
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                    uint8_t *st = stages + s * kStageBytes;
                    const uint64_t a_desc = sw128_desc(smem_addr(st + kOffA));
                    const uint64_t b_desc = sw128_desc(smem_addr(st));
#pragma unroll
                    for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
                        // +32 bytes along K inside the swizzle atom = +2 in the
                        // descriptor's 16-byte address units.
                        umma_bf16(d_tmem, a_desc + 2 * kk, b_desc + 2 * kk, (kb | kk) != 0);
                    }
                    umma_commit(&empty[s]);
                }
                if (!stop) umma_commit(&acc_full[j]);
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
    } else if (warp < 6) {
        // ------------------------------ dequantizers ------------------------------
        const int row = threadIdx.x - 64;  // token row of the tile, 0..127
        const uint32_t swz = row & 7;
        int it = 0;
        bool stop = false;
        for (int tile = blockIdx.x; tile < n_total && !stop; tile += gridDim.x) {
            for (int kb = 0; kb < n_k; ++kb, ++it) {
                const int s = it % kStages, r = it / kStages;
                // Warp-uniform outcome: the warp's later steps need all lanes.
                if (!__all_sync(0xffffffffu, mbar_wait_bounded(&full_tma[s], r & 1, p.timeout_ns,
                                                               p.status, abort_flag))) {
                    stop = true;
                    break;
                }
                uint8_t *st = stages + s * kStageBytes;
                const uint4 *src = reinterpret_cast<const uint4 *>(st + kOffCodes + row * 32);
                const uint4 c0 = src[0], c1 = src[1];
                const __half2 sz = *reinterpret_cast<const __half2 *>(st + kOffSz + row * 4);
                const float sc = __low2float(sz), zp = __high2float(sz);
                const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                uint8_t *arow = st + kOffA + (row >> 3) * 1024 + swz * 128;
#pragma unroll
                for (int cidx = 0; cidx < 8; ++cidx) {
                    // 8 channels: bytes 4c..4c+3, low nibble first.
                    const uint32_t w = words[cidx];
                    const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
                    uint32_t out[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float qe = small_uint_to_float((lo >> (8 * i)) & 0xFFu);
                        const float qo = small_uint_to_float((hi >> (8 * i)) & 0xFFu);
                        out[i] = pack_bf16x2(__fmaf_rn(qe, sc, zp), __fmaf_rn(qo, sc, zp));
                    }
                    *reinterpret_cast<uint4 *>(arow + ((cidx ^ swz) << 4)) =
                        make_uint4(out[0], out[1], out[2], out[3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&full_a[s]);
            }
        }
    } else {
        // ------------------------------ epilogue ----------------------------------
        const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
        const int row = quarter * 32 + lane;
        int lt = 0;
        for (int tile = blockIdx.x; tile < n_total; tile += gridDim.x, ++lt) {
            const int j = lt & 1, u = lt >> 1;
            // Warp-uniform outcome: tcgen05.ld needs the whole warp.
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(&acc_full[j], u & 1, p.timeout_ns,
                                                           p.status, abort_flag)))
                break;
            tc_fence_after();
            const TileCoord c = tile_coord(p, tile);
            const int t = c.t0 + row;
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + j * kAccCols;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                const int slot = c.n * 2 + half;  // K heads 0..H-1, then V heads
                const bool is_k = slot < p.H;
                const int h = is_k ? slot : slot - p.H;
                uint16_t *dst = (is_k ? p.k_out : p.v_out) +
                                ((static_cast<int64_t>(c.b) * p.H + h) * p.T + t) * kHeadDim;
                const uint32_t col = tbase + half * kHeadDim;
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
                    uint4 *d0 = reinterpret_cast<uint4 *>(dst + c32);
                    uint4 *d1 = reinterpret_cast<uint4 *>(dst + 64 + c32);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        d0[v] = make_uint4(pack_bf16x2(a[8 * v + 0], a[8 * v + 1]), pack_bf16x2(a[8 * v + 2], a[8 * v + 3]),
                                           pack_bf16x2(a[8 * v + 4], a[8 * v + 5]), pack_bf16x2(a[8 * v + 6], a[8 * v + 7]));
                        d1[v] = make_uint4(pack_bf16x2(bv[8 * v + 0], bv[8 * v + 1]), pack_bf16x2(bv[8 * v + 2], bv[8 * v + 3]),
                                           pack_bf16x2(bv[8 * v + 4], bv[8 * v + 5]), pack_bf16x2(bv[8 * v + 6], bv[8 * v + 7]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[j]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
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
                     kHeadDim / 2, kBK / 2, kBM, CU_TENSOR_MAP_SWIZZLE_NONE))
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
    if (cudaFuncSetAttribute(remat_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes)) != cudaSuccess)
        return KVQ_ERR_CUDA;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return KVQ_ERR_CUDA;
    const int64_t tiles = static_cast<int64_t>(p.m_tiles) * p.n_tiles;
    if (tiles >= (1LL << 31)) return KVQ_ERR_UNSUPPORTED;
    const int grid = static_cast<int>(std::min<int64_t>(tiles, sms));
    remat_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tm_w, tm_x, p);
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // namespace kvq
