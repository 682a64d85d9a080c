// kvq_common.cuh -- device helpers shared by the sm_100a kernels: bounded
// mbarrier waits, 1-D bulk copies (TMA engine), status reporting, number
// conversions. Internal header, not part of the C ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

constexpr int kHeadDim = 128;
constexpr int kWarp = 32;

// ---------------------------------------------------------------------------
// Host-side launch settings shared by the translation units.
// ---------------------------------------------------------------------------
struct DebugHooks {
    int64_t wait_timeout_ns;
    int32_t skip_tile;
};
DebugHooks &debug_hooks();

// ---------------------------------------------------------------------------
// Status word
// ---------------------------------------------------------------------------
__device__ __forceinline__ void status_or(int32_t *st, int32_t bits) {
    if (st != nullptr) atomicOr(st, bits);
}

// ---------------------------------------------------------------------------
// Timers and mbarriers (PTX). Every wait is bounded by a %globaltimer limit.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

// Make mbarrier initialisation visible to the async proxy (bulk copies).
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_addr(bar)),
        "r"(bytes)
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Same test, but a thread whose phase is not complete may be suspended (it
// issues nothing) until the phase completes or about `hint_ns` pass.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Suspend hint of the bounded waits: waiters sleep in hardware instead of
// re-polling; the timeout and the abort flag are checked once per wake-up.
constexpr uint32_t kWaitSleepNs = 200000;

// Wait until the phase of `bar` with the given parity has completed, or until
// `timeout_ns` passes (then OR KVQ_DEV_TIMEOUT into *status and raise the
// CTA's abort flag), or until another thread raised the abort flag.
// Returns true when the phase completed.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  int64_t timeout_ns, int32_t *status,
                                                  volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) return true;
        if (*abort_flag) return false;
        if (static_cast<int64_t>(global_timer_ns() - t0) > timeout_ns) {
            status_or(status, KVQ_DEV_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
    }
}

// Programmatic dependent launch: let the next kernel of the stream (launched
// with programmatic stream serialization) be scheduled now; and, in that
// kernel, wait until the previous grid has completed and its writes are
// visible. Both are no-ops without such a launch.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_prior_grid() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// 1-D bulk copy global -> shared through the TMA engine, completing on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16. No multicast.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// Named barrier among `nthreads` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// Number conversions
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_bits_to_float(uint32_t b16) {
    return __uint_as_float(b16 << 16);
}

// Small unsigned integer (< 2^23) to float exactly: place it in the
// mantissa of 2^23 and subtract 2^23.
__device__ __forceinline__ float small_uint_to_float(uint32_t c) {
    return __fsub_rn(__uint_as_float(0x4B000000u | c), 8388608.0f);
}

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Log-sum-exp combination of n partials (o_j, m_j, l_j) of one (sequence,
// query head) by a CTA of 128 * NG threads: thread t takes channel t % 128
// and the partials j = t / 128 (mod NG), so NG groups walk the partials side
// by side. Partial j's o row is at o_part + o0 + j * o_step (kHeadDim floats),
// its (m, l) at ml[m0 + j * m_step]. o = sum_j e_j o_j, l = sum_j e_j l_j with
// e_j = 2^(m_j - M), M = max_j m_j (log2 units); partials with m = -inf (no
// tokens) weigh 0. The groups' sums are added in group order. Results are
// valid in the threads of group 0 (t < 128).
template <int NG>
struct CombineSmem {
    float o[NG][kHeadDim];
    float l[NG];
    float red[NG * 4];
    float max;
};

template <int NG>
__device__ __forceinline__ void combine_partials(const float *o_part, const float2 *ml, int64_t o0,
                                                 int64_t o_step, int64_t m0, int64_t m_step, int n,
                                                 CombineSmem<NG> &sm, float &M, float &o, float &l) {
    const int t = threadIdx.x, d = t & (kHeadDim - 1), grp = t / kHeadDim;
    float m = -INFINITY;
    for (int j = t; j < n; j += NG * kHeadDim) m = fmaxf(m, ml[m0 + j * m_step].x);
#pragma unroll
    for (int k = 16; k > 0; k >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, k));
    if ((t & 31) == 0) sm.red[t >> 5] = m;
    __syncthreads();
    if (t == 0) {
        float mm = sm.red[0];
        for (int w = 1; w < NG * 4; ++w) mm = fmaxf(mm, sm.red[w]);
        sm.max = mm;
    }
    __syncthreads();
    M = sm.max;
    float oo = 0.0f, ll = 0.0f;
#pragma unroll 4
    for (int j = grp; j < n; j += NG) {
        const float2 v = ml[m0 + j * m_step];
        const float e = (v.x == -INFINITY) ? 0.0f : fast_exp2(v.x - M);
        oo = fmaf(e, o_part[o0 + j * o_step + d], oo);
        ll = fmaf(e, v.y, ll);
    }
    if constexpr (NG == 1) {
        o = oo;
        l = ll;
    } else {
        sm.o[grp][d] = oo;
        if (d == 0) sm.l[grp] = ll;
        __syncthreads();
        o = sm.o[0][d];
        l = sm.l[0];
#pragma unroll
        for (int g = 1; g < NG; ++g) {
            o += sm.o[g][d];
            l += sm.l[g];
        }
    }
}

// The same combination by a CTA of 32 * NW threads with one partial per warp
// at a time: warp w takes the partials j = w, w + NW, ..., lane i channels
// 4i..4i+3 of each, so every o load is 16 bytes and NW partials are read per
// step (the loop is unrolled, several steps in flight). o rows must be 16-byte
// aligned (o0 and o_step multiples of 4). The warps' sums are added in warp
// order; the results are valid in warp 0 (o = channels 4*lane..4*lane+3).
template <int NW>
struct CombineSmemW {
    float4 o[NW][32];
    float l[NW];
    float red[NW];
};

template <int NW>
__device__ __forceinline__ void combine_partials_w(const float *o_part, const float2 *ml, int64_t o0,
                                                   int64_t o_step, int64_t m0, int64_t m_step, int n,
                                                   CombineSmemW<NW> &sm, float &M, float4 &o, float &l) {
    const int t = threadIdx.x, w = t >> 5, lane = t & 31;
    float m = -INFINITY;
    for (int j = t; j < n; j += NW * 32) m = fmaxf(m, ml[m0 + j * m_step].x);
#pragma unroll
    for (int k = 16; k > 0; k >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, k));
    if (lane == 0) sm.red[w] = m;
    __syncthreads();
    float mm = sm.red[0];
#pragma unroll
    for (int k = 1; k < NW; ++k) mm = fmaxf(mm, sm.red[k]);
    M = mm;
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    float ll = 0.0f;
#pragma unroll 4
    for (int j = w; j < n; j += NW) {
        const float2 v = ml[m0 + j * m_step];
        const float4 ov = *reinterpret_cast<const float4 *>(o_part + o0 + j * o_step + 4 * lane);
        const float e = (v.x == -INFINITY) ? 0.0f : fast_exp2(v.x - M);
        acc.x = fmaf(e, ov.x, acc.x);
        acc.y = fmaf(e, ov.y, acc.y);
        acc.z = fmaf(e, ov.z, acc.z);
        acc.w = fmaf(e, ov.w, acc.w);
        ll = fmaf(e, v.y, ll);
    }
    sm.o[w][lane] = acc;
    if (lane == 0) sm.l[w] = ll;
    __syncthreads();
    o = sm.o[0][lane];
    l = sm.l[0];
#pragma unroll
    for (int k = 1; k < NW; ++k) {
        const float4 b = sm.o[k][lane];
        o.x += b.x; o.y += b.y; o.z += b.z; o.w += b.w;
        l += sm.l[k];
    }
}

}  // namespace kvq
