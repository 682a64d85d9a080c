// kvq_static_ws.cu -- decode attention for callers that cannot allocate
// device memory.
//
// kvq_decode_attention needs a workspace (split partial outputs, softmax
// statistics and an item counter). Some callers cannot provide one: a plain C
// host program or a plugin that runs inside another runtime which owns every
// device allocation, or a latency-bound decode loop that must not call
// cudaMalloc, which can synchronize the whole device. For them this file keeps
// the workspace in a fixed array in device global memory that the library
// itself declares, so the call below takes only inputs and outputs.
//
// Costs and limits: the array (kStaticBytes) is reserved on every GPU that
// loads the library, for the life of the process. All calls share it and it
// keeps whatever the previous call left; the launch path zeroes the one word
// that has to start at zero (the item counter) on the stream. Calls whose
// work overlaps on the GPU (other streams, or other host threads) race on the
// array.
#include <cuda.h>

#include <mutex>

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr size_t kStaticBytes = size_t(16) << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

// The shared scratch array. In host code this name is only a host-side handle
// for the symbol, never a device address; kernels get the address looked up
// below.
__device__ __align__(256) unsigned char g_static_workspace[kStaticBytes];

// The array's device address is valid in the context that loaded the module.
// The lookups are cached per device together with the context they were made
// in (read through the driver's cuCtxGetCurrent, reached via the runtime's
// entry-point query so the library needs no link to the driver), and made
// again when a different context is current on that device: a plugin that
// runs in its own context, or a context created after cudaDeviceReset.
using CtxGetCurrentFn = CUresult (*)(CUcontext *);

struct Cached {
    CUcontext ctx;
    void *ptr;
};
std::mutex g_lock;
Cached g_cache[kMaxDevices];
CtxGetCurrentFn g_ctx_get = nullptr;
bool g_ctx_get_looked_up = false;

// The current context, or nullptr when it cannot be read (then nothing is
// cached and every call looks the address up).
CUcontext current_context() {
    if (!g_ctx_get_looked_up) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_get = reinterpret_cast<CtxGetCurrentFn>(fn);
        g_ctx_get_looked_up = true;
    }
    CUcontext ctx = nullptr;
    if (g_ctx_get == nullptr || g_ctx_get(&ctx) != CUDA_SUCCESS) return nullptr;
    return ctx;
}

// Device address of the array in the current context of the current device.
// The first call on a device (and in each further context) performs this
// set-up.
kvq_status static_workspace(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
    std::lock_guard<std::mutex> guard(g_lock);
    CUcontext ctx = current_context();
    if (ctx != nullptr && g_cache[dev].ctx == ctx && g_cache[dev].ptr != nullptr) {
        *out = g_cache[dev].ptr;
        return KVQ_OK;
    }
    // the lookup also makes the device's primary context current on this
    // thread when no context was yet
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_workspace) != cudaSuccess || ptr == nullptr) return KVQ_ERR_CUDA;
    if (ctx == nullptr) ctx = current_context();
    g_cache[dev] = Cached{ctx, ptr};  // ctx == nullptr: never matches, looked up on every call
    *out = ptr;
    return KVQ_OK;
}

}  // namespace
}  // namespace kvq

using namespace kvq;

extern "C" {

kvq_status kvq_decode_attention_static(const kvq_cache_desc *desc, const void *q, kvq_dtype q_dtype,
                                       int32_t num_q_heads, const int32_t *seq_lens,
                                       int32_t num_seqs, int32_t max_seq_len, float softmax_scale,
                                       float *out, void *stream) {
    if (desc == nullptr || out == nullptr) return KVQ_ERR_INVALID_ARG;
    const size_t need = kvq_decode_workspace_size(desc, num_seqs, num_q_heads, max_seq_len);
    if (need == 0) return KVQ_ERR_INVALID_ARG;
    if (need > kStaticBytes) return KVQ_ERR_CAPACITY;  // larger than the fixed array
    void *ws = nullptr;
    const kvq_status s = static_workspace(&ws);
    if (s != KVQ_OK) return s;
    return kvq_decode_attention(desc, q, q_dtype, num_q_heads, seq_lens, num_seqs, max_seq_len,
                                softmax_scale, out, ws, kStaticBytes, stream);
}

}  // extern "C"
