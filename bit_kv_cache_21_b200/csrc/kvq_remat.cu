// kvq_remat.cu -- XQuant-style rematerialization of K and V from a cache of
// quantized layer inputs X ("XQuant: Breaking the Memory Wall for LLM
// Inference with KV Cache Rematerialization", Abstract), and RoPE tables.
#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

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
    (void)x; (void)w_kv; (void)n_kv_heads; (void)rope_cos; (void)rope_sin; (void)batch;
    (void)ctx_len; (void)k_out; (void)v_out; (void)stream;
    return KVQ_ERR_UNSUPPORTED;
}

}  // namespace kvq
