// kvq_internal.h -- host-side launchers shared between the translation units
// of libkvq.so. Internal; the public interface is include/kvq.h.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

// Rotation scale fp32(1/sqrt(block)) for a power-of-two block, 0 for none.
float hadamard_scale(int block);

// Quantized-residual split: tokens [0, R*floor((T-1)/R)) are quantized.
__host__ __device__ inline int quantized_len(int T, int R) { return (R <= 0) ? T : (T <= 0 ? 0 : R * ((T - 1) / R)); }

kvq_status launch_append(const kvq_cache_desc &d, const void *k_new, const void *v_new,
                         kvq_dtype dtype, const int32_t *cu_new, int32_t *seq_lens,
                         int num_seqs, int total_new, cudaStream_t stream);

// Token ranges of the splits, the same for every sequence: split j < n covers
// the tokens [j * chunk, (j + 1) * chunk) below the sequence's length; chunk
// is a multiple of the decode tiles. A sequence of length T has
// ceil(T / chunk) splits (at most n).
constexpr int kMaxDecodeSplits = 512;
struct SplitBounds {
    int n;      // splits of the longest sequence
    int chunk;  // tokens per split
};

// First token of split j (j <= n; clamped to the int range).
__host__ __device__ inline int split_begin(const SplitBounds &sp, int j) {
    const long long b = static_cast<long long>(j) * sp.chunk;
    return b < 0x7fffffffLL ? static_cast<int>(b) : 0x7fffffff;
}

// Number of splits of a sequence of length T (0 for T <= 0).
__host__ __device__ inline int splits_of(const SplitBounds &sp, int T) {
    if (T <= 0) return 0;
    const int n = static_cast<int>((static_cast<long long>(T) + sp.chunk - 1) / sp.chunk);
    return n < sp.n ? n : sp.n;
}

// Decode attention geometry chosen on the host from the sizes alone.
struct DecodePlan {
    SplitBounds splits;
    int n_split;    // splits of the longest sequence (partials per query head)
    size_t ws_part; // bytes of partial outputs
    size_t ws_ml;   // bytes of (m, l) pairs
    size_t ws_total;
};
bool plan_decode(const kvq_cache_desc &d, int num_seqs, int num_q_heads, int max_seq_len,
                 DecodePlan *plan);

kvq_status launch_decode_splitk(const kvq_cache_desc &d, const DecodePlan &plan, const void *q,
                                kvq_dtype q_dtype, int num_q_heads, const int32_t *seq_lens,
                                int num_seqs, int max_seq_len, float softmax_scale,
                                void *workspace, cudaStream_t stream);
// out_ml == nullptr: normalized output; else this cache's unnormalized
// partial into out and its (m, l) pairs into out_ml.
kvq_status launch_decode_merge(const kvq_cache_desc &d, const DecodePlan &plan, int num_q_heads,
                               const int32_t *seq_lens, int num_seqs, int max_seq_len,
                               float *out, float *out_ml, const void *workspace, cudaStream_t stream);
kvq_status launch_merge_partials(const float *parts, int n_part, int num_seqs, int num_q_heads, float *out,
                                 cudaStream_t stream);

kvq_status launch_remat(const kvq_cache_desc &x, const void *w_kv, int n_kv_heads,
                        const float *rope_cos, const float *rope_sin, int batch, int ctx_len,
                        void *k_out, void *v_out, cudaStream_t stream);
kvq_status launch_rope_tables(float *c, float *s, int n_pos, int head_dim, double theta,
                              cudaStream_t stream);
size_t remat_attention_workspace(int batch, int num_q_heads, int ctx_len);
kvq_status launch_remat_attention(const kvq_cache_desc &x, const void *w_kv, int n_kv_heads,
                                  const float *rope_cos, const float *rope_sin, int batch, int ctx_len,
                                  const void *q, kvq_dtype q_dtype, int num_q_heads, float softmax_scale,
                                  float *out, void *workspace, cudaStream_t stream);

}  // namespace kvq
