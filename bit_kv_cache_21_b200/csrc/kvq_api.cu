// kvq_api.cu -- the C ABI of libkvq.so: argument validation and dispatch to
// the kernel launchers. Validation failures launch nothing.
#include <math.h>

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {

DebugHooks &debug_hooks() {
    static DebugHooks h{1000000000LL, -1};
    return h;
}

float hadamard_scale(int block) {
    return block > 0 ? static_cast<float>(1.0 / sqrt(static_cast<double>(block))) : 0.0f;
}

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
bool token_group_ok(int g) { return g == 16 || g == 32 || g == 64 || g == 128; }

// Checks shared by every entry point. `need_v`: the call reads or writes V.
kvq_status validate_desc(const kvq_cache_desc *d, bool need_v) {
    if (d == nullptr) return KVQ_ERR_INVALID_ARG;
    if (d->head_dim != kHeadDim) return KVQ_ERR_UNSUPPORTED;
    if (d->num_kv_heads <= 0 || d->num_seqs <= 0 || d->reserved != 0) return KVQ_ERR_INVALID_ARG;
    if (d->hadamard_block_k != 0 && !(pow2(d->hadamard_block_k) && d->hadamard_block_k >= 2 &&
                                      d->hadamard_block_k <= kHeadDim))
        return KVQ_ERR_INVALID_ARG;
    auto bits_ok = [](int b) { return b == 2 || b == 4 || b == 16; };
    if (!bits_ok(d->bits_k) || (need_v && !bits_ok(d->bits_v))) return KVQ_ERR_INVALID_ARG;
    if (d->axis_k != KVQ_PER_TOKEN && d->axis_k != KVQ_PER_CHANNEL) return KVQ_ERR_INVALID_ARG;
    if (d->axis_v != KVQ_PER_TOKEN && d->axis_v != KVQ_PER_CHANNEL) return KVQ_ERR_INVALID_ARG;
    const bool bf16_k = d->bits_k == 16, bf16_v = need_v && d->bits_v == 16;
    const bool chan_v = need_v && d->axis_v == KVQ_PER_CHANNEL;
    if (need_v && bf16_k != bf16_v) return KVQ_ERR_UNSUPPORTED;
    if (bf16_k && (d->paged || d->residual_len || d->hadamard_block_k)) return KVQ_ERR_UNSUPPORTED;
    if (!bf16_k) {
        if (d->axis_k == KVQ_PER_TOKEN && !token_group_ok(d->group_k)) return KVQ_ERR_INVALID_ARG;
        if (need_v && !chan_v && !token_group_ok(d->group_v)) return KVQ_ERR_INVALID_ARG;
    }
    if (d->axis_k == KVQ_PER_CHANNEL) {
        if (bf16_k || d->paged || d->hadamard_block_k) return KVQ_ERR_UNSUPPORTED;
        if (d->residual_len != d->group_k) return KVQ_ERR_INVALID_ARG;
    }
    if (chan_v) {  // values grouped along tokens: one block of the window at a time
        if (bf16_v || d->paged || d->hadamard_block_k) return KVQ_ERR_UNSUPPORTED;
        if (d->residual_len != d->group_v) return KVQ_ERR_INVALID_ARG;
        if (d->bits_k != d->bits_v) return KVQ_ERR_UNSUPPORTED;
    }
    if (d->residual_len != 0) {
        if (!(d->residual_len == 64 || d->residual_len == 128 || d->residual_len == 256))
            return KVQ_ERR_INVALID_ARG;
        if (d->paged || d->hadamard_block_k || !need_v) return KVQ_ERR_UNSUPPORTED;
        if (d->k_res == nullptr || d->v_res == nullptr || !aligned16(d->k_res) || !aligned16(d->v_res))
            return KVQ_ERR_INVALID_ARG;
        if (d->capacity_tokens % d->residual_len != 0) return KVQ_ERR_INVALID_ARG;
    }
    if (d->paged) {
        if (!pow2(d->page_size) || d->page_size < 16 || d->page_size > 1024) return KVQ_ERR_INVALID_ARG;
        if (d->max_pages_per_seq <= 0 || d->num_pages <= 0 || d->block_table == nullptr)
            return KVQ_ERR_INVALID_ARG;
    } else {
        if (d->capacity_tokens <= 0 || d->capacity_tokens % 64 != 0) return KVQ_ERR_INVALID_ARG;
    }
    if (d->k_codes == nullptr || !aligned16(d->k_codes)) return KVQ_ERR_INVALID_ARG;
    if (!bf16_k && (d->k_sz == nullptr || !aligned16(d->k_sz))) return KVQ_ERR_INVALID_ARG;
    if (need_v) {
        if (d->v_codes == nullptr || !aligned16(d->v_codes)) return KVQ_ERR_INVALID_ARG;
        if (!bf16_v && (d->v_sz == nullptr || !aligned16(d->v_sz))) return KVQ_ERR_INVALID_ARG;
    }
    if (d->status != nullptr && (reinterpret_cast<uintptr_t>(d->status) & 3u)) return KVQ_ERR_INVALID_ARG;
    if (d->hadamard_signs != nullptr && (d->hadamard_block_k == 0 || !aligned16(d->hadamard_signs)))
        return KVQ_ERR_INVALID_ARG;
    if ((d->hybrid != 0 && d->hybrid != 1) || d->sink_len < 0 || d->sink_len > 64) return KVQ_ERR_INVALID_ARG;
    if (d->sink_len > 0) {
        if (!need_v || bf16_k || d->axis_k != KVQ_PER_TOKEN || d->residual_len != 0) return KVQ_ERR_UNSUPPORTED;
        if (d->k_sink == nullptr || d->v_sink == nullptr || !aligned16(d->k_sink) || !aligned16(d->v_sink))
            return KVQ_ERR_INVALID_ARG;
    }
    return KVQ_OK;
}

bool dtype_ok(int dt) { return dt == KVQ_BF16 || dt == KVQ_FP16 || dt == KVQ_FP32; }

kvq_status validate_decode(const kvq_cache_desc *d, const void *q, int q_dtype, int num_q_heads,
                           const int32_t *seq_lens, int num_seqs, int max_seq_len) {
    kvq_status s = validate_desc(d, true);
    if (s != KVQ_OK) return s;
    if (q == nullptr || !aligned16(q) || !dtype_ok(q_dtype) || seq_lens == nullptr)
        return KVQ_ERR_INVALID_ARG;
    if (num_seqs <= 0 || max_seq_len < 0 || num_q_heads <= 0) return KVQ_ERR_INVALID_ARG;
    if (num_q_heads % d->num_kv_heads != 0) return KVQ_ERR_INVALID_ARG;
    const int gqa = num_q_heads / d->num_kv_heads;
    if (gqa != 1 && gqa != 2 && gqa != 4) return KVQ_ERR_UNSUPPORTED;
    if (d->sink_len > 0 && num_seqs > d->num_seqs) return KVQ_ERR_INVALID_ARG;
    if (!d->paged) {
        if (num_seqs > d->num_seqs || max_seq_len > d->capacity_tokens) return KVQ_ERR_INVALID_ARG;
    } else if (static_cast<int64_t>(max_seq_len) >
               static_cast<int64_t>(d->max_pages_per_seq) * d->page_size) {
        return KVQ_ERR_INVALID_ARG;
    }
    return KVQ_OK;
}

}  // namespace
}  // namespace kvq

using namespace kvq;

extern "C" {

kvq_status kvq_quantize_append(const kvq_cache_desc *desc, const void *k_new, const void *v_new,
                               kvq_dtype dtype, const int32_t *cu_new, int32_t *seq_lens,
                               int32_t num_seqs, int32_t total_new_tokens, void *stream) {
    const bool need_v = desc != nullptr && desc->v_codes != nullptr;
    kvq_status s = validate_desc(desc, need_v);
    if (s != KVQ_OK) return s;
    if (desc->bits_k == 16) return KVQ_ERR_UNSUPPORTED;
    if (!dtype_ok(dtype) || cu_new == nullptr || seq_lens == nullptr) return KVQ_ERR_INVALID_ARG;
    if (num_seqs <= 0 || total_new_tokens < 0) return KVQ_ERR_INVALID_ARG;
    if ((!desc->paged || desc->sink_len > 0) && num_seqs > desc->num_seqs) return KVQ_ERR_INVALID_ARG;
    if (total_new_tokens == 0) return KVQ_OK;  // nothing to write, lengths unchanged
    if ((v_new != nullptr) != need_v) return KVQ_ERR_INVALID_ARG;
    if (k_new == nullptr || !aligned16(k_new) || (need_v && !aligned16(v_new)))
        return KVQ_ERR_INVALID_ARG;
    if (desc->residual_len > 0 && dtype != KVQ_BF16) return KVQ_ERR_UNSUPPORTED;
    return launch_append(*desc, k_new, v_new, dtype, cu_new, seq_lens, num_seqs, total_new_tokens,
                         static_cast<cudaStream_t>(stream));
}

size_t kvq_decode_workspace_size(const kvq_cache_desc *desc, int32_t num_seqs,
                                 int32_t num_q_heads, int32_t max_seq_len) {
    if (desc == nullptr) return 0;
    DecodePlan plan;
    if (!plan_decode(*desc, num_seqs, num_q_heads, max_seq_len, &plan)) return 0;
    return plan.ws_total;
}

kvq_status kvq_decode_splitk(const kvq_cache_desc *desc, const void *q, kvq_dtype q_dtype,
                             int32_t num_q_heads, const int32_t *seq_lens, int32_t num_seqs,
                             int32_t max_seq_len, float softmax_scale, void *workspace,
                             size_t workspace_bytes, void *stream) {
    kvq_status s = validate_decode(desc, q, q_dtype, num_q_heads, seq_lens, num_seqs, max_seq_len);
    if (s != KVQ_OK) return s;
    DecodePlan plan;
    if (!plan_decode(*desc, num_seqs, num_q_heads, max_seq_len, &plan)) return KVQ_ERR_INVALID_ARG;
    if (workspace == nullptr || !aligned16(workspace) || workspace_bytes < plan.ws_total)
        return workspace == nullptr || !aligned16(workspace) ? KVQ_ERR_INVALID_ARG : KVQ_ERR_CAPACITY;
    if (!isfinite(softmax_scale)) return KVQ_ERR_INVALID_ARG;
    return launch_decode_splitk(*desc, plan, q, q_dtype, num_q_heads, seq_lens, num_seqs,
                                max_seq_len, softmax_scale, workspace,
                                static_cast<cudaStream_t>(stream));
}

kvq_status kvq_decode_merge(const kvq_cache_desc *desc, int32_t num_q_heads,
                            const int32_t *seq_lens, int32_t num_seqs, int32_t max_seq_len,
                            float *out, const void *workspace, size_t workspace_bytes,
                            void *stream) {
    kvq_status s = validate_desc(desc, true);
    if (s != KVQ_OK) return s;
    if (out == nullptr || !aligned16(out) || seq_lens == nullptr || num_seqs <= 0 || num_q_heads <= 0 ||
        max_seq_len < 0)
        return KVQ_ERR_INVALID_ARG;
    DecodePlan plan;
    if (!plan_decode(*desc, num_seqs, num_q_heads, max_seq_len, &plan)) return KVQ_ERR_INVALID_ARG;
    if (workspace == nullptr || !aligned16(workspace) || workspace_bytes < plan.ws_total)
        return workspace == nullptr || !aligned16(workspace) ? KVQ_ERR_INVALID_ARG : KVQ_ERR_CAPACITY;
    return launch_decode_merge(*desc, plan, num_q_heads, seq_lens, num_seqs, max_seq_len, out,
                               nullptr, workspace, static_cast<cudaStream_t>(stream));
}

kvq_status kvq_decode_merge_partial(const kvq_cache_desc *desc, int32_t num_q_heads,
                                    const int32_t *seq_lens, int32_t num_seqs, int32_t max_seq_len,
                                    float *o_part, float *ml, const void *workspace,
                                    size_t workspace_bytes, void *stream) {
    kvq_status s = validate_desc(desc, true);
    if (s != KVQ_OK) return s;
    if (o_part == nullptr || ml == nullptr || !aligned16(o_part) || (reinterpret_cast<uintptr_t>(ml) & 7u) ||
        seq_lens == nullptr || num_seqs <= 0 || num_q_heads <= 0 || max_seq_len < 0)
        return KVQ_ERR_INVALID_ARG;
    DecodePlan plan;
    if (!plan_decode(*desc, num_seqs, num_q_heads, max_seq_len, &plan)) return KVQ_ERR_INVALID_ARG;
    if (workspace == nullptr || !aligned16(workspace) || workspace_bytes < plan.ws_total)
        return workspace == nullptr || !aligned16(workspace) ? KVQ_ERR_INVALID_ARG : KVQ_ERR_CAPACITY;
    return launch_decode_merge(*desc, plan, num_q_heads, seq_lens, num_seqs, max_seq_len, o_part, ml,
                               workspace, static_cast<cudaStream_t>(stream));
}

kvq_status kvq_merge_partials(const float *parts, int32_t n_part, int32_t num_seqs, int32_t num_q_heads,
                              float *out, void *stream) {
    if (parts == nullptr || out == nullptr || !aligned16(parts) || n_part <= 0 || num_seqs <= 0 ||
        num_q_heads <= 0 || num_seqs > 65535 || num_q_heads > 65535)
        return KVQ_ERR_INVALID_ARG;
    if (static_cast<int64_t>(num_seqs) * num_q_heads * (kHeadDim + 2) * n_part > (int64_t(1) << 40))
        return KVQ_ERR_INVALID_ARG;
    return launch_merge_partials(parts, n_part, num_seqs, num_q_heads, out, static_cast<cudaStream_t>(stream));
}

kvq_status kvq_decode_attention(const kvq_cache_desc *desc, const void *q, kvq_dtype q_dtype,
                                int32_t num_q_heads, const int32_t *seq_lens, int32_t num_seqs,
                                int32_t max_seq_len, float softmax_scale, float *out,
                                void *workspace, size_t workspace_bytes, void *stream) {
    if (out == nullptr || !aligned16(out)) return KVQ_ERR_INVALID_ARG;
    kvq_status s = kvq_decode_splitk(desc, q, q_dtype, num_q_heads, seq_lens, num_seqs,
                                     max_seq_len, softmax_scale, workspace, workspace_bytes, stream);
    if (s != KVQ_OK) return s;
    return kvq_decode_merge(desc, num_q_heads, seq_lens, num_seqs, max_seq_len, out, workspace,
                            workspace_bytes, stream);
}

kvq_status kvq_remat_kv(const kvq_cache_desc *x_cache, const void *w_kv, int32_t n_kv_heads,
                        const float *rope_cos, const float *rope_sin, int32_t batch,
                        int32_t ctx_len, void *k_out, void *v_out, void *stream) {
    kvq_status s = validate_desc(x_cache, false);
    if (s != KVQ_OK) return s;
    if (x_cache->paged || x_cache->bits_k != 4 || x_cache->group_k != 128 ||
        x_cache->axis_k != KVQ_PER_TOKEN || x_cache->hadamard_block_k != 0 ||
        x_cache->residual_len != 0)
        return KVQ_ERR_UNSUPPORTED;
    if (w_kv == nullptr || rope_cos == nullptr || rope_sin == nullptr || k_out == nullptr ||
        v_out == nullptr || !aligned16(w_kv) || !aligned16(k_out) || !aligned16(v_out) ||
        !aligned16(rope_cos) || !aligned16(rope_sin))
        return KVQ_ERR_INVALID_ARG;
    if (n_kv_heads <= 0 || batch <= 0 || batch > x_cache->num_seqs || ctx_len <= 0 ||
        ctx_len % 128 != 0 || ctx_len > x_cache->capacity_tokens)
        return KVQ_ERR_INVALID_ARG;
    return launch_remat(*x_cache, w_kv, n_kv_heads, rope_cos, rope_sin, batch, ctx_len, k_out,
                        v_out, static_cast<cudaStream_t>(stream));
}

size_t kvq_remat_attention_workspace_size(int32_t batch, int32_t num_q_heads, int32_t ctx_len) {
    if (batch <= 0 || num_q_heads <= 0 || ctx_len <= 0 || ctx_len % 128 != 0) return 0;
    return remat_attention_workspace(batch, num_q_heads, ctx_len);
}

kvq_status kvq_remat_attention(const kvq_cache_desc *x_cache, const void *w_kv, int32_t n_kv_heads,
                               const float *rope_cos, const float *rope_sin, int32_t batch, int32_t ctx_len,
                               const void *q, kvq_dtype q_dtype, int32_t num_q_heads, float softmax_scale,
                               float *out, void *workspace, size_t workspace_bytes, void *stream) {
    kvq_status s = validate_desc(x_cache, false);
    if (s != KVQ_OK) return s;
    if (x_cache->paged || x_cache->bits_k != 4 || x_cache->group_k != 128 ||
        x_cache->axis_k != KVQ_PER_TOKEN || x_cache->hadamard_block_k != 0 ||
        x_cache->residual_len != 0 || x_cache->sink_len != 0)
        return KVQ_ERR_UNSUPPORTED;
    if (w_kv == nullptr || rope_cos == nullptr || rope_sin == nullptr || q == nullptr || out == nullptr ||
        !aligned16(w_kv) || !aligned16(rope_cos) || !aligned16(rope_sin) || !aligned16(q) || !aligned16(out) ||
        !dtype_ok(q_dtype))
        return KVQ_ERR_INVALID_ARG;
    if (n_kv_heads <= 0 || batch <= 0 || batch > x_cache->num_seqs || ctx_len <= 0 || ctx_len % 128 != 0 ||
        ctx_len > x_cache->capacity_tokens || num_q_heads <= 0 || num_q_heads % n_kv_heads != 0 ||
        batch > 65535)
        return KVQ_ERR_INVALID_ARG;
    const int gqa = num_q_heads / n_kv_heads;
    if (gqa != 1 && gqa != 2 && gqa != 4) return KVQ_ERR_UNSUPPORTED;
    if (workspace == nullptr || !aligned16(workspace)) return KVQ_ERR_INVALID_ARG;
    if (workspace_bytes < remat_attention_workspace(batch, num_q_heads, ctx_len)) return KVQ_ERR_CAPACITY;
    return launch_remat_attention(*x_cache, w_kv, n_kv_heads, rope_cos, rope_sin, batch, ctx_len, q, q_dtype,
                                  num_q_heads, softmax_scale, out, workspace, static_cast<cudaStream_t>(stream));
}

kvq_status kvq_rope_tables(float *rope_cos, float *rope_sin, int32_t n_pos, int32_t head_dim,
                           double theta, void *stream) {
    if (rope_cos == nullptr || rope_sin == nullptr || n_pos <= 0 || head_dim <= 0 ||
        head_dim % 2 != 0 || !(theta > 1.0))
        return KVQ_ERR_INVALID_ARG;
    return launch_rope_tables(rope_cos, rope_sin, n_pos, head_dim, theta,
                              static_cast<cudaStream_t>(stream));
}

const char *kvq_status_string(kvq_status status) {
    switch (status) {
        case KVQ_OK: return "ok";
        case KVQ_ERR_INVALID_ARG: return "invalid argument";
        case KVQ_ERR_UNSUPPORTED: return "unsupported combination";
        case KVQ_ERR_CAPACITY: return "buffer too small";
        case KVQ_ERR_TIMEOUT: return "timed out";
        case KVQ_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

kvq_status kvq_debug_set(int32_t what, int64_t value) {
    switch (what) {
        case KVQ_DEBUG_WAIT_TIMEOUT_NS:
            debug_hooks().wait_timeout_ns = value > 0 ? value : 1000000000LL;
            return KVQ_OK;
        case KVQ_DEBUG_SKIP_TILE:
            debug_hooks().skip_tile = value < 0 ? -1 : static_cast<int32_t>(value);
            return KVQ_OK;
    }
    return KVQ_ERR_INVALID_ARG;
}

int32_t kvq_version(void) { return 100; }

}  // extern "C"
