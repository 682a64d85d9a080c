// kvq_decode.cu -- decode attention entry: the split plan, the choice of the
// split-K variant family, and the log-sum-exp merge of the splits. The split-K
// kernel itself is kvq_decode_kernel.cuh, instantiated by kvq_decode_*.cu.
#include "kvq_decode_kernel.cuh"

namespace kvq {

using namespace dec;

namespace {
// One CTA of 128 threads per (query head, sequence): combine the splits.
// Launched as a programmatic dependent of the split-K pass: its CTAs may start
// while that pass drains and wait here until its partials are complete.
__global__ void __launch_bounds__(128) decode_merge_kernel(const float *o_part, const float2 *ml,
                                                           const int32_t *seq_lens, float *out,
                                                           int Hq, int n_split, int chunk,
                                                           int max_seq_len) {
    __shared__ float s_max;
    pdl_wait_prior_grid();
    const int hq = blockIdx.x, seq = blockIdx.y, d = threadIdx.x;
    const int T = min(__ldg(seq_lens + seq), max_seq_len);
    const int nv = T > 0 ? (T + chunk - 1) / chunk : 0;
    const int64_t base = (static_cast<int64_t>(seq) * Hq + hq) * n_split;
    if (d < 32) {  // maximum over the splits, one warp
        float m = -INFINITY;
        for (int j = d; j < nv; j += 32) m = fmaxf(m, ml[base + j].x);
#pragma unroll
        for (int k = 16; k > 0; k >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, k));
        if (d == 0) s_max = m;
    }
    __syncthreads();
    const float M = s_max;
    float o = 0.0f, l = 0.0f;
    const float *op = o_part + base * kHeadDim + d;
#pragma unroll 4
    for (int j = 0; j < nv; ++j) {
        const float2 v = ml[base + j];
        const float e = (v.x == -INFINITY) ? 0.0f : fast_exp2(v.x - M);
        o = fmaf(e, op[static_cast<int64_t>(j) * kHeadDim], o);
        l = fmaf(e, v.y, l);
    }
    out[(static_cast<int64_t>(seq) * Hq + hq) * kHeadDim + d] = (l > 0.0f) ? o / l : 0.0f;
}

}  // namespace

bool plan_decode(const kvq_cache_desc &d, int num_seqs, int num_q_heads, int max_seq_len,
                 DecodePlan *plan) {
    if (num_seqs <= 0 || num_q_heads <= 0 || max_seq_len < 0 || d.num_kv_heads <= 0) return false;
    // About eight items per resident CTA (2 per SM) when every sequence is at
    // max_seq_len; chunks of 256..4096 tokens, a multiple of the tiles.
    const int64_t units = static_cast<int64_t>(num_seqs) * d.num_kv_heads;
    const int64_t target_items = 8 * 2 * 148;
    int64_t chunk = (units * std::max(1, max_seq_len) + target_items - 1) / target_items;
    chunk = ((chunk + kTileQ - 1) / kTileQ) * kTileQ;
    chunk = std::min<int64_t>(std::max<int64_t>(chunk, 256), 4096);
    plan->chunk = static_cast<int>(chunk);
    plan->n_split = static_cast<int>(std::max<int64_t>(1, (max_seq_len + chunk - 1) / chunk));
    const size_t rows = static_cast<size_t>(num_seqs) * num_q_heads * plan->n_split;
    plan->ws_part = rows * kHeadDim * sizeof(float);
    plan->ws_ml = rows * sizeof(float2);
    plan->ws_total = plan->ws_part + plan->ws_ml + 16;  // + the item counter
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
    p.signs = d.hadamard_block_k > 0 ? d.hadamard_signs : nullptr;
    p.k_sink = static_cast<const uint16_t *>(d.k_sink);
    p.v_sink = static_cast<const uint16_t *>(d.v_sink);
    p.sink_len = d.sink_len;
    p.o_part = static_cast<float *>(workspace);
    p.ml = reinterpret_cast<float2 *>(static_cast<uint8_t *>(workspace) + plan.ws_part);
    p.counter = reinterpret_cast<int *>(static_cast<uint8_t *>(workspace) + plan.ws_part + plan.ws_ml);
    p.status = d.status;
    p.S = num_seqs;
    p.H = d.num_kv_heads;
    p.Hq = num_q_heads;
    p.gk = (d.bits_k == 16 || d.axis_k == KVQ_PER_CHANNEL) ? kHeadDim : d.group_k;
    p.gv = (d.bits_v == 16 || d.axis_v == KVQ_PER_CHANNEL) ? kHeadDim : d.group_v;
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
    p.q_bytes = (q_dtype == KVQ_FP32) ? 4 : 2;
    const int gqa = num_q_heads / d.num_kv_heads;
    const StageLayout L = stage_layout(d, gqa, p.q_bytes);
    p.stage_bytes = L.bytes;
    p.off_ksz = L.off_ksz;
    p.off_vc = L.off_vc;
    p.off_vsz = L.off_vsz;
    p.off_q = L.off_q;
    p.off_hdr = L.off_hdr;
    p.bf_tile = L.bf_tile;
    p.bf_off_v = L.bf_off_v;
    p.timeout_ns = debug_hooks().wait_timeout_ns;
    p.skip_tile = debug_hooks().skip_tile;
    const int64_t max_items64 = static_cast<int64_t>(num_seqs) * d.num_kv_heads * plan.n_split;
    const int max_items = static_cast<int>(std::min<int64_t>(max_items64, 1 << 30));
    if (gqa != 1 && gqa != 2 && gqa != 4) return KVQ_ERR_UNSUPPORTED;
    if (d.bits_k != 16 && d.residual_len > 0)
        return (d.axis_v == KVQ_PER_CHANNEL) ? dispatch_innerq(d, p, gqa, max_items, stream)
                                             : dispatch_window(d, p, gqa, max_items, stream);
    if (d.bits_k != 16 && d.sink_len > 0) return dispatch_sink(d, p, gqa, max_items, stream);
    return dispatch_plain(d, p, gqa, max_items, stream);
}

kvq_status launch_decode_merge(const kvq_cache_desc &d, const DecodePlan &plan, int num_q_heads,
                               const int32_t *seq_lens, int num_seqs, int max_seq_len,
                               float *out, const void *workspace, cudaStream_t stream) {
    (void)d;
    const float *o_part = static_cast<const float *>(workspace);
    const float2 *ml =
        reinterpret_cast<const float2 *>(static_cast<const uint8_t *>(workspace) + plan.ws_part);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(num_q_heads, num_seqs);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int n_split = plan.n_split, chunk = plan.chunk;
    return cudaLaunchKernelEx(&cfg, decode_merge_kernel, o_part, ml, seq_lens, out, num_q_heads,
                              n_split, chunk, max_seq_len) == cudaSuccess
               ? KVQ_OK
               : KVQ_ERR_CUDA;
}

}  // namespace kvq
