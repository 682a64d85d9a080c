// kvq_decode.cu -- decode attention entry: the split plan, the choice of the
// split-K variant family, and the log-sum-exp merges (of the splits, and of
// partials from caches that hold other token ranges of the same sequences).
// The split-K kernel itself is kvq_decode_kernel.cuh, a template over GQA, the
// key mode (token-wise groups, KIVI's per-channel blocks, bf16), the value
// mode (token-wise groups, groups along tokens = one scale/zero per channel
// and R-token block, bf16), the code widths, compile-time group sizes and the
// item's bf16 tail (none, the recent window, the attention sinks); each family
// is instantiated in its own unit (kvq_decode_plain/window/innerq/sink.cu).
#include <cmath>

#include "kvq_decode_kernel.cuh"

namespace kvq {

using namespace dec;

namespace {
// One CTA of 32 * NW threads per (query head, sequence): combine the splits
// into the output, or (PARTIAL) into this cache's unnormalized partial
// (o, m, l) for a merge with the partials of other caches that hold other
// token ranges of the same sequences. Launched as a programmatic dependent of
// the split-K pass: its CTAs may start while that pass drains and wait here
// until its partials are complete. NW partials are read per step (one per
// warp, 16 bytes per lane): 4 warps for up to kMergeFewSplits splits, else 16
// (long sequences have few rows and many splits).
constexpr int kMergeFewSplits = 32;

// Split plan: SMs of the B200 whose resident CTAs the items are balanced over,
// items per resident CTA aimed at, and the longest split in tiles.
constexpr int kBalanceSms = 148;
constexpr double kMinItemsPerCta = 1.9, kMaxItemsPerCta = 4.5;
constexpr int kMaxSplitTiles = 8;

template <bool PARTIAL, int NW>
__global__ void __launch_bounds__(32 * NW) decode_merge_kernel(const float *o_part, const float2 *ml,
                                                           const int32_t *seq_lens, float *out,
                                                           float2 *out_ml, int Hq, int max_seq_len,
                                                           const SplitBounds sp) {
    __shared__ CombineSmemW<NW> sm;
    pdl_wait_prior_grid();
    const int hq = blockIdx.x, seq = blockIdx.y;
    const int T = min(__ldg(seq_lens + seq), max_seq_len);
    const int nv = splits_of(sp, T);
    const int n_split = sp.n;
    const int64_t row = static_cast<int64_t>(seq) * Hq + hq;
    float M, l;
    float4 o;
    combine_partials_w<NW>(o_part, ml, row * n_split * kHeadDim, kHeadDim, row * n_split, 1, nv, sm,
                                    M, o, l);
    if (threadIdx.x >= 32) return;
    float4 *dst = reinterpret_cast<float4 *>(out + row * kHeadDim) + threadIdx.x;
    if constexpr (PARTIAL) {
        *dst = o;
        if (threadIdx.x == 0) out_ml[row] = make_float2(M, l);
    } else {
        *dst = (l > 0.0f) ? make_float4(o.x / l, o.y / l, o.z / l, o.w / l) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
}

// One CTA of 128 threads per (query head, sequence): the output from n_part
// partials, part j = `rows` o rows of kHeadDim floats then `rows` (m, l)
// pairs, parts back to back (rows * (kHeadDim + 2) floats each).
__global__ void __launch_bounds__(128) merge_partials_kernel(const float *parts, int n_part, int rows,
                                                             float *out) {
    __shared__ CombineSmem<1> sm;
    const int64_t row = static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x;
    const int64_t part = static_cast<int64_t>(rows) * (kHeadDim + 2);  // floats per part
    const float2 *ml = reinterpret_cast<const float2 *>(parts + static_cast<int64_t>(rows) * kHeadDim);
    float M, o, l;
    combine_partials<1>(parts, ml, row * kHeadDim, part, row, part / 2, n_part, sm, M, o, l);
    out[row * kHeadDim + threadIdx.x] = (l > 0.0f) ? o / l : 0.0f;
}

}  // namespace

bool plan_decode(const kvq_cache_desc &d, int num_seqs, int num_q_heads, int max_seq_len,
                 DecodePlan *plan) {
    if (num_seqs <= 0 || num_q_heads <= 0 || max_seq_len < 0 || d.num_kv_heads <= 0) return false;
    // Every (sequence, KV head) unit is cut into splits of `chunk` tokens (1 to
    // kMaxSplitTiles whole 256-token tiles), the last one partial; the CTAs
    // claim the items split-major, so the partial splits come last. The chunk
    // balances the launch with every sequence at max_seq_len: the full items
    // should fill a whole number of rounds of the resident CTAs (two per SM
    // on the B200's 148 SMs), 1.9..4.5 items per CTA;
    // among the chunks that do, the most even one wins, then the one whose
    // trailing split is the smallest share of a chunk. With more work than
    // that the longest chunk is taken, with less the shortest. Measured on
    // B200 (split-K pass): llama8b-shaped step, 128 units of 8256 tokens:
    // 1024-token chunks 89.1 us, 768 94.4, 1280 95.3, 1536 95.9, 2048 97.9;
    // long_int2, 8 units of 131072: 1792 107.2 us, 1280 116.5, 1024 117.9,
    // 2048 122.6; paged_mix (ragged, split-K + merge): 2048 277.6 us, 3072
    // 282.5, 4096 304.9. The plan depends on the sizes alone, so the workspace
    // query and the launches agree.
    const int64_t units = static_cast<int64_t>(num_seqs) * d.num_kv_heads;
    const int64_t L = std::max(1, max_seq_len);
    const int64_t ctas = 2 * kBalanceSms;
    // at most kMaxDecodeSplits splits
    const int64_t m_floor = (L + static_cast<int64_t>(kMaxDecodeSplits) * kTileQ - 1) /
                            (static_cast<int64_t>(kMaxDecodeSplits) * kTileQ);
    int64_t m_best = -1;
    double best_even = -1.0, best_tail = 2.0;
    bool all_above = true;
    for (int64_t m = std::max<int64_t>(1, m_floor); m <= std::max<int64_t>(m_floor, kMaxSplitTiles); ++m) {
        const int64_t c = m * kTileQ;
        const double k = static_cast<double>(units * (L / c)) / static_cast<double>(ctas);
        if (k <= kMaxItemsPerCta) all_above = false;
        if (k < kMinItemsPerCta || k > kMaxItemsPerCta) continue;
        const double even = k / std::ceil(k);
        const double tail = static_cast<double>(L % c) / static_cast<double>(c);
        if (even > best_even + 1e-9 || (even > best_even - 1e-9 && tail < best_tail - 1e-9)) {
            best_even = even;
            best_tail = tail;
            m_best = m;
        }
    }
    if (m_best < 0) m_best = all_above ? std::max<int64_t>(m_floor, kMaxSplitTiles) : std::max<int64_t>(1, m_floor);
    int64_t chunk = m_best * kTileQ;
    if (d.bits_k == 16) {
        // bf16 caches (one CTA per SM, 66 KB stages): about eight items per SM
        // in 256..4096-token chunks measured best (remat leg's attention over
        // 64 units of 16384 tokens: 1024-token chunks 0.156-0.161 ms, 1792
        // 0.167 ms).
        chunk = (units * L + 8 * kBalanceSms - 1) / (8 * kBalanceSms);
        chunk = std::min<int64_t>(std::max<int64_t>((chunk + kTileQ - 1) / kTileQ * kTileQ, kTileQ), 4096);
        chunk = std::max(chunk, m_floor * kTileQ);
    }
    SplitBounds &sp = plan->splits;
    sp.chunk = static_cast<int>(chunk);
    sp.n = static_cast<int>((L + chunk - 1) / chunk);
    plan->n_split = sp.n;
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
    p.r_shift = 0;
    while (p.R > 0 && (1 << p.r_shift) < p.R) ++p.r_shift;  // R is a power of two (validated)
    p.paged = d.paged;
    p.page_size = d.page_size;
    p.max_pages = d.max_pages_per_seq;
    p.num_pages = d.num_pages;
    p.cap = d.capacity_tokens;
    p.sp = plan.splits;
    p.n_split = plan.n_split;
    p.max_seq_len = max_seq_len;
    p.q_dtype = q_dtype;
    p.q_bytes = (q_dtype == KVQ_FP32) ? 4 : 2;
    const int gqa = num_q_heads / d.num_kv_heads;
    const StageLayout L = stage_layout(d);
    p.stage_bytes = L.bytes;
    p.off_ksz = L.off_ksz;
    p.off_vc = L.off_vc;
    p.off_vsz = L.off_vsz;
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
                               float *out, float *out_ml, const void *workspace, cudaStream_t stream) {
    (void)d;
    const float *o_part = static_cast<const float *>(workspace);
    const float2 *ml =
        reinterpret_cast<const float2 *>(static_cast<const uint8_t *>(workspace) + plan.ws_part);
    const bool few = plan.n_split <= kMergeFewSplits;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(num_q_heads, num_seqs);
    cfg.blockDim = dim3(few ? 128 : 512);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    float2 *oml = reinterpret_cast<float2 *>(out_ml);
    const SplitBounds &sp = plan.splits;
    cudaError_t e;
    if (out_ml)
        e = few ? cudaLaunchKernelEx(&cfg, decode_merge_kernel<true, 4>, o_part, ml, seq_lens, out, oml, num_q_heads,
                                     max_seq_len, sp)
                : cudaLaunchKernelEx(&cfg, decode_merge_kernel<true, 16>, o_part, ml, seq_lens, out, oml,
                                     num_q_heads, max_seq_len, sp);
    else
        e = few ? cudaLaunchKernelEx(&cfg, decode_merge_kernel<false, 4>, o_part, ml, seq_lens, out, oml,
                                     num_q_heads, max_seq_len, sp)
                : cudaLaunchKernelEx(&cfg, decode_merge_kernel<false, 16>, o_part, ml, seq_lens, out, oml,
                                     num_q_heads, max_seq_len, sp);
    return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

kvq_status launch_merge_partials(const float *parts, int n_part, int num_seqs, int num_q_heads, float *out,
                                 cudaStream_t stream) {
    merge_partials_kernel<<<dim3(num_q_heads, num_seqs), 128, 0, stream>>>(parts, n_part, num_seqs * num_q_heads,
                                                                           out);
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // namespace kvq
