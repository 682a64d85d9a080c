// kvq_decode_sink.cu -- split-K decode variants for token-wise caches with the
// attention-sink window: a sequence's first sink_len tokens kept in bf16 and
// scored with the unrotated query (InnerQ, Abstract: high-precision windows
// for recent and attention-sink tokens).
#include "kvq_decode_kernel.cuh"

namespace kvq {
namespace dec {
namespace {

template <int GQA, int KB, int VB>
kvq_status sink_groups(const kvq_cache_desc &d, const DecodeParams &p, int max_items, cudaStream_t stream) {
    if constexpr (GQA == 4 && KB == 4 && VB == 4) {
        if (d.group_k == 128 && d.group_v == 128)  // llama-shaped INT4 caches
            return launch_variant<GQA, K_TOKEN, V_TOKEN, 4, 4, 128, 128, kTailSink>(p, max_items, stream);
    }
    return launch_variant<GQA, K_TOKEN, V_TOKEN, KB, VB, 0, 0, kTailSink>(p, max_items, stream);
}

template <int GQA>
kvq_status sink_gqa(const kvq_cache_desc &d, const DecodeParams &p, int max_items, cudaStream_t stream) {
    if (d.axis_k != KVQ_PER_TOKEN || d.axis_v != KVQ_PER_TOKEN) return KVQ_ERR_UNSUPPORTED;
    if (d.bits_k == 4 && d.bits_v == 4) return sink_groups<GQA, 4, 4>(d, p, max_items, stream);
    if (d.bits_k == 2 && d.bits_v == 2) return sink_groups<GQA, 2, 2>(d, p, max_items, stream);
    if (d.bits_k == 4 && d.bits_v == 2) return sink_groups<GQA, 4, 2>(d, p, max_items, stream);
    if (d.bits_k == 2 && d.bits_v == 4) return sink_groups<GQA, 2, 4>(d, p, max_items, stream);
    return KVQ_ERR_UNSUPPORTED;
}

}  // namespace

kvq_status dispatch_sink(const kvq_cache_desc &d, const DecodeParams &p, int gqa, int max_items,
                         cudaStream_t stream) {
    switch (gqa) {
        case 1: return sink_gqa<1>(d, p, max_items, stream);
        case 2: return sink_gqa<2>(d, p, max_items, stream);
        case 4: return sink_gqa<4>(d, p, max_items, stream);
        default: return KVQ_ERR_UNSUPPORTED;
    }
}

}  // namespace dec
}  // namespace kvq
