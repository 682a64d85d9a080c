// kvq_decode_innerq.cu -- split-K decode variants for caches whose values are
// grouped along tokens (one scale/zero per channel and R-token block of the
// recent window): InnerQ's inner-dimension grouping ("InnerQ: Hardware-Aware
// Tuning-Free Quantization of KV Cache for Large Language Models", Abstract),
// with token-wise keys (InnerQ's own layout) or KIVI's per-channel keys.
#include "kvq_decode_kernel.cuh"

namespace kvq {
namespace dec {
namespace {

template <int GQA, int B>
kvq_status innerq_bits(const kvq_cache_desc &d, const DecodeParams &p, int max_items, cudaStream_t stream) {
    if (d.axis_k == KVQ_PER_CHANNEL)
        return launch_variant<GQA, K_CHANNEL, V_CHANNEL, B, B, 0, 0, kTailWindow>(p, max_items, stream);
    if (d.group_k == 128)
        return launch_variant<GQA, K_TOKEN, V_CHANNEL, B, B, 128, 0, kTailWindow>(p, max_items, stream);
    if constexpr (GQA == 4) {
        if (d.group_k == 32)
            return launch_variant<GQA, K_TOKEN, V_CHANNEL, B, B, 32, 0, kTailWindow>(p, max_items, stream);
    }
    return launch_variant<GQA, K_TOKEN, V_CHANNEL, B, B, 0, 0, kTailWindow>(p, max_items, stream);
}

template <int GQA>
kvq_status innerq_gqa(const kvq_cache_desc &d, const DecodeParams &p, int max_items, cudaStream_t stream) {
    if (d.axis_v != KVQ_PER_CHANNEL || d.bits_k != d.bits_v) return KVQ_ERR_UNSUPPORTED;
    if (d.bits_v == 2) return innerq_bits<GQA, 2>(d, p, max_items, stream);
    if (d.bits_v == 4) return innerq_bits<GQA, 4>(d, p, max_items, stream);
    return KVQ_ERR_UNSUPPORTED;
}

}  // namespace

kvq_status dispatch_innerq(const kvq_cache_desc &d, const DecodeParams &p, int gqa, int max_items,
                           cudaStream_t stream) {
    switch (gqa) {
        case 1: return innerq_gqa<1>(d, p, max_items, stream);
        case 2: return innerq_gqa<2>(d, p, max_items, stream);
        case 4: return innerq_gqa<4>(d, p, max_items, stream);
        default: return KVQ_ERR_UNSUPPORTED;
    }
}

}  // namespace dec
}  // namespace kvq
