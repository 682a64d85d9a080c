// kvq_decode_window.cu -- split-K decode variants for caches with the bf16
// recent-token window and values grouped per token: KIVI's keys per channel
// over R-token blocks (KIVI Abstract), or token-wise keys.
#include "kvq_decode_kernel.cuh"

namespace kvq {
namespace dec {
namespace {

template <int GQA, int KB, int VB>
kvq_status kivi_groups(const kvq_cache_desc &d, const DecodeParams &p, int max_items, cudaStream_t stream) {
    if constexpr (GQA == 4 && KB == 2 && VB == 2) {
        if (d.group_v == 32)  // KIVI-style INT2
            return launch_variant<GQA, K_CHANNEL, V_TOKEN, 2, 2, 0, 32, kTailWindow>(p, max_items, stream);
    }
    if constexpr (GQA == 4 && KB == 4 && VB == 4) {
        if (d.group_v == 128)  // KIVI-style INT4 with 128-channel value groups
            return launch_variant<GQA, K_CHANNEL, V_TOKEN, 4, 4, 0, 128, kTailWindow>(p, max_items, stream);
    }
    return launch_variant<GQA, K_CHANNEL, V_TOKEN, KB, VB, 0, 0, kTailWindow>(p, max_items, stream);
}

template <int GQA>
kvq_status window_gqa(const kvq_cache_desc &d, const DecodeParams &p, int max_items, cudaStream_t stream) {
    if (d.axis_v != KVQ_PER_TOKEN) return KVQ_ERR_UNSUPPORTED;
    if (d.axis_k == KVQ_PER_CHANNEL) {
        if (d.bits_k == 2 && d.bits_v == 2) return kivi_groups<GQA, 2, 2>(d, p, max_items, stream);
        if (d.bits_k == 4 && d.bits_v == 4) return kivi_groups<GQA, 4, 4>(d, p, max_items, stream);
        if (d.bits_k == 2 && d.bits_v == 4) return kivi_groups<GQA, 2, 4>(d, p, max_items, stream);
        if (d.bits_k == 4 && d.bits_v == 2) return kivi_groups<GQA, 4, 2>(d, p, max_items, stream);
        return KVQ_ERR_UNSUPPORTED;
    }
    if (d.bits_k == 4 && d.bits_v == 4) {
        if constexpr (GQA == 4) {  // the plain family's compile-time group sizes
            if (d.group_k == 128 && d.group_v == 128)
                return launch_variant<GQA, K_TOKEN, V_TOKEN, 4, 4, 128, 128, kTailWindow>(p, max_items, stream);
            if (d.group_k == 32 && d.group_v == 32)
                return launch_variant<GQA, K_TOKEN, V_TOKEN, 4, 4, 32, 32, kTailWindow>(p, max_items, stream);
        }
        return launch_variant<GQA, K_TOKEN, V_TOKEN, 4, 4, 0, 0, kTailWindow>(p, max_items, stream);
    }
    if (d.bits_k == 2 && d.bits_v == 2)
        return launch_variant<GQA, K_TOKEN, V_TOKEN, 2, 2, 0, 0, kTailWindow>(p, max_items, stream);
    if (d.bits_k == 4 && d.bits_v == 2)
        return launch_variant<GQA, K_TOKEN, V_TOKEN, 4, 2, 0, 0, kTailWindow>(p, max_items, stream);
    if (d.bits_k == 2 && d.bits_v == 4)
        return launch_variant<GQA, K_TOKEN, V_TOKEN, 2, 4, 0, 0, kTailWindow>(p, max_items, stream);
    return KVQ_ERR_UNSUPPORTED;
}

}  // namespace

kvq_status dispatch_window(const kvq_cache_desc &d, const DecodeParams &p, int gqa, int max_items,
                           cudaStream_t stream) {
    switch (gqa) {
        case 1: return window_gqa<1>(d, p, max_items, stream);
        case 2: return window_gqa<2>(d, p, max_items, stream);
        case 4: return window_gqa<4>(d, p, max_items, stream);
        default: return KVQ_ERR_UNSUPPORTED;
    }
}

}  // namespace dec
}  // namespace kvq
