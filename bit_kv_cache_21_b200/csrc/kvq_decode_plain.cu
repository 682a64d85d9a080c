// kvq_decode_plain.cu -- split-K decode variants without a bf16 tail:
// token-wise key and value groups (contiguous or paged), and bf16 caches.
#include "kvq_decode_kernel.cuh"

namespace kvq {
namespace dec {
namespace {

// Compile-time group sizes for the common shapes, runtime ones otherwise.
template <int GQA, int KB, int VB>
kvq_status plain_groups(const kvq_cache_desc &d, const DecodeParams &p, int max_items, cudaStream_t stream) {
    if constexpr (GQA == 4 && KB == 4 && VB == 4) {
        if (d.group_k == 128 && d.group_v == 128)  // llama-shaped INT4 caches
            return launch_variant<GQA, K_TOKEN, V_TOKEN, 4, 4, 128, 128>(p, max_items, stream);
        if (d.group_k == 32 && d.group_v == 32)
            return launch_variant<GQA, K_TOKEN, V_TOKEN, 4, 4, 32, 32>(p, max_items, stream);
    }
    return launch_variant<GQA, K_TOKEN, V_TOKEN, KB, VB, 0, 0>(p, max_items, stream);
}

template <int GQA>
kvq_status plain_gqa(const kvq_cache_desc &d, const DecodeParams &p, int max_items, cudaStream_t stream) {
    if (d.bits_k == 16 && d.bits_v == 16)
        return launch_variant<GQA, K_BF16, V_BF16, 16, 16, 0, 0>(p, max_items, stream);
    if (d.axis_k != KVQ_PER_TOKEN || d.axis_v != KVQ_PER_TOKEN) return KVQ_ERR_UNSUPPORTED;
    if (d.bits_k == 4 && d.bits_v == 4) return plain_groups<GQA, 4, 4>(d, p, max_items, stream);
    if (d.bits_k == 2 && d.bits_v == 2) return plain_groups<GQA, 2, 2>(d, p, max_items, stream);
    if (d.bits_k == 4 && d.bits_v == 2) return plain_groups<GQA, 4, 2>(d, p, max_items, stream);
    if (d.bits_k == 2 && d.bits_v == 4) return plain_groups<GQA, 2, 4>(d, p, max_items, stream);
    return KVQ_ERR_UNSUPPORTED;
}

}  // namespace

kvq_status dispatch_plain(const kvq_cache_desc &d, const DecodeParams &p, int gqa, int max_items,
                          cudaStream_t stream) {
    switch (gqa) {
        case 1: return plain_gqa<1>(d, p, max_items, stream);
        case 2: return plain_gqa<2>(d, p, max_items, stream);
        case 4: return plain_gqa<4>(d, p, max_items, stream);
        default: return KVQ_ERR_UNSUPPORTED;
    }
}

}  // namespace dec
}  // namespace kvq
