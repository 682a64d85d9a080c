/*
 * kvq.h -- C ABI of the B200 (sm_100a) low-bit KV-cache library.
 *
 * Three operations, after the problem the method pages state:
 *   kvq_quantize_append   rotate (block-diagonal Hadamard), quantize (INT4 /
 *                         INT2 asymmetric groups, fp16 scale and zero) and pack
 *                         new K/V vectors into a contiguous or paged cache.
 *                         "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization
 *                         for Real-World LLM Serving", Abstract (token-wise
 *                         INT4 with block-diagonal Hadamard rotation in a fused
 *                         rotation-quantization kernel over paged layouts);
 *                         "InnerQ: Hardware-Aware Tuning-Free Quantization of
 *                         KV Cache for Large Language Models", Abstract (groups
 *                         along the inner dimension; a high-precision window of
 *                         recent tokens); KIVI, in the references of both pages
 *                         (keys per channel over token blocks, values per token).
 *   kvq_decode_attention  split-K grouped-query decode attention that reads the
 *                         packed cache directly; queries take the keys'
 *                         rotation. SAW-INT4 Abstract (fused attention
 *                         execution); "Dual-QK: Sharp Queries and Flat Keys for
 *                         Prunable 2-bit KV Caches", Abstract (the same
 *                         orthogonal transform on queries preserves q.k).
 *   kvq_remat_kv          rebuild K and V from a cache of quantized layer inputs
 *                         X with a tensor-core GEMM, RoPE on K. "XQuant:
 *                         Breaking the Memory Wall for LLM Inference with KV
 *                         Cache Rematerialization", Abstract.
 * and their compositions: kvq_remat_attention (the remat GEMM with decode
 * attention in its epilogue, K and V never stored), kvq_decode_merge_partial
 * and kvq_merge_partials (decode over token ranges held by several caches,
 * e.g. one per GPU).
 *
 * Conventions for every call:
 *   - The caller owns all memory. Pointers named d_* or documented "device" are
 *     device pointers; the library allocates nothing (decode attention takes a
 *     caller-provided workspace, see kvq_decode_workspace_size).
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*, NULL
 *     = the legacy default stream) and never synchronize.
 *   - Errors the host can see (bad sizes, NULL or misaligned pointers,
 *     unsupported combinations) return a non-zero kvq_status and launch
 *     nothing. A failed launch returns KVQ_ERR_CUDA.
 *   - Errors only the device can see (a token position outside the cache, a
 *     sequence longer than max_seq_len, a bounded wait that gave up) are OR-ed
 *     as KVQ_DEV_* bits into *desc->status when desc->status is non-NULL; the
 *     caller reads it after synchronizing. No kernel traps or asserts; a
 *     kernel that meets such an error skips the offending access.
 *   - All device pointers must be 16-byte aligned.
 *   - head_dim must be 128.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols (the library is built with hidden default visibility). */
#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

typedef enum {
    KVQ_OK = 0,
    KVQ_ERR_INVALID_ARG = 1, /* NULL, misaligned or out-of-range argument */
    KVQ_ERR_UNSUPPORTED = 2, /* valid but not implemented combination */
    KVQ_ERR_CAPACITY = 3,    /* workspace or static buffer too small */
    KVQ_ERR_TIMEOUT = 4,     /* reserved for host-side waits (none today) */
    KVQ_ERR_CUDA = 5         /* a CUDA runtime call or launch failed */
} kvq_status;

/* Bits OR-ed into *desc->status by kernels. */
#define KVQ_DEV_CAPACITY 0x1 /* a token position fell outside the cache */
#define KVQ_DEV_TIMEOUT 0x2  /* a bounded wait gave up (about 1 s) */
#define KVQ_DEV_SEQLEN 0x4   /* a sequence longer than max_seq_len */

typedef enum { KVQ_BF16 = 0, KVQ_FP16 = 1, KVQ_FP32 = 2 } kvq_dtype;

/* Quantization axis of a tensor's groups. */
typedef enum {
    KVQ_PER_TOKEN = 0,  /* G consecutive head_dim channels of one token */
    KVQ_PER_CHANNEL = 1 /* one channel over an aligned block of G tokens */
} kvq_axis;

/*
 * Cache descriptor. Layouts (S = num_seqs, H = num_kv_heads, D = head_dim,
 * Tc = capacity_tokens, P = num_pages, ps = page_size, row = D*bits/8 bytes;
 * half2 = {fp16 scale, fp16 zero}, scale in the low half):
 *
 *   bits 2 or 4, per-token groups (axis KVQ_PER_TOKEN), group G in {16,32,64,128}:
 *     contiguous  codes u8 [S][H][Tc][row]     sz half2 [S][H][Tc][D/G]
 *     paged       codes u8 [P][H][ps][row]     sz half2 [P][H][ps][D/G]
 *                 token t of sequence s lives in page block_table[s*max_pages_per_seq
 *                 + t/ps], slot t%ps.
 *   bits 2 or 4, per-channel key groups (axis_k KVQ_PER_CHANNEL, contiguous only,
 *   requires residual_len == group_k, a multiple of 64):
 *     codes u8 [S][H][Tc][row] (packed along channels)  sz half2 [S][H][Tc/G][D]
 *   bits 2 or 4, per-channel value groups (axis_v KVQ_PER_CHANNEL): the same
 *   layout for V, with residual_len == group_v and bits_v == bits_k. InnerQ
 *   ("InnerQ: Hardware-Aware Tuning-Free Quantization of KV Cache for Large
 *   Language Models", Abstract) groups each cache matrix along the inner
 *   dimension of its product with the attention vector: channels for q.K^T,
 *   tokens for p.V, so V's groups are one channel over an R-token block.
 *   bits 16 (unquantized bf16, contiguous only):
 *     codes bf16 [S][H][Tc][D]; sz unused (may be NULL).
 *   Packing: INT4 element 2i in the low nibble of byte i, 2i+1 in the high
 *   nibble; INT2 element 4i+j in bits 2j..2j+1 of byte i.
 *
 *   residual_len R > 0 keeps the most recent tokens in bf16 windows
 *     k_res, v_res bf16 [S][H][R][D]. A sequence of length T holds its first
 *     Tq = R*floor((T-1)/R) tokens quantized and tokens [Tq, T) in window slots
 *     0..T-Tq-1 (a full window is flushed as one block only when a further token
 *     arrives). Requires contiguous layout, bf16 appends, no rotation.
 *
 * hadamard_block_k: 0 = no rotation, else a power of two in [2, D]: each
 * block of that many consecutive channels of a key is multiplied by the
 * normalized Sylvester Hadamard matrix before quantization (fp32 butterflies
 * with half-widths 1, 2, 4, ... in that order, then one multiply by
 * fp32(1/sqrt(block))). Decode attention rotates queries by the same block.
 * Values are never rotated.
 */
typedef struct {
    int32_t num_seqs;          /* S: sequences the contiguous cache holds */
    int32_t num_kv_heads;      /* H */
    int32_t head_dim;          /* D, must be 128 */
    int32_t bits_k, bits_v;    /* 2, 4 or 16 */
    int32_t group_k, group_v;  /* group sizes (ignored for bits 16) */
    int32_t axis_k, axis_v;    /* kvq_axis of the key and value groups */
    int32_t hadamard_block_k;  /* 0 or power of two <= D */
    int32_t residual_len;      /* 0 or R (bf16 window length) */
    int32_t paged;             /* 0 contiguous, 1 paged */
    int32_t page_size;         /* tokens per page, power of two >= 16 */
    int32_t max_pages_per_seq; /* row stride of block_table */
    int32_t num_pages;         /* pages in the pool */
    int32_t capacity_tokens;   /* Tc (contiguous), multiple of 64 */
    int32_t reserved;          /* must be 0 */
    void *k_codes, *v_codes;   /* device */
    void *k_sz, *v_sz;         /* device, half2 */
    void *k_res, *v_res;       /* device, bf16 windows (residual_len > 0) */
    const int32_t *block_table;/* device [S][max_pages_per_seq] (paged) */
    int32_t *status;           /* device status word, may be NULL */
    const float *hadamard_signs;/* device [128] entries +1.0f / -1.0f, or NULL.
                                  With hadamard_block_k > 0 the keys (and the
                                  queries) take x -> H_blk diag(signs) x / sqrt(blk):
                                  the randomized Hadamard of "QuaRot: Outlier-Free
                                  4-Bit Inference in Rotated LLMs" (listed among the
                                  works the pages build on). Multiplying by +-1 is
                                  exact, and (H D)^T (H D) = blk I, so q.k is kept.
                                  Other values give a transform that is not
                                  orthogonal. Requires hadamard_block_k > 0. */
    void *k_sink, *v_sink;     /* device bf16 [num_seqs][H][sink_len][D], or NULL:
                                  the attention-sink window of "InnerQ: Hardware-Aware
                                  Tuning-Free Quantization of KV Cache for Large
                                  Language Models", Abstract (high-precision windows
                                  for recent tokens and attention sink tokens). */
    int32_t sink_len;          /* 0, or 1..64: a sequence's first sink_len tokens
                                  are kept in k_sink / v_sink as bf16 (the input
                                  rounded to nearest even) instead of being
                                  quantized, and attention reads them with the
                                  unrotated query. Token-wise keys and values
                                  without the recent window (residual_len == 0),
                                  contiguous or paged; their quantized rows stay
                                  unused. */
    int32_t hybrid;            /* 0, or 1: every quantized group of K and V takes
                                  the symmetric or the asymmetric grid, whichever
                                  reconstructs it with the smaller squared error
                                  (InnerQ, Abstract, "(i) hybrid quantization ...
                                  based on local statistics"; the page states no
                                  criterion, this is the library's). Symmetric:
                                  Qp = 2^(bits-1) - 1, C = 2^(bits-1),
                                  s = fp16_ru(max|x| / Qp), z = -C s, q =
                                  clamp(rint(x / s), -Qp, Qp) + C, so zero is a level.
                                  Error: fp32 e = x - fma(q, s, z), squares summed
                                  with fma over runs of 32 elements in order, runs
                                  added pairwise; ties keep the asymmetric grid.
                                  Readers of the cache see (s, z) pairs as always. */
} kvq_cache_desc;

/*
 * kvq_quantize_append -- append new tokens to every sequence of a batch.
 *
 * k_new, v_new: device [total_new_tokens][H][D] of `dtype`, the new tokens of
 *   sequence 0 first, then sequence 1, ... (ragged). v_new may be NULL when
 *   desc->v_codes is NULL (a K-only cache such as quantized layer inputs X).
 * cu_new: device int32 [num_seqs + 1], prefix sums of new tokens per sequence
 *   (cu_new[0] = 0, cu_new[num_seqs] = total_new_tokens).
 * seq_lens: device int32 [num_seqs], current lengths; token i of sequence s
 *   is written at position seq_lens[s] + i, and seq_lens[s] is advanced by the
 *   sequence's new count when the call's kernels finish (stream order).
 * Each (token, head) key vector is rotated (hadamard_block_k > 0) and both K
 * and V are quantized per the descriptor; with residual_len > 0 tokens pass
 * through the bf16 window and are quantized as whole blocks when it flushes.
 * Positions outside the cache (>= capacity_tokens, or past the sequence's
 * block-table row, or a page id outside [0, num_pages)) are skipped and set
 * KVQ_DEV_CAPACITY. total_new_tokens == 0 is a no-op.
 */
KVQ_API kvq_status kvq_quantize_append(const kvq_cache_desc *desc, const void *k_new,
                               const void *v_new, kvq_dtype dtype,
                               const int32_t *cu_new, int32_t *seq_lens,
                               int32_t num_seqs, int32_t total_new_tokens,
                               void *stream);

/*
 * kvq_decode_workspace_size -- bytes of workspace kvq_decode_attention needs
 * for these sizes (split-K partial outputs and softmax statistics). Returns 0
 * for invalid arguments.
 */
KVQ_API size_t kvq_decode_workspace_size(const kvq_cache_desc *desc, int32_t num_seqs,
                                 int32_t num_q_heads, int32_t max_seq_len);

/*
 * kvq_decode_attention -- one decode step of grouped-query attention over the
 * packed cache: for every sequence s and query head h (KV head
 * h / (num_q_heads / H)),
 *     out[s][h] = sum_t softmax_t(softmax_scale * q~ . k^_t) v^_t
 * over all t < seq_lens[s], where k^, v^ are the dequantized cache entries
 * (q*s+z; bf16 window tokens as stored) and q~ is q rotated like the keys.
 * q: device [num_seqs][num_q_heads][D] of q_dtype. out: device fp32
 * [num_seqs][num_q_heads][D]. A sequence of length 0 gives zeros.
 * max_seq_len bounds every seq_lens[s] (longer sequences set KVQ_DEV_SEQLEN
 * and attend to their first max_seq_len tokens). num_q_heads / H must be 1,
 * 2 or 4. workspace: device, >= kvq_decode_workspace_size(...) bytes, else
 * KVQ_ERR_CAPACITY. Runs kvq_decode_splitk then kvq_decode_merge.
 */
KVQ_API kvq_status kvq_decode_attention(const kvq_cache_desc *desc, const void *q,
                                kvq_dtype q_dtype, int32_t num_q_heads,
                                const int32_t *seq_lens, int32_t num_seqs,
                                int32_t max_seq_len, float softmax_scale,
                                float *out, void *workspace,
                                size_t workspace_bytes, void *stream);

/* First pass of kvq_decode_attention alone: per (sequence, KV head, split)
 * partial outputs and softmax statistics into the workspace. Same arguments
 * minus `out`. */
KVQ_API kvq_status kvq_decode_splitk(const kvq_cache_desc *desc, const void *q,
                             kvq_dtype q_dtype, int32_t num_q_heads,
                             const int32_t *seq_lens, int32_t num_seqs,
                             int32_t max_seq_len, float softmax_scale,
                             void *workspace, size_t workspace_bytes,
                             void *stream);

/* Second pass alone: log-sum-exp merge of the partials that kvq_decode_splitk
 * wrote with the same sizes into fp32 `out`. */
KVQ_API kvq_status kvq_decode_merge(const kvq_cache_desc *desc, int32_t num_q_heads,
                            const int32_t *seq_lens, int32_t num_seqs,
                            int32_t max_seq_len, float *out,
                            const void *workspace, size_t workspace_bytes,
                            void *stream);

/*
 * Token-range sharding of long sequences over several caches (one per GPU):
 * each cache holds a disjoint, contiguous token range of the same sequences
 * (lengths local to the cache), and softmax attention over the union is the
 * log-sum-exp combination of the per-cache partials, the same identity the
 * split-K merge uses inside one cache. A decode step is then kvq_decode_splitk
 * and kvq_decode_merge_partial on every cache, one all-gather of the partials
 * (e.g. NCCL; 130 floats per query head per cache), and kvq_merge_partials.
 *
 * kvq_decode_merge_partial -- as kvq_decode_merge, but writes this cache's
 * unnormalized partial: o_part fp32 [num_seqs][num_q_heads][D] holds
 * sum_t 2^(x_t - m) v^_t and ml fp32 [num_seqs][num_q_heads][2] holds (m, l),
 * with x_t = log2(e) * softmax_scale * q~ . k^_t, l = sum_t 2^(x_t - m) and m
 * a reference score: max_t x_t up to the kernel's lazy rescaling (m may sit
 * below the maximum by at most 8, so every weight stays <= 2^8). Only
 * o / l and l * 2^m carry meaning. A sequence with no tokens here gives
 * (-inf, 0) and zeros. o_part 16-byte and ml 8-byte aligned.
 */
KVQ_API kvq_status kvq_decode_merge_partial(const kvq_cache_desc *desc, int32_t num_q_heads,
                                            const int32_t *seq_lens, int32_t num_seqs,
                                            int32_t max_seq_len, float *o_part, float *ml,
                                            const void *workspace, size_t workspace_bytes,
                                            void *stream);

/*
 * kvq_merge_partials -- out[s][h] = sum_r 2^(m_r - M) o_r / sum_r 2^(m_r - M) l_r
 * over n_part partials (M = max_r m_r; zeros when every l_r is 0). `parts`:
 * device fp32, the n_part partials back to back, each num_seqs * num_q_heads
 * o rows [num_seqs][num_q_heads][D] followed by their (m, l) pairs
 * [num_seqs][num_q_heads][2] -- what an all-gather of one buffer per cache
 * gives when kvq_decode_merge_partial wrote o_part at its start and ml right
 * after the o rows. 16-byte aligned. out: device fp32 [num_seqs][num_q_heads][D].
 * num_seqs and num_q_heads at most 65535.
 */
KVQ_API kvq_status kvq_merge_partials(const float *parts, int32_t n_part, int32_t num_seqs,
                                      int32_t num_q_heads, float *out, void *stream);

/*
 * kvq_decode_attention_static -- kvq_decode_attention without a workspace
 * argument, for callers that cannot allocate device memory: a plain C program
 * or a plugin running inside a runtime that owns every device allocation, or a
 * decode loop that must not call cudaMalloc (it can synchronize the device).
 * The method pages have no counterpart; this is an interface convenience.
 * The workspace is a 16 MiB array in device global memory that the library
 * declares; it is reserved on every GPU that loads the library until the
 * process exits. Sizes whose workspace (kvq_decode_workspace_size) exceeds
 * 16 MiB are rejected with KVQ_ERR_CAPACITY before anything is launched.
 * The first call on a device looks up the array's device address (again
 * whenever another context is current on that device, e.g. after
 * cudaDeviceReset or inside a plugin's own context); make the first call in
 * each context before any stream capture. All calls share the
 * array and it keeps the previous call's contents (what must start at zero is
 * cleared on the stream by each call), so calls whose work overlaps on the GPU
 * -- on different streams or from different host threads -- race on it.
 * Other arguments, results and errors are those of kvq_decode_attention.
 */
KVQ_API kvq_status kvq_decode_attention_static(const kvq_cache_desc *desc, const void *q,
                                               kvq_dtype q_dtype, int32_t num_q_heads,
                                               const int32_t *seq_lens, int32_t num_seqs,
                                               int32_t max_seq_len, float softmax_scale,
                                               float *out, void *stream);

/*
 * kvq_remat_kv -- rematerialize K and V of `batch` sequences for positions
 * [0, ctx_len) from a cache of quantized layer inputs X.
 * x_cache: contiguous per-token cache holding X as hidden/128 "heads" of 128
 *   channels (num_kv_heads = hidden/128, bits_k = 4, group_k = 128, no
 *   rotation; only k_codes and k_sz are read), hidden a multiple of 128.
 * w_kv: device bf16 [2*n_kv_heads*128][hidden], the K projection rows
 *   followed by the V projection rows (a linear layer's weight layout).
 * rope_cos, rope_sin: device fp32 [ctx_len][64], cos/sin of position p times
 *   theta^(-2i/128) (kvq_rope_tables writes them).
 * k_out, v_out: device bf16 [batch][n_kv_heads][ctx_len][128] (the bits-16
 *   cache layout, so kvq_decode_attention can read them directly).
 * Computes x^ = bf16_rn(fp32(q*s + z)), [K V] = x^ W^T with fp32 accumulation
 * on the tensor cores, RoPE (rotate-half pairs i, i+64) on K, bf16 stores.
 * ctx_len must be a multiple of 128 and <= capacity_tokens.
 */
KVQ_API kvq_status kvq_remat_kv(const kvq_cache_desc *x_cache, const void *w_kv,
                        int32_t n_kv_heads, const float *rope_cos,
                        const float *rope_sin, int32_t batch, int32_t ctx_len,
                        void *k_out, void *v_out, void *stream);

/*
 * kvq_remat_attention -- rematerialization fused with decode attention
 * ("XQuant: Breaking the Memory Wall for LLM Inference with KV Cache
 * Rematerialization", Abstract: K and V are recomputed from the cached X
 * instead of being cached). Same arguments and requirements as kvq_remat_kv
 * for the X cache, W and the RoPE tables, and K, V are the same values
 * (fp32 accumulation, RoPE on K, rounded to bf16), but they never leave the
 * chip: each 128-token tile of a head's K and V, held in tensor memory, is
 * scored against the head's GQA query rows at once, and
 *     out[b][h] = sum_t softmax_t(softmax_scale * q[b][h] . k_t) v_t
 * over all t < ctx_len (no rotation; queries as given). q: device
 * [batch][num_q_heads][128] of q_dtype, num_q_heads / n_kv_heads in {1, 2, 4}.
 * out: device fp32 [batch][num_q_heads][128]. workspace: device, at least
 * kvq_remat_attention_workspace_size(batch, num_q_heads, ctx_len) bytes
 * (per 128-token tile and query head a partial of 130 floats), else
 * KVQ_ERR_CAPACITY. ctx_len a multiple of 128; batch <= 65535.
 */
KVQ_API size_t kvq_remat_attention_workspace_size(int32_t batch, int32_t num_q_heads, int32_t ctx_len);
KVQ_API kvq_status kvq_remat_attention(const kvq_cache_desc *x_cache, const void *w_kv,
                                       int32_t n_kv_heads, const float *rope_cos,
                                       const float *rope_sin, int32_t batch, int32_t ctx_len,
                                       const void *q, kvq_dtype q_dtype, int32_t num_q_heads,
                                       float softmax_scale, float *out, void *workspace,
                                       size_t workspace_bytes, void *stream);

/* kvq_rope_tables -- cos and sin tables fp32 [n_pos][head_dim/2]:
 * fp32 of cos/sin(p * theta^(-2i/head_dim)) evaluated in float64 on the
 * device. */
KVQ_API kvq_status kvq_rope_tables(float *rope_cos, float *rope_sin, int32_t n_pos,
                           int32_t head_dim, double theta, void *stream);

/* Human-readable name of a status code (static string). */
KVQ_API const char *kvq_status_string(kvq_status status);

/* Test hooks. KVQ_DEBUG_WAIT_TIMEOUT_NS sets the limit of every bounded
 * device wait launched afterwards (default 1e9 ns; <= 0 restores it).
 * KVQ_DEBUG_SKIP_TILE makes the next decode launches' producer skip staging
 * the tile with that index (-1 = off), so the consumers' bounded wait runs
 * out and sets KVQ_DEV_TIMEOUT. Not thread-safe; for tests only. */
#define KVQ_DEBUG_WAIT_TIMEOUT_NS 1
#define KVQ_DEBUG_SKIP_TILE 2
KVQ_API kvq_status kvq_debug_set(int32_t what, int64_t value);

/* Library version, major*10000 + minor*100 + patch. */
KVQ_API int32_t kvq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
