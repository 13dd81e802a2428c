/*
 * gqa_attn.h -- C ABI of libgqa_attn.so: fused multi-head attention forward
 * with grouped-query attention (GQA) and split-KV single-token decode, written
 * for NVIDIA B200 (sm_100a).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are caller-owned DEVICE buffers (allocated by the caller, e.g.
 *    with PyTorch), dense and row-major (C order).  Q, K, V and O hold bf16
 *    values (raw 16-bit storage); LSE holds float32; lengths hold int32.
 *    Every tensor base address must be 16-byte aligned.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Calls are asynchronous: they validate their arguments on the
 *    host, enqueue kernels on `stream` and return.  The library never
 *    synchronises a stream except in attn_last_device_status().
 *  - Errors detectable on the host are returned before anything is enqueued:
 *    ATTN_ERR_NULL for a NULL required pointer, ATTN_ERR_INVALID for
 *    inconsistent sizes or flags, ATTN_ERR_UNSUPPORTED for a head size the
 *    library was not built for, ATTN_ERR_CUDA when a CUDA call fails.
 *  - Errors found on the device (a bounded wait that ran out, a length
 *    outside the tensor) are recorded in a per-device status word and read
 *    back with attn_last_device_status().  Kernels never trap.
 *  - Query head h reads key/value head h / (Hq / Hkv): consecutive groups of
 *    Hq / Hkv query heads share one K/V head (GQA; Heads must be a multiple of
 *    Heads_KV -- Tylo.jl "Primitives" page, entry `flex_attention!`).
 */
#ifndef GQA_ATTN_H
#define GQA_ATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_NULL = 1,          /* a required pointer is NULL */
    ATTN_ERR_INVALID = 2,       /* sizes / flags inconsistent, misaligned pointer */
    ATTN_ERR_UNSUPPORTED = 3,   /* head size D not built (built: 64, 128) */
    ATTN_ERR_CUDA = 4,          /* a CUDA runtime / driver call failed */
    ATTN_ERR_TIMEOUT = 5,       /* device: a bounded wait ran out, kernel gave up */
    ATTN_ERR_DEVICE_BOUNDS = 6, /* device: a length exceeded the tensor, clamped */
    ATTN_ERR_SCRATCH_LIMIT = 7  /* attn_decode_noalloc: workspace above its fixed array */
} attn_status_t;

/*
 * attn_fwd -- fused attention forward, O = softmax(Q K^T * scale + mask) V.
 *
 * Defined by: Tylo.jl "Primitives" page, entry `attention!` (fused MHA with
 * GQA; keywords causal, input_pos = absolute position of the first query,
 * k_lengths / q_lengths = optional per-batch valid lengths; the softmax
 * statistics M/L are saved for the backward; Float32 accumulation), the
 * causal rule of entry `CausalMask` (a query sees keys at or before its own
 * absolute position), and the sliding window of the mlx-arsenal "Attention"
 * page, entry `sliding_window_mask` (at most window_size keys, the query's
 * own position included).
 *
 *   O     [out] bf16 (B, Hq, Sq, D)
 *   Q     [in]  bf16 (B, Hq, Sq, D)
 *   K, V  [in]  bf16 (B, Hkv, Sk, D)
 *   LSE   [out] float32 (B, Hq, Sq) or NULL (statistics not saved).
 *         LSE = M + ln L in natural-log units of the scaled scores, where
 *         M = max_j s_j and L = sum_j exp(s_j - M) over the visible keys.
 *   scale       multiplies Q K^T (the pages' default is 1/sqrt(D)).
 *   causal      0 or 1.  Key j is visible from query row i only if
 *               j <= input_pos + i.
 *   window      0 = no window; w > 0 (requires causal) keeps only keys with
 *               input_pos + i - w < j <= input_pos + i.
 *   input_pos   >= 0, absolute position of query row 0.
 *   k_lengths   int32 (B,) device array or NULL (= Sk): keys j >= k_lengths[b]
 *               are invisible.  Values above Sk are clamped to Sk and flagged
 *               ATTN_ERR_DEVICE_BOUNDS; negative values count as 0.
 *   Sizes: B, Sq, Sk >= 0; Hq, Hkv >= 1, Hq % Hkv == 0; D in {64, 128}.
 *
 * A query row that sees no key (k_length 0, or every key cut by the masks)
 * gets O = 0 and LSE = -inf.  Key/value rows at positions >= k_lengths[b]
 * contribute exactly zero, whatever they hold.
 */
attn_status_t attn_fwd(void *O, const void *Q, const void *K, const void *V, float *LSE,
                       int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale,
                       int causal, int window, int input_pos,
                       const int32_t *k_lengths, void *stream);

/*
 * attn_fwd_varlen -- attn_fwd plus per-batch valid query lengths.
 *
 * Same definition and arguments as attn_fwd, with q_lengths an int32 (B,)
 * device array or NULL (= Sq): query rows i >= q_lengths[b] are invalid and
 * get O = +0.0 (every bit zero) and LSE = -inf, whatever those rows of Q hold,
 * NaN and Inf included (Tylo.jl "Primitives" page, entry `attention!`, keyword
 * q_lengths).  attn_fwd(...) is attn_fwd_varlen(..., q_lengths=NULL).
 */
attn_status_t attn_fwd_varlen(void *O, const void *Q, const void *K, const void *V, float *LSE,
                              int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale,
                              int causal, int window, int input_pos,
                              const int32_t *k_lengths, const int32_t *q_lengths,
                              void *stream);

/*
 * attn_fwd_flex -- flex_attention! forward with one score mod and a document
 * mask (Tylo.jl "Primitives" page, entries `flex_attention!`,
 * `SoftCapScore`, `AliBiScore`, `DocumentMask`, `BlockMask`).
 *
 * Same tensors, masks and lengths as attn_fwd_varlen; on top of them, with
 * s = scale * <q_i, k_j> the scaled score of query row i and key j:
 *   softcap       > 0: s -> softcap * tanh(s / softcap)        (SoftCapScore)
 *   alibi_slopes  float32 (Hq,) device array or NULL:
 *                 s -> s + alibi_slopes[h] * ((input_pos + i) - j)  (AliBiScore)
 *                 At most one of softcap > 0 and alibi_slopes is given.
 *   doc_q, doc_kv int32 device arrays, (Sq,) ids of the query rows and (Sk,)
 *                 ids of the keys, both NULL or both given: the pair attends
 *                 only if the ids match (DocumentMask; shared by every batch
 *                 entry and head).
 *   block_mask    uint8 device array (ceil(Sq/64), ceil(Sk/64)) or NULL, one
 *                 state per 64x64 block of (query row, key): 0 = no pair of
 *                 the block attends (skipped), 2 = every pair attends (document
 *                 ids not checked), anything else = check each pair.  Build it
 *                 with attn_block_mask_document or attn_block_mask_build (the
 *                 page's build_block_mask); it must agree with the other masks.
 *   block_mask_per_head  0: one block_mask for every batch entry and head;
 *                 1: block_mask is (B, Hq, ceil(Sq/64), ceil(Sk/64)), one matrix
 *                 per (batch, query head) -- block-sparse prefill with the
 *                 masks of attn_rbs_block_mask.
 * A call with a block_mask and nothing else to apply (causal 0, no lengths, no
 * document ids, no score mod, Sk <= 65536) runs the block-sparse kernel, which
 * steps over the kept 64-key blocks of each 128-row query tile; it computes the
 * same function.
 * Limits: Sk <= 131072.  Errors as attn_fwd, plus ATTN_ERR_INVALID for a
 * negative or non-finite softcap, softcap together with ALiBi, or only one of
 * doc_q / doc_kv, and ATTN_ERR_UNSUPPORTED for a longer Sk.
 */
attn_status_t attn_fwd_flex(void *O, const void *Q, const void *K, const void *V, float *LSE,
                            int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale,
                            int causal, int window, int input_pos,
                            const int32_t *k_lengths, const int32_t *q_lengths,
                            float softcap, const float *alibi_slopes,
                            const int32_t *doc_q, const int32_t *doc_kv,
                            const uint8_t *block_mask, int block_mask_per_head, void *stream);

/*
 * attn_bwd -- backward of attn_fwd_varlen (Tylo.jl "Primitives" page, entry
 * `∇attention!`: from the output gradient, the inputs, the output and the
 * forward's saved softmax statistics, write the input gradients; overwrite).
 *
 *   dQ  [out] bf16 (B, Hq, Sq, D);  dK, dV [out] bf16 (B, Hkv, Sk, D)
 *   dO  [in]  bf16 (B, Hq, Sq, D), the output gradient
 *   Q, K, V, O [in] the forward's inputs and output
 *   LSE [in]  float32 (B, Hq, Sq) saved by the forward (LSE = M + ln L)
 *   scale, causal, window, input_pos, k_lengths, q_lengths: as in the forward
 *   (they must match it).
 * With P = exp(scale Q K^T - LSE) on the visible pairs: dV = P^T dO,
 * dS = P (dO V^T - rowsum(dO O)), dQ = scale dS K, dK = scale dS^T Q; dK / dV
 * of a KV head sum over the query heads it serves; keys never visible and
 * query rows past q_lengths get zero gradients (rows of dQ past q_lengths and
 * of dK, dV past k_lengths are +0.0).  Padding rows (Q, dO, O past q_lengths;
 * K, V past k_lengths) must hold finite values: they enter the tensor-core
 * products with weight zero, and zero times NaN or Inf is NaN.  Allocates a
 * stream-ordered workspace of B * Hq * Sq floats.  The dQ kernel runs on a
 * library-owned stream forked from `stream` and joined back to it with events,
 * so the call stays ordered on `stream` (and can be captured in a CUDA graph).
 * Errors as attn_fwd.
 */
attn_status_t attn_bwd(void *dQ, void *dK, void *dV, const void *dO, const void *Q, const void *K,
                       const void *V, const void *O, const float *LSE, int B, int Hq, int Hkv,
                       int Sq, int Sk, int D, float scale, int causal, int window, int input_pos,
                       const int32_t *k_lengths, const int32_t *q_lengths, void *stream);

/*
 * attn_rbs_block_mask -- block scores and block mask of block-sparse prefill
 * (mlx-arsenal "Radius-bounded block scores (RBS)" page: the block estimator of
 * "The idea", radius_bounded_block_scores and relative_block_mask of "What
 * mlx-arsenal ships", and the union of the recipe), 64-token blocks.
 *
 *   block_mask  [out] uint8 (B, Hq, ceil(Sq/64), ceil(Sk/64)) device array:
 *               2 = keep the block, 0 = skip it; pass it to attn_fwd_flex with
 *               block_mask_per_head = 1.
 *   base_scores, rescue_scores [out] float32, same shape, or NULL: the log
 *               block scores log sum_t exp(l_t) over the query block's tokens,
 *               l_base = <q, c> / sqrt(D), l_rescue = (<q, c> + |q| r beta) /
 *               sqrt(D), c / r the key block's centroid / radius, beta =
 *               clip((r - r_low) / (r_high - r_low), 0, 1) with r_low / r_high
 *               the median / 90th percentile of the KV head's block radii.
 *   Q (B, Hq, Sq, D), K (B, Hkv, Sk, D) bf16 device arrays (GQA: query head h
 *               scores the blocks of KV head h / (Hq / Hkv)).
 *   A block is kept when base >= row max + ln alpha_base, or rescue >= row max
 *   + ln alpha_rescue, or |qb - kb| < diagonal (the page uses 0.22, 0.18, 1).
 * Limits: Sk <= 131072, D in {64, 128}.  Allocates a stream-ordered workspace
 * of B * Hkv * ceil(Sk/64) * (D + 2) floats.
 */
attn_status_t attn_rbs_block_mask(uint8_t *block_mask, float *base_scores, float *rescue_scores,
                                  const void *Q, const void *K, int B, int Hq, int Hkv, int Sq,
                                  int Sk, int D, float alpha_base, float alpha_rescue,
                                  int diagonal, void *stream);

/*
 * attn_block_mask_build -- the page's build_block_mask (Tylo.jl "Primitives"
 * page, entry `build_block_mask`, TILE_M = TILE_N = 64) on the host.
 *
 *   out   [out] host uint8 (ceil(Sq/64), ceil(Sk/64)), caller-owned.  Block
 *         (qb, kb) gets 0 if keep is false for every (query row, key) pair of
 *         the block, 2 if it is true for every pair, 1 otherwise (pairs past
 *         Sq or Sk are not part of a block).
 *   keep  predicate on (q, kv): q = input_pos + i is the absolute position of
 *         query row i, kv the key position; nonzero = attend.
 * Returns ATTN_ERR_NULL / ATTN_ERR_INVALID on bad arguments.
 */
attn_status_t attn_block_mask_build(uint8_t *out, int Sq, int Sk, int input_pos,
                                    int (*keep)(int q, int kv, void *ctx), void *ctx);

/*
 * attn_block_mask_document -- attn_block_mask_build for the predicate
 * "doc_q[i] == doc_kv[kv], and the causal / window rule of attn_fwd holds"
 * (DocumentMask combined with CausalMask / the sliding window), with host
 * arrays doc_q (Sq,) and doc_kv (Sk,).
 */
attn_status_t attn_block_mask_document(uint8_t *out, int Sq, int Sk, int input_pos, int causal,
                                       int window, const int32_t *doc_q, const int32_t *doc_kv);

/*
 * attn_decode -- split-KV (Flash-Decoding) attention of one new query token per
 * head and sequence against a KV cache.
 *
 * Defined by: Tylo.jl "Primitives" page, entry `decode_attention!` (one query
 * vector per head and sequence, the KV cache processed in n_splits parallel
 * slices, lengths = valid KV length per sequence); scale is the page's default
 * qk_scale = 1/sqrt(D) (entry `flex_attention!`).  Slice s of sequence b
 * covers keys [s*C, min((s+1)*C, lengths[b])) with C = 64 * ceil(ceil(
 * lengths[b]/64) / n_splits); each slice yields a partial output and its
 * log-sum-exp, and a second kernel merges the slices by their log-sum-exp.
 *
 *   O        [out] bf16 (B, Hq, D)
 *   Q        [in]  bf16 (B, Hq, D)
 *   K, V     [in]  bf16 caches (B, Hkv, S_cap, D)
 *   lengths  [in]  int32 (B,) device array, required.  Values above S_cap are
 *                  clamped and flagged ATTN_ERR_DEVICE_BOUNDS; values <= 0
 *                  give O = 0 for that sequence.
 *   n_splits 1..64.
 *   Sizes: B >= 0; Hq, Hkv >= 1, Hq % Hkv == 0, Hq / Hkv <= 16;
 *          S_cap >= 0; D in {64, 128}.
 *
 * The per-slice partial results live in a workspace of
 * B * Hq * n_splits * (D + 4) floats that the call allocates and frees in
 * stream order on `stream`, from a memory pool the library keeps per device
 * (memory freed to it stays reserved for later calls).
 */
attn_status_t attn_decode(void *O, const void *Q, const void *K, const void *V,
                          const int32_t *lengths, int n_splits, void *stream,
                          int B, int Hq, int Hkv, int S_cap, int D);

/*
 * attn_decode_paged -- attn_decode over a paged KV cache (vllm-mlx
 * "attention" page: MLXAttentionBackend.get_kv_cache_shape gives the cache
 * shape (num_blocks, block_size, num_kv_heads, head_size); MLXAttentionMetadata
 * carries seq_lens and block_tables).
 *
 *   O       [out] bf16 (B, Hq, D)
 *   Q       [in]  bf16 (B, Hq, D), one new token per sequence
 *   K_cache, V_cache [in] bf16 (num_blocks, block_size, Hkv, D)
 *   block_tables [in] int32 (B, max_blocks_per_seq) device array: key j of
 *           sequence b is row j % block_size of block block_tables[b][j /
 *           block_size].  Entries past a sequence's last block are not read.
 *   seq_lens [in] int32 (B,) device array: keys 0 .. seq_lens[b]-1 attend.
 *           Values above max_blocks_per_seq * block_size are clamped and
 *           flagged ATTN_ERR_DEVICE_BOUNDS, as is a block index outside
 *           0 .. num_blocks-1 (that block then reads as zeros).
 *   n_splits, scale (1/sqrt(D)), GQA rule, workspace and errors as attn_decode.
 *   block_size: a power of two >= 8.
 */
attn_status_t attn_decode_paged(void *O, const void *Q, const void *K_cache, const void *V_cache,
                                const int32_t *block_tables, const int32_t *seq_lens, int n_splits,
                                void *stream, int B, int Hq, int Hkv, int num_blocks,
                                int block_size, int max_blocks_per_seq, int D);

/*
 * attn_decode_noalloc -- attn_decode for callers that cannot allocate device
 * memory.  The pages have no counterpart: it is attn_decode with a different
 * home for the per-slice workspace.
 *
 * Who needs it: attn_decode allocates and frees its workspace (stream
 * ordered, from the library's pool) on every call.  A serving loop that reserves all of its device memory up front and
 * forbids allocation afterwards (an allocation can fail once the memory is
 * spoken for, and its latency is not bounded), or a program whose device
 * memory belongs to another allocator, cannot let the library allocate.  This
 * entry point allocates nothing: it runs the same kernels with the workspace
 * in a fixed 16 MiB device array compiled into the library.
 *
 * Arguments, layouts, results and errors: as attn_decode, plus
 * ATTN_ERR_SCRATCH_LIMIT, returned before anything is enqueued, when the
 * workspace B * Hq * n_splits * (D + 4) * 4 bytes exceeds 16 MiB
 * (16777216 bytes; e.g. B 64, Hq 32, n_splits 8, D 128 needs 8.65 MB).
 *
 * Sharing rules: every GPU that loads the library holds the 16 MiB array until
 * the process exits, and all calls on one device share it.  Calls that can
 * overlap on the GPU (other streams, unordered host threads) race on it; issue
 * them on one stream or otherwise order them.  The array keeps the last call's
 * contents; nothing in it needs to start at zero.  The first call on a device,
 * made while that device is current, looks up the array's device address
 * (cudaGetSymbolAddress); make that first call before any stream capture.
 */
attn_status_t attn_decode_noalloc(void *O, const void *Q, const void *K, const void *V,
                                  const int32_t *lengths, int n_splits, void *stream,
                                  int B, int Hq, int Hkv, int S_cap, int D);

/* Human-readable name of a status code (static storage, never NULL). */
const char *attn_status_string(attn_status_t status);

/*
 * attn_last_device_status -- synchronise `stream`, then return and clear the
 * status word that kernels of this library set on the current device
 * (ATTN_OK if none did).  Returns ATTN_ERR_CUDA if the synchronisation failed.
 */
attn_status_t attn_last_device_status(void *stream);

/*
 * attn_check_bounded_wait -- diagnostic for the library's bounded waits.
 * Launches one block that waits on a barrier nobody completes, with a limit
 * of `limit_us` microseconds (1..2000000), through the same wait routine the
 * attention kernels use.  The kernel gives up, records ATTN_ERR_TIMEOUT in
 * the device status word and returns; read it with attn_last_device_status.
 * No page defines this; it exists to test the failure path without a hang.
 */
attn_status_t attn_check_bounded_wait(int limit_us, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GQA_ATTN_H */
