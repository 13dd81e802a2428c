// internal.h -- declarations shared by the library's translation units.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "gqa_attn.h"

namespace gqa {

// Encode a 3-D bf16 tensor map over a row-major (outer, rows, D) tensor with
// a (64, box_rows, 1) box and 128-byte swizzle; out-of-range rows read as 0.
attn_status_t make_tmap_bf16_3d(CUtensorMap *map, const void *base, uint64_t D, uint64_t rows,
                                uint64_t outer, uint32_t box_rows);

// Encode a 3-D bf16 tensor map over a paged cache viewed as (rows, heads, D)
// row-major, with a (64, 1, box_rows) box and 128-byte swizzle: one box is
// box_rows consecutive cache rows of one head, 64 columns wide.
attn_status_t make_tmap_bf16_paged(CUtensorMap *map, const void *base, uint64_t D, uint64_t heads,
                                   uint64_t rows, uint32_t box_rows);

// The same cache with D = 128 viewed as (rows, heads, 2, 64): one (64, 2, 1, box_rows) box
// copies both 64-column halves of box_rows rows, stored row by row (half 0, half 1).
attn_status_t make_tmap_bf16_paged_wide(CUtensorMap *map, const void *base, uint64_t heads,
                                        uint64_t rows, uint32_t box_rows);

struct FwdArgs {
    void *O;
    const void *Q, *K, *V;
    float *LSE;
    const int32_t *k_lengths, *q_lengths;
    int B, Hq, Hkv, Sq, Sk, D;
    float scale;
    int causal, window, input_pos;
    // flex_attention! extras; flex = 0 selects the plain kernel
    int flex = 0;
    float softcap = 0.f;
    const float *alibi_slopes = nullptr;
    const int32_t *doc_q = nullptr, *doc_kv = nullptr;
    const uint8_t *block_mask = nullptr;
    int block_mask_per_head = 0;  // block_mask is (B, Hq, nqb, nkb) instead of (nqb, nkb)
};

// Longest KV sequence the flex kernel takes, in 128-key tiles (its per-CTA list
// of visited tiles lives in shared memory).
constexpr int kFlexMaxKvTiles = 1024;

// Block-sparse prefill kernel (BlockMask alone, no score mod, no DocumentMask,
// not causal, no lengths): longest key sequence it takes, in 64-key blocks (its
// per-CTA list of visited blocks lives in shared memory).  Other flex calls, and
// longer sequences, run on the flex kernel's list path.
constexpr int kBsparseMaxKvBlocks = 1024;
bool bsparse_eligible(const FwdArgs &a);
attn_status_t launch_fwd_bsparse(const FwdArgs &a, cudaStream_t stream);

struct DecodeArgs {
    void *O;
    const void *Q, *K, *V;
    const int32_t *lengths;
    int n_splits;
    int B, Hq, Hkv, S_cap, D;
    float *workspace;  // B * Hq * n_splits * (D + 4) floats
    // paged KV cache (block_tables != nullptr): K/V are (num_blocks, block_size,
    // Hkv, D) and S_cap = max_blocks * block_size
    const int32_t *block_tables = nullptr;
    int num_blocks = 0, block_size = 0, max_blocks = 0;
};

// Backward of the forward (Tylo.jl `∇attention!`).
struct BwdArgs {
    void *dQ, *dK, *dV;
    const void *dO, *Q, *K, *V, *O;
    const float *LSE;
    const int32_t *k_lengths, *q_lengths;
    int B, Hq, Hkv, Sq, Sk, D;
    float scale;
    int causal, window, input_pos;
    float *delta;  // workspace (B, Hq, Sq)
};

attn_status_t launch_bwd(const BwdArgs &a, cudaStream_t stream);
// dK / dV and dQ on tcgen05 (after the delta workspace is written).
attn_status_t launch_bwd_tc(const BwdArgs &a, cudaStream_t stream);

// Block scores + block mask of block-sparse prefill (RBS page of mlx-arsenal).
struct RbsArgs {
    const void *Q, *K;
    int B, Hq, Hkv, Sq, Sk, D;
    float alpha_base, alpha_rescue;
    int diagonal;
    uint8_t *mask;                     // (B, Hq, nqb, nkb) BlockMask states 2 / 0
    float *base_scores, *rescue_scores;  // (B, Hq, nqb, nkb) or nullptr
    float *cent, *rad, *beta;          // workspace: (B, Hkv, nkb, D), (B, Hkv, nkb) x 2
};

attn_status_t launch_rbs(const RbsArgs &a, cudaStream_t stream);

// Device address of the status word on the current device (looked up once per
// device), or nullptr if the lookup failed.
int *device_status_word();

attn_status_t launch_fwd(const FwdArgs &a, cudaStream_t stream);
attn_status_t launch_decode(const DecodeArgs &a, cudaStream_t stream);
attn_status_t launch_wait_probe(int limit_us, cudaStream_t stream);

// Once per (device, kernel), thread-safe: check that the kernel was built with
// `required_regs` registers per thread (skipped when negative), raise its
// dynamic shared-memory limit to `smem_bytes` on the current device and, with
// max_smem_carveout, ask for the largest shared-memory carveout (kernels that
// run several CTAs per SM, each with a large dynamic allocation).
cudaError_t kernel_setup(const void *func, int smem_bytes, int required_regs = -1,
                         bool max_smem_carveout = false);

// Bounded-wait limit used by the attention kernels (nanoseconds of global time).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

}  // namespace gqa
