// block_mask.cu -- host builders of the coarse block mask that attn_fwd_flex
// uses to skip tiles: the build_block_mask of the Tylo.jl "Primitives" page
// (entry `build_block_mask`, TILE_M = TILE_N = 64; entry `BlockMask`: per
// query block, the key blocks holding any unmasked pair and which of them are
// fully unmasked).  Plain host code; no device work.
#include <cstdint>

#include "gqa_attn.h"

namespace {

constexpr int kTile = 64;

// Classify one 64x64 block from a predicate on (local query row, key).
template <class Keep>
uint8_t classify(int qb, int kb, int Sq, int Sk, const Keep &keep) {
    const int i0 = qb * kTile, i1 = (i0 + kTile < Sq) ? i0 + kTile : Sq;
    const int j0 = kb * kTile, j1 = (j0 + kTile < Sk) ? j0 + kTile : Sk;
    bool any = false, all = true;
    for (int i = i0; i < i1; ++i) {
        for (int j = j0; j < j1; ++j) {
            if (keep(i, j))
                any = true;
            else
                all = false;
            if (any && !all) return 1;
        }
    }
    return any ? 2 : 0;
}

template <class Keep>
void fill(uint8_t *out, int Sq, int Sk, const Keep &keep) {
    const int n_qb = (Sq + kTile - 1) / kTile, n_kb = (Sk + kTile - 1) / kTile;
    for (int qb = 0; qb < n_qb; ++qb)
        for (int kb = 0; kb < n_kb; ++kb) out[(long long)qb * n_kb + kb] = classify(qb, kb, Sq, Sk, keep);
}

}  // namespace

extern "C" {

attn_status_t attn_block_mask_build(uint8_t *out, int Sq, int Sk, int input_pos,
                                    int (*keep)(int q, int kv, void *ctx), void *ctx) {
    if (Sq < 0 || Sk < 0 || input_pos < 0) return ATTN_ERR_INVALID;
    if ((long long)Sq * Sk == 0) return ATTN_OK;
    if (!out || !keep) return ATTN_ERR_NULL;
    fill(out, Sq, Sk, [&](int i, int j) { return keep(input_pos + i, j, ctx) != 0; });
    return ATTN_OK;
}

attn_status_t attn_block_mask_document(uint8_t *out, int Sq, int Sk, int input_pos, int causal,
                                       int window, const int32_t *doc_q, const int32_t *doc_kv) {
    if (Sq < 0 || Sk < 0 || input_pos < 0 || window < 0) return ATTN_ERR_INVALID;
    if (causal != 0 && causal != 1) return ATTN_ERR_INVALID;
    if (window > 0 && !causal) return ATTN_ERR_INVALID;
    if ((long long)Sq * Sk == 0) return ATTN_OK;
    if (!out || !doc_q || !doc_kv) return ATTN_ERR_NULL;
    fill(out, Sq, Sk, [&](int i, int j) {
        const long long q = (long long)input_pos + i;
        if (causal && j > q) return false;
        if (window > 0 && j <= q - window) return false;
        return doc_q[i] == doc_kv[j];
    });
    return ATTN_OK;
}

}  // extern "C"
