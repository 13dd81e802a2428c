// attn_decode.cu -- split-KV (Flash-Decoding) single-token attention for sm_100a.
//
// Defined on the Tylo.jl "Primitives" page, entry `decode_attention!`: one
// query vector per (sequence, head), the KV cache of each sequence processed
// in n_splits parallel slices of TILE_N = 64-key tiles, `lengths` = valid KV
// length per sequence; scale 1/sqrt(D) (the page's default qk_scale).
//
// Kernel 1 (split): one CTA per (split s, KV head, sequence).  All G = Hq/Hkv
// query heads that share the KV head are processed together so every K/V byte
// is read from HBM once per split.  A producer thread streams 64-key K and V
// tiles into a ring of shared-memory stages with TMA (128-byte swizzle, so the
// consumers' ldmatrix reads are bank-conflict free).  Four consumer warps each
// take 16 keys of every tile and run the two small contractions on the tensor
// cores with warp-level mma.sync (M = 16 rows hold the G <= 16 query heads;
// tcgen05's smallest M is 64, a poor fit for 4 query rows).  Each warp keeps
// its own fp32 online-softmax state; the four are merged in shared memory and
// the slice's normalised partial output and log-sum-exp are written to the
// workspace.
//
// Paged variant (vllm-mlx "attention" page: KV cache of shape (num_blocks,
// block_size, num_kv_heads, head_size), metadata seq_lens and block_tables):
// the same kernels, with each 64-key tile gathered by TMA from the blocks the
// sequence's block table names, block_size (or 64) rows of one head per copy.
// At D = 128 the cache is viewed as (rows, heads, 2, 64), so one copy brings both
// 64-column halves of those rows (stored row by row, each half 128-byte swizzled):
// half the copies of two 64-column boxes, 707 -> 674 us on the B64 paged workload
// with 16-token blocks, bitwise the same.
//
// Kernel 2 (combine): one warp per (sequence, query head) merges the slices:
// LSE = log sum_s exp(lse_s), O = sum_s exp(lse_s - LSE) o_s; empty slices
// (lse = -inf) weigh nothing, and a sequence with no valid key gets O = 0.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace gqa {

namespace {

constexpr int TN = 64;           // keys per tile (the pages' TILE_N)
constexpr int kConsumers = 4;    // consumer warps, 16 keys each per tile
constexpr int kDecThreads = 32 * (kConsumers + 1);
constexpr int kMaxGroup = 16;    // query heads per KV head handled by one CTA

template <int D>
struct DecCfg {
    static constexpr int NS = 3;               // ring stages
    static constexpr int NBOX = D / 64;
    static constexpr int BOX = TN * 128;        // bytes of one 64-column box
    static constexpr int TILE = TN * D * 2;     // bytes of one K (or V) tile
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = NS * TILE;
    static constexpr int OFF_BAR = 2 * NS * TILE;
    static constexpr int N_BARS = 2 * NS;       // full[NS], empty[NS]
    static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
    // merge area (reuses the ring once every tile is consumed)
    static constexpr int MERGE_BYTES = kConsumers * kMaxGroup * (D + 2) * 4;
    static_assert(MERGE_BYTES <= 2 * NS * TILE, "merge area must fit in the ring");
    static constexpr int WS_STRIDE = D + 4;     // floats per partial: o[D], lse, pad
};

struct DecParams {
    const __nv_bfloat16 *Q;
    float *ws;
    const int32_t *lengths;
    int B, Hq, Hkv, S_cap, group, n_splits;
    float scale_log2;
    uint64_t wait_limit_ns;
    int *status;  // device status word
    // paged cache only
    const int32_t *block_tables;  // (B, max_blocks)
    int max_blocks, block_shift, num_blocks, box_rows;
};

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }

// 4-D tiled TMA load (the paged cache's wide view below), no cluster multicast.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const void *tmap, uint32_t bar, int x,
                                            int y, int z, int w) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(x), "r"(y), "r"(z), "r"(w)
        : "memory");
}

// Byte offset of 16-byte chunk `chunk` (0 .. D/8-1) of tile row `row` inside a
// tile stored as D/64 TMA boxes of (64 rows x 128 bytes), 128-byte swizzled.
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
    return (chunk >> 3) * (TN * 128) + row * 128 + (((chunk & 7) ^ (row & 7)) << 4);
}

// The same for a tile whose rows hold both 64-column halves in turn (paged cache,
// D = 128, one TMA box per chunk of rows): 128-byte segment s = 2 row + half.
template <bool kWide>
__device__ __forceinline__ uint32_t swz_t(int row, int chunk) {
    if constexpr (kWide) {
        const int s = 2 * row + (chunk >> 3);
        return s * 128 + (((chunk & 7) ^ (s & 7)) << 4);
    } else {
        return swz(row, chunk);
    }
}

template <int D, bool kPaged>
__global__ void __launch_bounds__(kDecThreads)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const DecParams p) {
    using C = DecCfg<D>;
    constexpr bool kWide = kPaged && D == 128;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    auto full = [&](int s) -> uint32_t { return sbase + C::OFF_BAR + 8 * s; };
    auto empty = [&](int s) -> uint32_t { return sbase + C::OFF_BAR + 8 * (C::NS + s); };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC);

    const int split = blockIdx.x;
    const int hkv = blockIdx.y;
    const int b = blockIdx.z;
    const int G = p.group;
    const int h0 = hkv * G;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Programmatic dependent launch: every global read or write below comes after
    // the previous kernel on the stream has finished; the combine may launch at
    // once (its own wait covers all of this grid).
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    int len = p.lengths[b];
    if (len > p.S_cap) {
        if (threadIdx.x == 0 && split == 0 && hkv == 0) record_status(p.status, ATTN_ERR_DEVICE_BOUNDS);
        len = p.S_cap;
    }
    if (len < 0) len = 0;
    const int n_all = (len + TN - 1) / TN;
    const int per = (n_all + p.n_splits - 1) / p.n_splits;
    const int k0 = split * per * TN;
    const int k1 = min(k0 + per * TN, len);

    float *ws_base = p.ws + ((long long)(b * p.Hq + h0) * p.n_splits + split) * C::WS_STRIDE;
    const long long ws_head = (long long)p.n_splits * C::WS_STRIDE;
    // checked build: the workspace entries of this CTA's G heads lie inside it
    const long long ws_end = (long long)p.B * p.Hq * p.n_splits * C::WS_STRIDE;
    const bool ws_ok = in_range(
        ((long long)(b * p.Hq + h0 + G - 1) * p.n_splits + split) * C::WS_STRIDE + D < ws_end,
        p.status, nullptr);

    if (k0 >= k1) {  // empty slice: weight zero in the combine
        for (int h = threadIdx.x; h < G && ws_ok; h += blockDim.x) ws_base[h * ws_head + D] = neg_inf();
        return;
    }
    const int t_begin = k0 / TN;
    const int n_tiles = (k1 + TN - 1) / TN - t_begin;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), kConsumers);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kConsumers) {
        // ===================== TMA producer =====================
        if (lane == 0) {
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            // paged: block ids of a tile's chunks, loaded one tile ahead so that the
            // block-table reads overlap the previous tile's copies instead of each
            // copy waiting for its own read (block_size >= 8: at most TN / 8 chunks)
            constexpr int kMaxChunks = TN / 8;
            int ids[kMaxChunks];
            auto load_ids = [&](int it2) {
                if constexpr (kPaged) {
                    const int row2 = (t_begin + it2) * TN;
                    const int n2 = (min(TN, len - row2) + p.box_rows - 1) / p.box_rows;
                    const int32_t *bt = p.block_tables + (long long)b * p.max_blocks;
#pragma unroll
                    for (int k = 0; k < kMaxChunks; ++k)
                        ids[k] = k < n2 ? bt[(row2 + k * p.box_rows) >> p.block_shift] : 0;
                }
            };
            if (n_tiles > 0) load_ids(0);
            for (int it = 0; it < n_tiles; ++it) {
                const int st = it % C::NS;
                const int use = it / C::NS;
                if (use > 0 &&
                    !mbar_wait(empty(st), (use - 1) & 1, abort_flag, p.wait_limit_ns, p.status))
                    break;
                const int row = (t_begin + it) * TN;
                if constexpr (!kPaged) {
                    if (!in_range(box_ok(0, row, b * p.Hkv + hkv, D, p.S_cap, (long long)p.B * p.Hkv,
                                         TN) &&
                                      row >= 0 && row < p.S_cap,
                                  p.status, abort_flag))
                        break;
                    mbar_arrive_expect_tx(full(st), 2 * C::TILE);
                    for (int c = 0; c < C::NBOX; ++c) {
                        tma_load_3d(sbase + C::OFF_K + st * C::TILE + c * C::BOX, &tmK, full(st),
                                    c * 64, row, b * p.Hkv + hkv);
                        tma_load_3d(sbase + C::OFF_V + st * C::TILE + c * C::BOX, &tmV, full(st),
                                    c * 64, row, b * p.Hkv + hkv);
                    }
                } else {
                    // Gather the tile's valid keys chunk by chunk: key j of the sequence
                    // is cache row block_tables[b][j / block_size] * block_size +
                    // j % block_size.  Chunks past the length are not loaded; the
                    // consumers mask those keys and zero those V rows.
                    const int br = p.box_rows;
                    const int n_chunks = (min(TN, len - row) + br - 1) / br;
                    int cur[kMaxChunks];
#pragma unroll
                    for (int k = 0; k < kMaxChunks; ++k) cur[k] = ids[k];
                    if (it + 1 < n_tiles) load_ids(it + 1);
                    mbar_arrive_expect_tx(full(st), 2 * n_chunks * br * 128 * C::NBOX);
#pragma unroll
                    for (int k = 0; k < kMaxChunks; ++k) {
                        if (k >= n_chunks) break;
                        const int j = row + k * br;
                        const int blk = cur[k];
                        if (blk < 0 || blk >= p.num_blocks) record_status(p.status, ATTN_ERR_DEVICE_BOUNDS);
                        // an out-of-range block reads as zeros (outside the tensor map)
                        const int prow = blk * (1 << p.block_shift) + (j & ((1 << p.block_shift) - 1));
                        // checked build: the chunk stays inside its tile of the ring (an
                        // out-of-range block is the documented zero-filled case)
                        if (!in_range(k * br + br <= TN && hkv < p.Hkv, p.status, abort_flag)) break;
                        if constexpr (kWide) {
                            const uint32_t off = st * C::TILE + k * br * 256;
                            tma_load_4d(sbase + C::OFF_K + off, &tmK, full(st), 0, 0, hkv, prow);
                            tma_load_4d(sbase + C::OFF_V + off, &tmV, full(st), 0, 0, hkv, prow);
                        } else {
                            for (int c = 0; c < C::NBOX; ++c) {
                                const uint32_t off = st * C::TILE + c * C::BOX + k * br * 128;
                                tma_load_3d(sbase + C::OFF_K + off, &tmK, full(st), c * 64, hkv, prow);
                                tma_load_3d(sbase + C::OFF_V + off, &tmV, full(st), c * 64, hkv, prow);
                            }
                        }
                    }
                }
            }
        }
    } else {
        // ===================== consumers =====================
        const int g = lane >> 2;  // fragment row (query head within the group)
        const int t = lane & 3;
        // Q as m16n8k16 A fragments: rows = query heads (zero past G), k = d.
        uint32_t qa[D / 16][4];
        {
            const __nv_bfloat16 *q_lo = p.Q + (long long)(b * p.Hq + h0 + g) * D;
            const __nv_bfloat16 *q_hi = p.Q + (long long)(b * p.Hq + h0 + g + 8) * D;
            const bool lo_ok = g < G, hi_ok = g + 8 < G;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const int c0 = kk * 16 + 2 * t;
                qa[kk][0] = lo_ok ? *reinterpret_cast<const uint32_t *>(q_lo + c0) : 0u;
                qa[kk][1] = hi_ok ? *reinterpret_cast<const uint32_t *>(q_hi + c0) : 0u;
                qa[kk][2] = lo_ok ? *reinterpret_cast<const uint32_t *>(q_lo + c0 + 8) : 0u;
                qa[kk][3] = hi_ok ? *reinterpret_cast<const uint32_t *>(q_hi + c0 + 8) : 0u;
            }
        }
        float o[D / 8][4];
#pragma unroll
        for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
        float m_run[2] = {neg_inf(), neg_inf()};  // rows g, g + 8 (log2 units)
        float l_run[2] = {0.f, 0.f};              // this lane's partial row sums

        // ldmatrix lane roles
        const int mi = lane >> 3, rr = lane & 7;
        bool ok = true;
        for (int it = 0; it < n_tiles; ++it) {
            const int st = it % C::NS;
            if (!warp_wait(full(st), (it / C::NS) & 1, abort_flag, p.wait_limit_ns, p.status)) {
                ok = false;
                break;
            }
            const int key0 = (t_begin + it) * TN + warp * 16;  // first key of this warp
            if (key0 < k1) {
                const uint32_t kb = sbase + C::OFF_K + st * C::TILE;
                const uint32_t vb = sbase + C::OFF_V + st * C::TILE;
                // ---- S = Q K^T over this warp's 16 keys ----
                float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                {
                    const int krow = warp * 16 + (mi >> 1) * 8 + rr;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        uint32_t b0, b1, b2, b3;
                        ldmatrix_x4(kb + swz_t<kWide>(krow, 2 * kk + (mi & 1)), b0, b1, b2, b3);
                        mma_m16n8k16(sc[0], qa[kk], b0, b1);
                        mma_m16n8k16(sc[1], qa[kk], b2, b3);
                    }
                }
                // ---- mask keys past the slice end; online softmax (exp2 domain) ----
                float mt[2] = {neg_inf(), neg_inf()};
#pragma unroll
                for (int nb = 0; nb < 2; ++nb)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int key = key0 + nb * 8 + 2 * t + (e & 1);
                        const float x = key < k1 ? sc[nb][e] * p.scale_log2 : neg_inf();
                        sc[nb][e] = x;
                        mt[e >> 1] = fmaxf(mt[e >> 1], x);
                    }
                float alpha[2], m_use[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    mt[h] = fmaxf(mt[h], __shfl_xor_sync(0xffffffffu, mt[h], 1));
                    mt[h] = fmaxf(mt[h], __shfl_xor_sync(0xffffffffu, mt[h], 2));
                    const float m_new = fmaxf(m_run[h], mt[h]);
                    m_use[h] = (m_new == neg_inf()) ? 0.f : m_new;
                    alpha[h] = fast_exp2(m_run[h] - m_use[h]);
                    m_run[h] = m_new;
                }
                float pr[2][4];
#pragma unroll
                for (int nb = 0; nb < 2; ++nb)
#pragma unroll
                    for (int e = 0; e < 4; ++e) pr[nb][e] = fast_exp2(sc[nb][e] - m_use[e >> 1]);
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    l_run[h] = l_run[h] * alpha[h] + pr[0][2 * h] + pr[0][2 * h + 1] +
                               pr[1][2 * h] + pr[1][2 * h + 1];
#pragma unroll
                for (int n = 0; n < D / 8; ++n) {
                    o[n][0] *= alpha[0];
                    o[n][1] *= alpha[0];
                    o[n][2] *= alpha[1];
                    o[n][3] *= alpha[1];
                }
                uint32_t pa[4];
                pa[0] = pack_bf16x2(pr[0][0], pr[0][1]);
                pa[1] = pack_bf16x2(pr[0][2], pr[0][3]);
                pa[2] = pack_bf16x2(pr[1][0], pr[1][1]);
                pa[3] = pack_bf16x2(pr[1][2], pr[1][3]);
                // Cache rows at or past the sequence length may hold anything; their
                // weights are 0, but 0 * NaN is NaN, so zero this warp's such V rows.
                const bool tail = key0 + 16 > len && key0 < p.S_cap;
                if (tail) {
                    const int rows_from = max(len - key0, 0);
                    for (int idx = lane; idx < 16 * (D / 8); idx += 32) {
                        const int rrow = idx / (D / 8), ch = idx % (D / 8);
                        if (rrow >= rows_from)
                            *reinterpret_cast<uint4 *>(smem + C::OFF_V + st * C::TILE +
                                                       swz_t<kWide>(warp * 16 + rrow, ch)) =
                                make_uint4(0, 0, 0, 0);
                    }
                    __syncwarp();
                }
                // ---- O += P V over this warp's 16 keys ----
                {
                    const int vrow = warp * 16 + (mi & 1) * 8 + rr;
#pragma unroll
                    for (int dp = 0; dp < D / 16; ++dp) {
                        uint32_t b0, b1, b2, b3;
                        ldmatrix_x4_trans(vb + swz_t<kWide>(vrow, 2 * dp + (mi >> 1)), b0, b1, b2, b3);
                        mma_m16n8k16(o[2 * dp], pa, b0, b1);
                        mma_m16n8k16(o[2 * dp + 1], pa, b2, b3);
                    }
                }
                if (tail) fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty(st));
        }

        // ---- merge the four warps' states (ring memory is free now) ----
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsumers) : "memory");
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 1);
            l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 2);
        }
        float *mrg = reinterpret_cast<float *>(smem);
        // layout: [warp][row 0..15][D] outputs, then m[warp][16], l[warp][16]
        float *mo = mrg;
        float *mm = mrg + kConsumers * kMaxGroup * D;
        float *ml = mm + kConsumers * kMaxGroup;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
            const int col = n * 8 + 2 * t;
            mo[(warp * kMaxGroup + g) * D + col] = o[n][0];
            mo[(warp * kMaxGroup + g) * D + col + 1] = o[n][1];
            mo[(warp * kMaxGroup + g + 8) * D + col] = o[n][2];
            mo[(warp * kMaxGroup + g + 8) * D + col + 1] = o[n][3];
        }
        if (t == 0) {
            mm[warp * kMaxGroup + g] = m_run[0];
            mm[warp * kMaxGroup + g + 8] = m_run[1];
            ml[warp * kMaxGroup + g] = l_run[0];
            ml[warp * kMaxGroup + g + 8] = l_run[1];
        }
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsumers) : "memory");
        if (ok && !*abort_flag && ws_ok) {
            for (int idx = threadIdx.x; idx < G * D; idx += 32 * kConsumers) {
                const int h = idx / D, d = idx % D;
                float M = neg_inf();
#pragma unroll
                for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, mm[w * kMaxGroup + h]);
                float acc = 0.f, lsum = 0.f;
#pragma unroll
                for (int w = 0; w < kConsumers; ++w) {
                    const float wt = fast_exp2(mm[w * kMaxGroup + h] - M);
                    acc += wt * mo[(w * kMaxGroup + h) * D + d];
                    lsum += wt * ml[w * kMaxGroup + h];
                }
                float *dst = ws_base + h * ws_head;
                dst[d] = acc / lsum;
                if (d == 0) dst[D] = (M + __log2f(lsum)) * 0.69314718055994531f;
            }
        } else {
            // A bounded wait ran out: the slice weighs nothing in the combine, so
            // whatever the workspace held before (another call's partials) never
            // reaches O.
            for (int h = threadIdx.x; h < G && ws_ok; h += 32 * kConsumers)
                ws_base[h * ws_head + D] = neg_inf();
        }
    }
    if (*abort_flag) drain_delay(2000000);
    __syncthreads();
}

template <int D>
__global__ void __launch_bounds__(128)
    decode_combine_kernel(__nv_bfloat16 *__restrict__ O, const float *__restrict__ ws, int BH,
                          int n_splits) {
    constexpr int WS = DecCfg<D>::WS_STRIDE;
    const int idx = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    // the split kernel's partials are complete and visible after this wait
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (idx >= BH) return;
    const float *part = ws + (long long)idx * n_splits * WS;
    float M = neg_inf();
    for (int s = lane; s < n_splits; s += 32) M = fmaxf(M, part[s * WS + D]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    constexpr int PER = D / 32;  // output elements per lane
    float acc[PER];
#pragma unroll
    for (int k = 0; k < PER; ++k) acc[k] = 0.f;
    __nv_bfloat16 *out = O + (long long)idx * D + lane * PER;
    if (M == neg_inf()) {  // no valid key in any slice
#pragma unroll
        for (int k = 0; k < PER; ++k) out[k] = __float2bfloat16_rn(0.f);
        return;
    }
    float wsum = 0.f;
    for (int s = 0; s < n_splits; ++s) {
        const float lse = part[s * WS + D];
        if (lse == neg_inf()) continue;
        const float w = __expf(lse - M);
        wsum += w;
        const float *src = part + s * WS + lane * PER;
#pragma unroll
        for (int k = 0; k < PER; ++k) acc[k] += w * src[k];
    }
    const float inv = 1.f / wsum;
#pragma unroll
    for (int k = 0; k < PER; k += 2) {
        __nv_bfloat162 v = __floats2bfloat162_rn(acc[k] * inv, acc[k + 1] * inv);
        *reinterpret_cast<__nv_bfloat162 *>(out + k) = v;
    }
}

template <int D, bool kPaged>
attn_status_t launch_decode_d(const DecodeArgs &a, cudaStream_t stream) {
    using C = DecCfg<D>;
    CUtensorMap tk, tv;
    attn_status_t st;
    const uint32_t box_rows = kPaged ? static_cast<uint32_t>(min(a.block_size, TN)) : TN;
    if constexpr (kPaged) {
        const uint64_t rows = (uint64_t)a.num_blocks * a.block_size;
        if (D == 128) {
            if ((st = make_tmap_bf16_paged_wide(&tk, a.K, a.Hkv, rows, box_rows)) != ATTN_OK) return st;
            if ((st = make_tmap_bf16_paged_wide(&tv, a.V, a.Hkv, rows, box_rows)) != ATTN_OK) return st;
        } else {
            if ((st = make_tmap_bf16_paged(&tk, a.K, D, a.Hkv, rows, box_rows)) != ATTN_OK) return st;
            if ((st = make_tmap_bf16_paged(&tv, a.V, D, a.Hkv, rows, box_rows)) != ATTN_OK) return st;
        }
    } else {
        if ((st = make_tmap_bf16_3d(&tk, a.K, D, a.S_cap, (uint64_t)a.B * a.Hkv, TN)) != ATTN_OK)
            return st;
        if ((st = make_tmap_bf16_3d(&tv, a.V, D, a.S_cap, (uint64_t)a.B * a.Hkv, TN)) != ATTN_OK)
            return st;
    }
    if (kernel_setup(reinterpret_cast<const void *>(decode_split_kernel<D, kPaged>), C::SMEM_BYTES) !=
        cudaSuccess)
        return ATTN_ERR_CUDA;
    DecParams p;
    p.Q = static_cast<const __nv_bfloat16 *>(a.Q);
    p.ws = a.workspace;
    p.lengths = a.lengths;
    p.B = a.B;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.S_cap = a.S_cap;
    p.group = a.Hq / a.Hkv;
    p.n_splits = a.n_splits;
    p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
    p.wait_limit_ns = kWaitLimitNs;
    p.status = device_status_word();
    if (!p.status) return ATTN_ERR_CUDA;
    p.block_tables = a.block_tables;
    p.max_blocks = a.max_blocks;
    p.num_blocks = a.num_blocks;
    p.box_rows = static_cast<int>(box_rows);
    p.block_shift = 0;
    while (kPaged && (1 << p.block_shift) < a.block_size) ++p.block_shift;
    // Both kernels are launched with programmatic dependent launch (each waits for
    // its predecessor on the stream before touching global memory).
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.n_splits, a.Hkv, a.B);
    cfg.blockDim = dim3(kDecThreads, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, decode_split_kernel<D, kPaged>, tk, tv, p) != cudaSuccess)
        return ATTN_ERR_CUDA;
    const int BH = a.B * a.Hq;
    cfg.gridDim = dim3((BH + 3) / 4, 1, 1);
    cfg.blockDim = dim3(128, 1, 1);
    cfg.dynamicSmemBytes = 0;
    if (cudaLaunchKernelEx(&cfg, decode_combine_kernel<D>, static_cast<__nv_bfloat16 *>(a.O),
                           static_cast<const float *>(a.workspace), BH, a.n_splits) != cudaSuccess)
        return ATTN_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

size_t decode_workspace_floats(int B, int Hq, int n_splits, int D) {
    return (size_t)B * Hq * n_splits * (D + 4);
}

attn_status_t launch_decode(const DecodeArgs &a, cudaStream_t stream) {
    if (a.B == 0) return ATTN_OK;
    if (a.block_tables) {
        if (a.D == 128) return launch_decode_d<128, true>(a, stream);
        if (a.D == 64) return launch_decode_d<64, true>(a, stream);
        return ATTN_ERR_UNSUPPORTED;
    }
    if (a.D == 128) return launch_decode_d<128, false>(a, stream);
    if (a.D == 64) return launch_decode_d<64, false>(a, stream);
    return ATTN_ERR_UNSUPPORTED;
}

}  // namespace gqa
