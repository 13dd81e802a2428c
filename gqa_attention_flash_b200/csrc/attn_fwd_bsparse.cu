// attn_fwd_bsparse.cu -- block-sparse prefill forward for sm_100a: attention over
// the kept 64x64 blocks of a BlockMask, one 64-key block per step.
//
// Computes the rows of O = softmax(Q K^T * scale + mask) V and their
// log-sum-exp (Tylo.jl "Primitives" page, entry `attention!`) where the mask
// keeps exactly the (query, key) pairs of the kept 64x64 blocks: the BlockMask
// of the same page (entries `BlockMask` and `build_block_mask`, 64-row by
// 64-key blocks) applied by `flex_attention!` with no score mod and no
// DocumentMask, which is how block-sparse prefill applies the block mask of the
// mlx-arsenal "Radius-bounded block scores (RBS)" page.  A block state of 0
// skips the block; any other state keeps all of its pairs.
//
// Work item: one 128-row query tile (two 64-row query blocks) of one (query head,
// batch).  The CTA visits, in order, the 64-key blocks that either of its query
// blocks keeps; the rows of a query block mask out the keys of a visited block
// that their own row of the BlockMask skips.  At 10 % block density a 128 x 128
// tile is visited about three times as often as a 64 x 64 block, a 128 x 64 step
// about twice, which is why the steps here are 64 keys wide.
//
// Two CTAs per SM (256 TMEM columns and under 113 KB of shared memory each), so
// that the softmax of one overlaps the tensor-core work of the other.  6 warps:
//   warps 0-3  softmax, one query row per thread (= TMEM lane), and the epilogue
//   warp 4     builds the block list (whole warp), then TMA producer (lane 0):
//              Q once, K_j and V_j into NS-stage rings released separately (a K
//              stage when S_j is done, a V stage when P_j V_j is done)
//   warp 5     TMEM owner and MMA issuer (lane 0):
//              S_j = Q K_j^T into S buffer j % 2 (smem x smem, N = 64),
//              O += P_j V_j (P_j read from TMEM, written over S_j as bf16)
// Issue order S_0, S_1, P_0 V_0, S_2, P_1 V_1, S_3, ...: the softmax of S_{j+1}
// runs while P_j V_j and S_{j+2} are on the tensor core.  TMEM: S0 | S1 | O.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace gqa {

namespace {

constexpr int SP_BM = 128;          // query rows per CTA (two 64-row query blocks)
constexpr int SP_BN = 64;           // keys per step (one BlockMask block)
constexpr int kSpWarpTma = 4;
constexpr int kSpWarpMma = 5;
constexpr int kSpThreads = 192;
constexpr uint32_t kSpTmemCols = 256;

template <int D>
struct SpCfg {
    static constexpr int NBOX = D / 64;              // 64-column TMA boxes per row
    static constexpr int Q_BOX = SP_BM * 128;        // bytes of one (128 rows x 64 cols) box
    static constexpr int KV_BOX = SP_BN * 128;       // bytes of one (64 rows x 64 cols) box
    static constexpr int Q_BYTES = SP_BM * D * 2;
    static constexpr int KV_BYTES = SP_BN * D * 2;
    static constexpr int NS = (D == 128) ? 2 : 4;    // depth of the K ring and of the V ring
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + NS * KV_BYTES;
    static constexpr int BAR_QFULL = 0;
    static constexpr int BAR_KFULL = 1;              // [NS]
    static constexpr int BAR_KEMPTY = 1 + NS;        // [NS]
    static constexpr int BAR_VFULL = 1 + 2 * NS;     // [NS]
    static constexpr int BAR_VEMPTY = 1 + 3 * NS;    // [NS]
    static constexpr int BAR_SFULL = 1 + 4 * NS;     // [2] one per S buffer
    static constexpr int BAR_PFULL = 3 + 4 * NS;
    static constexpr int BAR_ODONE = 4 + 4 * NS;
    static constexpr int N_BARS = 5 + 4 * NS;
    static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;   // tmem slot, abort flag, list count
    static constexpr int OFF_LIST = OFF_MISC + 16;
    static constexpr int SMEM_BYTES = OFF_LIST + 2 * kBsparseMaxKvBlocks + 1024;  // + alignment
    static constexpr uint32_t S_COL0 = 0, O_COL = 2 * SP_BN;
};
// two CTAs per SM: 2 x (dynamic + 1 KB reserved per block) within 228 KB
static_assert(2 * (SpCfg<128>::SMEM_BYTES + 1024) <= 233472, "two CTAs per SM must fit");
static_assert(2 * (SpCfg<64>::SMEM_BYTES + 1024) <= 233472, "two CTAs per SM must fit");
static_assert(SpCfg<128>::O_COL + 128 <= kSpTmemCols, "TMEM columns");
static_assert(kBsparseMaxKvBlocks <= 1024, "block index must fit 10 bits of a list entry");

struct SpParams {
    __nv_bfloat16 *O;
    float *LSE;
    const uint8_t *bmask;     // (n_qb, n_kb) states, one matrix per (batch, query head) if per_head
    int per_head;
    int B, Hq, Hkv, Sq, Sk, group, n_qt, n_qb, n_kb;
    float scale_log2;         // scale * log2(e)
    uint64_t wait_limit_ns;
    int *status;
};

__device__ __forceinline__ float sp_neg_inf() { return __int_as_float(0xff800000); }

// Bring a 3-D tile of a tensor map into L2 ahead of its load (no shared memory,
// no completion to wait for); x is a multiple of 64 elements.
__device__ __forceinline__ void tma_prefetch_3d(const void *tmap, int x, int y, int z,
                                                uint64_t policy) {
    asm volatile(
        "cp.async.bulk.prefetch.tensor.3d.L2.global.tile.L2::cache_hint [%0, {%1, %2, %3}], %4;" ::"l"(
            reinterpret_cast<uint64_t>(tmap)),
        "r"(x), "r"(y), "r"(z), "l"(policy)
        : "memory");
}

// Key blocks whose K and V tiles are prefetched into L2 ahead of the block loaded.
constexpr int kSpPrefetch = 4;

template <int D>
__global__ void __launch_bounds__(kSpThreads, 2)
    attn_fwd_bsparse_kernel(const __grid_constant__ CUtensorMap tmQ,
                            const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV, const SpParams p) {
    using C = SpCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8 * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    int *count_slot = reinterpret_cast<int *>(smem + C::OFF_MISC + 8);
    // visited key blocks in order: bits 0-9 the block index, bit 14 / 15 set when
    // query block 0 / 1 of the tile keeps it
    uint16_t *list = reinterpret_cast<uint16_t *>(smem + C::OFF_LIST);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    int w = blockIdx.x;
    const int qt = w % p.n_qt;
    w /= p.n_qt;
    const int hq = w % p.Hq;
    const int b = w / p.Hq;
    const int hkv = hq / p.group;

    // ---- set-up ----
    if (threadIdx.x == 0) {
        mbar_init(bar(C::BAR_QFULL), 1);
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(bar(C::BAR_KFULL + s), 1);
            mbar_init(bar(C::BAR_KEMPTY + s), 1);
            mbar_init(bar(C::BAR_VFULL + s), 1);
            mbar_init(bar(C::BAR_VEMPTY + s), 1);
        }
        mbar_init(bar(C::BAR_SFULL), 1);
        mbar_init(bar(C::BAR_SFULL + 1), 1);
        mbar_init(bar(C::BAR_PFULL), SP_BM);
        mbar_init(bar(C::BAR_ODONE), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // Programmatic dependent launch: launch and set-up overlap the previous kernel
    // (the block scores that write the mask); every global access below follows
    // its completion.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (warp == kSpWarpTma) {
        // The key blocks either query block of the tile keeps, in order (ballot
        // compaction, 32 blocks per round).
        const uint8_t *bm = p.bmask;
        if (p.per_head) bm += (size_t)(b * p.Hq + hq) * p.n_qb * p.n_kb;
        const int qb0 = 2 * qt, qb1 = 2 * qt + 1;
        const uint8_t *row0 = bm + (size_t)qb0 * p.n_kb;
        const uint8_t *row1 = qb1 < p.n_qb ? bm + (size_t)qb1 * p.n_kb : nullptr;
        int count = 0;
        for (int base = 0; base < p.n_kb; base += 32) {
            const int kb = base + lane;
            uint32_t k0 = 0, k1 = 0;
            if (kb < p.n_kb) {
                k0 = row0[kb] != 0 ? 1u : 0u;
                if (row1) k1 = row1[kb] != 0 ? 1u : 0u;
            }
            const uint32_t vote = __ballot_sync(0xffffffffu, (k0 | k1) != 0);
            if (k0 | k1)
                list[count + __popc(vote & ((1u << lane) - 1u))] =
                    static_cast<uint16_t>(kb | (k0 << 14) | (k1 << 15));
            count += __popc(vote);
        }
        if (lane == 0) *count_slot = count;
    } else if (warp == kSpWarpMma) {
        tmem_alloc(smem_u32(tmem_slot), kSpTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n = *count_slot;

    if (warp == kSpWarpTma) {
        // ===================== TMA producer =====================
        if (lane == 0 && n > 0) {
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            // Q is read once; the K / V blocks of a head serve all its query tiles.
            const uint64_t pol_q = l2_policy_evict_first(), pol_kv = l2_policy_evict_last();
            const int zq = b * p.Hq + hq, zk = b * p.Hkv + hkv;
            bool ok = in_range(box_ok(0, qt * SP_BM, zq, D, p.Sq, (long long)p.B * p.Hq, SP_BM),
                               p.status, abort_flag);
            if (ok) {
                mbar_arrive_expect_tx(bar(C::BAR_QFULL), C::Q_BYTES);
                for (int c = 0; c < C::NBOX; ++c)
                    tma_load_3d_hint(sbase + C::OFF_Q + c * C::Q_BOX, &tmQ, bar(C::BAR_QFULL), c * 64,
                                     qt * SP_BM, zq, pol_q);
            }
            // Checked build: the block lies inside K and V.
            auto kv_row_of = [&](int j, int &row) -> bool {
                row = (list[j] & 0x3FF) * SP_BN;
                return in_range(box_ok(0, row, zk, D, p.Sk, (long long)p.B * p.Hkv, SP_BN) &&
                                    row < p.Sk,
                                p.status, abort_flag);
            };
            auto prefetch = [&](int j) {
                int row;
                if (j < n && kv_row_of(j, row)) {
                    for (int c = 0; c < C::NBOX; ++c) {
                        tma_prefetch_3d(&tmK, c * 64, row, zk, pol_kv);
                        tma_prefetch_3d(&tmV, c * 64, row, zk, pol_kv);
                    }
                }
            };
            // K stage st is free once S of the block NS earlier is done; V stage st once
            // P V of that block is done.
            auto load_k = [&](int j) -> bool {
                const int st = j % C::NS;
                const uint32_t use = static_cast<uint32_t>(j / C::NS);
                int row;
                if (!kv_row_of(j, row)) return false;
                if (use > 0 && !mbar_wait(bar(C::BAR_KEMPTY + st), (use - 1) & 1, abort_flag,
                                          p.wait_limit_ns, p.status))
                    return false;
                mbar_arrive_expect_tx(bar(C::BAR_KFULL + st), C::KV_BYTES);
                for (int c = 0; c < C::NBOX; ++c)
                    tma_load_3d_hint(sbase + C::OFF_K + st * C::KV_BYTES + c * C::KV_BOX, &tmK,
                                     bar(C::BAR_KFULL + st), c * 64, row, zk, pol_kv);
                prefetch(j + kSpPrefetch);
                return true;
            };
            auto load_v = [&](int j) -> bool {
                const int st = j % C::NS;
                const uint32_t use = static_cast<uint32_t>(j / C::NS);
                int row;
                if (!kv_row_of(j, row)) return false;
                if (use > 0 && !mbar_wait(bar(C::BAR_VEMPTY + st), (use - 1) & 1, abort_flag,
                                          p.wait_limit_ns, p.status))
                    return false;
                mbar_arrive_expect_tx(bar(C::BAR_VFULL + st), C::KV_BYTES);
                for (int c = 0; c < C::NBOX; ++c)
                    tma_load_3d_hint(sbase + C::OFF_V + st * C::KV_BYTES + c * C::KV_BOX, &tmV,
                                     bar(C::BAR_VFULL + st), c * 64, row, zk, pol_kv);
                return true;
            };
            for (int j = 1; ok && j < kSpPrefetch; ++j) prefetch(j);
            // K runs one block ahead of V: S_{j+1} is needed before P_j V_j, and the
            // stage K_{j+1} reuses is released (S_{j-1} done) before the one V_j
            // reuses (P_{j-2} V_{j-2} done), so neither ring waits behind the other.
            if (ok) ok = load_k(0);
            for (int j = 0; ok && j < n; ++j) {
                if (j + 1 < n) ok = load_k(j + 1);
                if (ok) ok = load_v(j);
            }
        }
    } else if (warp == kSpWarpMma) {
        // ===================== MMA issuer =====================
        if (lane == 0 && n > 0) {
            constexpr uint32_t idS = idesc_bf16_f32(SP_BM, SP_BN, 0, 0);
            constexpr uint32_t idO = idesc_bf16_f32(SP_BM, D, 0, 1);
            bool ok = mbar_wait(bar(C::BAR_QFULL), 0, abort_flag, p.wait_limit_ns, p.status);
            auto issue_s = [&](int j) -> bool {
                const int st = j % C::NS;
                if (!mbar_wait(bar(C::BAR_KFULL + st), (j / C::NS) & 1, abort_flag, p.wait_limit_ns,
                               p.status))
                    return false;
                tc_fence_after();
                const uint32_t qa = sbase + C::OFF_Q, ka = sbase + C::OFF_K + st * C::KV_BYTES;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t col = (kk & 3) * 32;
                    mma_ss(tmem + C::S_COL0 + (j & 1) * SP_BN,
                           smem_desc_sw128(qa + (kk >> 2) * C::Q_BOX + col, 16, 1024),
                           smem_desc_sw128(ka + (kk >> 2) * C::KV_BOX + col, 16, 1024), idS,
                           kk > 0 ? 1u : 0u);
                }
                mma_commit(bar(C::BAR_SFULL + (j & 1)));
                mma_commit(bar(C::BAR_KEMPTY + st));
                return true;
            };
            auto issue_pv = [&](int j) -> bool {
                const int st = j % C::NS;
                if (!mbar_wait(bar(C::BAR_PFULL), j & 1, abort_flag, p.wait_limit_ns, p.status))
                    return false;
                if (!mbar_wait(bar(C::BAR_VFULL + st), (j / C::NS) & 1, abort_flag, p.wait_limit_ns,
                               p.status))
                    return false;
                tc_fence_after();
                const uint32_t va = sbase + C::OFF_V + st * C::KV_BYTES;
#pragma unroll
                for (int kk = 0; kk < SP_BN / 16; ++kk)
                    mma_ts(tmem + C::O_COL, tmem + C::S_COL0 + (j & 1) * SP_BN + kk * 8,
                           smem_desc_sw128(va + kk * 16 * 128, C::KV_BOX, 1024), idO,
                           (j > 0 || kk > 0) ? 1u : 0u);
                mma_commit(bar(C::BAR_ODONE));
                mma_commit(bar(C::BAR_VEMPTY + st));
                return true;
            };
            if (ok) ok = issue_s(0);
            if (ok && n > 1) ok = issue_s(1);
            for (int j = 0; ok && j < n; ++j) {
                ok = issue_pv(j);
                if (ok && j + 2 < n) ok = issue_s(j + 2);
            }
        }
    } else {
        // ===================== softmax and epilogue =====================
        const int r = threadIdx.x;                 // row within the tile = TMEM lane
        const uint32_t qh = static_cast<uint32_t>(r >> 6);  // query block of the row (warp-uniform)
        const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const float sl2 = p.scale_log2;
        float m_used = sp_neg_inf();  // max subtracted so far (log2 units)
        float l = 0.f;
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            const uint32_t e = list[j];
            const int kv0 = static_cast<int>(e & 0x3FFu) * SP_BN;
            // visible keys of this block for this row: [0, c_hi)
            const int c_hi = ((e >> (14 + qh)) & 1u) ? min(SP_BN, p.Sk - kv0) : 0;
            const uint32_t s_addr = trow + C::S_COL0 + (j & 1) * SP_BN;
            if (!warp_wait(bar(C::BAR_SFULL + (j & 1)), (j >> 1) & 1, abort_flag, p.wait_limit_ns,
                           p.status)) {
                ok = false;
                break;
            }
            float alpha = 1.f;
            bool resc = false;
            if (c_hi == 0) {
                // this row's query block does not keep the key block (the other one
                // does): every score is masked, so P = 0 and m, l stay as they are --
                // the same bits the full pass below would produce, without its work
                const uint32_t z[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                tc_fence_after();  // after S_j has landed in these columns
                tmem_st16(s_addr, z);
                tmem_st16(s_addr + 16, z);
            } else {
                tc_fence_after();
                uint32_t sr[2][32];
                tmem_ld32(s_addr, sr[0]);
                tmem_ld32(s_addr + 32, sr[1]);
                tmem_wait_ld();
                reg_fence32(sr[0]);
                reg_fence32(sr[1]);
                float *s = reinterpret_cast<float *>(&sr[0][0]);
                if (c_hi < SP_BN) {
#pragma unroll
                    for (int c = 0; c < SP_BN; ++c) s[c] = c < c_hi ? s[c] : sp_neg_inf();
                }
                // online softmax in the exp2 domain; O is rescaled only when the row max
                // grows by more than 2^8
                // row max: four independent chains of three-input maxima
                float mx[4];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    float a = fmax3(s[16 * g], s[16 * g + 1], s[16 * g + 2]);
#pragma unroll
                    for (int c = 16 * g + 3; c < 16 * g + 15; c += 2) a = fmax3(a, s[c], s[c + 1]);
                    mx[g] = fmaxf(a, s[16 * g + 15]);
                }
                const float m_new = fmax3(mx[0], mx[1], fmaxf(mx[2], mx[3])) * sl2;
                if (m_new > m_used + 8.f) {
                    alpha = fast_exp2(m_used - m_new);
                    m_used = m_new;
                    resc = true;
                }
                const float neg_m = (m_used == sp_neg_inf()) ? 0.f : -m_used;
                const uint64_t sl2x2 = f2_pack(sl2, sl2), negm2 = f2_pack(neg_m, neg_m);
                uint64_t sum2 = f2_pack(0.f, 0.f);
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        float x0, x1;
                        f2_unpack(f2_fma(f2_pack(s[c * 32 + 2 * k], s[c * 32 + 2 * k + 1]), sl2x2, negm2),
                                  x0, x1);
                        const float p0 = fast_exp2(x0);
                        const float p1 = fast_exp2(x1);
                        sum2 = f2_add(sum2, f2_pack(p0, p1));
                        pk[k] = pack_bf16x2(p0, p1);
                    }
                    tmem_st16(s_addr + c * 16, pk);
                }
                float sum0, sum1;
                f2_unpack(sum2, sum0, sum1);
                l = l * alpha + (sum0 + sum1);
            }
            // P_{j-1} V_{j-1} must be complete before O is rescaled, and before P_j is
            // handed over (this also keeps every barrier below one phase ahead at most).
            if (j > 0) {
                if (!warp_wait(bar(C::BAR_ODONE), (j - 1) & 1, abort_flag, p.wait_limit_ns,
                               p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (__any_sync(0xffffffffu, resc)) {
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t v[32];
                        tmem_ld32(trow + C::O_COL + c * 32, v);
                        tmem_wait_ld();
                        reg_fence32(v);
#pragma unroll
                        for (int k = 0; k < 32; ++k)
                            v[k] = __float_as_uint(__uint_as_float(v[k]) * alpha);
                        tmem_st32(trow + C::O_COL + c * 32, v);
                    }
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(C::BAR_PFULL));
        }

        // epilogue
        const int row = qt * SP_BM + r;
        const bool row_in = row < p.Sq;
        bool have = ok && n > 0;
        if (have && !warp_wait(bar(C::BAR_ODONE), (n - 1) & 1, abort_flag, p.wait_limit_ns, p.status))
            have = false;
        const bool out_valid = have && l > 0.f;
        const float inv_l = out_valid ? 1.f / l : 0.f;
        __nv_bfloat16 *orow = p.O + ((long long)(b * p.Hq + hq) * p.Sq + row) * D;
        if (have) {
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(trow + C::O_COL + c * 32, v);
                tmem_wait_ld();
                reg_fence32(v);
                uint32_t o16[16];
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    o16[k] = out_valid ? pack_bf16x2(__uint_as_float(v[2 * k]) * inv_l,
                                                     __uint_as_float(v[2 * k + 1]) * inv_l)
                                       : 0u;
                if (row_in) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        dst[k] = make_uint4(o16[4 * k], o16[4 * k + 1], o16[4 * k + 2], o16[4 * k + 3]);
                }
            }
        } else if (row_in && !*abort_flag) {
            uint4 *dst = reinterpret_cast<uint4 *>(orow);
#pragma unroll
            for (int k = 0; k < D / 8; ++k) dst[k] = make_uint4(0, 0, 0, 0);
        }
        if (row_in && p.LSE && !*abort_flag)
            p.LSE[(long long)(b * p.Hq + hq) * p.Sq + row] =
                out_valid ? m_used * 0.69314718055994531f + logf(l) : sp_neg_inf();
    }

    // ---- teardown ----
    if (*abort_flag) drain_delay(2000000);  // let copies / MMAs in flight land
    tc_fence_before();
    __syncthreads();
    if (warp == kSpWarpMma) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kSpTmemCols);
    }
}

template <int D>
attn_status_t launch_bsparse_d(const FwdArgs &a, cudaStream_t stream) {
    using C = SpCfg<D>;
    CUtensorMap tq, tk, tv;
    attn_status_t st;
    if ((st = make_tmap_bf16_3d(&tq, a.Q, D, a.Sq, (uint64_t)a.B * a.Hq, SP_BM)) != ATTN_OK) return st;
    if ((st = make_tmap_bf16_3d(&tk, a.K, D, a.Sk, (uint64_t)a.B * a.Hkv, SP_BN)) != ATTN_OK) return st;
    if ((st = make_tmap_bf16_3d(&tv, a.V, D, a.Sk, (uint64_t)a.B * a.Hkv, SP_BN)) != ATTN_OK) return st;
    const void *fn = reinterpret_cast<const void *>(attn_fwd_bsparse_kernel<D>);
    if (kernel_setup(fn, C::SMEM_BYTES, -1, true) != cudaSuccess) return ATTN_ERR_CUDA;
    SpParams p;
    p.O = static_cast<__nv_bfloat16 *>(a.O);
    p.LSE = a.LSE;
    p.bmask = a.block_mask;
    p.per_head = a.block_mask_per_head;
    p.B = a.B;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.Sq = a.Sq;
    p.Sk = a.Sk;
    p.group = a.Hq / a.Hkv;
    p.n_qt = (a.Sq + SP_BM - 1) / SP_BM;
    p.n_qb = (a.Sq + 63) / 64;
    p.n_kb = (a.Sk + 63) / 64;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.wait_limit_ns = kWaitLimitNs;
    p.status = device_status_word();
    if (!p.status) return ATTN_ERR_CUDA;
    const long long grid = (long long)p.n_qt * a.Hq * a.B;
    if (grid == 0) return ATTN_OK;
    if (grid > 0x7fffffffll) return ATTN_ERR_INVALID;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(kSpThreads, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, attn_fwd_bsparse_kernel<D>, tq, tk, tv, p) != cudaSuccess)
        return ATTN_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

bool bsparse_eligible(const FwdArgs &a) {
    return a.flex && a.block_mask && !a.doc_q && !a.doc_kv && a.softcap == 0.f && !a.alibi_slopes &&
           !a.causal && a.window == 0 && !a.k_lengths && !a.q_lengths && a.Sk > 0 &&
           (a.Sk + 63) / 64 <= kBsparseMaxKvBlocks;
}

attn_status_t launch_fwd_bsparse(const FwdArgs &a, cudaStream_t stream) {
    if (a.D == 128) return launch_bsparse_d<128>(a, stream);
    if (a.D == 64) return launch_bsparse_d<64>(a, stream);
    return ATTN_ERR_UNSUPPORTED;
}

}  // namespace gqa
