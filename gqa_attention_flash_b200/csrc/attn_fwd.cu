// attn_fwd.cu -- fused GQA attention forward for sm_100a.
//
// Computes the rows of O = softmax(Q K^T * scale + mask) V and their
// log-sum-exp, as defined on the Tylo.jl "Primitives" page (entry `attention!`:
// fused MHA with GQA, causal, input_pos, k_lengths / q_lengths, saved softmax
// statistics M/L, Float32 accumulation) with the sliding window of the
// mlx-arsenal "Attention" page (entry `sliding_window_mask`).
//
// Work item: a pair of 128-row query tiles of one (query head, batch).  The grid
// has one CTA per item, in launch order heaviest causal pairs first with the
// query heads of one KV group adjacent.  When every item does the same work (no
// causal mask, no window) and the last round of items would fill at most half of
// the SMs, those last pairs run as two single-tile items each, so that round is
// twice as wide (64x64-token image workload: 0.305 -> 0.294 ms, bitwise the same).
// The kernel is persistent: a running
// CTA takes over the items of CTAs not yet launched (cluster launch control), so
// about one CTA per SM runs and the next item's Q and first K/V tiles load and its
// first S products run while the current item finishes.  The two query tiles of
// an item share every K/V tile the CTA loads, and their softmax runs alternate with
// the tensor core (while warpgroup 0 turns S0 into P0, the tensor core computes
// P1 V and the next S1, and the other way round).  12 warps:
//   warps 0-3  softmax of query tile 0 (one row per thread = TMEM lane)
//   warps 4-7  softmax of query tile 1
//   warp 8     TMA producer and work scheduler: the query tiles of each item
//              into a ring of three Q slots, K_j / V_j into an NS-stage ring, the
//              launch-control request for the next item and its hand-over to the
//              other roles
//   warp 9     MMA issuer (one thread) and TMEM owner:
//              S_t = Q_t K_j^T (smem x smem -> TMEM), O_t += P_t V_j (P_t read
//              from TMEM, written there by the softmax over S_t)
//   warps 10-11 idle
// The block launches with 168 registers per thread; the producer warpgroup
// (warps 8-11) drops to 88 and the two softmax warpgroups rise to 208
// (128 * 88 + 256 * 208 = 384 * 168).  Every translation unit is compiled as a
// whole program: with relocatable device code ptxas would ignore setmaxnreg.
// TMEM (512 columns): S0 | S1 | O0 | O1.  Each query tile visits only the KV
// tiles that hold a key it can see (whole-tile skipping for causal, window and
// length masks -- Tylo `flex_attention!` keyword block_sparse); the
// per-element mask is applied on boundary tiles only.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace gqa {

namespace {

constexpr int BM = 128;         // query rows per query tile (= TMEM lanes)
constexpr int BN = 128;         // keys per KV tile
constexpr int kTiles = 2;       // query tiles per CTA
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;     // per thread at launch (checked on the host)
constexpr int kListMax = kFlexMaxKvTiles;  // flex: KV tiles per CTA list
constexpr uint32_t kProducerRegs = 88;
constexpr uint32_t kSoftmaxRegs = 208;
static_assert(128 * kProducerRegs + 256 * kSoftmaxRegs <= kThreads * kLaunchRegs,
              "register split must use exactly the launch allocation");

template <int D, bool kList>
struct FwdCfg {
    static constexpr int NS = (D == 128) ? 2 : 4;  // K/V ring depth
    // Q tile slots.  Persistent CTAs rotate the tiles of consecutive work items
    // through three slots, so the next item's first query tile loads while the
    // current item still runs; a flex list CTA handles one item and needs two.
    static constexpr int NQ = kList ? 2 : 3;
    static constexpr int NBOX = D / 64;             // 64-column TMA boxes per row
    static constexpr int BOX = 128 * 128;            // bytes of one (128 rows x 64 cols) box
    static constexpr int Q_BYTES = BM * D * 2;       // one query tile
    static constexpr int KV_BYTES = BN * D * 2;      // one K or V tile
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + NQ * Q_BYTES;
    static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + NS * KV_BYTES;
    static constexpr int BAR_QFULL = 0;              // [NQ] Q slot loaded
    static constexpr int BAR_QFREE = NQ;             // [NQ] last S MMA reading the slot done
    static constexpr int BAR_KFULL = 2 * NQ;         // [NS]
    static constexpr int BAR_VFULL = 2 * NQ + NS;    // [NS]
    static constexpr int BAR_EMPTY = 2 * NQ + 2 * NS;  // [NS]
    static constexpr int BAR_SFULL = 2 * NQ + 3 * NS;  // [2]
    static constexpr int BAR_PFULL = BAR_SFULL + 2;    // [2]
    static constexpr int BAR_ODONE = BAR_PFULL + 2;    // [2]
    static constexpr int BAR_CLC = BAR_ODONE + 2;      // [2] launch-control responses
    static constexpr int BAR_IFULL = BAR_CLC + 2;      // [2] next-item slots
    static constexpr int BAR_IEMPTY = BAR_IFULL + 2;   // [2]
    static constexpr int N_BARS = BAR_IEMPTY + 2;
    static constexpr int OFF_CLC = (OFF_BAR + N_BARS * 8 + 15) / 16 * 16;  // 2 x 16-byte responses
    static constexpr int OFF_ITEM = OFF_CLC + 32;                         // 2 x next item index
    static constexpr int OFF_MISC = OFF_ITEM + 16;                        // tmem slot, abort flag
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
    // flex_attention! only: count + list of the KV tiles the CTA visits
    // and, per query tile, the entries it uses
    static constexpr int OFF_LIST = OFF_MISC + 16;
    static constexpr int OFF_TLIST = OFF_LIST + 4 * (kListMax + 1);  // [2]
    static constexpr int SMEM_BYTES_FLEX = OFF_TLIST + 2 * 4 * (kListMax + 1) + 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    // consumers of a next-item slot: the MMA thread and lane 0 of each softmax warp
    static constexpr uint32_t ITEM_READERS = 1 + 8;
    __host__ __device__ static constexpr uint32_t s_col(int t) { return t * BN; }
    __host__ __device__ static constexpr uint32_t o_col(int t) { return 2 * BN + t * D; }
};
static_assert(FwdCfg<128, false>::SMEM_BYTES <= 232448, "forward shared memory above 227 KB");
static_assert(FwdCfg<128, true>::SMEM_BYTES_FLEX <= 232448, "flex shared memory above 227 KB");
static_assert(FwdCfg<64, true>::SMEM_BYTES_FLEX <= 232448, "flex shared memory above 227 KB");

struct FwdParams {
    __nv_bfloat16 *O;
    float *LSE;
    const int32_t *k_lengths;
    const int32_t *q_lengths;
    int B, Hq, Hkv, Sq, Sk, group, n_pairs;
    int n_split;       // the last n_split pair items run as two single-tile items each
    float scale_log2;  // scale * log2(e)
    int causal, window, input_pos;
    uint64_t wait_limit_ns;
    int *status;  // device status word
    // flex_attention! (read only by the flex instantiation)
    float scale;             // natural-log scale of the scores
    float softcap;           // > 0: SoftCapScore(cap)
    float softcap_k;         // scale / cap
    float softcap_c;         // cap log2(e)
    const float *alibi;      // AliBiScore slopes, one per query head, or null
    const int32_t *doc_q;    // DocumentMask ids per local query row, or null
    const int32_t *doc_kv;   // ... per key, or null
    const uint8_t *bmask;    // BlockMask states of 64x64 blocks (n_qb, n_kb), or null
    int n_qb, n_kb;
    int bmask_per_head;      // bmask holds one (n_qb, n_kb) matrix per (batch, query head)
};

// flex_attention!: 2-bit states of the four 64x64 blocks of the 128x128 tile
// (query tile qt, KV tile u): 0 = nothing visible, 1 = some pairs visible (apply
// the document mask), 2 = every pair the block mask covers is visible.  State of
// block (query half qs, key half ks) sits at bits 2 * (2 qs + ks).  Blocks past
// the ends of the BlockMask are 0.
__device__ __forceinline__ uint32_t flex_states(const FwdParams &p, const uint8_t *bm, int qt,
                                                int u) {
    uint32_t st = 0;
#pragma unroll
    for (int qs = 0; qs < 2; ++qs)
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            const int qb = 2 * qt + qs, kb = 2 * u + ks;
            uint32_t v = 0;
            if (qb < p.n_qb && kb < p.n_kb) {
                if (bm) {
                    const uint32_t m = bm[(size_t)qb * p.n_kb + kb];
                    v = m == 0 ? 0u : (m == 2 ? 2u : 1u);
                } else {
                    v = p.doc_q ? 1u : 2u;
                }
            }
            st |= v << (2 * (2 * qs + ks));
        }
    return st;
}

// SoftCapScore in log2 units for a raw dot product d (s = scale d):
//   cap tanh(s / cap) log2e = c tanh(k d),  k = scale / cap,  c = cap log2e,
// with the hyperbolic tangent of the special-function unit (tanh.approx.f32): one
// operation per score instead of an exp2 and a reciprocal (18 % faster on the
// soft-capped document workload), within the parity tolerances of every soft-capped
// test case (caps 2 to 50).  The softmax keeps t = tanh(k d) and applies c in the
// exponent's FMA and to the row max (c > 0, so max(c t) = c max(t)): one multiply
// per score fewer (LLM shape with a cap of 50: 0.856 -> 0.821 ms).
__device__ __forceinline__ float tanh_approx(float x) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(x));
    return t;
}

// a * b on both fp32 halves of a packed pair.
__device__ __forceinline__ uint64_t f2_mul_fwd(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }

// One work item: a pair of 128-row query tiles of one (query head, batch) and
// the KV tiles they see.
struct FwdItem {
    int pair, hq, b, hkv;
    int qt0;                 // query tile of the item's tile 0 (tile 1 is qt0 + 1)
    bool single;             // one query tile only (a split pair): tile 1 is not the item's
    int k_end, q_end;
    int lo0, hi0, lo1, hi1;  // KV tiles [lo_t, hi_t) that query tile t sees
    int ql0, ql1;            // last valid row of query tile t
    int u_lo, u_hi, n_u;     // KV tiles the item loads (union of both ranges)
    bool act0, act1;         // query tile t sees at least one key
    bool rev;                // KV tiles visited last to first (ALiBi, negative slope)
};

__device__ __forceinline__ bool item_uses(const FwdItem &it, int t, int u) {
    return t ? (u >= it.lo1 && u < it.hi1) : (u >= it.lo0 && u < it.hi0);
}

// Work item w, in launch order: heaviest causal query-tile pairs first, the query
// heads of one KV group adjacent (they share K/V through L2).  Step a1: the
// visible KV tile range of each query tile (whole-tile skipping).
template <int kMode>
__device__ __forceinline__ void fwd_item(const FwdParams &p, int w, FwdItem &it, bool report) {
    // The last n_split pair items of the launch order are split in two: item
    // n_full + 2 x + h is query tile h of pair item n_full + x.
    const int n_full = p.n_pairs * p.Hq * p.B - p.n_split;
    int half = 0;
    it.single = false;
    if (w >= n_full) {
        half = (w - n_full) & 1;
        w = n_full + ((w - n_full) >> 1);
        it.single = true;
    }
    it.hq = w % p.Hq;
    w /= p.Hq;
    it.b = w % p.B;
    w /= p.B;
    it.pair = p.n_pairs - 1 - w;
    it.qt0 = it.pair * kTiles + half;
    it.hkv = it.hq / p.group;
    int k_end = p.Sk, q_end = p.Sq;
    if (p.k_lengths) {
        int kl = p.k_lengths[it.b];
        if (kl > p.Sk) {
            if (report && it.hq == 0 && it.pair == 0) record_status(p.status, ATTN_ERR_DEVICE_BOUNDS);
            kl = p.Sk;
        }
        k_end = kl > 0 ? kl : 0;
    }
    if (p.q_lengths) {
        int ql = p.q_lengths[it.b];
        if (ql > p.Sq) {
            if (report && it.hq == 0 && it.pair == 0) record_status(p.status, ATTN_ERR_DEVICE_BOUNDS);
            ql = p.Sq;
        }
        q_end = ql > 0 ? ql : 0;
    }
    it.k_end = k_end;
    it.q_end = q_end;
    // Tile t (0, 1) covers rows [q0_t, q0_t + 128) and sees KV tiles [lo_t, hi_t).
#pragma unroll
    for (int t = 0; t < kTiles; ++t) {
        const int q0 = (it.qt0 + t) * BM;
        int lo_t = 0, hi_t = 0, qlast = q0;
        if (q0 < q_end && k_end > 0 && !(t == 1 && it.single)) {
            qlast = min(q0 + BM - 1, q_end - 1);
            long long hi = k_end;
            if (p.causal) hi = min(hi, (long long)p.input_pos + qlast + 1);
            long long lo = 0;
            if (p.window > 0) lo = max(0ll, (long long)p.input_pos + q0 - p.window + 1);
            if (hi > lo) {
                lo_t = static_cast<int>(lo / BN);
                hi_t = static_cast<int>((hi + BN - 1) / BN);
            }
        }
        if (t == 0) { it.lo0 = lo_t; it.hi0 = hi_t; it.ql0 = qlast; }
        else { it.lo1 = lo_t; it.hi1 = hi_t; it.ql1 = qlast; }
    }
    it.act0 = it.hi0 > it.lo0;
    it.act1 = it.hi1 > it.lo1;
    it.u_lo = it.act0 ? (it.act1 ? min(it.lo0, it.lo1) : it.lo0) : it.lo1;
    it.u_hi = it.act0 ? (it.act1 ? max(it.hi0, it.hi1) : it.hi0) : it.hi1;
    it.n_u = (it.act0 || it.act1) ? it.u_hi - it.u_lo : 0;
    // AliBiScore with a negative slope: the bias grows towards the query, so the
    // KV tiles are visited nearest first; the running max is then found at once
    // and the lazy rescale of O stays rare.  (The softmax does not depend on the
    // visiting order.)
    it.rev = false;
    if constexpr (kMode == 3) it.rev = p.alibi[it.hq] < 0.f;
}

// kMode: score mod of flex_attention!: 0 = none, 2 = SoftCapScore, 3 = AliBiScore.
// kList: the CTA visits the KV tiles of a per-CTA list built from the BlockMask
// and applies the block states / DocumentMask per element; without it, the KV
// tiles of the analytic ranges in order (attention! is <D, 0, false>).
//
// Without a list the kernel is persistent: the grid has one CTA per work item,
// but a running CTA takes over the items of CTAs not yet launched (cluster launch
// control), in launch order, so about one CTA per SM runs and the next item's Q
// and first K/V tiles load and its first S products run while the current item
// finishes.  Every barrier phase below is counted across items.
template <int D, int kMode, bool kList>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
    using C = FwdCfg<D, kList>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8 * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    volatile int *item_slot = reinterpret_cast<volatile int *>(smem + C::OFF_ITEM);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    FwdItem it;
    // flex: [0] = number of KV tiles the CTA visits, then one entry per tile:
    // bits 0-15 the KV tile index, bits 16-23 / 24-31 the block states of query
    // tile 0 / 1 (0 when that query tile skips the KV tile).
    uint32_t *kv_list = reinterpret_cast<uint32_t *>(smem + C::OFF_LIST);
    // per query tile t: [0] = count, then entries g | u << 10 | states << 20 |
    // (query tile 0 uses it) << 28, in visiting order
    uint32_t *tile_list = reinterpret_cast<uint32_t *>(smem + C::OFF_TLIST);

    // ---- set-up ----
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NQ; ++s) {
            mbar_init(bar(C::BAR_QFULL + s), 1);
            mbar_init(bar(C::BAR_QFREE + s), 1);
        }
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(bar(C::BAR_KFULL + s), 1);
            mbar_init(bar(C::BAR_VFULL + s), 1);
            mbar_init(bar(C::BAR_EMPTY + s), 1);
        }
        for (int t = 0; t < kTiles; ++t) {
            mbar_init(bar(C::BAR_SFULL + t), 1);
            mbar_init(bar(C::BAR_PFULL + t), BM);
            mbar_init(bar(C::BAR_ODONE + t), 1);
            mbar_init(bar(C::BAR_CLC + t), 1);
            mbar_init(bar(C::BAR_IFULL + t), 1);
            mbar_init(bar(C::BAR_IEMPTY + t), C::ITEM_READERS);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    // Programmatic dependent launch: the launch and the set-up above overlap the
    // previous kernel on the stream; every global read or write below comes after
    // that kernel has finished.  The next kernel may start its own set-up at once
    // (its wait covers all of this grid).
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if constexpr (kList) {
        fwd_item<kMode>(p, blockIdx.x, it, false);
        // The KV tiles this CTA visits: inside a query tile's analytic range and
        // holding a visible block (BlockMask of flex_attention!), in order.
        if (warp == kWarpTma) {
            const uint8_t *bm = p.bmask;
            if (bm && p.bmask_per_head) bm += (size_t)(it.b * p.Hq + it.hq) * p.n_qb * p.n_kb;
            int count = 0;
            for (int base = it.u_lo; it.n_u > 0 && base < it.u_hi; base += 32) {
                const int u = base + lane;
                uint32_t e = 0;
                if (u < it.u_hi) {
                    const uint32_t s0 = item_uses(it, 0, u) ? flex_states(p, bm, it.qt0, u) : 0u;
                    const uint32_t s1 =
                        item_uses(it, 1, u) ? flex_states(p, bm, it.qt0 + 1, u) : 0u;
                    if (s0 | s1) e = static_cast<uint32_t>(u) | (s0 << 16) | (s1 << 24);
                }
                const uint32_t vote = __ballot_sync(0xffffffffu, e != 0);
                if (e != 0) kv_list[1 + count + __popc(vote & ((1u << lane) - 1u))] = e;
                count += __popc(vote);
            }
            if constexpr (kMode == 3) {
                if (it.rev) {
                    __syncwarp();
                    for (int j = lane; j < count / 2; j += 32) {
                        const uint32_t x = kv_list[1 + j];
                        kv_list[1 + j] = kv_list[count - j];
                        kv_list[count - j] = x;
                    }
                    __syncwarp();
                }
            }
            __syncwarp();
#pragma unroll
            for (int t = 0; t < kTiles; ++t) {
                uint32_t *tl = tile_list + t * (kListMax + 1);
                int n_t_list = 0;
                for (int base = 0; base < count; base += 32) {
                    const int g = base + lane;
                    uint32_t x = 0;
                    bool use = false;
                    if (g < count) {
                        const uint32_t e = kv_list[1 + g];
                        const uint32_t st = (e >> (16 + 8 * t)) & 0xFFu;
                        use = st != 0;
                        x = static_cast<uint32_t>(g) | ((e & 0x3FFu) << 10) | (st << 20) |
                            ((((e >> 16) & 0xFFu) != 0 ? 1u : 0u) << 28);
                    }
                    const uint32_t vote = __ballot_sync(0xffffffffu, use);
                    if (use) tl[1 + n_t_list + __popc(vote & ((1u << lane) - 1u))] = x;
                    n_t_list += __popc(vote);
                }
                if (lane == 0) tl[0] = static_cast<uint32_t>(n_t_list);
            }
            if (lane == 0) kv_list[0] = static_cast<uint32_t>(count);
        }
    }
    if (warp == kWarpMma) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // KV tiles the current item loads (the flex list CTA handles one item)
    auto n_loads = [&](const FwdItem &x) -> int {
        return kList ? static_cast<int>(kv_list[0]) : x.n_u;
    };

    if (warp >= 8) {
      regs_dec<kProducerRegs>();
      fwd_item<kMode>(p, blockIdx.x, it, false);
      if (warp == kWarpTma) {
        // ===================== TMA producer and work scheduler =====================
        if (lane == 0) {
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            // L2 policies: each Q tile is read once (evict first); the K / V tiles of a
            // KV head serve every query tile and query head of its group (evict last).
            // DRAM traffic of the LLM workload: 393 -> 335 MB per launch (322 MB of
            // inputs and outputs), at the same speed.
            const uint64_t pol_q = l2_policy_evict_first(), pol_kv = l2_policy_evict_last();
            bool more = !kList;  // launch-control requests still allowed
            bool ok = true;
            uint32_t qi = 0;     // Q tiles loaded so far: slot qi % NQ, use qi / NQ
            uint32_t gi = 0;     // K/V ring entries loaded so far
            for (int k = 0;; ++k) {
                const int cs = k & 1;
                if (more) {  // ask for the next item now; the answer is read after the loads
                    mbar_arrive_expect_tx(bar(C::BAR_CLC + cs), 16);
                    clc_try_cancel(sbase + C::OFF_CLC + 16 * cs, bar(C::BAR_CLC + cs));
                }
                const int n_load = n_loads(it);
                auto load_q = [&](int t) -> bool {
                    // checked build: the query tile lies inside Q
                    if (!in_range(box_ok(0, (it.qt0 + t) * BM, it.b * p.Hq + it.hq, D, p.Sq,
                                         (long long)p.B * p.Hq, BM) &&
                                      it.pair >= 0 && it.pair < p.n_pairs,
                                  p.status, abort_flag))
                        return false;
                    const uint32_t slot = qi % C::NQ, use = qi / C::NQ;
                    if (use > 0 && !mbar_wait(bar(C::BAR_QFREE + slot), (use - 1) & 1, abort_flag,
                                              p.wait_limit_ns, p.status))
                        return false;
                    mbar_arrive_expect_tx(bar(C::BAR_QFULL + slot), C::Q_BYTES);
                    for (int c = 0; c < C::NBOX; ++c)
                        tma_load_3d_hint(sbase + C::OFF_Q + slot * C::Q_BYTES + c * C::BOX, &tmQ,
                                         bar(C::BAR_QFULL + slot), c * 64, (it.qt0 + t) * BM,
                                         it.b * p.Hq + it.hq, pol_q);
                    ++qi;
                    return true;
                };
                auto load_kv = [&](int g) -> bool {
                    const uint32_t st = gi % C::NS, use = gi / C::NS;
                    if (use > 0 && !mbar_wait(bar(C::BAR_EMPTY + st), (use - 1) & 1, abort_flag,
                                              p.wait_limit_ns, p.status))
                        return false;
                    const int kv_row =
                        (kList ? static_cast<int>(kv_list[1 + g] & 0xFFFFu)
                               : (it.rev ? it.u_hi - 1 - g : it.u_lo + g)) * BN;
                    // checked build: the K / V tile lies inside K and V
                    if (!in_range(box_ok(0, kv_row, it.b * p.Hkv + it.hkv, D, p.Sk,
                                         (long long)p.B * p.Hkv, BN) &&
                                      kv_row >= 0 && kv_row < p.Sk,
                                  p.status, abort_flag))
                        return false;
                    mbar_arrive_expect_tx(bar(C::BAR_KFULL + st), C::KV_BYTES);
                    for (int c = 0; c < C::NBOX; ++c)
                        tma_load_3d_hint(sbase + C::OFF_K + st * C::KV_BYTES + c * C::BOX, &tmK,
                                         bar(C::BAR_KFULL + st), c * 64, kv_row,
                                         it.b * p.Hkv + it.hkv, pol_kv);
                    mbar_arrive_expect_tx(bar(C::BAR_VFULL + st), C::KV_BYTES);
                    for (int c = 0; c < C::NBOX; ++c)
                        tma_load_3d_hint(sbase + C::OFF_V + st * C::KV_BYTES + c * C::BOX, &tmV,
                                         bar(C::BAR_VFULL + st), c * 64, kv_row,
                                         it.b * p.Hkv + it.hkv, pol_kv);
                    ++gi;
                    return true;
                };
                if (ok && n_load > 0) {
                    // Q0, the first K/V tile, then Q1 (its slot may still be in use by
                    // the previous item's last S products) and the other K/V tiles.
                    if (it.act0) ok = load_q(0);
                    if (ok) ok = load_kv(0);
                    if (ok && it.act1) ok = load_q(1);
                    for (int g = 1; ok && g < n_load; ++g) ok = load_kv(g);
                }
                int wn = -1;
                if (more) {
                    if (ok && mbar_wait(bar(C::BAR_CLC + cs), (k >> 1) & 1, abort_flag,
                                        p.wait_limit_ns, p.status)) {
                        wn = clc_cancelled_x(sbase + C::OFF_CLC + 16 * cs);
                        fence_proxy_async_smem();  // the slot is rewritten by a later request
                        if (wn >= static_cast<int>(gridDim.x)) {  // never expected: stop safely
                            record_status(p.status, ATTN_ERR_DEVICE_BOUNDS);
                            wn = -1;
                        }
                    } else {
                        ok = false;
                    }
                    if (wn < 0) more = false;
                }
                // hand the next item (or -1 = stop) to the MMA thread and the softmax warps
                if (k >= 2 && !mbar_wait(bar(C::BAR_IEMPTY + cs), ((k - 2) >> 1) & 1, abort_flag,
                                         p.wait_limit_ns, p.status))
                    ok = false;
                item_slot[cs] = ok ? wn : -1;
                mbar_arrive(bar(C::BAR_IFULL + cs));
                if (!ok || wn < 0) break;
                fwd_item<kMode>(p, wn, it, false);
            }
        }
      } else if (warp == kWarpMma) {
        // ===================== MMA issuer =====================
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16_f32(BM, BN, 0, 0);
            constexpr uint32_t idO = idesc_bf16_f32(BM, D, 0, 1);
            bool ok = true;
            uint32_t qi = 0;                // Q tiles consumed so far (same order as loaded)
            uint32_t gi = 0;                // ring entries of the previous items
            uint32_t npv0 = 0, npv1 = 0;    // P_t handed over so far (P_FULL phases)
            for (int k = 0; ok; ++k) {
                const int n_load = n_loads(it);
                // Q slot of each active tile; waited for at its first S product
                uint32_t qs0 = 0, qs1 = 0, qu0 = 0, qu1 = 0;
                if (it.act0) { qs0 = qi % C::NQ; qu0 = qi / C::NQ; ++qi; }
                if (it.act1) { qs1 = qi % C::NQ; qu1 = qi / C::NQ; ++qi; }
                bool qr0 = false, qr1 = false;
                // g: index of the KV tile in the item's load order; i: the query tile's
                // own iteration index within the item.
                auto issue_s = [&](int t, int g, bool last) -> bool {
                    const uint32_t qs = t ? qs1 : qs0;
                    if (!(t ? qr1 : qr0)) {
                        if (!mbar_wait(bar(C::BAR_QFULL + qs), (t ? qu1 : qu0) & 1, abort_flag,
                                       p.wait_limit_ns, p.status))
                            return false;
                        if (t) qr1 = true; else qr0 = true;
                    }
                    const uint32_t ge = gi + g;
                    const int st = ge % C::NS;
                    if (!mbar_wait(bar(C::BAR_KFULL + st), (ge / C::NS) & 1, abort_flag,
                                   p.wait_limit_ns, p.status))
                        return false;
                    tc_fence_after();
                    const uint32_t qa = sbase + C::OFF_Q + qs * C::Q_BYTES;
                    const uint32_t ka = sbase + C::OFF_K + st * C::KV_BYTES;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                        mma_ss(tmem + C::s_col(t), smem_desc_sw128(qa + off, 16, 1024),
                               smem_desc_sw128(ka + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(bar(C::BAR_SFULL + t));
                    if (!kList && last) mma_commit(bar(C::BAR_QFREE + qs));  // slot free for a later item
                    return true;
                };
                auto issue_pv = [&](int t, int g, int i) -> bool {
                    const uint32_t ge = gi + g;
                    const int st = ge % C::NS;
                    const uint32_t np = t ? npv1++ : npv0++;
                    if (!mbar_wait(bar(C::BAR_PFULL + t), np & 1, abort_flag, p.wait_limit_ns, p.status))
                        return false;
                    if (!mbar_wait(bar(C::BAR_VFULL + st), (ge / C::NS) & 1, abort_flag,
                                   p.wait_limit_ns, p.status))
                        return false;
                    tc_fence_after();
                    const uint32_t va = sbase + C::OFF_V + st * C::KV_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk)
                        mma_ts(tmem + C::o_col(t), tmem + C::s_col(t) + kk * 8,
                               smem_desc_sw128(va + kk * 16 * 128, C::BOX, 1024), idO,
                               (i > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(bar(C::BAR_ODONE + t));
                    return true;
                };
                if (n_load > 0) {
                    if constexpr (!kList) {
                        // last KV tile of query tile t in visiting order
                        auto last_of = [&](int t, int u) -> bool {
                            return it.rev ? u == (t ? it.lo1 : it.lo0) : u == (t ? it.hi1 : it.hi0) - 1;
                        };
                        const int u_first = it.rev ? it.u_hi - 1 : it.u_lo;
#pragma unroll
                        for (int t = 0; t < kTiles; ++t)
                            if (ok && item_uses(it, t, u_first)) ok = issue_s(t, 0, last_of(t, u_first));
                        for (int g = 0; ok && g < it.n_u; ++g) {
                            const int u = it.rev ? it.u_hi - 1 - g : it.u_lo + g;
                            const int un = it.rev ? u - 1 : u + 1;
#pragma unroll
                            for (int t = 0; t < kTiles; ++t) {
                                if (ok && item_uses(it, t, u))
                                    ok = issue_pv(t, g, it.rev ? (t ? it.hi1 : it.hi0) - 1 - u
                                                               : u - (t ? it.lo1 : it.lo0));
                                if (ok && g + 1 < it.n_u && item_uses(it, t, un))
                                    ok = issue_s(t, g + 1, last_of(t, un));
                            }
                            if (ok) mma_commit(bar(C::BAR_EMPTY + (gi + g) % C::NS));
                        }
                    } else {
                        // Same order over the listed KV tiles: P_t V_g, then S_t for the next
                        // listed tile when tile t uses it; a tile that resumes after a gap
                        // issues its S when its next listed tile comes up.
                        int it0 = 0, it1 = 0;
                        bool sq0 = false, sq1 = false;  // S of tile t already issued for this g
                        for (int g = 0; ok && g < n_load; ++g) {
                            const uint32_t e = kv_list[1 + g];
                            const uint32_t en = g + 1 < n_load ? kv_list[2 + g] : 0u;
#pragma unroll
                            for (int t = 0; t < kTiles; ++t) {
                                if (!ok || ((e >> (16 + 8 * t)) & 0xFFu) == 0) continue;
                                if (!(t ? sq1 : sq0)) ok = issue_s(t, g, false);
                                if (ok) ok = issue_pv(t, g, t ? it1 : it0);
                                if (t) ++it1; else ++it0;
                                const bool next = ok && ((en >> (16 + 8 * t)) & 0xFFu) != 0;
                                if (next) ok = issue_s(t, g + 1, false);
                                if (t) sq1 = next; else sq0 = next;
                            }
                            if (ok) mma_commit(bar(C::BAR_EMPTY + (gi + g) % C::NS));
                        }
                    }
                }
                gi += n_load;
                // next item (or -1 = stop)
                if (!ok || !mbar_wait(bar(C::BAR_IFULL + (k & 1)), (k >> 1) & 1, abort_flag,
                                      p.wait_limit_ns, p.status))
                    break;
                const int wn = item_slot[k & 1];
                mbar_arrive(bar(C::BAR_IEMPTY + (k & 1)));
                if (wn < 0) break;
                fwd_item<kMode>(p, wn, it, false);
            }
        }
      }
    } else {
        // ===================== softmax / correction / epilogue =====================
        regs_inc<kSoftmaxRegs>();
        fwd_item<kMode>(p, blockIdx.x, it, threadIdx.x == 0);
        const int t = warp >> 2;                 // query tile of this warpgroup
        const int r = threadIdx.x & (BM - 1);    // row within the tile = TMEM lane
        const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const uint32_t s_addr = trow + (t ? C::s_col(1) : C::s_col(0));
        const uint32_t o_addr = trow + (t ? C::o_col(1) : C::o_col(0));
        const uint32_t bar_s = bar(C::BAR_SFULL + t), bar_p = bar(C::BAR_PFULL + t),
                       bar_o = bar(C::BAR_ODONE + t);
        // Factor from the values the softmax holds to log2 units, applied to the row max
        // and in the exponent's FMA: scale log2 e for raw scores; for the soft cap, whose
        // values are tanh(k d), the cap c = cap log2 e; 1 for ALiBi, whose scale is folded
        // into its scores before the max.
        const float sl2 = kMode == 2 ? p.softcap_c : (kMode == 3 ? 1.f : p.scale_log2);
        const uint32_t *my_list = tile_list + t * (kListMax + 1);
        bool ok = true;
        uint32_t n_it = 0;  // S_t tiles of the previous items (S_FULL / O_DONE phases)
        uint32_t gi = 0;    // ring entries of the previous items
        for (int k = 0;; ++k) {
            const int row = (it.qt0 + t) * BM + r;
            const int q0 = (it.qt0 + t) * BM;
            const long long pos = (long long)p.input_pos + row;  // absolute position
            // this tile's range, selected without runtime-indexed arrays
            const int my_lo = t ? it.lo1 : it.lo0;
            const int my_hi = t ? it.hi1 : it.hi0;
            const int my_qlast = t ? it.ql1 : it.ql0;
            const int k_end = it.k_end, q_end = it.q_end;
            float m_used = neg_inf();  // max subtracted so far (log2 units)
            float l = 0.f;
            int doc_row = -1;
            if constexpr (kList) {
                if (p.doc_q && row < p.Sq) doc_row = p.doc_q[row];
            }
            // AliBiScore in log2 units: s * scale * log2e + slope * log2e * (pos - kv0 - c)
            float al_a = 0.f, al_b = 0.f;
            if constexpr (kMode == 3) {
                al_b = p.alibi[it.hq] * 1.4426950408889634f;
                al_a = p.scale_log2;
            }

            // KV tiles of this query tile: its analytic range, or (flex) the listed
            // tiles whose block states for this query tile are not all 0.
            const int n_iter =
                kList ? static_cast<int>(my_list[0]) : (my_hi > my_lo ? my_hi - my_lo : 0);
            int n_done = 0;  // KV tiles this query tile has processed in this item
            for (int i = 0; i < n_iter; ++i) {
                int u, g;  // KV tile and its load index within the item
                uint32_t my_st = 0;
                bool tile0_uses;  // query tile 0 also visits this KV tile
                if constexpr (kList) {
                    const uint32_t e = my_list[1 + i];
                    g = static_cast<int>(e & 0x3FFu);
                    u = static_cast<int>((e >> 10) & 0x3FFu);
                    my_st = (e >> 20) & 0xFFu;
                    tile0_uses = (e >> 28) != 0;
                } else {
                    u = it.rev ? my_hi - 1 - i : my_lo + i;
                    g = it.rev ? it.u_hi - 1 - u : u - it.u_lo;
                    tile0_uses = item_uses(it, 0, u);
                }
                const int kv0 = u * BN;
                if (!warp_wait(bar_s, (n_it + i) & 1, abort_flag, p.wait_limit_ns, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t sr[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + c * 32, sr[c]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c) reg_fence32(sr[c]);
                float *s = reinterpret_cast<float *>(&sr[0][0]);
                // flex_attention! score mods on s = scale <q, k>, then log2 units
                if constexpr (kMode == 2) {
                    // 16 columns at a time: the fence after each group also redefines the
                    // next group's inputs, so at most 16 elements' temporaries are live
                    uint32_t *flat = &sr[0][0];
                    const uint64_t k2 = f2_pack(p.softcap_k, p.softcap_k);
#pragma unroll
                    for (int gp = 0; gp < BN / 16; ++gp) {
#pragma unroll
                        for (int c = 16 * gp; c < 16 * gp + 16; c += 2) {
                            float x0, x1;
                            f2_unpack(f2_mul_fwd(f2_pack(s[c], s[c + 1]), k2), x0, x1);
                            s[c] = tanh_approx(x0);
                            s[c + 1] = tanh_approx(x1);
                        }
                        const int f0 = gp < BN / 16 - 1 ? 16 * gp : BN - 32;
                        reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(flat + f0));
                    }
                } else if constexpr (kMode == 3) {
                    const float t0 = al_b * static_cast<float>(pos - kv0);  // bias of key kv0
#pragma unroll
                    for (int c = 0; c < BN; ++c)
                        s[c] = fmaf(s[c], al_a, fmaf(-al_b, static_cast<float>(c), t0));
                }
                // step a5: per-element mask on boundary tiles only
                const bool edge = (kv0 + BN > k_end) ||
                                  (p.causal && (long long)kv0 + BN - 1 > (long long)p.input_pos + q0) ||
                                  (p.window > 0 &&
                                   (long long)kv0 <= (long long)p.input_pos + my_qlast - p.window) ||
                                  (kList && my_st != 0xAAu);
                if (edge) {
                    long long hi = k_end;
                    if (p.causal) hi = min(hi, pos + 1);
                    const long long lo = p.window > 0 ? pos - p.window + 1 : 0;
                    const int c_hi = static_cast<int>(max(-1ll, min((long long)BN, hi - kv0)));
                    const int c_lo = static_cast<int>(max(-1ll, min((long long)BN, lo - kv0)));
                    if constexpr (kList) {
                        // One visibility bit per key, 32 keys per word: the analytic range,
                        // the block state of this row's 64-row half for the key's half
                        // (0: none, 2: all), and for state 1 the document ids.  The ids
                        // of the tile's keys are read once per warp (one per lane) and
                        // passed around with shuffles; this keeps the unrolled per-key
                        // code as small as the plain path's.
                        const uint32_t qs = static_cast<uint32_t>(r >> 6);
                        uint32_t vm[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int lo_j = min(max(c_lo - 32 * j, 0), 32);
                            const int hi_j = min(max(c_hi - 32 * j, 0), 32);
                            const uint32_t below_hi = hi_j >= 32 ? 0xffffffffu : ((1u << hi_j) - 1u);
                            const uint32_t below_lo = lo_j >= 32 ? 0xffffffffu : ((1u << lo_j) - 1u);
                            uint32_t m = below_hi & ~below_lo;
                            const uint32_t st = (my_st >> (4 * qs + 2 * (j >> 1))) & 3u;
                            if (st == 0) m = 0;
                            if (st == 1 && p.doc_kv) {  // uniform: st depends on the warp only
                                const int kc = kv0 + 32 * j + lane;
                                const int dv = kc < p.Sk ? p.doc_kv[kc] : 0;
                                const int dv0 = __shfl_sync(0xffffffffu, dv, 0);
                                uint32_t same = 0;
                                if (__all_sync(0xffffffffu, dv == dv0)) {
                                    // the 32 keys belong to one document (packed documents
                                    // leave most chunks so): one compare for the row
                                    same = dv0 == doc_row ? 0xffffffffu : 0u;
                                } else {
#pragma unroll 1
                                    for (int c = 0; c < 32; ++c)
                                        same |= (__shfl_sync(0xffffffffu, dv, c) == doc_row ? 1u : 0u) << c;
                                }
                                m &= same;
                            }
                            vm[j] = m;
                        }
#pragma unroll
                        for (int c = 0; c < BN; ++c)
                            s[c] = ((vm[c >> 5] >> (c & 31)) & 1u) ? s[c] : neg_inf();
                    } else {
#pragma unroll
                        for (int c = 0; c < BN; ++c) s[c] = (c >= c_lo && c < c_hi) ? s[c] : neg_inf();
                    }
                }
                // step a6: online softmax in the exp2 domain with lazy rescaling
                float mx0 = s[0], mx1 = s[1];
#pragma unroll
                for (int c = 2; c < BN; c += 2) {
                    mx0 = fmaxf(mx0, s[c]);
                    mx1 = fmaxf(mx1, s[c + 1]);
                }
                const float m_new = fmaxf(mx0, mx1) * sl2;
                float alpha = 1.f;
                bool resc = false;
                if (m_new > m_used + 8.f) {
                    alpha = fast_exp2(m_used - m_new);
                    m_used = m_new;
                    resc = true;
                }
                const float neg_m = (m_used == neg_inf()) ? 0.f : -m_used;
                // exponent arguments and the two running sums on packed fp32 pairs (one
                // f32x2 FMA / add per two scores; same roundings as the scalar forms)
                const uint64_t sl2x2 = f2_pack(sl2, sl2), negm2 = f2_pack(neg_m, neg_m);
                uint64_t sum2 = f2_pack(0.f, 0.f);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
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
                // O correction.  S_t(i) completing implies P_t(i-1) V has completed (same
                // issuing thread, in order), so O_t is quiet until we arrive on P_FULL.
                if (i > 0 && __any_sync(0xffffffffu, resc)) {
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t v[32];
                        tmem_ld32(o_addr + c * 32, v);
                        tmem_wait_ld();
                        reg_fence32(v);
#pragma unroll
                        for (int k = 0; k < 32; ++k)
                            v[k] = __float_as_uint(__uint_as_float(v[k]) * alpha);
                        tmem_st32(o_addr + c * 32, v);
                    }
                }
                // Key rows at or past k_end inside this tile may hold anything; their
                // weights are exactly 0, but 0 * NaN is NaN, so zero those V rows (done
                // by the first query tile that uses this KV tile).
                if (k_end < p.Sk && k_end > kv0 && k_end < kv0 + BN && (t == 0 || !tile0_uses)) {
                    const uint32_t ge = gi + g;
                    const int st = ge % C::NS;
                    if (!warp_wait(bar(C::BAR_VFULL + st), (ge / C::NS) & 1, abort_flag,
                                   p.wait_limit_ns, p.status)) {
                        ok = false;
                    } else {
                        if (r >= k_end - kv0 && r < p.Sk - kv0) {
#pragma unroll
                            for (int c = 0; c < C::NBOX; ++c) {
                                uint4 *dst = reinterpret_cast<uint4 *>(
                                    smem + C::OFF_V + st * C::KV_BYTES + c * C::BOX + r * 128);
#pragma unroll
                                for (int k = 0; k < 8; ++k) dst[k] = make_uint4(0, 0, 0, 0);
                            }
                        }
                        fence_proxy_async_smem();
                    }
                    __syncwarp();
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar_p);
                if (!ok) break;
                n_done = i + 1;
            }

            // step a8: epilogue
            // a split pair's other tile belongs to the other single-tile item
            const bool row_in = row < p.Sq && !(t == 1 && it.single);
            bool have = ok && n_done > 0;
            if (have && !warp_wait(bar_o, (n_it + n_done - 1) & 1, abort_flag, p.wait_limit_ns,
                                   p.status))
                have = false;
            const bool out_valid = have && row < q_end && l > 0.f;
            const float inv_l = out_valid ? 1.f / l : 0.f;
            __nv_bfloat16 *orow = p.O + ((long long)(it.b * p.Hq + it.hq) * p.Sq + row) * D;
            if (have) {
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld32(o_addr + c * 32, v);
                    tmem_wait_ld();
                    reg_fence32(v);
                    // Rows past q_lengths ran the whole chain on whatever the padding of
                    // Q holds (NaN included); their output is selected, not scaled, to
                    // +0.0 so nothing of that padding reaches O.
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
                            dst[k] = make_uint4(o16[4 * k], o16[4 * k + 1], o16[4 * k + 2],
                                                o16[4 * k + 3]);
                    }
                }
            } else if (row_in && !*abort_flag) {
                uint4 *dst = reinterpret_cast<uint4 *>(orow);
#pragma unroll
                for (int k = 0; k < D / 8; ++k) dst[k] = make_uint4(0, 0, 0, 0);
            }
            if (row_in && p.LSE && !*abort_flag) {
                p.LSE[(long long)(it.b * p.Hq + it.hq) * p.Sq + row] =
                    out_valid ? m_used * 0.69314718055994531f + logf(l) : neg_inf();
            }
            n_it += n_done;
            gi += n_loads(it);
            if (!ok) break;
            // next item (or -1 = stop)
            if (!warp_wait(bar(C::BAR_IFULL + (k & 1)), (k >> 1) & 1, abort_flag, p.wait_limit_ns,
                           p.status))
                break;
            const int wn = item_slot[k & 1];
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::BAR_IEMPTY + (k & 1)));
            if (wn < 0) break;
            fwd_item<kMode>(p, wn, it, false);
        }
    }

    // ---- teardown ----
    if (*abort_flag) drain_delay(2000000);  // let copies / MMAs in flight land
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int D, int kMode, bool kList>
attn_status_t launch_fwd_d(const FwdArgs &a, cudaStream_t stream) {
    using C = FwdCfg<D, kList>;
    constexpr int kSmem = kList ? C::SMEM_BYTES_FLEX : C::SMEM_BYTES;
    CUtensorMap tq, tk, tv;
    attn_status_t st;
    if ((st = make_tmap_bf16_3d(&tq, a.Q, D, a.Sq, (uint64_t)a.B * a.Hq, BM)) != ATTN_OK) return st;
    if ((st = make_tmap_bf16_3d(&tk, a.K, D, a.Sk, (uint64_t)a.B * a.Hkv, BN)) != ATTN_OK) return st;
    if ((st = make_tmap_bf16_3d(&tv, a.V, D, a.Sk, (uint64_t)a.B * a.Hkv, BN)) != ATTN_OK) return st;
    // The register hand-over inside the kernel assumes exactly kLaunchRegs
    // registers per thread at launch; refuse to launch a build where it differs.
    if (kernel_setup(reinterpret_cast<const void *>(attn_fwd_kernel<D, kMode, kList>), kSmem,
                     kLaunchRegs) != cudaSuccess)
        return ATTN_ERR_CUDA;
    FwdParams p;
    p.O = static_cast<__nv_bfloat16 *>(a.O);
    p.LSE = a.LSE;
    p.k_lengths = a.k_lengths;
    p.q_lengths = a.q_lengths;
    p.B = a.B;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.Sq = a.Sq;
    p.Sk = a.Sk;
    p.group = a.Hq / a.Hkv;
    p.n_pairs = (a.Sq + kTiles * BM - 1) / (kTiles * BM);
    p.n_split = 0;
    if (!kList && !a.causal && a.window == 0) {
        // Items of equal work: when the last round of CTAs would be at most half full,
        // its pair items run as single-tile items instead, filling it twice as wide.
        int dev = 0, n_sm = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
            n_sm > 0) {
            const long long items = (long long)p.n_pairs * a.Hq * a.B;
            const long long rem = items % n_sm;
            if (items > n_sm && 2 * rem <= n_sm) p.n_split = static_cast<int>(rem);
        }
    }
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.causal = a.causal;
    p.window = a.window;
    p.input_pos = a.input_pos;
    p.wait_limit_ns = kWaitLimitNs;
    p.status = device_status_word();
    p.scale = a.scale;
    p.softcap = a.softcap;
    p.softcap_k = a.softcap > 0.f ? a.scale / a.softcap : 0.f;
    p.softcap_c = a.softcap * 1.4426950408889634f;
    p.alibi = a.alibi_slopes;
    p.doc_q = a.doc_q;
    p.doc_kv = a.doc_kv;
    p.bmask = a.block_mask;
    p.bmask_per_head = a.block_mask_per_head;
    p.n_qb = (a.Sq + 63) / 64;
    p.n_kb = (a.Sk + 63) / 64;
    if (!p.status) return ATTN_ERR_CUDA;
    const long long grid = (long long)p.n_pairs * a.Hq * a.B + p.n_split;
    if (grid == 0) return ATTN_OK;
    if (grid > 0x7fffffffll) return ATTN_ERR_INVALID;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, attn_fwd_kernel<D, kMode, kList>, tq, tk, tv, p) != cudaSuccess)
        return ATTN_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

attn_status_t launch_fwd(const FwdArgs &a, cudaStream_t stream) {
    const int mode = !a.flex ? 0 : (a.softcap > 0.f ? 2 : (a.alibi_slopes ? 3 : 0));
    const bool list = a.flex && (a.block_mask || a.doc_q);
#define GQA_LAUNCH(DD)                                                            \
    do {                                                                          \
        if (list) {                                                               \
            if (mode == 0) return launch_fwd_d<DD, 0, true>(a, stream);           \
            if (mode == 2) return launch_fwd_d<DD, 2, true>(a, stream);           \
            return launch_fwd_d<DD, 3, true>(a, stream);                          \
        }                                                                         \
        if (mode == 0) return launch_fwd_d<DD, 0, false>(a, stream);              \
        if (mode == 2) return launch_fwd_d<DD, 2, false>(a, stream);              \
        return launch_fwd_d<DD, 3, false>(a, stream);                             \
    } while (0)
    if (a.D == 128) GQA_LAUNCH(128);
    if (a.D == 64) GQA_LAUNCH(64);
#undef GQA_LAUNCH
    return ATTN_ERR_UNSUPPORTED;
}

}  // namespace gqa
