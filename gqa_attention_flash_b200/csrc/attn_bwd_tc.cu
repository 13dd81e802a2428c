// attn_bwd_tc.cu -- dK / dV and dQ kernels of the attention backward on the
// fifth-generation tensor cores (tcgen05.mma, TMEM accumulators, TMA-fed operands).
//
// Tylo.jl "Primitives" page, entry `∇attention!`: with P = exp(S * scale - LSE) on
// the visible pairs of the forward's masks and delta_i = sum_d dO_id O_id,
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - delta),  dQ = scale dS K,
//   dK = scale dS^T Q  (a KV head sums the gradients of its query heads).
//
// bwd_dkdv_tc_kernel: one CTA per (128-key tile, KV head, batch), 10 warps.
//   warps 0-7  elementwise: warp w owns TMEM lanes 32 (w % 4) .. +31 (one key row
//              per thread) and query columns 64 (w / 4) .. +63; turns S^T into
//              P^T and dP^T into dS^T (bf16, written back over their own columns)
//              and writes its half of the dK, dV rows
//   warp 8     TMA: K, V of the tile once, then Q, dO of every (query head of the
//              group, 128-row query tile that sees the key tile) into a 2-slot
//              ring whose Q and dO halves are released separately (after dK and
//              after dV); it also copies that tile's -LSE (log2 units) and -delta
//              next to them
//   warp 9     MMA issuer and TMEM owner
//   TMEM (512 columns): S^T | dP^T | dV | dK.
//   Tensor-pipe order per ring item t: dP^T(t), [P^T(t) ready] dV += P^T dO,
//   S^T(t+1), [dS^T(t) ready] dK += dS^T Q -- so P^T(t+1) is computed while dK(t)
//   and dP^T(t+1) run, and dS^T(t) while dV(t) and S^T(t+1) run.  P^T is released
//   in two halves: each elementwise warp stores and signals the first 32 of its 64
//   query columns before it computes the other 32, and dV issues the K-steps of
//   the first halves (query columns 0-31, 64-95) while the rest is computed (4 %
//   faster on the LLM causal backward than one release).
// bwd_dq_tc_kernel: one CTA per (128-row query tile, query head, batch), same
//   roles over the visible 128-key tiles, Q and dO resident, K in a 3-slot and V
//   in a 2-slot ring; TMEM: S0 | S1 | dP | dQ, dS (bf16) written over its own S
//   buffer.  Order: S(0), dP(0), S(1), then per key tile g: [dS(g) ready]
//   dQ += dS(g) K(g), dP(g+1), S(g+2).
// The elementwise arithmetic runs on packed fp32 pairs (f32x2 FMA / add / mul).
// dS is recomputed by the dQ kernel rather than reduced with atomics.  The two
// kernels are independent: dQ runs on a library-owned side stream forked from and
// joined back to the caller's stream with events, so each kernel's last wave
// overlaps the other's work (3 % on the LLM causal backward, bitwise the same).
// The side stream and its events are shared per device; a mutex keeps the
// fork / launch / join sequence of concurrent callers from interleaving.  Key,
// value, query and output-gradient rows past the lengths are read as MMA
// operands with weight exactly zero, so they must hold finite values: zero times
// NaN or Inf is NaN, which would reach the gradients of valid rows.  The rows of
// dQ past q_lengths and of dK, dV past k_lengths are themselves written as +0.0
// by selection.
#include <cuda_bf16.h>

#include <mutex>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace gqa {

namespace {

constexpr int TB = 128;         // rows per tile (keys or queries)
constexpr int kEltWarps = 8;
constexpr int kEltThreads = 32 * kEltWarps;
constexpr int kWarpTmaB = 8;
constexpr int kWarpMmaB = 9;
constexpr int kThreadsTc = 320;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct TcCfg {
    static constexpr int NBOX = D / 64;
    static constexpr int BOX = TB * 128;          // bytes of one (128 rows x 64 cols) box
    static constexpr int TILE = TB * D * 2;       // one 128-row tile
    static constexpr int NS = 2;                  // ring stages
    // resident pair: K, V (dkdv) or Q, dO (dq); ring stages: Q, dO (+ LSE, delta) or K, V
    static constexpr int OFF_R0 = 0;
    static constexpr int OFF_R1 = TILE;
    static constexpr int STAGE = 2 * TILE + 2 * TB * 4;
    static constexpr int OFF_S = 2 * TILE;
    __host__ __device__ static constexpr int stage(int s) { return OFF_S + s * STAGE; }
    static constexpr int OFF_BAR = OFF_S + NS * STAGE;
    // barriers: resident; per ring slot full / empty of its Q half and of its dO
    // half (they are released at different points); s_full, dp_full, p_done (first
    // half of P^T), ds_full, done, p_done2 (second half of P^T)
    static constexpr int BAR_RES = 0, BAR_FULLQ = 1, BAR_EMPTYQ = 1 + NS, BAR_FULLD = 1 + 2 * NS,
                         BAR_EMPTYD = 1 + 3 * NS, BAR_SFULL = 1 + 4 * NS, BAR_DPFULL = 2 + 4 * NS,
                         BAR_PDONE = 3 + 4 * NS, BAR_DSFULL = 4 + 4 * NS, BAR_DONE = 5 + 4 * NS,
                         BAR_PDONE2 = 6 + 4 * NS, N_BARS = 7 + 4 * NS;
    static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
    // TMEM columns
    static constexpr uint32_t COL_S = 0, COL_DP = TB, COL_A = 2 * TB, COL_B = 2 * TB + D;
};

struct TcParams {
    const float *LSE, *delta;
    __nv_bfloat16 *dQ, *dK, *dV;
    const int32_t *k_lengths, *q_lengths;
    int B, Hq, Hkv, Sq, Sk, group;
    float scale, scale_log2;
    int causal, window, input_pos;
    uint64_t wait_limit_ns;
    int *status;
};

__device__ __forceinline__ float ninf() { return __int_as_float(0xff800000); }

// a * b on both fp32 halves of a packed pair (see f2_fma / f2_add).
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ void tc_lengths(const TcParams &p, int b, int &k_end, int &q_end) {
    k_end = p.Sk;
    q_end = p.Sq;
    if (p.k_lengths) {
        int kl = p.k_lengths[b];
        if (kl > p.Sk) {
            if (threadIdx.x == 0) record_status(p.status, ATTN_ERR_DEVICE_BOUNDS);
            kl = p.Sk;
        }
        k_end = kl > 0 ? kl : 0;
    }
    if (p.q_lengths) {
        int ql = p.q_lengths[b];
        if (ql > p.Sq) {
            if (threadIdx.x == 0) record_status(p.status, ATTN_ERR_DEVICE_BOUNDS);
            ql = p.Sq;
        }
        q_end = ql > 0 ? ql : 0;
    }
}

// Visible pairs (query i, key j): i < q_end, j < k_end, causal j <= input_pos + i,
// window j > input_pos + i - window.  For one key row j and the query tile at q0:
// the visible tile columns are [lo, hi) (lo >= hi: none).
__device__ __forceinline__ void cols_of_key(const TcParams &p, int j, int q0, int k_end, int q_end,
                                            int &lo, int &hi) {
    long long l = 0, h = min(TB, q_end - q0);
    if (p.causal) l = max(l, (long long)j - p.input_pos - q0);
    if (p.window > 0) h = min(h, (long long)j + p.window - p.input_pos - q0);
    if (j >= k_end) h = 0;
    lo = static_cast<int>(max(0ll, min(l, (long long)TB)));
    hi = static_cast<int>(max(0ll, h));
}

// For one query row i and the key tile at kv0: visible tile columns [lo, hi).
__device__ __forceinline__ void cols_of_query(const TcParams &p, int i, int kv0, int k_end, int q_end,
                                              int &lo, int &hi) {
    const long long pos = (long long)p.input_pos + i;
    long long l = 0, h = min(TB, k_end - kv0);
    if (p.causal) h = min(h, pos - kv0 + 1);
    if (p.window > 0) l = max(l, pos - p.window - kv0 + 1);
    if (i >= q_end) h = 0;
    lo = static_cast<int>(max(0ll, min(l, (long long)TB)));
    hi = static_cast<int>(max(0ll, h));
}

// 16 K-steps of D = 128 (8 for D = 64) of an M128 x N128 product with both
// operands K-major in 128-byte-swizzled TMA tiles.
template <int D>
__device__ __forceinline__ void mma_kmajor(uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem) {
    using C = TcCfg<D>;
    constexpr uint32_t id = idesc_bf16_f32(TB, TB, 0, 0);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
        mma_ss(d_tmem, smem_desc_sw128(a_smem + off, 16, 1024), smem_desc_sw128(b_smem + off, 16, 1024),
               id, kk > 0 ? 1u : 0u);
    }
}

// D[128 x D] (+)= A[128 x 128 from TMEM, bf16 pairs] * B[128 rows of the tile x D]
// with B MN-major (the tile's rows are the K index).  kSplit: A's K index 0..63
// sits in columns 0..31 and 64..127 in columns 64..95 (each elementwise warp half
// packs over its own fp32 columns); otherwise K pairs are contiguous.
template <int D, bool kSplit>
__device__ __forceinline__ void mma_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_smem,
                                           bool accumulate) {
    using C = TcCfg<D>;
    constexpr uint32_t id = idesc_bf16_f32(TB, D, 0, 1);
#pragma unroll
    for (int kk = 0; kk < TB / 16; ++kk) {
        const uint32_t a_col = kSplit ? (kk >> 2) * 64 + (kk & 3) * 8 : kk * 8;
        mma_ts(d_tmem, a_tmem + a_col, smem_desc_sw128(b_smem + kk * 16 * 128, C::BOX, 1024), id,
               (accumulate || kk > 0) ? 1u : 0u);
    }
}

// Half r of the K-steps of mma_tmem_a<D, true>: K-steps 4 k + 2 r, 4 k + 2 r + 1 (k = 0, 1),
// i.e. A's K index 32 r .. 32 r + 31 and 64 + 32 r .. 64 + 32 r + 31.
template <int D>
__device__ __forceinline__ void mma_tmem_a_half(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_smem,
                                                bool accumulate, int r) {
    using C = TcCfg<D>;
    constexpr uint32_t id = idesc_bf16_f32(TB, D, 0, 1);
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int kk = 4 * k + 2 * r + e;
            const uint32_t a_col = (kk >> 2) * 64 + (kk & 3) * 8;
            mma_ts(d_tmem, a_tmem + a_col, smem_desc_sw128(b_smem + kk * 16 * 128, C::BOX, 1024), id,
                   (accumulate || kk > 0) ? 1u : 0u);
        }
}

// Shared set-up: barriers (the elementwise warps' arrival barriers count 256
// arrivals, the others one), TMEM allocation (warp 9), 512 columns.
template <class C>
__device__ __forceinline__ uint32_t tc_setup(uint8_t *smem, uint32_t sbase) {
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::N_BARS; ++i)
            mbar_init(sbase + C::OFF_BAR + 8 * i,
                      (i == C::BAR_PDONE || i == C::BAR_PDONE2 || i == C::BAR_DSFULL) ? kEltThreads : 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if ((threadIdx.x >> 5) == kWarpMmaB) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return *tmem_slot;
}

// Shared teardown: let work in flight land after a give-up, free TMEM.
template <class C>
__device__ __forceinline__ void tc_teardown(uint8_t *smem, uint32_t tmem) {
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    if (*abort_flag) drain_delay(2000000);
    tc_fence_before();
    __syncthreads();
    if ((threadIdx.x >> 5) == kWarpMmaB) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Write columns [c0, c0 + D/2) of this thread's TMEM lane of an fp32 accumulator,
// times `mul`, as bf16 to dst[c0 ..).
template <int D>
__device__ __forceinline__ void tc_store_half(uint32_t taddr, __nv_bfloat16 *dst, int c0, float mul,
                                              bool store, bool valid) {
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
        uint32_t v[32];
        tmem_ld32(taddr + c0 + c * 32, v);
        tmem_wait_ld();
        reg_fence32(v);
        // rows past the lengths are +0.0 by selection (their accumulators saw
        // only zero weights, but zero times a non-finite operand is NaN)
        uint32_t o16[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
            o16[k] = valid ? pack_bf16x2(__uint_as_float(v[2 * k]) * mul,
                                         __uint_as_float(v[2 * k + 1]) * mul)
                           : 0u;
        if (store) {
            uint4 *d4 = reinterpret_cast<uint4 *>(dst + c0 + c * 32);
#pragma unroll
            for (int k = 0; k < 4; ++k) d4[k] = make_uint4(o16[4 * k], o16[4 * k + 1], o16[4 * k + 2], o16[4 * k + 3]);
        }
    }
}

template <int D>
__device__ __forceinline__ void tc_zero_half(__nv_bfloat16 *dst, int c0) {
    uint4 *d4 = reinterpret_cast<uint4 *>(dst + c0);
#pragma unroll
    for (int k = 0; k < D / 16; ++k) d4[k] = make_uint4(0, 0, 0, 0);
}

// ---------------------------------------------------------------------------------
// dK, dV of one 128-key tile
// ---------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kThreadsTc, 1)
    bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                       const TcParams p) {
    using C = TcCfg<D>;
    // (KV head, batch) pairs in chunks of 4; inside a chunk the key tiles in
    // increasing order with the pairs fastest: under a causal mask the heaviest
    // tiles go first, and the Q / dO rows one wave reads (a few chunks) stay in L2
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8 * i; };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pairs = p.Hkv * p.B, n_kt = (p.Sk + TB - 1) / TB;
    const int G = min(4, pairs), full = pairs / G;
    const int chunk = min(static_cast<int>(blockIdx.x / (G * n_kt)), full);
    const int size = chunk < full ? G : pairs - full * G;
    const int local = static_cast<int>(blockIdx.x) - chunk * G * n_kt;
    const int kt = local / size, pair = chunk * G + local % size;
    const int hkv = pair % p.Hkv, b = pair / p.Hkv;
    const int kv0 = kt * TB;
    int k_end, q_end;
    tc_lengths(p, b, k_end, q_end);
    // query tiles that hold a row seeing a key of this tile
    int i_lo = 0, i_hi = q_end;
    if (kv0 >= k_end) i_hi = 0;
    if (p.causal) i_lo = max(0, kv0 - p.input_pos);
    if (p.window > 0) i_hi = static_cast<int>(min((long long)i_hi, (long long)kv0 + TB + p.window - p.input_pos));
    const int qt_lo = i_lo / TB, qt_hi = i_hi > i_lo ? (i_hi + TB - 1) / TB : qt_lo;
    const int n_qt = qt_hi - qt_lo, n_it = p.group * n_qt;

    const uint32_t tmem = tc_setup<C>(smem, sbase);

    if (warp == kWarpTmaB) {
        // ===================== TMA producer =====================
        if (n_it > 0) {
            if (lane == 0) {
                prefetch_tensormap(&tmQ);
                prefetch_tensormap(&tmK);
                prefetch_tensormap(&tmV);
                prefetch_tensormap(&tmdO);
                // checked build: the resident K / V tile lies inside the tensors
                if (in_range(box_ok(0, kv0, b * p.Hkv + hkv, D, p.Sk, (long long)p.B * p.Hkv, TB) &&
                                 kv0 >= 0 && kv0 < p.Sk,
                             p.status, abort_flag))
                    mbar_arrive_expect_tx(bar(C::BAR_RES), 2 * C::TILE);
                for (int c = 0; c < C::NBOX && !*abort_flag; ++c) {
                    tma_load_3d(sbase + C::OFF_R0 + c * C::BOX, &tmK, bar(C::BAR_RES), c * 64, kv0,
                                b * p.Hkv + hkv);
                    tma_load_3d(sbase + C::OFF_R1 + c * C::BOX, &tmV, bar(C::BAR_RES), c * 64, kv0,
                                b * p.Hkv + hkv);
                }
            }
            for (int it = 0; it < n_it; ++it) {
                const int st = it % C::NS, use = it / C::NS;
                const int hq = hkv * p.group + it / n_qt;
                const int q0 = (qt_lo + it % n_qt) * TB;
                const long long qrow = (long long)(b * p.Hq + hq) * p.Sq;
                // checked build: this item's Q / dO tiles and LSE / delta rows exist
                if (!in_range(hq < p.Hq && box_ok(0, q0, b * p.Hq + hq, D, p.Sq, (long long)p.B * p.Hq,
                                                  TB) && q0 >= 0 && q0 < p.Sq,
                              p.status, abort_flag))
                    break;
                // the tile's -LSE (log2 units) and -delta, loaded before the slot is free
                float lr[TB / 32], dr[TB / 32];
#pragma unroll
                for (int k = 0; k < TB / 32; ++k) {
                    const int i = q0 + lane + 32 * k;
                    const bool ok = i < p.Sq;
                    lr[k] = ok ? -p.LSE[qrow + i] * kLog2e : -ninf();
                    dr[k] = ok ? -p.delta[qrow + i] : 0.f;
                }
                // dO half: free once dV of the slot's previous item has run
                if (use > 0 && !warp_wait(bar(C::BAR_EMPTYD + st), (use - 1) & 1, abort_flag,
                                          p.wait_limit_ns, p.status))
                    break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar(C::BAR_FULLD + st), C::TILE);
                    for (int c = 0; c < C::NBOX; ++c)
                        tma_load_3d(sbase + C::stage(st) + C::TILE + c * C::BOX, &tmdO,
                                    bar(C::BAR_FULLD + st), c * 64, q0, b * p.Hq + hq);
                }
                // Q half and the rows: free once dK of the slot's previous item has run
                if (use > 0 && !warp_wait(bar(C::BAR_EMPTYQ + st), (use - 1) & 1, abort_flag,
                                          p.wait_limit_ns, p.status))
                    break;
                float *rows = reinterpret_cast<float *>(smem + C::stage(st) + 2 * C::TILE);
#pragma unroll
                for (int k = 0; k < TB / 32; ++k) {
                    rows[lane + 32 * k] = lr[k];
                    rows[TB + lane + 32 * k] = dr[k];
                }
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar(C::BAR_FULLQ + st), C::TILE);
                    for (int c = 0; c < C::NBOX; ++c)
                        tma_load_3d(sbase + C::stage(st) + c * C::BOX, &tmQ, bar(C::BAR_FULLQ + st),
                                    c * 64, q0, b * p.Hq + hq);
                }
                __syncwarp();
            }
        }
    } else if (warp == kWarpMmaB) {
        // ===================== MMA issuer =====================
        if (lane == 0 && n_it > 0) {
            bool ok = mbar_wait(bar(C::BAR_RES), 0, abort_flag, p.wait_limit_ns, p.status) &&
                      mbar_wait(bar(C::BAR_FULLQ), 0, abort_flag, p.wait_limit_ns, p.status);
            if (ok) {
                tc_fence_after();
                mma_kmajor<D>(tmem + C::COL_S, sbase + C::OFF_R0, sbase + C::stage(0));  // S^T = K Q^T
                mma_commit(bar(C::BAR_SFULL));
            }
            for (int it = 0; ok && it < n_it; ++it) {
                const int st = it % C::NS;
                const uint32_t q_s = sbase + C::stage(st), do_s = q_s + C::TILE;
                if (!(ok = mbar_wait(bar(C::BAR_FULLD + st), (it / C::NS) & 1, abort_flag,
                                     p.wait_limit_ns, p.status)))
                    break;
                tc_fence_after();
                mma_kmajor<D>(tmem + C::COL_DP, sbase + C::OFF_R1, do_s);  // dP^T = V dO^T
                mma_commit(bar(C::BAR_DPFULL));
                // dV += P^T dO in two halves of its K-steps: the query columns 0-31 and
                // 64-95 of P^T are released first, 32-63 and 96-127 after them
                if (!(ok = mbar_wait(bar(C::BAR_PDONE), it & 1, abort_flag, p.wait_limit_ns, p.status)))
                    break;
                tc_fence_after();
                mma_tmem_a_half<D>(tmem + C::COL_A, tmem + C::COL_S, do_s, it > 0, 0);
                if (!(ok = mbar_wait(bar(C::BAR_PDONE2), it & 1, abort_flag, p.wait_limit_ns, p.status)))
                    break;
                tc_fence_after();
                mma_tmem_a_half<D>(tmem + C::COL_A, tmem + C::COL_S, do_s, true, 1);
                mma_commit(bar(C::BAR_EMPTYD + st));
                if (it + 1 < n_it) {
                    const int st1 = (it + 1) % C::NS;
                    if (!(ok = mbar_wait(bar(C::BAR_FULLQ + st1), ((it + 1) / C::NS) & 1, abort_flag,
                                         p.wait_limit_ns, p.status)))
                        break;
                    tc_fence_after();
                    mma_kmajor<D>(tmem + C::COL_S, sbase + C::OFF_R0, sbase + C::stage(st1));
                    mma_commit(bar(C::BAR_SFULL));
                }
                if (!(ok = mbar_wait(bar(C::BAR_DSFULL), it & 1, abort_flag, p.wait_limit_ns, p.status)))
                    break;
                tc_fence_after();
                mma_tmem_a<D, true>(tmem + C::COL_B, tmem + C::COL_DP, q_s, it > 0);  // dK += dS^T Q
                mma_commit(bar(C::BAR_EMPTYQ + st));
            }
            if (ok) mma_commit(bar(C::BAR_DONE));
        }
    } else {
        // ===================== P^T, dS^T and the epilogue =====================
        const int quad = warp & 3, half = warp >> 2;
        const int r = quad * 32 + lane;  // key row of the tile = TMEM lane
        const int j = kv0 + r;
        const int cb = half * 64;        // first query column of this warp
        const uint32_t trow = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        bool ok = true;
        for (int it = 0; it < n_it; ++it) {
            const int st = it % C::NS;
            // S^T(it) in TMEM; the producer's plain stores of LSE / delta are
            // published by its arrive on the stage's full barrier
            if (!warp_wait(bar(C::BAR_SFULL), it & 1, abort_flag, p.wait_limit_ns, p.status) ||
                !warp_wait(bar(C::BAR_FULLQ + st), (it / C::NS) & 1, abort_flag, p.wait_limit_ns,
                           p.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int q0 = (qt_lo + it % n_qt) * TB;
            const float *rows = reinterpret_cast<const float *>(smem + C::stage(st) + 2 * C::TILE);
            int lo, hi;
            cols_of_key(p, j, q0, k_end, q_end, lo, hi);
            lo -= cb;
            hi -= cb;
            float pr[64];
            {
                uint32_t sv[2][32];
                tmem_ld32(trow + C::COL_S + cb, sv[0]);
                tmem_ld32(trow + C::COL_S + cb + 32, sv[1]);
                tmem_wait_ld();
                reg_fence32(sv[0]);
                reg_fence32(sv[1]);
                // exponent arguments on packed fp32 pairs (rows[] holds -LSE * log2 e)
                const float4 *l4 = reinterpret_cast<const float4 *>(rows + cb);
                const uint64_t sl2x2 = f2_pack(p.scale_log2, p.scale_log2);
                // two halves of the warp's 64 columns, each released to the dV product as
                // soon as it is in TMEM
#pragma unroll
                for (int c = 0; c < 2; ++c) {
#pragma unroll
                    for (int q = 8 * c; q < 8 * c + 8; ++q) {
                        const float4 l = l4[q];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int x = 4 * q + 2 * h;
                            float x0, x1;
                            f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[x >> 5][x & 31]),
                                                     __uint_as_float(sv[x >> 5][(x + 1) & 31])),
                                             sl2x2, h ? f2_pack(l.z, l.w) : f2_pack(l.x, l.y)),
                                      x0, x1);
                            const float v0 = fast_exp2(x0), v1 = fast_exp2(x1);
                            pr[x] = (x >= lo && x < hi) ? v0 : 0.f;
                            pr[x + 1] = (x + 1 >= lo && x + 1 < hi) ? v1 : 0.f;
                        }
                    }
                    uint32_t pk[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) pk[k] = pack_bf16x2(pr[32 * c + 2 * k], pr[32 * c + 2 * k + 1]);
                    tmem_st16(trow + C::COL_S + cb + 16 * c, pk);
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(bar(c ? C::BAR_PDONE2 : C::BAR_PDONE));
                }
            }
            if (!warp_wait(bar(C::BAR_DPFULL), it & 1, abort_flag, p.wait_limit_ns, p.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            {
                uint32_t dv[2][32];
                tmem_ld32(trow + C::COL_DP + cb, dv[0]);
                tmem_ld32(trow + C::COL_DP + cb + 32, dv[1]);
                tmem_wait_ld();
                reg_fence32(dv[0]);
                reg_fence32(dv[1]);
                // dS^T = P^T (dP^T - delta) on packed pairs (rows[TB..] holds -delta)
                const float4 *d4 = reinterpret_cast<const float4 *>(rows + TB + cb);
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const float4 dl = d4[q];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int x = 4 * q + 2 * h;
                        const uint64_t t2 = f2_add(f2_pack(__uint_as_float(dv[x >> 5][x & 31]),
                                                           __uint_as_float(dv[x >> 5][(x + 1) & 31])),
                                                   h ? f2_pack(dl.z, dl.w) : f2_pack(dl.x, dl.y));
                        f2_unpack(f2_mul(f2_pack(pr[x], pr[x + 1]), t2), pr[x], pr[x + 1]);
                    }
                }
            }
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t pk[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) pk[k] = pack_bf16x2(pr[32 * c + 2 * k], pr[32 * c + 2 * k + 1]);
                tmem_st16(trow + C::COL_DP + cb + 16 * c, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(C::BAR_DSFULL));
        }
        const bool have = ok && n_it > 0 &&
                          warp_wait(bar(C::BAR_DONE), 0, abort_flag, p.wait_limit_ns, p.status);
        const long long krow = (long long)(b * p.Hkv + hkv) * p.Sk + j;
        if (have) {
            tc_fence_after();
            tc_store_half<D>(trow + C::COL_A, p.dV + krow * D, half * (D / 2), 1.f, j < p.Sk,
                             j < k_end);
            tc_store_half<D>(trow + C::COL_B, p.dK + krow * D, half * (D / 2), p.scale, j < p.Sk,
                             j < k_end);
        } else if (j < p.Sk && !*abort_flag) {
            tc_zero_half<D>(p.dV + krow * D, half * (D / 2));
            tc_zero_half<D>(p.dK + krow * D, half * (D / 2));
        }
    }
    tc_teardown<C>(smem, tmem);
}

// ---------------------------------------------------------------------------------
// dQ of one 128-row query tile
// ---------------------------------------------------------------------------------
// Shared memory of the dQ kernel: Q and dO resident, three K slots and two V
// slots (K of a tile is read last, by dQ += dS K, and first, by the next-but-one
// S, so it gets the deeper ring).
template <int D>
struct DqCfg {
    static constexpr int NBOX = D / 64;
    static constexpr int BOX = TB * 128;
    static constexpr int TILE = TB * D * 2;
    static constexpr int NK = 3, NV = 2;
    static constexpr int OFF_Q = 0, OFF_DO = TILE;
    __host__ __device__ static constexpr int k_slot(int s) { return 2 * TILE + s * TILE; }
    __host__ __device__ static constexpr int v_slot(int s) { return (2 + NK) * TILE + s * TILE; }
    static constexpr int OFF_BAR = (2 + NK + NV) * TILE;
    static constexpr int BAR_RES = 0, BAR_FULLK = 1, BAR_EMPTYK = 1 + NK, BAR_FULLV = 1 + 2 * NK,
                         BAR_EMPTYV = 1 + 2 * NK + NV, BAR_SFULL = 1 + 2 * NK + 2 * NV,  // two
                         BAR_DPFULL = 3 + 2 * NK + 2 * NV, BAR_DSFULL = 4 + 2 * NK + 2 * NV,
                         BAR_DONE = 5 + 2 * NK + 2 * NV, BAR_PDONE = -1, BAR_PDONE2 = -1,
                         N_BARS = 6 + 2 * NK + 2 * NV;
    static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
    // TMEM: two S buffers (dS written over its own S), dP, dQ
    static constexpr uint32_t COL_S = 0, COL_DP = 2 * TB, COL_DQ = 3 * TB;
};

template <int D>
__global__ void __launch_bounds__(kThreadsTc, 1)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                     const TcParams p, int n_qt_total) {
    using C = DqCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8 * i; };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // heaviest causal query tiles first, the query heads of one KV group adjacent
    int bid = blockIdx.x;
    const int hq = bid % p.Hq;
    bid /= p.Hq;
    const int b = bid % p.B;
    bid /= p.B;
    const int qt = n_qt_total - 1 - bid;
    const int hkv = hq / p.group;
    const int q0 = qt * TB;
    int k_end, q_end;
    tc_lengths(p, b, k_end, q_end);
    int lo = 0, hi = 0;  // key tiles holding a key some row of this tile sees
    if (q0 < q_end && k_end > 0) {
        const int qlast = min(q0 + TB - 1, q_end - 1);
        long long h = k_end;
        if (p.causal) h = min(h, (long long)p.input_pos + qlast + 1);
        long long l = 0;
        if (p.window > 0) l = max(0ll, (long long)p.input_pos + q0 - p.window + 1);
        if (h > l) {
            lo = static_cast<int>(l / TB);
            hi = static_cast<int>((h + TB - 1) / TB);
        }
    }
    const int n_kt = hi - lo;

    const uint32_t tmem = tc_setup<C>(smem, sbase);

    if (warp == kWarpTmaB) {
        // ===================== TMA producer =====================
        if (lane == 0 && n_kt > 0) {
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            prefetch_tensormap(&tmdO);
            // checked build: the resident Q / dO tile lies inside the tensors
            if (in_range(box_ok(0, q0, b * p.Hq + hq, D, p.Sq, (long long)p.B * p.Hq, TB) && q0 >= 0 &&
                             q0 < p.Sq,
                         p.status, abort_flag))
                mbar_arrive_expect_tx(bar(C::BAR_RES), 2 * C::TILE);
            for (int c = 0; c < C::NBOX && !*abort_flag; ++c) {
                tma_load_3d(sbase + C::OFF_Q + c * C::BOX, &tmQ, bar(C::BAR_RES), c * 64, q0,
                            b * p.Hq + hq);
                tma_load_3d(sbase + C::OFF_DO + c * C::BOX, &tmdO, bar(C::BAR_RES), c * 64, q0,
                            b * p.Hq + hq);
            }
            for (int g = 0; g < n_kt; ++g) {
                const int kv0 = (lo + g) * TB;
                const int ks = g % C::NK, ku = g / C::NK, vs = g % C::NV, vu = g / C::NV;
                if (!in_range(box_ok(0, kv0, b * p.Hkv + hkv, D, p.Sk, (long long)p.B * p.Hkv, TB) &&
                                  kv0 >= 0 && kv0 < p.Sk,
                              p.status, abort_flag))
                    break;
                if (ku > 0 && !mbar_wait(bar(C::BAR_EMPTYK + ks), (ku - 1) & 1, abort_flag,
                                         p.wait_limit_ns, p.status))
                    break;
                mbar_arrive_expect_tx(bar(C::BAR_FULLK + ks), C::TILE);
                for (int c = 0; c < C::NBOX; ++c)
                    tma_load_3d(sbase + C::k_slot(ks) + c * C::BOX, &tmK, bar(C::BAR_FULLK + ks), c * 64,
                                kv0, b * p.Hkv + hkv);
                if (vu > 0 && !mbar_wait(bar(C::BAR_EMPTYV + vs), (vu - 1) & 1, abort_flag,
                                         p.wait_limit_ns, p.status))
                    break;
                mbar_arrive_expect_tx(bar(C::BAR_FULLV + vs), C::TILE);
                for (int c = 0; c < C::NBOX; ++c)
                    tma_load_3d(sbase + C::v_slot(vs) + c * C::BOX, &tmV, bar(C::BAR_FULLV + vs), c * 64,
                                kv0, b * p.Hkv + hkv);
            }
        }
    } else if (warp == kWarpMmaB) {
        // ===================== MMA issuer =====================
        // order: S(0), dP(0), S(1), then per tile g: [dS(g)] dQ += dS(g) K(g), dP(g+1),
        // S(g+2) -- S(g+2) reuses the TMEM buffer of S(g) / dS(g) after dQ(g) read it
        if (lane == 0 && n_kt > 0) {
            auto issue_s = [&](int g) -> bool {
                const int ks = g % C::NK;
                if (!mbar_wait(bar(C::BAR_FULLK + ks), (g / C::NK) & 1, abort_flag, p.wait_limit_ns,
                               p.status))
                    return false;
                tc_fence_after();
                mma_kmajor<D>(tmem + C::COL_S + (g & 1) * TB, sbase + C::OFF_Q, sbase + C::k_slot(ks));
                mma_commit(bar(C::BAR_SFULL + (g & 1)));
                return true;
            };
            auto issue_dp = [&](int g) -> bool {
                const int vs = g % C::NV;
                if (!mbar_wait(bar(C::BAR_FULLV + vs), (g / C::NV) & 1, abort_flag, p.wait_limit_ns,
                               p.status))
                    return false;
                tc_fence_after();
                mma_kmajor<D>(tmem + C::COL_DP, sbase + C::OFF_DO, sbase + C::v_slot(vs));
                mma_commit(bar(C::BAR_DPFULL));
                mma_commit(bar(C::BAR_EMPTYV + vs));
                return true;
            };
            bool ok = mbar_wait(bar(C::BAR_RES), 0, abort_flag, p.wait_limit_ns, p.status) && issue_s(0) &&
                      issue_dp(0) && (n_kt < 2 || issue_s(1));
            for (int g = 0; ok && g < n_kt; ++g) {
                if (!(ok = mbar_wait(bar(C::BAR_DSFULL), g & 1, abort_flag, p.wait_limit_ns, p.status)))
                    break;
                tc_fence_after();
                mma_tmem_a<D, true>(tmem + C::COL_DQ, tmem + C::COL_S + (g & 1) * TB,
                                    sbase + C::k_slot(g % C::NK), g > 0);  // dQ += dS K
                mma_commit(bar(C::BAR_EMPTYK + g % C::NK));
                if (g + 1 < n_kt && !(ok = issue_dp(g + 1))) break;
                if (g + 2 < n_kt && !(ok = issue_s(g + 2))) break;
            }
            if (ok) mma_commit(bar(C::BAR_DONE));
        }
    } else {
        // ===================== P, dS and the epilogue =====================
        const int quad = warp & 3, half = warp >> 2;
        const int r = quad * 32 + lane;  // query row of the tile = TMEM lane
        const int i = q0 + r;
        const int cb = half * 64;        // first key column of this warp
        const uint32_t trow = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const long long qrow = (long long)(b * p.Hq + hq) * p.Sq;
        const float lse2 = i < p.Sq ? p.LSE[qrow + i] * kLog2e : 0.f;
        const float del = i < p.Sq ? p.delta[qrow + i] : 0.f;
        bool ok = true;
        for (int g = 0; g < n_kt; ++g) {
            if (!warp_wait(bar(C::BAR_SFULL + (g & 1)), (g >> 1) & 1, abort_flag, p.wait_limit_ns,
                           p.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t t_s = trow + C::COL_S + (g & 1) * TB + cb;
            const int kv0 = (lo + g) * TB;
            int clo, chi;
            cols_of_query(p, i, kv0, k_end, q_end, clo, chi);
            clo -= cb;
            chi -= cb;
            float pr[64];
            {
                uint32_t sv[2][32];
                tmem_ld32(t_s, sv[0]);
                tmem_ld32(t_s + 32, sv[1]);
                tmem_wait_ld();
                reg_fence32(sv[0]);
                reg_fence32(sv[1]);
                const uint64_t sl2x2 = f2_pack(p.scale_log2, p.scale_log2), nl2 = f2_pack(-lse2, -lse2);
#pragma unroll
                for (int x = 0; x < 64; x += 2) {
                    float x0, x1;
                    f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[x >> 5][x & 31]),
                                             __uint_as_float(sv[x >> 5][(x + 1) & 31])),
                                     sl2x2, nl2),
                              x0, x1);
                    const float v0 = fast_exp2(x0), v1 = fast_exp2(x1);
                    pr[x] = (x >= clo && x < chi) ? v0 : 0.f;
                    pr[x + 1] = (x + 1 >= clo && x + 1 < chi) ? v1 : 0.f;
                }
            }
            if (!warp_wait(bar(C::BAR_DPFULL), g & 1, abort_flag, p.wait_limit_ns, p.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            {
                uint32_t dv[2][32];
                tmem_ld32(trow + C::COL_DP + cb, dv[0]);
                tmem_ld32(trow + C::COL_DP + cb + 32, dv[1]);
                tmem_wait_ld();
                reg_fence32(dv[0]);
                reg_fence32(dv[1]);
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t pk[16];
                    const uint64_t nd2 = f2_pack(-del, -del);
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const int x = 32 * c + 2 * k;
                        float d0, d1;
                        f2_unpack(f2_mul(f2_pack(pr[x], pr[x + 1]),
                                         f2_add(f2_pack(__uint_as_float(dv[c][2 * k]),
                                                        __uint_as_float(dv[c][2 * k + 1])),
                                                nd2)),
                                  d0, d1);
                        pk[k] = pack_bf16x2(d0, d1);
                    }
                    tmem_st16(t_s + 16 * c, pk);  // dS over this warp's own S columns
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(C::BAR_DSFULL));
        }
        const bool have = ok && n_kt > 0 &&
                          warp_wait(bar(C::BAR_DONE), 0, abort_flag, p.wait_limit_ns, p.status);
        if (have) {
            tc_fence_after();
            tc_store_half<D>(trow + C::COL_DQ, p.dQ + (qrow + i) * D, half * (D / 2), p.scale, i < p.Sq,
                             i < q_end);
        } else if (i < p.Sq && !*abort_flag) {
            tc_zero_half<D>(p.dQ + (qrow + i) * D, half * (D / 2));
        }
    }
    tc_teardown<C>(smem, tmem);
}

struct SideStream {
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    std::mutex mu;
};

// One side stream (and its fork / join events) per device, made on first use.
SideStream *side_stream() {
    static std::mutex mu;
    static SideStream *per_dev[64] = {};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!per_dev[dev]) {
        SideStream *ss = new SideStream();
        if (cudaStreamCreateWithFlags(&ss->s, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&ss->fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&ss->join, cudaEventDisableTiming) != cudaSuccess)
            return nullptr;
        per_dev[dev] = ss;
    }
    return per_dev[dev];
}

template <int D>
attn_status_t launch_bwd_tc_d(const BwdArgs &a, cudaStream_t stream) {
    using C = TcCfg<D>;
    CUtensorMap tq, tk, tv, tdo;
    attn_status_t st;
    if ((st = make_tmap_bf16_3d(&tq, a.Q, D, a.Sq, (uint64_t)a.B * a.Hq, TB)) != ATTN_OK) return st;
    if ((st = make_tmap_bf16_3d(&tdo, a.dO, D, a.Sq, (uint64_t)a.B * a.Hq, TB)) != ATTN_OK) return st;
    if ((st = make_tmap_bf16_3d(&tk, a.K, D, a.Sk, (uint64_t)a.B * a.Hkv, TB)) != ATTN_OK) return st;
    if ((st = make_tmap_bf16_3d(&tv, a.V, D, a.Sk, (uint64_t)a.B * a.Hkv, TB)) != ATTN_OK) return st;
    if (kernel_setup(reinterpret_cast<const void *>(bwd_dkdv_tc_kernel<D>), C::SMEM) != cudaSuccess ||
        kernel_setup(reinterpret_cast<const void *>(bwd_dq_tc_kernel<D>), DqCfg<D>::SMEM) !=
            cudaSuccess)
        return ATTN_ERR_CUDA;
    TcParams p;
    p.LSE = a.LSE;
    p.delta = a.delta;
    p.dQ = static_cast<__nv_bfloat16 *>(a.dQ);
    p.dK = static_cast<__nv_bfloat16 *>(a.dK);
    p.dV = static_cast<__nv_bfloat16 *>(a.dV);
    p.k_lengths = a.k_lengths;
    p.q_lengths = a.q_lengths;
    p.B = a.B;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.Sq = a.Sq;
    p.Sk = a.Sk;
    p.group = a.Hq / a.Hkv;
    p.scale = a.scale;
    p.scale_log2 = a.scale * kLog2e;
    p.causal = a.causal;
    p.window = a.window;
    p.input_pos = a.input_pos;
    p.wait_limit_ns = kWaitLimitNs;
    p.status = device_status_word();
    if (!p.status) return ATTN_ERR_CUDA;
    const int n_qt = (a.Sq + TB - 1) / TB;
    const long long grid = (long long)n_qt * a.Hq * a.B;
    if (grid > 0x7fffffffll) return ATTN_ERR_INVALID;
    // dK/dV and dQ are independent: run dQ on a side stream so that each kernel's
    // last wave overlaps the other's work.
    SideStream *ss = side_stream();
    if (!ss) return ATTN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(ss->mu);
    if (cudaEventRecord(ss->fork, stream) != cudaSuccess ||
        cudaStreamWaitEvent(ss->s, ss->fork, 0) != cudaSuccess)
        return ATTN_ERR_CUDA;
    bwd_dq_tc_kernel<D><<<static_cast<unsigned>(grid), kThreadsTc, DqCfg<D>::SMEM, ss->s>>>(tq, tk, tv, tdo, p,
                                                                                    n_qt);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    if (a.Sk > 0) {
        const long long grid_kv = (long long)((a.Sk + TB - 1) / TB) * a.Hkv * a.B;
        if (grid_kv > 0x7fffffffll) return ATTN_ERR_INVALID;
        bwd_dkdv_tc_kernel<D><<<static_cast<unsigned>(grid_kv), kThreadsTc, C::SMEM, stream>>>(
            tq, tk, tv, tdo, p);
        if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    }
    if (cudaEventRecord(ss->join, ss->s) != cudaSuccess ||
        cudaStreamWaitEvent(stream, ss->join, 0) != cudaSuccess)
        return ATTN_ERR_CUDA;
    return ATTN_OK;
}

}  // namespace

attn_status_t launch_bwd_tc(const BwdArgs &a, cudaStream_t stream) {
    if (a.D == 128) return launch_bwd_tc_d<128>(a, stream);
    if (a.D == 64) return launch_bwd_tc_d<64>(a, stream);
    return ATTN_ERR_UNSUPPORTED;
}

}  // namespace gqa
