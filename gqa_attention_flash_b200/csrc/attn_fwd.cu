// attn_fwd.cu -- fused GQA attention forward for sm_100a.
//
// Computes, per (batch b, query head hq, 128-row query tile), the rows of
// O = softmax(Q K^T * scale + mask) V and their log-sum-exp, as defined on the
// Tylo.jl "Primitives" page (entry `attention!`: fused MHA with GQA, causal,
// input_pos, k_lengths / q_lengths, saved softmax statistics M/L, Float32
// accumulation) with the sliding window of the mlx-arsenal "Attention" page
// (entry `sliding_window_mask`).
//
// One CTA per (query tile, hq, b); 6 warps with fixed roles:
//   warps 0-3  softmax: one thread per query row (TMEM lane), online softmax
//              in fp32 in the exp2 domain, P written back to TMEM as bf16,
//              lazy O rescaling, epilogue O / L -> bf16 and LSE.
//   warp 4     TMA producer: Q once, then K_j / V_j into an NS-stage ring.
//   warp 5     MMA issuer (one thread): S_j = Q K_j^T into one of two TMEM S
//              buffers, O += P_j V_j with P read from TMEM; owns the TMEM
//              allocation.
// Only the KV tiles that hold a visible key are visited (whole-tile skipping
// for causal / window / length masks, Tylo `flex_attention!` keyword
// block_sparse); the per-element mask is applied on boundary tiles only.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace gqa {

namespace {

constexpr int BM = 128;  // query rows per tile (= TMEM lanes)
constexpr int BN = 128;  // keys per KV tile
constexpr int kThreads = 192;

template <int D>
struct FwdCfg {
    static constexpr int NS = (D == 128) ? 2 : 4;  // K/V ring depth
    static constexpr int NBOX = D / 64;             // 64-column TMA boxes per row
    static constexpr int BOX_Q = BM * 128;           // bytes of one Q box
    static constexpr int BOX_KV = BN * 128;          // bytes of one K or V box
    static constexpr int Q_BYTES = BM * D * 2;
    static constexpr int KV_BYTES = BN * D * 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + NS * KV_BYTES;
    // barriers: q_full, k_full[NS], v_full[NS], kv_empty[NS], s_full[2], p_full[2], o_done
    static constexpr int BAR_Q = 0;
    static constexpr int BAR_KFULL = 1;
    static constexpr int BAR_VFULL = 1 + NS;
    static constexpr int BAR_EMPTY = 1 + 2 * NS;
    static constexpr int BAR_SFULL = 1 + 3 * NS;
    static constexpr int BAR_PFULL = 3 + 3 * NS;
    static constexpr int BAR_ODONE = 5 + 3 * NS;
    static constexpr int N_BARS = 6 + 3 * NS;
    static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;  // tmem slot, abort flag
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t O_COL = 256;  // S buffers at columns 0 and 128
};

struct FwdParams {
    __nv_bfloat16 *O;
    float *LSE;
    const int32_t *k_lengths;
    const int32_t *q_lengths;
    int B, Hq, Hkv, Sq, Sk, group, n_qtiles;
    float scale_log2;  // scale * log2(e)
    int causal, window, input_pos;
    uint64_t wait_limit_ns;
};

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
    using C = FwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8 * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- which tile: heaviest causal query tiles first, sibling heads adjacent ----
    int bid = blockIdx.x;
    const int hq = bid % p.Hq;
    bid /= p.Hq;
    const int b = bid % p.B;
    bid /= p.B;
    const int qt = p.n_qtiles - 1 - bid;
    const int hkv = hq / p.group;
    const int q0 = qt * BM;

    // ---- visible KV range of this tile (step a1: whole-tile skipping) ----
    int k_end = p.Sk, q_end = p.Sq;
    if (p.k_lengths) {
        int kl = p.k_lengths[b];
        if (kl > p.Sk) {
            if (threadIdx.x == 0 && hq == 0 && qt == 0) record_status(ATTN_ERR_DEVICE_BOUNDS);
            kl = p.Sk;
        }
        k_end = kl > 0 ? kl : 0;
    }
    if (p.q_lengths) {
        int ql = p.q_lengths[b];
        if (ql > p.Sq) {
            if (threadIdx.x == 0 && hq == 0 && qt == 0) record_status(ATTN_ERR_DEVICE_BOUNDS);
            ql = p.Sq;
        }
        q_end = ql > 0 ? ql : 0;
    }
    int n_tiles = 0, t_begin = 0, q_last = q0;
    if (q0 < q_end && k_end > 0) {
        q_last = min(q0 + BM - 1, q_end - 1);
        long long hi = k_end;
        if (p.causal) hi = min(hi, (long long)p.input_pos + q_last + 1);
        long long lo = 0;
        if (p.window > 0) lo = max(0ll, (long long)p.input_pos + q0 - p.window + 1);
        if (hi > lo) {
            t_begin = static_cast<int>(lo / BN);
            n_tiles = static_cast<int>((hi + BN - 1) / BN) - t_begin;
        }
    }

    // ---- set-up ----
    if (threadIdx.x == 0) {
        mbar_init(bar(C::BAR_Q), 1);
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(bar(C::BAR_KFULL + s), 1);
            mbar_init(bar(C::BAR_VFULL + s), 1);
            mbar_init(bar(C::BAR_EMPTY + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(C::BAR_SFULL + s), 1);
            mbar_init(bar(C::BAR_PFULL + s), BM);
        }
        mbar_init(bar(C::BAR_ODONE), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (n_tiles > 0 && warp == 4) {
        // ===================== TMA producer =====================
        if (lane == 0) {
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            mbar_arrive_expect_tx(bar(C::BAR_Q), C::Q_BYTES);
            for (int c = 0; c < C::NBOX; ++c)
                tma_load_3d(sbase + C::OFF_Q + c * C::BOX_Q, &tmQ, bar(C::BAR_Q), c * 64, q0,
                            b * p.Hq + hq);
            for (int it = 0; it < n_tiles; ++it) {
                const int st = it % C::NS;
                const int use = it / C::NS;
                if (use > 0 &&
                    !mbar_wait(bar(C::BAR_EMPTY + st), (use - 1) & 1, abort_flag, p.wait_limit_ns))
                    break;
                const int kv_row = (t_begin + it) * BN;
                mbar_arrive_expect_tx(bar(C::BAR_KFULL + st), C::KV_BYTES);
                for (int c = 0; c < C::NBOX; ++c)
                    tma_load_3d(sbase + C::OFF_K + st * C::KV_BYTES + c * C::BOX_KV, &tmK,
                                bar(C::BAR_KFULL + st), c * 64, kv_row, b * p.Hkv + hkv);
                mbar_arrive_expect_tx(bar(C::BAR_VFULL + st), C::KV_BYTES);
                for (int c = 0; c < C::NBOX; ++c)
                    tma_load_3d(sbase + C::OFF_V + st * C::KV_BYTES + c * C::BOX_KV, &tmV,
                                bar(C::BAR_VFULL + st), c * 64, kv_row, b * p.Hkv + hkv);
            }
        }
    } else if (n_tiles > 0 && warp == 5) {
        // ===================== MMA issuer =====================
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16_f32(BM, BN, 0, 0);
            constexpr uint32_t idO = idesc_bf16_f32(BM, D, 0, 1);
            auto issue_s = [&](int it) -> bool {
                const int st = it % C::NS;
                const int buf = it & 1;
                if (!mbar_wait(bar(C::BAR_KFULL + st), (it / C::NS) & 1, abort_flag,
                               p.wait_limit_ns))
                    return false;
                tc_fence_after();
                const uint32_t qa = sbase + C::OFF_Q;
                const uint32_t ka = sbase + C::OFF_K + st * C::KV_BYTES;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::BOX_Q + (kk & 3) * 32;
                    const uint64_t da = smem_desc_sw128(qa + off, 16, 1024);
                    const uint64_t db = smem_desc_sw128(ka + off, 16, 1024);
                    mma_ss(tmem + buf * BN, da, db, idS, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar(C::BAR_SFULL + buf));
                return true;
            };
            auto issue_pv = [&](int it) -> bool {
                const int st = it % C::NS;
                const int buf = it & 1;
                if (!mbar_wait(bar(C::BAR_PFULL + buf), (it >> 1) & 1, abort_flag, p.wait_limit_ns))
                    return false;
                if (!mbar_wait(bar(C::BAR_VFULL + st), (it / C::NS) & 1, abort_flag,
                               p.wait_limit_ns))
                    return false;
                tc_fence_after();
                const uint32_t va = sbase + C::OFF_V + st * C::KV_BYTES;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint64_t db = smem_desc_sw128(va + kk * 16 * 128, C::BOX_KV, 1024);
                    mma_ts(tmem + C::O_COL, tmem + buf * BN + kk * 8, db, idO,
                           (it > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(bar(C::BAR_EMPTY + st));
                mma_commit(bar(C::BAR_ODONE));
                return true;
            };
            if (mbar_wait(bar(C::BAR_Q), 0, abort_flag, p.wait_limit_ns) && issue_s(0)) {
                for (int it = 0; it < n_tiles; ++it) {
                    if (it + 1 < n_tiles && !issue_s(it + 1)) break;
                    if (!issue_pv(it)) break;
                }
            }
        }
    } else if (warp < 4) {
        // ===================== softmax / correction / epilogue =====================
        const int r = threadIdx.x;             // query row within the tile = TMEM lane
        const int row = q0 + r;                // query row within the sequence
        const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const long long pos = (long long)p.input_pos + row;  // absolute position
        float m_used = neg_inf();              // max subtracted so far (log2 units)
        float l = 0.f;
        bool ok = true;

        for (int it = 0; it < n_tiles; ++it) {
            const int buf = it & 1;
            const int kv0 = (t_begin + it) * BN;
            if (!warp_wait(bar(C::BAR_SFULL + buf), (it >> 1) & 1, abort_flag, p.wait_limit_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float s[BN];
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(trow + buf * BN + c * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 32; ++k) s[c * 32 + k] = __uint_as_float(v[k]);
            }
            // step a5: per-element mask on boundary tiles only
            const bool edge = (kv0 + BN > k_end) ||
                              (p.causal && (long long)kv0 + BN - 1 > (long long)p.input_pos + q0) ||
                              (p.window > 0 &&
                               (long long)kv0 <= (long long)p.input_pos + q_last - p.window);
            if (edge) {
                long long hi = k_end;
                if (p.causal) hi = min(hi, pos + 1);
                long long lo = p.window > 0 ? pos - p.window + 1 : 0;
                const int c_hi = static_cast<int>(max(-1ll, min((long long)BN, hi - kv0)));
                const int c_lo = static_cast<int>(max(-1ll, min((long long)BN, lo - kv0)));
#pragma unroll
                for (int c = 0; c < BN; ++c) s[c] = (c >= c_lo && c < c_hi) ? s[c] : neg_inf();
            }
            // step a6: online softmax in the exp2 domain, lazy rescaling
            float mx = s[0];
#pragma unroll
            for (int c = 1; c < BN; ++c) mx = fmaxf(mx, s[c]);
            const float m_new = mx * p.scale_log2;
            float alpha = 1.f;
            bool resc = false;
            if (m_new > m_used + 8.f) {
                alpha = fast_exp2(m_used - m_new);
                m_used = m_new;
                resc = true;
            }
            const float m_eff = (m_used == neg_inf()) ? 0.f : m_used;
            float sum = 0.f;
            uint32_t pk[BN / 2];
#pragma unroll
            for (int c = 0; c < BN / 2; ++c) {
                const float p0 = fast_exp2(fmaf(s[2 * c], p.scale_log2, -m_eff));
                const float p1 = fast_exp2(fmaf(s[2 * c + 1], p.scale_log2, -m_eff));
                sum += p0 + p1;
                pk[c] = pack_bf16x2(p0, p1);
            }
            l = l * alpha + sum;
#pragma unroll
            for (int c = 0; c < BN / 64; ++c) {
                uint32_t v[32];
#pragma unroll
                for (int k = 0; k < 32; ++k) v[k] = pk[c * 32 + k];
                tmem_st32(trow + buf * BN + c * 32, v);
            }
            // Key rows at or past k_end inside this tile may hold anything; their
            // weights are exactly 0, but 0 * NaN is NaN, so zero those V rows.
            if (k_end < p.Sk && k_end > kv0 && k_end < kv0 + BN) {
                const int st = it % C::NS;
                if (!warp_wait(bar(C::BAR_VFULL + st), (it / C::NS) & 1, abort_flag,
                               p.wait_limit_ns)) {
                    ok = false;
                }
                if (ok && r >= k_end - kv0 && r < p.Sk - kv0) {
#pragma unroll
                    for (int c = 0; c < C::NBOX; ++c) {
                        uint4 *dst = reinterpret_cast<uint4 *>(smem + C::OFF_V + st * C::KV_BYTES +
                                                               c * C::BOX_KV + r * 128);
#pragma unroll
                        for (int k = 0; k < 8; ++k) dst[k] = make_uint4(0, 0, 0, 0);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
            }
            // O correction: only when some row of this warp moved its max by > 8
            if (ok && it > 0 && __any_sync(0xffffffffu, resc)) {
                if (!warp_wait(bar(C::BAR_ODONE), (it - 1) & 1, abort_flag, p.wait_limit_ns)) {
                    ok = false;
                } else {
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t v[32];
                        tmem_ld32(trow + C::O_COL + c * 32, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 32; ++k)
                            v[k] = __float_as_uint(__uint_as_float(v[k]) * alpha);
                        tmem_st32(trow + C::O_COL + c * 32, v);
                    }
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(C::BAR_PFULL + buf));
            if (!ok) break;
        }

        // step a8: epilogue
        const bool row_in = row < p.Sq;
        bool have = ok && n_tiles > 0;
        if (have &&
            !warp_wait(bar(C::BAR_ODONE), (n_tiles - 1) & 1, abort_flag, p.wait_limit_ns))
            have = false;
        const bool out_valid = have && row < q_end && l > 0.f;
        const float inv_l = out_valid ? 1.f / l : 0.f;
        __nv_bfloat16 *orow = p.O + ((long long)(b * p.Hq + hq) * p.Sq + row) * D;
        if (have) {
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(trow + C::O_COL + c * 32, v);
                tmem_wait_ld();
                uint32_t o16[16];
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    o16[k] = pack_bf16x2(__uint_as_float(v[2 * k]) * inv_l,
                                         __uint_as_float(v[2 * k + 1]) * inv_l);
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
            p.LSE[(long long)(b * p.Hq + hq) * p.Sq + row] =
                out_valid ? m_used * 0.69314718055994531f + logf(l) : neg_inf();
        }
    }

    // ---- teardown ----
    if (*abort_flag) drain_delay(2000000);  // let copies / MMAs in flight land
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int D>
attn_status_t launch_fwd_d(const FwdArgs &a, cudaStream_t stream) {
    using C = FwdCfg<D>;
    CUtensorMap tq, tk, tv;
    attn_status_t st;
    if ((st = make_tmap_bf16_3d(&tq, a.Q, D, a.Sq, (uint64_t)a.B * a.Hq, BM)) != ATTN_OK) return st;
    if ((st = make_tmap_bf16_3d(&tk, a.K, D, a.Sk, (uint64_t)a.B * a.Hkv, BN)) != ATTN_OK) return st;
    if ((st = make_tmap_bf16_3d(&tv, a.V, D, a.Sk, (uint64_t)a.B * a.Hkv, BN)) != ATTN_OK) return st;
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM_BYTES) != cudaSuccess)
            return ATTN_ERR_CUDA;
        configured = true;
    }
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
    p.n_qtiles = (a.Sq + BM - 1) / BM;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.causal = a.causal;
    p.window = a.window;
    p.input_pos = a.input_pos;
    p.wait_limit_ns = kWaitLimitNs;
    const long long grid = (long long)p.n_qtiles * a.Hq * a.B;
    if (grid == 0) return ATTN_OK;
    if (grid > 0x7fffffffll) return ATTN_ERR_INVALID;
    attn_fwd_kernel<D><<<static_cast<unsigned>(grid), kThreads, C::SMEM_BYTES, stream>>>(tq, tk, tv,
                                                                                          p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

attn_status_t launch_fwd(const FwdArgs &a, cudaStream_t stream) {
    if (a.D == 128) return launch_fwd_d<128>(a, stream);
    if (a.D == 64) return launch_fwd_d<64>(a, stream);
    return ATTN_ERR_UNSUPPORTED;
}

}  // namespace gqa
