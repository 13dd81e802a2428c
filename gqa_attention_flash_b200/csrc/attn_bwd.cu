// attn_bwd.cu -- backward of the fused GQA attention forward for sm_100a.
//
// Tylo.jl "Primitives" page, entry `∇attention!`: from the output gradient dO,
// the inputs, the output O and the saved softmax statistics (here LSE = M + ln L)
// write dQ, dK, dV.  With P = exp(S * scale - LSE) (S = Q K^T) on the visible
// pairs of the forward's masks:
//   delta_i = sum_d dO_id O_id                       (= sum_j P_ij dP_ij)
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - delta),  dQ = scale dS K,
//   dK = scale dS^T Q; a KV head collects the gradients of its query heads.
//
// Three kernels, 64-row tiles, warp-level bf16 mma.sync (m16n8k16, fp32
// accumulate) fed from shared memory by ldmatrix:
//   bwd_delta_kernel  one warp per query row: delta_i.
//   bwd_dkdv_kernel   one CTA per (64-key tile, KV head, batch); four warps own
//                     16 keys each and keep their dK / dV rows in registers while
//                     the CTA walks every query tile of every query head of the
//                     group that can see the key tile: S^T = K Q^T, P^T, dV +=
//                     P^T dO, dP^T = V dO^T, dS^T, dK += dS^T Q.
//   bwd_dq_kernel     one CTA per (64-row query tile, query head, batch); four
//                     warps own 16 rows each and walk the visible key tiles:
//                     S = Q K^T, P, dP = dO V^T, dS, dQ += dS K.
// dS and P are recomputed in both kernels instead of exchanging dQ partials
// through atomics.  P and dS enter the second product of each pair as bf16, like
// P in the forward.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace gqa {

namespace {

constexpr int kT = 64;          // rows per tile (queries or keys)
constexpr int kWarps = 4;       // 16 rows each
constexpr int kThreadsBwd = 32 * kWarps;

struct BwdParams {
    const __nv_bfloat16 *Q, *K, *V, *dO, *O;
    const float *LSE;
    float *delta;  // (B, Hq, Sq) workspace
    __nv_bfloat16 *dQ, *dK, *dV;
    const int32_t *k_lengths, *q_lengths;
    int B, Hq, Hkv, Sq, Sk, group;
    float scale, scale_log2;
    int causal, window, input_pos;
    int *status;
};

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }

// Byte offset of 16-byte chunk c of row `row` in a 64-row tile stored as D/64
// boxes of (64 rows x 128 bytes) with the 128-byte XOR swizzle (conflict-free
// ldmatrix along rows and along columns).
__device__ __forceinline__ uint32_t swz(int row, int c) {
    return (c >> 3) * (kT * 128) + row * 128 + (((c & 7) ^ (row & 7)) << 4);
}

// Copy rows [r0, r0 + 64) of a row-major (rows, D) bf16 matrix into a swizzled
// tile; rows at or past n_rows are zero.
template <int D>
__device__ __forceinline__ void load_tile(uint8_t *dst, const __nv_bfloat16 *src, int r0,
                                          int n_rows) {
    constexpr int CH = D / 8;  // 16-byte chunks per row
    for (int idx = threadIdx.x; idx < kT * CH; idx += kThreadsBwd) {
        const int row = idx / CH, c = idx % CH;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r0 + row < n_rows)
            v = *reinterpret_cast<const uint4 *>(src + (long long)(r0 + row) * D + c * 8);
        *reinterpret_cast<uint4 *>(dst + swz(row, c)) = v;
    }
}

// Asynchronous 16-byte global -> shared copies (zero-filled when `valid` is false;
// the source address is then only a placeholder inside the tensor).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// load_tile with cp.async: rows [r0, r0 + 64) into the swizzled tile at `dst`.
template <int D>
__device__ __forceinline__ void load_tile_async(uint32_t dst, const __nv_bfloat16 *src, int r0,
                                                int n_rows) {
    constexpr int CH = D / 8;
    for (int idx = threadIdx.x; idx < kT * CH; idx += kThreadsBwd) {
        const int row = idx / CH, c = idx % CH;
        const bool ok = r0 + row < n_rows;
        cp_async16(dst + swz(row, c), src + (long long)(ok ? r0 + row : 0) * D + c * 8, ok);
    }
}

// Asynchronous 4-byte copy (zero-filled when `valid` is false).
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src),
                 "r"(valid ? 4 : 0)
                 : "memory");
}

// Lengths of batch entry b, clamped to the tensor (a length past it is flagged).
__device__ __forceinline__ void bwd_lengths(const BwdParams &p, int b, int &k_end, int &q_end) {
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

// Key j visible from query row i (the forward's masks).
__device__ __forceinline__ bool visible(const BwdParams &p, int i, int j, int k_end, int q_end) {
    if (i >= q_end || j >= k_end) return false;
    const long long pos = (long long)p.input_pos + i;
    if (p.causal && j > pos) return false;
    if (p.window > 0 && j <= pos - p.window) return false;
    return true;
}

// ---------------------------------------------------------------------------------
// delta_i = <dO_i, O_i>
// ---------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const BwdParams p, long long rows) {
    const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    const __nv_bfloat16 *go = p.dO + r * D, *o = p.O + r * D;
    float acc = 0.f;
    for (int d = lane * 2; d < D; d += 64) {
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(go + d);
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(o + d);
        acc = fmaf(__low2float(a), __low2float(b), acc);
        acc = fmaf(__high2float(a), __high2float(b), acc);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) p.delta[r] = acc;
}

// A fragments (16 rows x k16) of rows [r0, r0 + 16) of a swizzled tile, chunk pair kk.
__device__ __forceinline__ void ld_a(uint32_t (&a)[4], uint32_t tile, int r0, int kk, int lane) {
    const int mi = lane >> 3, rr = lane & 7;
    ldmatrix_x4(tile + swz(r0 + (mi & 1) * 8 + rr, 2 * kk + (mi >> 1)), a[0], a[1], a[2], a[3]);
}

// B fragments of two n8 tiles (rows [n0, n0 + 16) of the tile as the n index, the
// row's columns as k): b0, b1 for rows n0..n0+7, b2, b3 for n0+8..n0+15.
__device__ __forceinline__ void ld_b_rows(uint32_t (&b)[4], uint32_t tile, int n0, int kk, int lane) {
    const int mi = lane >> 3, rr = lane & 7;
    ldmatrix_x4(tile + swz(n0 + (mi >> 1) * 8 + rr, 2 * kk + (mi & 1)), b[0], b[1], b[2], b[3]);
}

// B fragments with the tile's rows as the k index (rows [k0, k0 + 16)) and its
// columns as n: b0, b1 for column chunk 2 dp, b2, b3 for chunk 2 dp + 1.
__device__ __forceinline__ void ld_b_cols(uint32_t (&b)[4], uint32_t tile, int k0, int dp, int lane) {
    const int mi = lane >> 3, rr = lane & 7;
    ldmatrix_x4_trans(tile + swz(k0 + (mi & 1) * 8 + rr, 2 * dp + (mi >> 1)), b[0], b[1], b[2],
                      b[3]);
}

// A fragment (16 x k16) from two adjacent m16n8 accumulators (n-tiles 2k, 2k+1).
__device__ __forceinline__ void c_to_a(uint32_t (&a)[4], const float (&lo)[4], const float (&hi)[4]) {
    a[0] = pack_bf16x2(lo[0], lo[1]);
    a[1] = pack_bf16x2(lo[2], lo[3]);
    a[2] = pack_bf16x2(hi[0], hi[1]);
    a[3] = pack_bf16x2(hi[2], hi[3]);
}

template <int D>
struct BwdCfg {
    static constexpr int TILE = kT * D * 2;  // bytes of one 64-row tile
    static constexpr int OFF_A = 0;          // K (dkdv) or Q (dq), resident
    static constexpr int OFF_B = TILE;       // V or dO, resident
    // two stages of streamed tiles: Q and dO (dkdv) or K and V (dq), then 64 LSE
    // and 64 delta floats (dkdv)
    static constexpr int STAGE = 2 * TILE + 2 * kT * 4;
    static constexpr int OFF_S = 2 * TILE;
    __host__ __device__ static constexpr int stage(int s) { return OFF_S + s * STAGE; }
    static constexpr int SMEM = OFF_S + 2 * STAGE + 1024;
};

// ---------------------------------------------------------------------------------
// dK, dV of one 64-key tile
// ---------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kThreadsBwd, 1) bwd_dkdv_kernel(const BwdParams p) {
    using C = BwdCfg<D>;
    constexpr int NT = D / 8;  // n8 tiles along D
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    const int kt = blockIdx.x, hkv = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int kv0 = kt * kT;
    int k_end, q_end;
    bwd_lengths(p, b, k_end, q_end);

    const long long kv_base = (long long)(b * p.Hkv + hkv) * p.Sk;
    load_tile<D>(smem + C::OFF_A, p.K + kv_base * D, kv0, p.Sk);
    load_tile<D>(smem + C::OFF_B, p.V + kv_base * D, kv0, p.Sk);

    float dk[NT][4], dv[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) dk[n][e] = dv[n][e] = 0.f;

    // query rows that can see a key of this tile
    int i_lo = 0, i_hi = q_end;
    if (kv0 >= k_end) i_hi = 0;
    if (p.causal) i_lo = max(0, kv0 - p.input_pos);
    if (p.window > 0) i_hi = min(i_hi, kv0 + kT + p.window - p.input_pos);
    const int qt_lo = i_lo / kT, qt_hi = i_hi > i_lo ? (i_hi + kT - 1) / kT : qt_lo;

    // (query head, query tile) pairs in order, the next one's Q, dO, LSE and delta
    // copied asynchronously into the other stage while this one is computed
    const int n_qt = qt_hi - qt_lo;
    const int n_it = p.group * n_qt;
    auto issue = [&](int it) {
        const int hq = hkv * p.group + it / n_qt;
        const int q0 = (qt_lo + it % n_qt) * kT;
        const long long qb = (long long)(b * p.Hq + hq) * p.Sq;
        const uint32_t st = sb + C::stage(it & 1);
        load_tile_async<D>(st, p.Q + qb * D, q0, p.Sq);
        load_tile_async<D>(st + C::TILE, p.dO + qb * D, q0, p.Sq);
        if (threadIdx.x < kT) {
            const int i = q0 + threadIdx.x;
            const bool ok = i < p.Sq;
            cp_async4(st + 2 * C::TILE + 4 * threadIdx.x, p.LSE + qb + (ok ? i : 0), ok);
            cp_async4(st + 2 * C::TILE + 4 * (kT + threadIdx.x), p.delta + qb + (ok ? i : 0), ok);
        }
        cp_async_commit();
    };
    if (n_it > 0) issue(0);
    for (int it = 0; it < n_it; ++it) {
        {
            if (it + 1 < n_it)
                issue(it + 1);
            else
                cp_async_commit();  // empty group: the wait below always leaves one pending
            cp_async_wait<1>();
            __syncthreads();
            const int q0 = (qt_lo + it % n_qt) * kT;
            const uint32_t so = C::stage(it & 1);
            const uint32_t tq = sb + so, tdo = sb + so + C::TILE;
            const float *lse_s = reinterpret_cast<const float *>(smem + so + 2 * C::TILE);
            const float *del_s = lse_s + kT;

            // S^T (16 keys of this warp x 64 queries)
            float st[8][4];
#pragma unroll
            for (int n = 0; n < 8; ++n) st[n][0] = st[n][1] = st[n][2] = st[n][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                uint32_t a[4];
                ld_a(a, sb + C::OFF_A, warp * 16, kk, lane);
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t bq[4];
                    ld_b_rows(bq, tq, np * 16, kk, lane);
                    mma_m16n8k16(st[2 * np], a, bq[0], bq[1]);
                    mma_m16n8k16(st[2 * np + 1], a, bq[2], bq[3]);
                }
            }
            // P^T on the visible pairs
#pragma unroll
            for (int n = 0; n < 8; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = kv0 + warp * 16 + g + (e >> 1) * 8;
                    const int il = n * 8 + 2 * t + (e & 1);
                    const float lse = lse_s[il] * 1.4426950408889634f;
                    const bool vis = visible(p, q0 + il, j, k_end, q_end) && lse != neg_inf();
                    st[n][e] = vis ? fast_exp2(fmaf(st[n][e], p.scale_log2, -lse)) : 0.f;
                }
            // dV += P^T dO
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
                uint32_t a[4];
                c_to_a(a, st[2 * kq], st[2 * kq + 1]);
#pragma unroll
                for (int dp = 0; dp < D / 16; ++dp) {
                    uint32_t bo[4];
                    ld_b_cols(bo, tdo, kq * 16, dp, lane);
                    mma_m16n8k16(dv[2 * dp], a, bo[0], bo[1]);
                    mma_m16n8k16(dv[2 * dp + 1], a, bo[2], bo[3]);
                }
            }
            // dP^T = V dO^T, then dS^T = P^T (dP^T - delta)
            float dpt[8][4];
#pragma unroll
            for (int n = 0; n < 8; ++n) dpt[n][0] = dpt[n][1] = dpt[n][2] = dpt[n][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                uint32_t a[4];
                ld_a(a, sb + C::OFF_B, warp * 16, kk, lane);
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t bq[4];
                    ld_b_rows(bq, tdo, np * 16, kk, lane);
                    mma_m16n8k16(dpt[2 * np], a, bq[0], bq[1]);
                    mma_m16n8k16(dpt[2 * np + 1], a, bq[2], bq[3]);
                }
            }
#pragma unroll
            for (int n = 0; n < 8; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    dpt[n][e] = st[n][e] * (dpt[n][e] - del_s[n * 8 + 2 * t + (e & 1)]);
            // dK += dS^T Q
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
                uint32_t a[4];
                c_to_a(a, dpt[2 * kq], dpt[2 * kq + 1]);
#pragma unroll
                for (int dp = 0; dp < D / 16; ++dp) {
                    uint32_t bq[4];
                    ld_b_cols(bq, tq, kq * 16, dp, lane);
                    mma_m16n8k16(dk[2 * dp], a, bq[0], bq[1]);
                    mma_m16n8k16(dk[2 * dp + 1], a, bq[2], bq[3]);
                }
            }
        }
        __syncthreads();  // every warp is done with this stage before it is refilled
    }
    cp_async_wait<0>();
    // write dK (scaled) and dV rows of this warp's 16 keys
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int j = kv0 + warp * 16 + g + half * 8;
        if (j >= p.Sk) continue;
        __nv_bfloat16 *dkr = p.dK + (kv_base + j) * D;
        __nv_bfloat16 *dvr = p.dV + (kv_base + j) * D;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int col = n * 8 + 2 * t;
            *reinterpret_cast<uint32_t *>(dkr + col) =
                pack_bf16x2(dk[n][2 * half] * p.scale, dk[n][2 * half + 1] * p.scale);
            *reinterpret_cast<uint32_t *>(dvr + col) = pack_bf16x2(dv[n][2 * half], dv[n][2 * half + 1]);
        }
    }
}

// ---------------------------------------------------------------------------------
// dQ of one 64-row query tile
// ---------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kThreadsBwd, 1) bwd_dq_kernel(const BwdParams p) {
    using C = BwdCfg<D>;
    constexpr int NT = D / 8;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    const int qt = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
    const int hkv = hq / p.group;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int q0 = qt * kT;
    int k_end, q_end;
    bwd_lengths(p, b, k_end, q_end);
    const long long q_base = (long long)(b * p.Hq + hq) * p.Sq;
    const long long kv_base = (long long)(b * p.Hkv + hkv) * p.Sk;

    load_tile<D>(smem + C::OFF_A, p.Q + q_base * D, q0, p.Sq);
    load_tile<D>(smem + C::OFF_B, p.dO + q_base * D, q0, p.Sq);
    // this lane's rows: q0 + warp * 16 + g (+ 8)
    float lse2[2], del[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int i = q0 + warp * 16 + g + h * 8;
        lse2[h] = i < p.Sq ? p.LSE[q_base + i] * 1.4426950408889634f : neg_inf();
        del[h] = i < p.Sq ? p.delta[q_base + i] : 0.f;
    }

    float dq[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) dq[n][0] = dq[n][1] = dq[n][2] = dq[n][3] = 0.f;

    // key tiles holding a key some row of this tile sees
    int lo = 0, hi = 0;
    if (q0 < q_end && k_end > 0) {
        const int qlast = min(q0 + kT - 1, q_end - 1);
        long long h = k_end;
        if (p.causal) h = min(h, (long long)p.input_pos + qlast + 1);
        long long l = 0;
        if (p.window > 0) l = max(0ll, (long long)p.input_pos + q0 - p.window + 1);
        if (h > l) {
            lo = static_cast<int>(l / kT);
            hi = static_cast<int>((h + kT - 1) / kT);
        }
    }
    // key tiles in order, the next one's K and V copied asynchronously into the
    // other stage while this one is computed
    auto issue = [&](int kt) {
        const uint32_t st = sb + C::stage((kt - lo) & 1);
        load_tile_async<D>(st, p.K + kv_base * D, kt * kT, p.Sk);
        load_tile_async<D>(st + C::TILE, p.V + kv_base * D, kt * kT, p.Sk);
        cp_async_commit();
    };
    if (hi > lo) issue(lo);
    for (int kt = lo; kt < hi; ++kt) {
        const int kv0 = kt * kT;
        if (kt + 1 < hi)
            issue(kt + 1);
        else
            cp_async_commit();  // empty group: the wait below always leaves one pending
        cp_async_wait<1>();
        __syncthreads();
        const uint32_t tk = sb + C::stage((kt - lo) & 1), tv = tk + C::TILE;
        // S (16 rows of this warp x 64 keys)
        float s[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            uint32_t a[4];
            ld_a(a, sb + C::OFF_A, warp * 16, kk, lane);
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t bk[4];
                ld_b_rows(bk, tk, np * 16, kk, lane);
                mma_m16n8k16(s[2 * np], a, bk[0], bk[1]);
                mma_m16n8k16(s[2 * np + 1], a, bk[2], bk[3]);
            }
        }
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = q0 + warp * 16 + g + (e >> 1) * 8;
                const int j = kv0 + n * 8 + 2 * t + (e & 1);
                const float l2 = lse2[e >> 1];
                const bool vis = visible(p, i, j, k_end, q_end) && l2 != neg_inf();
                s[n][e] = vis ? fast_exp2(fmaf(s[n][e], p.scale_log2, -l2)) : 0.f;
            }
        // dP = dO V^T, dS = P (dP - delta)
        float dps[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n) dps[n][0] = dps[n][1] = dps[n][2] = dps[n][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            uint32_t a[4];
            ld_a(a, sb + C::OFF_B, warp * 16, kk, lane);
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t bv[4];
                ld_b_rows(bv, tv, np * 16, kk, lane);
                mma_m16n8k16(dps[2 * np], a, bv[0], bv[1]);
                mma_m16n8k16(dps[2 * np + 1], a, bv[2], bv[3]);
            }
        }
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) dps[n][e] = s[n][e] * (dps[n][e] - del[e >> 1]);
        // dQ += dS K
#pragma unroll
        for (int kq = 0; kq < 4; ++kq) {
            uint32_t a[4];
            c_to_a(a, dps[2 * kq], dps[2 * kq + 1]);
#pragma unroll
            for (int dp = 0; dp < D / 16; ++dp) {
                uint32_t bk[4];
                ld_b_cols(bk, tk, kq * 16, dp, lane);
                mma_m16n8k16(dq[2 * dp], a, bk[0], bk[1]);
                mma_m16n8k16(dq[2 * dp + 1], a, bk[2], bk[3]);
            }
        }
        __syncthreads();  // every warp is done with this stage before it is refilled
    }
    cp_async_wait<0>();
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int i = q0 + warp * 16 + g + half * 8;
        if (i >= p.Sq) continue;
        __nv_bfloat16 *dqr = p.dQ + (q_base + i) * D;
#pragma unroll
        for (int n = 0; n < NT; ++n)
            *reinterpret_cast<uint32_t *>(dqr + n * 8 + 2 * t) =
                pack_bf16x2(dq[n][2 * half] * p.scale, dq[n][2 * half + 1] * p.scale);
    }
}

template <int D>
attn_status_t launch_bwd_d(const BwdArgs &a, cudaStream_t stream) {
    using C = BwdCfg<D>;
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM) != cudaSuccess ||
            cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM) != cudaSuccess)
            return ATTN_ERR_CUDA;
        configured = true;
    }
    BwdParams p;
    p.Q = static_cast<const __nv_bfloat16 *>(a.Q);
    p.K = static_cast<const __nv_bfloat16 *>(a.K);
    p.V = static_cast<const __nv_bfloat16 *>(a.V);
    p.dO = static_cast<const __nv_bfloat16 *>(a.dO);
    p.O = static_cast<const __nv_bfloat16 *>(a.O);
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
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.causal = a.causal;
    p.window = a.window;
    p.input_pos = a.input_pos;
    p.status = device_status_word();
    if (!p.status) return ATTN_ERR_CUDA;
    const long long rows = (long long)a.B * a.Hq * a.Sq;
    bwd_delta_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(p, rows);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    return launch_bwd_tc(a, stream);
}

}  // namespace

attn_status_t launch_bwd(const BwdArgs &a, cudaStream_t stream) {
    if (a.D == 128) return launch_bwd_d<128>(a, stream);
    if (a.D == 64) return launch_bwd_d<64>(a, stream);
    return ATTN_ERR_UNSUPPORTED;
}

}  // namespace gqa
