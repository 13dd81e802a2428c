// block_scores.cu -- block scores and block mask of block-sparse prefill, as on
// the mlx-arsenal "Radius-bounded block scores (RBS)" page (sections "The idea"
// and "What mlx-arsenal ships": radius_bounded_block_scores, relative_block_mask,
// and the recipe's union of both branches with a diagonal band).
//
// Kernels, 64-token blocks:
//   rbs_centroid_kernel  one CTA per (key block, KV head, batch): centroid c (fp32
//                        mean of the block's keys) and radius r = max |k - c|_2.
//   rbs_beta_kernel      (only above 64 key blocks) one CTA per (KV head, batch):
//                        sorts the head's radii, takes the median and the 90th
//                        percentile (linear interpolation between order
//                        statistics) and writes beta = clip((r - r_low) /
//                        (r_high - r_low), 0, 1) (1 for r > r_low, else 0, when
//                        the two coincide).  Up to 64 key blocks the scores kernel
//                        does the same with one warp (warp_radius_quantiles).
//   rbs_scores_kernel    one CTA per run of consecutive query blocks of a (query
//                        head, batch): up to 64 key blocks the runs are sized to
//                        about one wave of CTAs and share the head's staged
//                        centroids, the next query block loading while the current
//                        one is scored; above that, one query block.  For every
//                        query block and key block, l_base = <q, c> / sqrt(D) and l_rescue =
//                        (<q, c> + |q| r beta) / sqrt(D) for the block's query
//                        tokens, log-sum-exp over the tokens, then the row's
//                        relative mask: keep where score >= row max + ln alpha in
//                        either branch, or |qb - kb| < diagonal.  <q, c> for the
//                        64 tokens and 64 key blocks at a time is a 64 x 64 x D
//                        product on the tensor cores (warp-level bf16 MMA, fp32
//                        accumulation), taken transposed (key blocks as MMA rows)
//                        so that each key block's log-sum-exp over the tokens stays
//                        inside one warp, with each centroid split into a bf16 high
//                        part and a bf16 remainder, so the two products together
//                        carry the fp32 centroid to ~2^-17 relative (the queries
//                        are bf16 already).
// The mask is written as BlockMask states (2 = keep the whole block, 0 = skip),
// one (nqb, nkb) matrix per (batch, query head), ready for attn_fwd_flex.
#include <cuda_bf16.h>

#include <map>
#include <mutex>
#include <algorithm>
#include <utility>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace gqa {

namespace {

constexpr int kBlk = 64;

// 16-byte asynchronous copy global -> shared (cp.async); src_bytes 0 writes zeros.
// Every copy a thread issues is in flight at once, so staging a tile costs one
// memory round trip instead of one per loop iteration.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// Close the group of copies issued so far; wait until at most N groups are pending.
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int D>
__global__ void __launch_bounds__(128)
    rbs_centroid_kernel(const __nv_bfloat16 *__restrict__ K, __nv_bfloat16 *__restrict__ cent_hi,
                        __nv_bfloat16 *__restrict__ cent_lo, float *__restrict__ rad, int Hkv, int Sk,
                        int nkb) {
    __shared__ __align__(16) __nv_bfloat16 kblk[kBlk * D];  // the key block, read once
    __shared__ float c[D];
    __shared__ float part[128 / (D / 2)][D];
    __shared__ float rmax_w[4];
    const int kb = blockIdx.x, hkv = blockIdx.y, b = blockIdx.z;
    const int j0 = kb * kBlk, n = min(kBlk, Sk - j0);
    const __nv_bfloat16 *Kb = K + ((long long)(b * Hkv + hkv) * Sk + j0) * D;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the scores kernel may start launching now (it waits for this grid's results)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    for (int i = tid; i < n * D / 8; i += blockDim.x)  // 16-byte copies (rows are 16B-aligned)
        cp_async16(smem_u32(kblk) + 16 * i, reinterpret_cast<const uint4 *>(Kb) + i, 16);
    cp_async_wait_all();
    __syncthreads();
    // Keys as packed bf16 pairs; sums on packed fp32 pairs.
    constexpr int P = D / 2;                 // column pairs per row
    constexpr int G = 128 / P;               // row groups of the column sums
    const uint32_t *kw = reinterpret_cast<const uint32_t *>(kblk);
    auto bf2 = [](uint32_t u) {              // (lo, hi) bf16 -> packed fp32 pair
        return f2_pack(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
    };
    {
        // column sums: thread tid sums pair tid % P over rows tid / P, + G, ...
        const int pc = tid % P, g = tid / P;
        uint64_t a0 = f2_pack(0.f, 0.f), a1 = f2_pack(0.f, 0.f);
        int j = g;
        for (; j + G < n; j += 2 * G) {
            a0 = f2_add(a0, bf2(kw[j * P + pc]));
            a1 = f2_add(a1, bf2(kw[(j + G) * P + pc]));
        }
        if (j < n) a0 = f2_add(a0, bf2(kw[j * P + pc]));
        float lo, hi;
        f2_unpack(f2_add(a0, a1), lo, hi);
        part[g][2 * pc] = lo;
        part[g][2 * pc + 1] = hi;
    }
    __syncthreads();
    if (tid < D) {
        float sum = 0.f;
#pragma unroll
        for (int g = 0; g < G; ++g) sum += part[g][tid];
        c[tid] = sum / static_cast<float>(n);
    }
    __syncthreads();
    // |k - c|^2 of the warp's 16 rows (rows warp, warp + 4, ...): each lane sums its
    // column pairs (lane, lane + 32, ...) for all 16 rows, then one transposing
    // reduction across the lanes leaves each lane with one row's total (16 shuffles
    // instead of 5 per row)
    constexpr int kRowsPerWarp = kBlk / 4;
    constexpr int kPairsPerLane = P / 32;
    uint64_t cpair[kPairsPerLane];
#pragma unroll
    for (int q = 0; q < kPairsPerLane; ++q) cpair[q] = f2_pack(c[2 * (lane + 32 * q)], c[2 * (lane + 32 * q) + 1]);
    const uint64_t neg1 = f2_pack(-1.f, -1.f);
    float ss[kRowsPerWarp];
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
        const int j = warp + 4 * i;
        uint64_t acc = f2_pack(0.f, 0.f);
        if (j < n) {
#pragma unroll
            for (int q = 0; q < kPairsPerLane; ++q) {
                const uint64_t e = f2_fma(cpair[q], neg1, bf2(kw[j * P + lane + 32 * q]));
                acc = f2_fma(e, e, acc);
            }
        }
        float lo, hi;
        f2_unpack(acc, lo, hi);
        ss[i] = lo + hi;  // rows past n hold 0
    }
    // transposing reduction: after the step with lane bit m, a lane keeps the rows
    // whose index bit matches its lane bit and adds its partner's partial sums
#pragma unroll
    for (int half = kRowsPerWarp / 2, bitl = 16; half >= 1; half >>= 1, bitl >>= 1) {
        const bool up = (lane & bitl) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = up ? ss[i] : ss[i + half];
            const float keep = up ? ss[i + half] : ss[i];
            ss[i] = keep + __shfl_xor_sync(0xffffffffu, send, bitl);
        }
    }
    float tot = ss[0] + __shfl_xor_sync(0xffffffffu, ss[0], 1);  // lanes 2r, 2r + 1 hold one row
    float rm = sqrtf(tot);
#pragma unroll
    for (int o = 2; o < 32; o <<= 1) rm = fmaxf(rm, __shfl_xor_sync(0xffffffffu, rm, o));
    if (lane == 0) rmax_w[warp] = rm;
    const long long row = (long long)(b * Hkv + hkv) * nkb + kb;
    if (tid < D) {  // the centroid as bf16 high part + bf16 remainder
        const __nv_bfloat16 hi = __float2bfloat16_rn(c[tid]);
        cent_hi[row * D + tid] = hi;
        cent_lo[row * D + tid] = __float2bfloat16_rn(c[tid] - __bfloat162float(hi));
    }
    __syncthreads();
    if (tid == 0) rad[row] = fmaxf(fmaxf(rmax_w[0], rmax_w[1]), fmaxf(rmax_w[2], rmax_w[3]));
}

// Radii of one head sorted in shared memory (bitonic, padded to a power of two).
__global__ void __launch_bounds__(256)
    rbs_beta_kernel(const float *__restrict__ rad, float *__restrict__ beta, int nkb, int n_pow2) {
    extern __shared__ float v[];
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const long long base = (long long)blockIdx.x * nkb;
    for (int i = threadIdx.x; i < n_pow2; i += blockDim.x)
        v[i] = i < nkb ? rad[base + i] : __int_as_float(0x7f800000);  // +inf pads sort last
    __syncthreads();
    for (int k = 2; k <= n_pow2; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < n_pow2; i += blockDim.x) {
                const int x = i ^ j;
                if (x > i) {
                    const bool up = (i & k) == 0;
                    const float a = v[i], c = v[x];
                    if ((a > c) == up) {
                        v[i] = c;
                        v[x] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
    auto quantile = [&](float q) {
        const float pos = q * static_cast<float>(nkb - 1);
        const int lo = static_cast<int>(floorf(pos));
        const int hi = min(lo + 1, nkb - 1);
        return v[lo] + (pos - static_cast<float>(lo)) * (v[hi] - v[lo]);
    };
    const float r_low = quantile(0.5f), r_high = quantile(0.9f);
    for (int i = threadIdx.x; i < nkb; i += blockDim.x) {
        const float r = rad[base + i];
        float bt;
        if (r_high > r_low)
            bt = fminf(fmaxf((r - r_low) / (r_high - r_low), 0.f), 1.f);
        else
            bt = r > r_low ? 1.f : 0.f;
        beta[base + i] = bt;
    }
}

// Median and 90th percentile (linear interpolation between order statistics) of
// n <= 64 radii, by one warp: bitonic sort of 64 values held two per lane (+inf
// pads sort last), then the same arithmetic as rbs_beta_kernel.
__device__ __forceinline__ void warp_radius_quantiles(const float *rad, int n, float &r_low,
                                                      float &r_high) {
    const int lane = threadIdx.x & 31;
    const float inf = __int_as_float(0x7f800000);
    float v0 = lane < n ? rad[lane] : inf, v1 = lane + 32 < n ? rad[lane + 32] : inf;
    for (int k = 2; k <= 64; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j == 32) {  // elements lane and lane + 32, both ascending (k = 64)
                const float a = fminf(v0, v1), b = fmaxf(v0, v1);
                v0 = a;
                v1 = b;
                continue;
            }
            const float p0 = __shfl_xor_sync(0xffffffffu, v0, j);
            const float p1 = __shfl_xor_sync(0xffffffffu, v1, j);
            const bool lower = (lane & j) == 0;
            const bool up0 = (lane & k) == 0, up1 = ((lane + 32) & k) == 0;
            v0 = (lower == up0) ? fminf(v0, p0) : fmaxf(v0, p0);
            v1 = (lower == up1) ? fminf(v1, p1) : fmaxf(v1, p1);
        }
    }
    auto at = [&](int i) {
        const float a = __shfl_sync(0xffffffffu, v0, i & 31), b = __shfl_sync(0xffffffffu, v1, i & 31);
        return i < 32 ? a : b;
    };
    auto quantile = [&](float q) {
        const float pos = q * static_cast<float>(n - 1);
        const int lo = static_cast<int>(floorf(pos));
        const int hi = min(lo + 1, n - 1);
        const float vlo = at(lo), vhi = at(hi);
        return vlo + (pos - static_cast<float>(lo)) * (vhi - vlo);
    };
    r_low = quantile(0.5f);
    r_high = quantile(0.9f);
}

struct ScoreParams {
    const __nv_bfloat16 *Q;
    const __nv_bfloat16 *cent_hi, *cent_lo;
    const float *rad, *beta;  // beta == nullptr: the kernel derives it (nkb <= 64)
    uint8_t *mask;
    float *base_out, *rescue_out;  // optional
    int Hq, Hkv, group, Sq, nqb, nkb;
    float ln_alpha_base, ln_alpha_rescue;
    int diagonal;
    int qb_per_cta;  // query blocks scored by one CTA
};

// Byte offset of 16-byte chunk c of row `row` in a 64-row bf16 tile stored as
// D/64 boxes of (64 rows x 128 bytes) with the 128-byte XOR swizzle, so that
// ldmatrix reads of 8 rows at one chunk hit 8 different bank groups.
__device__ __forceinline__ uint32_t swz64(int row, int c) {
    return static_cast<uint32_t>((c >> 3) * (64 * 128) + row * 128 + (((c & 7) ^ (row & 7)) << 4));
}

// Rows [0, n) of a row-major (., D) bf16 matrix into a swizzled 64-row tile
// (rows n..63 zero), 16-byte asynchronous copies spread over the block's
// threads; the caller waits (cp_async_wait_all) and synchronises.
template <int D>
__device__ __forceinline__ void stage64(uint8_t *tile, const __nv_bfloat16 *src, int n) {
    constexpr int kChunks = D / 8;
    const uint32_t t = smem_u32(tile);
    for (int i = threadIdx.x; i < 64 * kChunks; i += blockDim.x) {
        const int row = i / kChunks, c = i % kChunks;
        const bool in = row < n;
        cp_async16(t + swz64(row, c),
                   reinterpret_cast<const uint4 *>(src + (long long)(in ? row : 0) * D) + c, in ? 16u : 0u);
    }
}

// kRun: the CTA scores a run of p.qb_per_cta query blocks (with the next one's load in
// flight); otherwise the single query block blockIdx.x.
template <int D, bool kRun>
__global__ void __launch_bounds__(128) rbs_scores_kernel(const ScoreParams p) {
    extern __shared__ __align__(1024) uint8_t smraw[];
    constexpr int kKs = D / 16;           // k-steps of 16
    constexpr int kTile = 64 * D * 2;     // bytes of one staged 64-row tile
    constexpr int kChunks = D / 8;        // 16-byte chunks per row
    // query blocks: the current one and (runs of several) the next
    constexpr int n_qbuf = kRun ? 2 : 1;
    uint8_t *q_tiles = smraw;
    uint8_t *ch_tile = smraw + n_qbuf * kTile;        // centroids of a 64-block group: high parts
    uint8_t *cl_tile = smraw + (n_qbuf + 1) * kTile;  // ... remainders
    float *sb = reinterpret_cast<float *>(smraw + (n_qbuf + 2) * kTile);  // [nkb] base scores of this row
    float *sr = sb + p.nkb;               // [nkb] rescue scores
    __shared__ float red2[2][4];
    __shared__ float rb_s[64];  // radius * beta of the key blocks of the current group
    __shared__ float qn_s[64];  // |q| of the block's tokens
    __shared__ float quant_s[2];  // median and 90th percentile of the head's radii
    // this CTA: query blocks qb0 .. qb0 + n_qb - 1 of one (query head, batch); they share
    // the head's key-block centroids, staged once when they fit one group of 64
    const int qb0 = kRun ? blockIdx.x * p.qb_per_cta : blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
    const int n_qb = kRun ? min(p.qb_per_cta, p.nqb - qb0) : 1;
    const int hkv = hq / p.group;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int mi = lane >> 3, rr = lane & 7;  // ldmatrix: matrix of this lane's address, its row
    const long long hrow = (long long)(b * p.Hkv + hkv) * p.nkb;
    // log2 units: scores scaled by log2(e) / sqrt(D), converted back at the end
    const float k2 = rsqrtf(static_cast<float>(D)) * 1.4426950408889634f;
    const float ninf = __int_as_float(0xff800000);
    const uint32_t hs = smem_u32(ch_tile), ls = smem_u32(cl_tile);
    const __nv_bfloat16 *Qh = p.Q + (long long)(b * p.Hq + hq) * p.Sq * D;
    auto rows_of = [&](int qb) { return min(kBlk, p.Sq - qb * kBlk); };
    if (n_qb <= 0) return;
    stage64<D>(q_tiles, Qh + (long long)qb0 * kBlk * D, rows_of(qb0));
    cp_async_commit();
    // Launched as a programmatic dependent of the centroid (or beta) kernel: the first
    // query block is an input of the call and is staged while that grid finishes;
    // centroids, radii and beta are read only after it has completed.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // the block-sparse attention that reads this mask may start its set-up now
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (!p.beta) {
        // beta of the head's key blocks from its radii (rbs_beta_kernel's rule, here
        // for nkb <= 64 so that the estimator needs no separate sorting launch)
        if (warp == 0) {
            float lo, hi;
            warp_radius_quantiles(p.rad + hrow, p.nkb, lo, hi);
            if (lane == 0) {
                quant_s[0] = lo;
                quant_s[1] = hi;
            }
        }
        __syncthreads();
    }
    const int n_groups = (p.nkb + 63) / 64;
    for (int qi = 0; qi < n_qb; ++qi) {
        const int qb = qb0 + qi, n_rows = rows_of(qb);
        const uint8_t *q_tile = q_tiles + (qi & 1) * kTile;
        const uint32_t qs = smem_u32(q_tile);
        // The product is taken transposed, S^T = C Q^T: warp w holds the 16 key blocks
        // 16 w .. 16 w + 15 of a group (MMA rows) against all 64 tokens (MMA columns),
        // so the log-sum-exp over the tokens of a key block runs over 16 values in each
        // thread and then across the 4 lanes that share the row -- no cross-warp step.
        float qn[8][2];  // |q| of this thread's tokens 8 j + 2 t + e
        for (int gi = 0; gi < n_groups; ++gi) {
            const int g0 = 64 * gi, nk = min(64, p.nkb - g0);
            if (qi == 0 || n_groups > 1) {
                stage64<D>(ch_tile, p.cent_hi + (hrow + g0) * D, nk);
                stage64<D>(cl_tile, p.cent_lo + (hrow + g0) * D, nk);
                if (tid < 64) {
                    float rbv = 0.f;
                    if (tid < nk) {
                        const float r = p.rad[hrow + g0 + tid];
                        float bt;
                        if (p.beta) {
                            bt = p.beta[hrow + g0 + tid];
                        } else {
                            const float r_low = quant_s[0], r_high = quant_s[1];
                            if (r_high > r_low)
                                bt = fminf(fmaxf((r - r_low) / (r_high - r_low), 0.f), 1.f);
                            else
                                bt = r > r_low ? 1.f : 0.f;
                        }
                        rbv = r * bt;
                    }
                    rb_s[tid] = rbv;
                }
            }
            cp_async_commit();
            // the next query block loads while this one is scored (its buffer was last
            // read before the barrier that ended the previous block)
            if (kRun && gi == 0 && qi + 1 < n_qb) {
                stage64<D>(q_tiles + ((qi + 1) & 1) * kTile, Qh + (long long)(qb + 1) * kBlk * D,
                           rows_of(qb + 1));
                cp_async_commit();
                cp_async_wait_group<1>();  // all but that prefetch
            } else {
                cp_async_wait_group<0>();
            }
            __syncthreads();
            if (gi == 0) {
                // |q| of token tid / 2: each of two threads sums the squares of half the row
                const int row = tid >> 1;
                float q2 = 0.f;
#pragma unroll
                for (int c = (tid & 1) * (kChunks / 2); c < (tid & 1) * (kChunks / 2) + kChunks / 2; ++c) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(q_tile + swz64(row, c));
                    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162 *>(&w4[e]);
                        const float x = __low2float(h), y = __high2float(h);
                        q2 = fmaf(x, x, fmaf(y, y, q2));
                    }
                }
                q2 += __shfl_xor_sync(0xffffffffu, q2, 1);
                if ((tid & 1) == 0) qn_s[row] = sqrtf(q2);
                __syncthreads();
#pragma unroll
                for (int j = 0; j < 8; ++j)
#pragma unroll
                    for (int e = 0; e < 2; ++e) qn[j][e] = qn_s[8 * j + 2 * t + e];
            }
            float acc[8][4];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < kKs; ++kk) {
                uint32_t ah[4], al[4];
                const uint32_t aoff = swz64(warp * 16 + (mi & 1) * 8 + rr, 2 * kk + (mi >> 1));
                ldmatrix_x4(hs + aoff, ah[0], ah[1], ah[2], ah[3]);
                ldmatrix_x4(ls + aoff, al[0], al[1], al[2], al[3]);
#pragma unroll
                for (int jp = 0; jp < 4; ++jp) {  // token n-tiles 2 jp, 2 jp + 1
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4(qs + swz64(16 * jp + (mi >> 1) * 8 + rr, 2 * kk + (mi & 1)), b0, b1, b2, b3);
                    mma_m16n8k16(acc[2 * jp], ah, b0, b1);
                    mma_m16n8k16(acc[2 * jp], al, b0, b1);
                    mma_m16n8k16(acc[2 * jp + 1], ah, b2, b3);
                    mma_m16n8k16(acc[2 * jp + 1], al, b2, b3);
                }
            }
            // rows g and g + 8 of the warp's tile: key blocks g0 + 16 warp + g (+ 8)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int col = warp * 16 + g + 8 * h;
                const float rb = rb_s[col];
                float vb[16], vr[16];
                float mb = ninf, mr = ninf;
#pragma unroll
                for (int j = 0; j < 8; ++j)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const bool in = 8 * j + 2 * t + e < n_rows;
                        const float sdot = acc[j][2 * h + e];
                        vb[2 * j + e] = in ? sdot * k2 : ninf;
                        vr[2 * j + e] = in ? fmaf(qn[j][e], rb, sdot) * k2 : ninf;
                        mb = fmaxf(mb, vb[2 * j + e]);
                        mr = fmaxf(mr, vr[2 * j + e]);
                    }
                mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 1));
                mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 2));
                mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, 1));
                mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, 2));
                // n_rows >= 1, so both maxima are finite here
                float eb = 0.f, er = 0.f;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    eb += fast_exp2(vb[i] - mb);
                    er += fast_exp2(vr[i] - mr);
                }
                eb += __shfl_xor_sync(0xffffffffu, eb, 1);
                eb += __shfl_xor_sync(0xffffffffu, eb, 2);
                er += __shfl_xor_sync(0xffffffffu, er, 1);
                er += __shfl_xor_sync(0xffffffffu, er, 2);
                if (t == 0 && g0 + col < p.nkb) {
                    sb[g0 + col] = (mb + __log2f(eb)) * 0.69314718055994531f;
                    sr[g0 + col] = (mr + __log2f(er)) * 0.69314718055994531f;
                }
            }
            __syncthreads();
        }
        // relative masks of the row: keep where score >= row max + ln alpha
        float mb = __int_as_float(0xff800000), mr = mb;
        for (int kb = tid; kb < p.nkb; kb += blockDim.x) {
            mb = fmaxf(mb, sb[kb]);
            mr = fmaxf(mr, sr[kb]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
            mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, o));
        }
        if (lane == 0) {
            red2[0][warp] = mb;
            red2[1][warp] = mr;
        }
        __syncthreads();
        mb = red2[0][0];
        mr = red2[1][0];
#pragma unroll
        for (int w = 1; w < 4; ++w) {
            mb = fmaxf(mb, red2[0][w]);
            mr = fmaxf(mr, red2[1][w]);
        }
        const long long orow = ((long long)(b * p.Hq + hq) * p.nqb + qb) * p.nkb;
        for (int kb = tid; kb < p.nkb; kb += blockDim.x) {
            const bool band = abs(qb - kb) < p.diagonal;
            const bool keep = sb[kb] >= mb + p.ln_alpha_base || sr[kb] >= mr + p.ln_alpha_rescue || band;
            p.mask[orow + kb] = keep ? 2 : 0;
            if (p.base_out) p.base_out[orow + kb] = sb[kb];
            if (p.rescue_out) p.rescue_out[orow + kb] = sr[kb];
        }
        __syncthreads();  // sb, sr and red2 are rewritten for the next query block
    }
}

// Resident scores CTAs per SM for a dynamic shared-memory size, and the SM count of
// the current device; cached per (device, size), as the launcher asks on every call.
template <int D>
cudaError_t scores_occupancy(size_t smem, int &per_sm, int &n_sm) {
    static std::mutex mu;
    static std::map<std::pair<int, size_t>, std::pair<int, int>> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find({dev, smem});
    if (it == cache.end()) {
        if ((e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return e;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rbs_scores_kernel<D, true>,
                                                               128, smem)) != cudaSuccess)
            return e;
        it = cache.emplace(std::make_pair(dev, smem), std::make_pair(per_sm, n_sm)).first;
    }
    per_sm = it->second.first;
    n_sm = it->second.second;
    return cudaSuccess;
}

template <int D>
attn_status_t launch_rbs_d(const RbsArgs &a, cudaStream_t stream) {
    const int nqb = (a.Sq + kBlk - 1) / kBlk, nkb = (a.Sk + kBlk - 1) / kBlk;
    // the fp32 centroid workspace holds the bf16 high parts and then the remainders
    __nv_bfloat16 *cent_hi = reinterpret_cast<__nv_bfloat16 *>(a.cent);
    __nv_bfloat16 *cent_lo = cent_hi + (size_t)a.B * a.Hkv * nkb * D;
    rbs_centroid_kernel<D><<<dim3(nkb, a.Hkv, a.B), 128, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(a.K), cent_hi, cent_lo, a.rad, a.Hkv, a.Sk, nkb);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    // Up to 64 key blocks the scores kernel derives beta itself (one warp sorts the
    // head's radii); longer sequences sort in a launch of their own.
    const bool own_beta = nkb > 64;
    if (own_beta) {
        int n_pow2 = 1;
        while (n_pow2 < nkb) n_pow2 <<= 1;
        rbs_beta_kernel<<<a.B * a.Hkv, 256, n_pow2 * sizeof(float), stream>>>(a.rad, a.beta, nkb,
                                                                              n_pow2);
        if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    }
    ScoreParams p;
    p.Q = static_cast<const __nv_bfloat16 *>(a.Q);
    p.cent_hi = cent_hi;
    p.cent_lo = cent_lo;
    p.rad = a.rad;
    p.beta = own_beta ? a.beta : nullptr;
    p.mask = a.mask;
    p.base_out = a.base_scores;
    p.rescue_out = a.rescue_scores;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.group = a.Hq / a.Hkv;
    p.Sq = a.Sq;
    p.nqb = nqb;
    p.nkb = nkb;
    p.ln_alpha_base = logf(a.alpha_base);
    p.ln_alpha_rescue = logf(a.alpha_rescue);
    p.diagonal = a.diagonal;
    // two query-block buffers for runs of several query blocks, else one
    auto smem_for = [&](int n_qbuf) {
        return (n_qbuf + 2) * (size_t)64 * D * 2 + sizeof(float) * 2 * (size_t)nkb;
    };
    size_t smem = smem_for(1);
    if (kernel_setup(reinterpret_cast<const void *>(rbs_scores_kernel<D, false>), 100 * 1024) !=
            cudaSuccess ||
        kernel_setup(reinterpret_cast<const void *>(rbs_scores_kernel<D, true>), 100 * 1024) !=
            cudaSuccess)
        return ATTN_ERR_CUDA;
    // Query blocks per CTA.  Up to 64 key blocks (one centroid group): as few as keep
    // about one wave of CTAs resident at once, so each CTA stages its head's centroids
    // once for several query blocks and overlaps the next block's load with the current
    // block's scores (45 -> 41 us for the estimator on a B1 H32 S4096 image workload).
    // With more key blocks the groups are restaged for every query block anyway, and one
    // query block per CTA keeps more CTAs in flight (runs measured 13-17 % slower there).
    p.qb_per_cta = 1;
    if (nkb <= 64) {
        int per_sm = 0, n_sm = 0;
        if (scores_occupancy<D>(smem_for(2), per_sm, n_sm) != cudaSuccess) return ATTN_ERR_CUDA;
        const long long rows = (long long)nqb * a.Hq * a.B;
        const long long slots = (long long)std::max(1, n_sm) * std::max(1, per_sm);
        p.qb_per_cta =
            static_cast<int>(std::min((long long)nqb, std::max(1ll, (rows + slots - 1) / slots)));
        if (p.qb_per_cta > 1) smem = smem_for(2);
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((nqb + p.qb_per_cta - 1) / p.qb_per_cta, a.Hq, a.B);
    cfg.blockDim = dim3(128, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = p.qb_per_cta > 1 ? cudaLaunchKernelEx(&cfg, rbs_scores_kernel<D, true>, p)
                                           : cudaLaunchKernelEx(&cfg, rbs_scores_kernel<D, false>, p);
    if (e != cudaSuccess) return ATTN_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

attn_status_t launch_rbs(const RbsArgs &a, cudaStream_t stream) {
    if (a.D == 128) return launch_rbs_d<128>(a, stream);
    if (a.D == 64) return launch_rbs_d<64>(a, stream);
    return ATTN_ERR_UNSUPPORTED;
}

}  // namespace gqa
