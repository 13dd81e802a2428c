// block_scores.cu -- block scores and block mask of block-sparse prefill, as on
// the mlx-arsenal "Radius-bounded block scores (RBS)" page (sections "The idea"
// and "What mlx-arsenal ships": radius_bounded_block_scores, relative_block_mask,
// and the recipe's union of both branches with a diagonal band).
//
// Three small kernels, 64-token blocks:
//   rbs_centroid_kernel  one CTA per (key block, KV head, batch): centroid c (fp32
//                        mean of the block's keys) and radius r = max |k - c|_2.
//   rbs_beta_kernel      one CTA per (KV head, batch): sorts the head's radii,
//                        takes the median and the 90th percentile (linear
//                        interpolation between order statistics) and writes
//                        beta = clip((r - r_low) / (r_high - r_low), 0, 1)
//                        (1 for r > r_low, else 0, when the two coincide).
//   rbs_scores_kernel    one CTA per (query block, query head, batch): for every
//                        key block, l_base = <q, c> / sqrt(D) and l_rescue =
//                        (<q, c> + |q| r beta) / sqrt(D) for the block's query
//                        tokens, log-sum-exp over the tokens, then the row's
//                        relative mask: keep where score >= row max + ln alpha in
//                        either branch, or |qb - kb| < diagonal.
// The mask is written as BlockMask states (2 = keep the whole block, 0 = skip),
// one (nqb, nkb) matrix per (batch, query head), ready for attn_fwd_flex.
#include <cuda_bf16.h>

#include "internal.h"

namespace gqa {

namespace {

constexpr int kBlk = 64;

template <int D>
__global__ void __launch_bounds__(128)
    rbs_centroid_kernel(const __nv_bfloat16 *__restrict__ K, float *__restrict__ cent,
                        float *__restrict__ rad, int Hkv, int Sk, int nkb) {
    __shared__ __align__(16) __nv_bfloat16 kblk[kBlk * D];  // the key block, read once
    __shared__ float c[D];
    __shared__ float rmax_w[4];
    const int kb = blockIdx.x, hkv = blockIdx.y, b = blockIdx.z;
    const int j0 = kb * kBlk, n = min(kBlk, Sk - j0);
    const __nv_bfloat16 *Kb = K + ((long long)(b * Hkv + hkv) * Sk + j0) * D;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < n * D / 8; i += blockDim.x)  // 16-byte loads (rows are 16B-aligned)
        reinterpret_cast<uint4 *>(kblk)[i] = reinterpret_cast<const uint4 *>(Kb)[i];
    __syncthreads();
    if (tid < D) {
        float acc = 0.f;
#pragma unroll 8
        for (int j = 0; j < n; ++j) acc += __bfloat162float(kblk[j * D + tid]);
        c[tid] = acc / static_cast<float>(n);
    }
    __syncthreads();
    float rm = 0.f;
    for (int j = warp; j < n; j += 4) {
        float ss = 0.f;
        for (int d = lane; d < D; d += 32) {
            const float e = __bfloat162float(kblk[j * D + d]) - c[d];
            ss = fmaf(e, e, ss);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        rm = fmaxf(rm, sqrtf(ss));
    }
    if (lane == 0) rmax_w[warp] = rm;
    const long long row = (long long)(b * Hkv + hkv) * nkb + kb;
    if (tid < D) cent[row * D + tid] = c[tid];
    __syncthreads();
    if (tid == 0) rad[row] = fmaxf(fmaxf(rmax_w[0], rmax_w[1]), fmaxf(rmax_w[2], rmax_w[3]));
}

// Radii of one head sorted in shared memory (bitonic, padded to a power of two).
__global__ void __launch_bounds__(256)
    rbs_beta_kernel(const float *__restrict__ rad, float *__restrict__ beta, int nkb, int n_pow2) {
    extern __shared__ float v[];
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

struct ScoreParams {
    const __nv_bfloat16 *Q;
    const float *cent, *rad, *beta;
    uint8_t *mask;
    float *base_out, *rescue_out;  // optional
    int Hq, Hkv, group, Sq, nqb, nkb;
    float ln_alpha_base, ln_alpha_rescue;
    int diagonal;
};

template <int D>
__global__ void __launch_bounds__(256) rbs_scores_kernel(const ScoreParams p) {
    extern __shared__ float sm[];
    constexpr int kLd = kBlk + 1;         // padded row: conflict-free transposed stores
    float *qT = sm;                       // [D][kLd] query block, transposed
    constexpr int kCg = 64;               // key blocks per group (8 per warp)
    constexpr int kCld = kCg + 4;         // padded row of the transposed centroids
    float *qn = qT + D * kLd;             // [64] |q_t|
    float *cT = qn + kBlk;                // [D][kCld] centroids of one group, transposed
    float *sb = cT + D * kCld;            // [nkb] base scores of this row
    float *sr = sb + p.nkb;               // [nkb] rescue scores
    __shared__ float red[2][8];
    const int qb = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
    const int hkv = hq / p.group;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int i0 = qb * kBlk, n_rows = min(kBlk, p.Sq - i0);
    const __nv_bfloat16 *Qb = p.Q + ((long long)(b * p.Hq + hq) * p.Sq + i0) * D;
    for (int idx = tid; idx < kBlk * D; idx += blockDim.x) {
        const int t = idx / D, d = idx % D;
        qT[d * kLd + t] = t < n_rows ? __bfloat162float(Qb[(long long)t * D + d]) : 0.f;
    }
    __syncthreads();
    if (tid < kBlk) {
        float ss = 0.f;
        for (int d = 0; d < D; ++d) ss = fmaf(qT[d * kLd + tid], qT[d * kLd + tid], ss);
        qn[tid] = sqrtf(ss);
    }
    __syncthreads();
    const float inv_sqrt_d = rsqrtf(static_cast<float>(D));
    const long long hrow = (long long)(b * p.Hkv + hkv) * p.nkb;
    const bool v0 = lane < n_rows, v1 = lane + 32 < n_rows;
    const float ninf = __int_as_float(0xff800000);
    // Key blocks in groups of 64: the group's centroids are staged transposed in
    // shared memory; warp w takes 8 of them and each lane 2 query rows, so every
    // shared-memory read feeds 4 or 16 FMAs (register blocking).
    for (int g0 = 0; g0 < p.nkb; g0 += kCg) {
        for (int idx = tid; idx < kCg * D; idx += blockDim.x) {
            const int j = idx / D, d = idx % D;
            cT[d * kCld + j] = g0 + j < p.nkb ? p.cent[(hrow + g0 + j) * D + d] : 0.f;
        }
        __syncthreads();
        float acc0[8], acc1[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc0[j] = acc1[j] = 0.f;
#pragma unroll 4
        for (int d = 0; d < D; ++d) {
            const float q0 = qT[d * kLd + lane], q1 = qT[d * kLd + lane + 32];
            const float4 ca = *reinterpret_cast<const float4 *>(cT + d * kCld + 8 * warp);
            const float4 cb = *reinterpret_cast<const float4 *>(cT + d * kCld + 8 * warp + 4);
            const float cv[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                acc0[j] = fmaf(q0, cv[j], acc0[j]);
                acc1[j] = fmaf(q1, cv[j], acc1[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int kb = g0 + 8 * warp + j;
            if (kb >= p.nkb) break;  // warp-uniform
            const float rb = p.rad[hrow + kb] * p.beta[hrow + kb];
            const float b0 = v0 ? acc0[j] * inv_sqrt_d : ninf, b1 = v1 ? acc1[j] * inv_sqrt_d : ninf;
            const float r0 = v0 ? fmaf(qn[lane], rb, acc0[j]) * inv_sqrt_d : ninf;
            const float r1 = v1 ? fmaf(qn[lane + 32], rb, acc1[j]) * inv_sqrt_d : ninf;
            float mb = fmaxf(b0, b1), mr = fmaxf(r0, r1);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
                mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, o));
            }
            float eb = __expf(b0 - mb) + __expf(b1 - mb), er = __expf(r0 - mr) + __expf(r1 - mr);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                eb += __shfl_xor_sync(0xffffffffu, eb, o);
                er += __shfl_xor_sync(0xffffffffu, er, o);
            }
            if (lane == 0) {
                sb[kb] = mb + __logf(eb);
                sr[kb] = mr + __logf(er);
            }
        }
        __syncthreads();
    }
    __syncthreads();
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
        red[0][warp] = mb;
        red[1][warp] = mr;
    }
    __syncthreads();
    mb = red[0][0];
    mr = red[1][0];
#pragma unroll
    for (int w = 1; w < 8; ++w) {
        mb = fmaxf(mb, red[0][w]);
        mr = fmaxf(mr, red[1][w]);
    }
    const long long orow = ((long long)(b * p.Hq + hq) * p.nqb + qb) * p.nkb;
    for (int kb = tid; kb < p.nkb; kb += blockDim.x) {
        const bool band = abs(qb - kb) < p.diagonal;
        const bool keep = sb[kb] >= mb + p.ln_alpha_base || sr[kb] >= mr + p.ln_alpha_rescue || band;
        p.mask[orow + kb] = keep ? 2 : 0;
        if (p.base_out) p.base_out[orow + kb] = sb[kb];
        if (p.rescue_out) p.rescue_out[orow + kb] = sr[kb];
    }
}

template <int D>
attn_status_t launch_rbs_d(const RbsArgs &a, cudaStream_t stream) {
    const int nqb = (a.Sq + kBlk - 1) / kBlk, nkb = (a.Sk + kBlk - 1) / kBlk;
    rbs_centroid_kernel<D><<<dim3(nkb, a.Hkv, a.B), 128, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(a.K), a.cent, a.rad, a.Hkv, a.Sk, nkb);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    int n_pow2 = 1;
    while (n_pow2 < nkb) n_pow2 <<= 1;
    rbs_beta_kernel<<<a.B * a.Hkv, 256, n_pow2 * sizeof(float), stream>>>(a.rad, a.beta, nkb,
                                                                          n_pow2);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    ScoreParams p;
    p.Q = static_cast<const __nv_bfloat16 *>(a.Q);
    p.cent = a.cent;
    p.rad = a.rad;
    p.beta = a.beta;
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
    const size_t smem = sizeof(float) * ((size_t)D * (kBlk + 1) + kBlk + (size_t)D * (64 + 4) +
                                         2 * (size_t)nkb);
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(rbs_scores_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 100 * 1024) != cudaSuccess)
            return ATTN_ERR_CUDA;
        configured = true;
    }
    rbs_scores_kernel<D><<<dim3(nqb, a.Hq, a.B), 256, smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

attn_status_t launch_rbs(const RbsArgs &a, cudaStream_t stream) {
    if (a.D == 128) return launch_rbs_d<128>(a, stream);
    if (a.D == 64) return launch_rbs_d<64>(a, stream);
    return ATTN_ERR_UNSUPPORTED;
}

}  // namespace gqa
