// attn_bwd.cu -- backward of the fused GQA attention forward for sm_100a: the
// row statistic delta and the launch of the tensor-core gradient kernels.
//
// Tylo.jl "Primitives" page, entry `∇attention!`: from the output gradient dO,
// the inputs, the output O and the saved softmax statistics (here LSE = M + ln L)
// write dQ, dK, dV.  With P = exp(S * scale - LSE) (S = Q K^T) on the visible
// pairs of the forward's masks:
//   delta_i = sum_d dO_id O_id                       (= sum_j P_ij dP_ij)
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - delta),  dQ = scale dS K,
//   dK = scale dS^T Q; a KV head collects the gradients of its query heads.
//
// bwd_delta_kernel (one warp per query row) writes delta to the workspace; the
// dK / dV and dQ kernels (attn_bwd_tc.cu) then run on the fifth-generation
// tensor cores.
#include <cuda_bf16.h>

#include "internal.h"

namespace gqa {

namespace {

// delta_i = <dO_i, O_i> over rows of D bf16 values.
template <int D>
__global__ void __launch_bounds__(256)
    bwd_delta_kernel(const __nv_bfloat16 *dO, const __nv_bfloat16 *O, float *delta, long long rows) {
    const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    const __nv_bfloat16 *go = dO + r * D, *o = O + r * D;
    float acc = 0.f;
    for (int d = lane * 2; d < D; d += 64) {
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(go + d);
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(o + d);
        acc = fmaf(__low2float(a), __low2float(b), acc);
        acc = fmaf(__high2float(a), __high2float(b), acc);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) delta[r] = acc;
}

template <int D>
attn_status_t launch_bwd_d(const BwdArgs &a, cudaStream_t stream) {
    const long long rows = (long long)a.B * a.Hq * a.Sq;
    if (rows > 0) {
        const long long blocks = (rows + 7) / 8;
        if (blocks > 0x7fffffffll) return ATTN_ERR_INVALID;
        bwd_delta_kernel<D><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
            static_cast<const __nv_bfloat16 *>(a.dO), static_cast<const __nv_bfloat16 *>(a.O), a.delta,
            rows);
        if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    }
    return launch_bwd_tc(a, stream);
}

}  // namespace

attn_status_t launch_bwd(const BwdArgs &a, cudaStream_t stream) {
    if (a.D == 128) return launch_bwd_d<128>(a, stream);
    if (a.D == 64) return launch_bwd_d<64>(a, stream);
    return ATTN_ERR_UNSUPPORTED;
}

}  // namespace gqa
