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
// bwd_delta_kernel (D / 8 threads per query row) writes delta to the workspace; the
// dK / dV and dQ kernels (attn_bwd_tc.cu) then run on the fifth-generation
// tensor cores.
#include <cuda_bf16.h>

#include "internal.h"

namespace gqa {

namespace {

// delta_i = <dO_i, O_i> over rows of D bf16 values: D / 8 threads per row, one
// 16-byte load of each operand per thread, then a shuffle sum over the row's lanes.
template <int D>
__global__ void __launch_bounds__(256)
    bwd_delta_kernel(const __nv_bfloat16 *dO, const __nv_bfloat16 *O, float *delta, long long rows) {
    constexpr int kTpr = D / 8;          // threads per row
    constexpr int kRpb = 256 / kTpr;     // rows per block
    const long long r = (long long)blockIdx.x * kRpb + threadIdx.x / kTpr;
    const int c = threadIdx.x % kTpr;
    float acc = 0.f;
    if (r < rows) {
        const uint4 a = __ldg(reinterpret_cast<const uint4 *>(dO + r * D) + c);
        const uint4 b = __ldg(reinterpret_cast<const uint4 *>(O + r * D) + c);
        const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162 *>(&wa[e]);
            const __nv_bfloat162 y = *reinterpret_cast<const __nv_bfloat162 *>(&wb[e]);
            acc = fmaf(__low2float(x), __low2float(y), acc);
            acc = fmaf(__high2float(x), __high2float(y), acc);
        }
    }
#pragma unroll
    for (int off = kTpr / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (r < rows && c == 0) delta[r] = acc;
}

template <int D>
attn_status_t launch_bwd_d(const BwdArgs &a, cudaStream_t stream) {
    const long long rows = (long long)a.B * a.Hq * a.Sq;
    if (rows > 0) {
        const long long blocks = (rows + 256 / (D / 8) - 1) / (256 / (D / 8));
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
