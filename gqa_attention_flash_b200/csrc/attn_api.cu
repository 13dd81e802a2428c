// attn_api.cu -- the library's C ABI (declared in include/gqa_attn.h):
// host-side argument validation, TMA descriptor encoding, the per-device status
// word, and the workspaces (from a per-device pool the library owns).
#include <nvtx3/nvToolsExt.h>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <set>
#include <utility>

#include <cuda.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace gqa {

__device__ int g_status = 0;

namespace {
std::mutex g_status_mutex;
int *g_status_ptr[64] = {};
}  // namespace

int *device_status_word() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(g_status_mutex);
    if (g_status_ptr[dev] == nullptr) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_status) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = static_cast<int *>(ptr);
    }
    return g_status_ptr[dev];
}

size_t decode_workspace_floats(int B, int Hq, int n_splits, int D);

namespace {
std::mutex g_setup_mutex;
std::set<std::pair<int, const void *>> g_setup_done;
}  // namespace

cudaError_t kernel_setup(const void *func, int smem_bytes, int required_regs, bool max_smem_carveout) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_setup_done.count({dev, func})) return cudaSuccess;
    if (required_regs >= 0) {
        cudaFuncAttributes fa;
        if ((e = cudaFuncGetAttributes(&fa, func)) != cudaSuccess) return e;
        if (fa.numRegs != required_regs) return cudaErrorInvalidValue;
    }
    if ((e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes)) !=
        cudaSuccess)
        return e;
    if (max_smem_carveout &&
        (e = cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout,
                                  cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
        return e;
    g_setup_done.insert({dev, func});
    return cudaSuccess;
}

namespace {
std::mutex g_pool_mutex;
cudaMemPool_t g_pool[64] = {};
bool g_pool_made[64] = {};
}  // namespace

// Stream-ordered workspace from a memory pool the library owns on each device
// (made on first use).  Its release threshold is the maximum, so memory freed
// back to it stays reserved for the next call instead of returning to the driver
// at every synchronisation; the default pool, which other code in the process may
// use, keeps its own settings.
cudaError_t workspace_alloc(void **ptr, size_t bytes, cudaStream_t stream) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    cudaMemPool_t pool;
    {
        std::lock_guard<std::mutex> lock(g_pool_mutex);
        if (!g_pool_made[dev]) {
            cudaMemPoolProps props = {};
            props.allocType = cudaMemAllocationTypePinned;
            props.handleTypes = cudaMemHandleTypeNone;
            props.location.type = cudaMemLocationTypeDevice;
            props.location.id = dev;
            if ((e = cudaMemPoolCreate(&g_pool[dev], &props)) != cudaSuccess) return e;
            uint64_t keep = UINT64_MAX;
            if ((e = cudaMemPoolSetAttribute(g_pool[dev], cudaMemPoolAttrReleaseThreshold, &keep)) !=
                cudaSuccess)
                return e;
            g_pool_made[dev] = true;
        }
        pool = g_pool[dev];
    }
    return cudaMallocFromPoolAsync(ptr, bytes, pool, stream);
}

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

attn_status_t make_tmap_bf16_3d(CUtensorMap *map, const void *base, uint64_t D, uint64_t rows,
                                uint64_t outer, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return ATTN_ERR_CUDA;
    const cuuint64_t dims[3] = {D, rows > 0 ? rows : 1, outer > 0 ? outer : 1};
    const cuuint64_t strides[2] = {D * 2, D * 2 * (rows > 0 ? rows : 1)};
    const cuuint32_t box[3] = {64, box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_INVALID;
}

attn_status_t make_tmap_bf16_paged(CUtensorMap *map, const void *base, uint64_t D, uint64_t heads,
                                   uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return ATTN_ERR_CUDA;
    const cuuint64_t dims[3] = {D, heads, rows > 0 ? rows : 1};
    const cuuint64_t strides[2] = {D * 2, D * 2 * heads};
    const cuuint32_t box[3] = {64, 1, box_rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_INVALID;
}

attn_status_t make_tmap_bf16_paged_wide(CUtensorMap *map, const void *base, uint64_t heads,
                                        uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return ATTN_ERR_CUDA;
    const cuuint64_t dims[4] = {64, 2, heads, rows > 0 ? rows : 1};
    const cuuint64_t strides[3] = {128, 256, 256 * heads};
    const cuuint32_t box[4] = {64, 2, 1, box_rows};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_INVALID;
}

namespace {

__global__ void wait_probe_kernel(uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // Nobody arrives on `bar`: the bounded wait must give up and record the status.
    warp_wait(b, 0, &abort_flag, limit_ns, &g_status);
    __syncthreads();
}

}  // namespace

attn_status_t launch_wait_probe(int limit_us, cudaStream_t stream) {
    wait_probe_kernel<<<1, 32, 0, stream>>>(static_cast<uint64_t>(limit_us) * 1000ull);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace gqa

using namespace gqa;

namespace {
// NVTX range around an ABI call (host side: the enqueue of its kernels), so that
// a profiler's timeline names the calls; no cost without a tool attached.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};
}  // namespace

namespace {

attn_status_t validate_fwd(void *O, const void *Q, const void *K, const void *V, float *LSE, int B,
                           int Hq, int Hkv, int Sq, int Sk, int D, float scale, int causal,
                           int window, int input_pos) {
    if (B < 0 || Sq < 0 || Sk < 0 || Hq < 1 || Hkv < 1 || input_pos < 0 || window < 0)
        return ATTN_ERR_INVALID;
    if (Hq % Hkv != 0) return ATTN_ERR_INVALID;
    if (causal != 0 && causal != 1) return ATTN_ERR_INVALID;
    if (window > 0 && !causal) return ATTN_ERR_INVALID;
    if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    const long long rows_q = (long long)B * Hq * Sq, rows_k = (long long)B * Hkv * Sk;
    if (rows_q > 0 && (!O || !Q)) return ATTN_ERR_NULL;
    if (rows_q > 0 && Sk > 0 && (!K || !V)) return ATTN_ERR_NULL;
    if (!aligned16(O) || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(LSE))
        return ATTN_ERR_INVALID;
    // TMA coordinates are 32-bit and each dimension must stay below 2^32 elements.
    if ((long long)B * Hq > 0x7fffffffll || (long long)B * Hkv > 0x7fffffffll)
        return ATTN_ERR_INVALID;
    (void)rows_k;
    (void)LSE;
    return ATTN_OK;
}

}  // namespace

extern "C" {

attn_status_t attn_fwd_varlen(void *O, const void *Q, const void *K, const void *V, float *LSE,
                              int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale,
                              int causal, int window, int input_pos, const int32_t *k_lengths,
                              const int32_t *q_lengths, void *stream) {
    NvtxRange nvtx_range("attn_fwd_varlen");
    attn_status_t st =
        validate_fwd(O, Q, K, V, LSE, B, Hq, Hkv, Sq, Sk, D, scale, causal, window, input_pos);
    if (st != ATTN_OK) return st;
    if ((long long)B * Hq * Sq == 0) return ATTN_OK;
    FwdArgs a;
    a.O = O;
    a.Q = Q;
    a.K = K;
    a.V = V;
    a.LSE = LSE;
    a.k_lengths = k_lengths;
    a.q_lengths = q_lengths;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.Sq = Sq;
    a.Sk = Sk;
    a.D = D;
    a.scale = scale;
    a.causal = causal;
    a.window = window;
    a.input_pos = input_pos;
    if (Sk == 0) {
        // No key at all: every row is empty.  The kernel handles k_end = 0 but
        // needs a valid K/V tensor map; use the query tensor as a stand-in.
        a.K = Q;
        a.V = Q;
        a.Sk = 0;
    }
    return launch_fwd(a, static_cast<cudaStream_t>(stream));
}

attn_status_t attn_fwd(void *O, const void *Q, const void *K, const void *V, float *LSE, int B,
                       int Hq, int Hkv, int Sq, int Sk, int D, float scale, int causal, int window,
                       int input_pos, const int32_t *k_lengths, void *stream) {
    NvtxRange nvtx_range("attn_fwd");
    return attn_fwd_varlen(O, Q, K, V, LSE, B, Hq, Hkv, Sq, Sk, D, scale, causal, window,
                           input_pos, k_lengths, nullptr, stream);
}

attn_status_t attn_fwd_flex(void *O, const void *Q, const void *K, const void *V, float *LSE,
                            int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale,
                            int causal, int window, int input_pos,
                            const int32_t *k_lengths, const int32_t *q_lengths,
                            float softcap, const float *alibi_slopes,
                            const int32_t *doc_q, const int32_t *doc_kv,
                            const uint8_t *block_mask, int block_mask_per_head, void *stream) {
    NvtxRange nvtx_range("attn_fwd_flex");
    attn_status_t st =
        validate_fwd(O, Q, K, V, LSE, B, Hq, Hkv, Sq, Sk, D, scale, causal, window, input_pos);
    if (st != ATTN_OK) return st;
    if (!(softcap >= 0.f) || !std::isfinite(softcap)) return ATTN_ERR_INVALID;
    if (softcap > 0.f && alibi_slopes) return ATTN_ERR_INVALID;
    if ((doc_q == nullptr) != (doc_kv == nullptr)) return ATTN_ERR_INVALID;
    if (block_mask_per_head != 0 && block_mask_per_head != 1) return ATTN_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(alibi_slopes) | reinterpret_cast<uintptr_t>(doc_q) |
         reinterpret_cast<uintptr_t>(doc_kv)) & 3u)
        return ATTN_ERR_INVALID;
    if ((long long)Sk > (long long)gqa::kFlexMaxKvTiles * 128) return ATTN_ERR_UNSUPPORTED;
    if ((long long)B * Hq * Sq == 0) return ATTN_OK;
    FwdArgs a;
    a.O = O;
    a.Q = Q;
    a.K = K;
    a.V = V;
    a.LSE = LSE;
    a.k_lengths = k_lengths;
    a.q_lengths = q_lengths;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.Sq = Sq;
    a.Sk = Sk;
    a.D = D;
    a.scale = scale;
    a.causal = causal;
    a.window = window;
    a.input_pos = input_pos;
    a.flex = 1;
    a.softcap = softcap;
    a.alibi_slopes = alibi_slopes;
    a.doc_q = doc_q;
    a.doc_kv = doc_kv;
    a.block_mask = block_mask;
    a.block_mask_per_head = block_mask_per_head;
    if (Sk == 0) {
        a.K = Q;  // stand-in tensor map; no key is visible
        a.V = Q;
        a.doc_kv = nullptr;
        a.doc_q = nullptr;
        a.block_mask = nullptr;
    }
    if (gqa::bsparse_eligible(a)) return gqa::launch_fwd_bsparse(a, static_cast<cudaStream_t>(stream));
    return launch_fwd(a, static_cast<cudaStream_t>(stream));
}

attn_status_t attn_decode(void *O, const void *Q, const void *K, const void *V,
                          const int32_t *lengths, int n_splits, void *stream, int B, int Hq,
                          int Hkv, int S_cap, int D) {
    NvtxRange nvtx_range("attn_decode");
    if (B < 0 || Hq < 1 || Hkv < 1 || S_cap < 0 || n_splits < 1 || n_splits > 64)
        return ATTN_ERR_INVALID;
    if (Hq % Hkv != 0 || Hq / Hkv > 16) return ATTN_ERR_INVALID;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if (B == 0) return ATTN_OK;
    if (!O || !Q || !lengths) return ATTN_ERR_NULL;
    if (S_cap > 0 && (!K || !V)) return ATTN_ERR_NULL;
    if (!aligned16(O) || !aligned16(Q) || !aligned16(K) || !aligned16(V) ||
        (reinterpret_cast<uintptr_t>(lengths) & 3u))
        return ATTN_ERR_INVALID;
    if ((long long)B * Hkv > 0x7fffffffll) return ATTN_ERR_INVALID;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t bytes = decode_workspace_floats(B, Hq, n_splits, D) * sizeof(float);
    void *ws = nullptr;
    if (workspace_alloc(&ws, bytes, s) != cudaSuccess) return ATTN_ERR_CUDA;
    DecodeArgs a;
    a.O = O;
    a.Q = Q;
    a.K = S_cap > 0 ? K : Q;
    a.V = S_cap > 0 ? V : Q;
    a.lengths = lengths;
    a.n_splits = n_splits;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.S_cap = S_cap;
    a.D = D;
    a.workspace = static_cast<float *>(ws);
    attn_status_t st = launch_decode(a, s);
    if (cudaFreeAsync(ws, s) != cudaSuccess && st == ATTN_OK) st = ATTN_ERR_CUDA;
    return st;
}

attn_status_t attn_bwd(void *dQ, void *dK, void *dV, const void *dO, const void *Q, const void *K,
                       const void *V, const void *O, const float *LSE, int B, int Hq, int Hkv,
                       int Sq, int Sk, int D, float scale, int causal, int window, int input_pos,
                       const int32_t *k_lengths, const int32_t *q_lengths, void *stream) {
    NvtxRange nvtx_range("attn_bwd");
    attn_status_t st =
        validate_fwd(const_cast<void *>(O), Q, K, V, nullptr, B, Hq, Hkv, Sq, Sk, D, scale, causal,
                     window, input_pos);
    if (st != ATTN_OK) return st;
    const long long rows_q = (long long)B * Hq * Sq, rows_k = (long long)B * Hkv * Sk;
    if (rows_q > 0 && (!dQ || !dO || !LSE)) return ATTN_ERR_NULL;
    if (rows_k > 0 && (!dK || !dV)) return ATTN_ERR_NULL;
    if (!aligned16(dQ) || !aligned16(dK) || !aligned16(dV) || !aligned16(dO) ||
        (reinterpret_cast<uintptr_t>(LSE) & 3u))
        return ATTN_ERR_INVALID;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (rows_q == 0) {  // no query: dK = dV = 0
        if (rows_k > 0) {
            const size_t bytes = (size_t)rows_k * D * 2;
            if (cudaMemsetAsync(dK, 0, bytes, s) != cudaSuccess ||
                cudaMemsetAsync(dV, 0, bytes, s) != cudaSuccess)
                return ATTN_ERR_CUDA;
        }
        return ATTN_OK;
    }
    void *ws = nullptr;
    if (workspace_alloc(&ws, (size_t)rows_q * sizeof(float), s) != cudaSuccess) return ATTN_ERR_CUDA;
    BwdArgs a;
    a.dQ = dQ;
    a.dK = dK;
    a.dV = dV;
    a.dO = dO;
    a.Q = Q;
    a.K = K;
    a.V = V;
    a.O = O;
    a.LSE = LSE;
    a.k_lengths = k_lengths;
    a.q_lengths = q_lengths;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.Sq = Sq;
    a.Sk = Sk;
    a.D = D;
    a.scale = scale;
    a.causal = causal;
    a.window = window;
    a.input_pos = input_pos;
    a.delta = static_cast<float *>(ws);
    st = launch_bwd(a, s);
    if (cudaFreeAsync(ws, s) != cudaSuccess && st == ATTN_OK) st = ATTN_ERR_CUDA;
    return st;
}

attn_status_t attn_rbs_block_mask(uint8_t *block_mask, float *base_scores, float *rescue_scores,
                                  const void *Q, const void *K, int B, int Hq, int Hkv, int Sq,
                                  int Sk, int D, float alpha_base, float alpha_rescue,
                                  int diagonal, void *stream) {
    NvtxRange nvtx_range("attn_rbs_block_mask");
    if (B < 0 || Hq < 1 || Hkv < 1 || Sq < 0 || Sk < 0 || diagonal < 0) return ATTN_ERR_INVALID;
    if (Hq % Hkv != 0) return ATTN_ERR_INVALID;
    if (!(alpha_base > 0.f) || !(alpha_rescue > 0.f) || !std::isfinite(alpha_base) ||
        !std::isfinite(alpha_rescue))
        return ATTN_ERR_INVALID;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if ((long long)Sk > 131072) return ATTN_ERR_UNSUPPORTED;
    if ((long long)B * Hq * Sq == 0 || Sk == 0) return ATTN_OK;
    if (!block_mask || !Q || !K) return ATTN_ERR_NULL;
    if (!aligned16(Q) || !aligned16(K) ||
        ((reinterpret_cast<uintptr_t>(base_scores) | reinterpret_cast<uintptr_t>(rescue_scores)) & 3u))
        return ATTN_ERR_INVALID;
    const long long nkb = (Sk + 63) / 64;
    const size_t ws_floats = (size_t)B * Hkv * nkb * (D + 2);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    void *ws = nullptr;
    if (workspace_alloc(&ws, ws_floats * sizeof(float), s) != cudaSuccess) return ATTN_ERR_CUDA;
    RbsArgs a;
    a.Q = Q;
    a.K = K;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.Sq = Sq;
    a.Sk = Sk;
    a.D = D;
    a.alpha_base = alpha_base;
    a.alpha_rescue = alpha_rescue;
    a.diagonal = diagonal;
    a.mask = block_mask;
    a.base_scores = base_scores;
    a.rescue_scores = rescue_scores;
    a.cent = static_cast<float *>(ws);
    a.rad = a.cent + (size_t)B * Hkv * nkb * D;
    a.beta = a.rad + (size_t)B * Hkv * nkb;
    attn_status_t st = launch_rbs(a, s);
    if (cudaFreeAsync(ws, s) != cudaSuccess && st == ATTN_OK) st = ATTN_ERR_CUDA;
    return st;
}

attn_status_t attn_decode_paged(void *O, const void *Q, const void *K_cache, const void *V_cache,
                                const int32_t *block_tables, const int32_t *seq_lens, int n_splits,
                                void *stream, int B, int Hq, int Hkv, int num_blocks,
                                int block_size, int max_blocks_per_seq, int D) {
    NvtxRange nvtx_range("attn_decode_paged");
    if (B < 0 || Hq < 1 || Hkv < 1 || num_blocks < 1 || max_blocks_per_seq < 0 || n_splits < 1 ||
        n_splits > 64)
        return ATTN_ERR_INVALID;
    if (block_size < 8 || block_size > 65536 || (block_size & (block_size - 1)) != 0)
        return ATTN_ERR_INVALID;
    if (Hq % Hkv != 0 || Hq / Hkv > 16) return ATTN_ERR_INVALID;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if ((long long)num_blocks * block_size > 0x7fffffffll ||
        (long long)max_blocks_per_seq * block_size > 0x7fffffffll)
        return ATTN_ERR_INVALID;
    if (B == 0) return ATTN_OK;
    if (!O || !Q || !K_cache || !V_cache || !seq_lens || (max_blocks_per_seq > 0 && !block_tables))
        return ATTN_ERR_NULL;
    if (!aligned16(O) || !aligned16(Q) || !aligned16(K_cache) || !aligned16(V_cache) ||
        ((reinterpret_cast<uintptr_t>(seq_lens) | reinterpret_cast<uintptr_t>(block_tables)) & 3u))
        return ATTN_ERR_INVALID;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t bytes = decode_workspace_floats(B, Hq, n_splits, D) * sizeof(float);
    void *ws = nullptr;
    if (workspace_alloc(&ws, bytes, s) != cudaSuccess) return ATTN_ERR_CUDA;
    DecodeArgs a;
    a.O = O;
    a.Q = Q;
    a.K = K_cache;
    a.V = V_cache;
    a.lengths = seq_lens;
    a.n_splits = n_splits;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.S_cap = max_blocks_per_seq * block_size;
    a.D = D;
    a.workspace = static_cast<float *>(ws);
    a.block_tables = block_tables;
    a.num_blocks = num_blocks;
    a.block_size = block_size;
    a.max_blocks = max_blocks_per_seq;
    attn_status_t st = launch_decode(a, s);
    if (cudaFreeAsync(ws, s) != cudaSuccess && st == ATTN_OK) st = ATTN_ERR_CUDA;
    return st;
}

const char *attn_status_string(attn_status_t status) {
    switch (status) {
        case ATTN_OK: return "ATTN_OK";
        case ATTN_ERR_NULL: return "ATTN_ERR_NULL: a required pointer is NULL";
        case ATTN_ERR_INVALID: return "ATTN_ERR_INVALID: inconsistent sizes, flags or alignment";
        case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED: head size not built (64, 128)";
        case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA: a CUDA call failed";
        case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT: a bounded device wait ran out";
        case ATTN_ERR_DEVICE_BOUNDS: return "ATTN_ERR_DEVICE_BOUNDS: a length exceeded its tensor";
        case ATTN_ERR_SCRATCH_LIMIT:
            return "ATTN_ERR_SCRATCH_LIMIT: workspace exceeds the 16 MiB fixed array of "
                   "attn_decode_noalloc";
    }
    return "unknown attn_status_t";
}

attn_status_t attn_last_device_status(void *stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return ATTN_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
    return static_cast<attn_status_t>(v);
}

attn_status_t attn_check_bounded_wait(int limit_us, void *stream) {
    if (limit_us < 1 || limit_us > 2000000) return ATTN_ERR_INVALID;
    return launch_wait_probe(limit_us, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
