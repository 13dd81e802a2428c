// attn_decode_noalloc.cu -- split-KV decode for callers that must not allocate.
//
// attn_decode() obtains its per-slice workspace from a stream-ordered allocator on every
// call.  Some callers cannot allow that: a serving loop that reserves all of its
// device memory up front and forbids any allocation afterwards (an allocation
// can fail once the memory is spoken for, and its latency is not bounded), or a
// host program whose memory is owned by another allocator the library must not
// bypass.  For them, attn_decode_noalloc() runs the same split and combine
// kernels with the workspace taken from one fixed array compiled into the
// library instead of from the allocator.
//
// The array is file-scope device memory of kNoAllocScratchBytes (16 MiB).  Every
// GPU that loads the library keeps it until the process exits, and every call
// on a device shares it:
//   - calls that may run at the same time on the GPU (different streams, or
//     different host threads without ordering) race on it and must be
//     serialised by the caller, e.g. by issuing them on one stream;
//   - it keeps whatever the last call left; the split kernel writes every
//     entry the combine kernel reads (an empty slice, or one whose bounded wait
//     ran out, writes a log-sum-exp of -inf and so weighs nothing), so nothing
//     needs clearing between calls.
// In host code the array's name is only a host-side stand-in, so its device
// address is looked up with cudaGetSymbolAddress, once per device, on the first
// call made while that device is current; that first call should come before
// any stream capture begins.
#include <nvtx3/nvToolsExt.h>
#include <mutex>

#include <cuda_runtime.h>

#include "internal.h"

namespace gqa {

size_t decode_workspace_floats(int B, int Hq, int n_splits, int D);

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

std::mutex g_setup_mutex;
float *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once).
attn_status_t scratch_for_current_device(float **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
            return ATTN_ERR_CUDA;
        g_scratch_ptr[dev] = static_cast<float *>(ptr);
    }
    *out = g_scratch_ptr[dev];
    return ATTN_OK;
}

}  // namespace

}  // namespace gqa

using namespace gqa;

extern "C" attn_status_t attn_decode_noalloc(void *O, const void *Q, const void *K, const void *V,
                                             const int32_t *lengths, int n_splits, void *stream,
                                             int B, int Hq, int Hkv, int S_cap, int D) {
    // NVTX range around the call (host side), as for the other entry points
    nvtxRangePushA("attn_decode_noalloc");
    struct Pop {
        ~Pop() { nvtxRangePop(); }
    } pop_at_return;
    // Same argument checks as attn_decode.
    if (B < 0 || Hq < 1 || Hkv < 1 || S_cap < 0 || n_splits < 1 || n_splits > 64)
        return ATTN_ERR_INVALID;
    if (Hq % Hkv != 0 || Hq / Hkv > 16) return ATTN_ERR_INVALID;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if (B == 0) return ATTN_OK;
    if (!O || !Q || !lengths) return ATTN_ERR_NULL;
    if (S_cap > 0 && (!K || !V)) return ATTN_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(O) | reinterpret_cast<uintptr_t>(Q) |
         reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(V)) & 15u ||
        (reinterpret_cast<uintptr_t>(lengths) & 3u))
        return ATTN_ERR_INVALID;
    if ((long long)B * Hkv > 0x7fffffffll) return ATTN_ERR_INVALID;
    // The workspace must fit in the fixed array.
    if (decode_workspace_floats(B, Hq, n_splits, D) * sizeof(float) > kNoAllocScratchBytes)
        return ATTN_ERR_SCRATCH_LIMIT;
    float *scratch = nullptr;
    attn_status_t st = scratch_for_current_device(&scratch);
    if (st != ATTN_OK) return st;
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
    a.workspace = scratch;
    return launch_decode(a, static_cast<cudaStream_t>(stream));
}
