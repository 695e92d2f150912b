// moe_permute_static_ws: the token permutation for callers that cannot allocate.
//
// Some callers only ever receive the tensors of a call (inputs and outputs) and
// have no way to hand this library a workspace: for example an inference
// engine's plugin "execute" hook that owns a fixed memory pool and forbids device
// allocation while a request runs, since an allocation there would stall the
// stream or fragment the pool.  This entry point runs the same permutation
// kernels as moe_permute, but keeps their per-chunk histogram in a file-scope
// device array instead of a caller-provided workspace.  It allocates nothing.
//
// The array holds (tokens / 256) x E int32 counters: at most 256 chunks of 256
// tokens and 256 experts, i.e. 65536 tokens, 256 KiB per device.  Every GPU
// that loads this library keeps it until the process exits.
#include <mutex>

#include "kernels.h"
#include "moe.h"

namespace {

constexpr int kStaticMaxTokens = MOE_PERMUTE_STATIC_MAX_TOKENS;
constexpr size_t kStaticWords = (size_t)(kStaticMaxTokens / moe::kPermuteChunk) * MOE_MAX_EXPERTS;

// The histogram scratch.  Shared by every call on a device and never cleared:
// each call's histogram kernel overwrites every entry it later reads.
static __device__ __align__(256) int32_t g_permute_scratch[kStaticWords];

constexpr int kMaxDev = 64;
std::mutex g_lookup_mu;
int32_t* g_scratch_ptr[kMaxDev] = {};

// In host code g_permute_scratch names a host-side stand-in, not device memory,
// so its device address is looked up per device (with that device current).
// Only a successful lookup is kept: a call that failed (for example one made
// during a stream capture) leaves the next call free to try again.
int32_t* scratch_for(int dev) {
    std::lock_guard<std::mutex> lock(g_lookup_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_permute_scratch) == cudaSuccess) g_scratch_ptr[dev] = static_cast<int32_t*>(p);
        else cudaGetLastError();
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" moe_status_t moe_permute_static_ws(const void* v, moe_dtype_t v_dt, const int32_t* topk_idx, int32_t T,
                                              int32_t d, int32_t E, int32_t k, int32_t* counts, int32_t* offsets,
                                              int32_t* slot_token, int32_t* token_slot, void* xp,
                                              int32_t* dev_status, moe_stream_t stream) {
    if (T < 0 || d <= 0 || E <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
    if (k > MOE_MAX_TOP_K || E > MOE_MAX_EXPERTS || k > E || d % 8 != 0) return MOE_ERR_UNSUPPORTED;
    if (T > kStaticMaxTokens) return MOE_ERR_UNSUPPORTED;  // beyond the static histogram's capacity
    if (v_dt != MOE_F32 && v_dt != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!v || !topk_idx || !slot_token || !token_slot || !xp ||
                  (reinterpret_cast<uintptr_t>(v) & 15u) || (reinterpret_cast<uintptr_t>(xp) & 15u)))
        return MOE_ERR_INVALID_ARG;
    int dev = 0, sms = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    if (major != 10) return MOE_ERR_DEVICE;
    int32_t* hist = scratch_for(dev);
    if (!hist) return MOE_ERR_CUDA;
    moe::Ctx c{reinterpret_cast<cudaStream_t>(stream), sms, dev};
    cudaError_t e = moe::launch_permute(c, v, v_dt, topk_idx, T, d, E, k, counts, offsets, slot_token, token_slot, xp,
                                        hist, dev_status);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}
