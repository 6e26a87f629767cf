// Routing and permutation for callers that cannot allocate device memory.
//
// Some callers of this library cannot call cudaMalloc or hand the library a
// workspace: code embedded in a host runtime that owns every device
// allocation up front (a serving engine with a fixed memory plan, a plugin
// inside another framework), or code on a path where an allocation is not
// allowed at all.  moe_route_permute_noalloc serves them: it runs the same
// three routing kernels as moe_route_permute, but their scratch (the status
// word and the per-chunk expert histograms) lives in one file-scope device
// array that the library owns for the life of the process.  The caller
// still passes the inputs and the outputs.
//
// Limits and sharing rules:
//  * at most kNoAllocMaxPairs = 65536 (token, slot) pairs (T * k) and
//    MOE_MAX_EXPERTS experts; larger calls return MOE_ERR_INVALID_ARG;
//  * every GPU that loads the library holds the array (about 256 KB) until
//    the process exits;
//  * every call uses the same array and leaves its contents behind; calls
//    whose kernels overlap on the GPU (different streams, no ordering
//    between them) race on it and give undefined results;
//  * the first call on a device looks up the array's device address on that
//    device; make that first call before any stream capture begins.
#include <cuda_runtime.h>

#include <mutex>

#include "moefp8.h"
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr int kNoAllocMaxPairs = 65536;
constexpr int kNoAllocChunks = kNoAllocMaxPairs / moe::kRouteChunk;
// status word, padded to 64 ints, then the chunk histograms
constexpr int kNoAllocStatusInts = 64;
constexpr int kNoAllocInts = kNoAllocStatusInts + kNoAllocChunks * MOE_MAX_EXPERTS;

static __device__ __align__(256) int32_t g_route_scratch[kNoAllocInts];

constexpr int kMaxDevices = 64;
int32_t* g_scratch_addr[kMaxDevices];  // device address of g_route_scratch per device
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device.  In host code
// the array's name only stands in for the symbol; the address has to be
// asked for once per device with that device current.
int32_t* scratch_on_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr) return nullptr;
        g_scratch_addr[dev] = static_cast<int32_t*>(p);
    }
    return g_scratch_addr[dev];
}

}  // namespace

extern "C" int moe_route_permute_noalloc(const int32_t* topk_ids, int T, int k, int E,
                                         int32_t* m_indptr, int32_t* perm, int32_t* inv_perm,
                                         moe_stream_t stream) {
    if (T < 0 || k < 1 || E < 1 || E > MOE_MAX_EXPERTS) return MOE_ERR_INVALID_ARG;
    if (static_cast<long long>(T) * k > kNoAllocMaxPairs) return MOE_ERR_INVALID_ARG;
    if (!m_indptr || (T > 0 && (!topk_ids || !perm))) return MOE_ERR_INVALID_ARG;
    int32_t* scratch = scratch_on_current_device();
    if (!scratch) return MOE_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // the status word accumulates with atomics: it must start at zero; the
    // histograms are fully rewritten by every call
    if (cudaMemsetAsync(scratch, 0, sizeof(int32_t) * kNoAllocStatusInts, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    moe::RouteArgs ra{topk_ids, T, k, E, m_indptr, perm, inv_perm,
                      scratch + kNoAllocStatusInts, scratch};
    return moe::launch_route_permute(ra, s);
}
