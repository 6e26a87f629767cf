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
//  * the first call on a device, and the first after a cudaDeviceReset of
//    it, looks up the array's device address in that device's context; make
//    that call before any stream capture begins.
#include <cuda.h>
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

// The device address of g_route_scratch is looked up once per CUDA context:
// cudaDeviceReset destroys the device's context (and the module holding the
// array), and the next context loads the module again, possibly elsewhere.
// The context's process-unique id (cuCtxGetId) tells the two apart.
struct ScratchAddr {
    unsigned long long ctx_id;
    int32_t* ptr;
};
ScratchAddr g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Id of the context current on this thread, or 0 when it cannot be read.
unsigned long long current_ctx_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(f);
    });
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of the scratch array in the current device's context.  In
// host code the array's name only stands in for the symbol; the address has
// to be asked for with that device (and context) current.
int32_t* scratch_on_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    // make the device's primary context current (no allocation), so that its id can be read
    if (cudaSetDevice(dev) != cudaSuccess) return nullptr;
    const unsigned long long id = current_ctx_id();
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    ScratchAddr& a = g_scratch_addr[dev];
    if (a.ptr == nullptr || id == 0 || a.ctx_id != id) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr) return nullptr;
        a.ptr = static_cast<int32_t*>(p);
        a.ctx_id = id;
    }
    return a.ptr;
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
