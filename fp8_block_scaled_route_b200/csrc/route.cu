// Routing and permutation: groups the T*k (token, slot) pairs by expert.
//
// The grouped layout is the m_indptr prefix array of the grouped GEMM
// interface on the page "FlashInfer SM120 MoE GEMM 최적화: 웨이브+잔여물 비용
// 모델 도입" (flashinfer PR #4318, "코드 분석 1."): rows of A grouped by
// expert, m_indptr[e] the first row of expert e.  Grouping is a stable
// counting sort on the pair id p = t*k + j, so the result is unique and
// bit-reproducible.
//
// Three launches (one for inputs of at most 8 chunks), no atomics on the
// output order:
//  1. route_hist:    one 1024-pair chunk per CTA -> per-chunk expert histogram
//  2. route_scan:    one CTA: per-expert exclusive scan over chunks, then the
//                    exclusive scan over experts -> m_indptr and the first
//                    output row of every (chunk, expert)
//  3. route_scatter: one warp per chunk walks its pairs in order, 32 at a
//                    time; lanes with the same expert are ranked with
//                    one warp ballot per expert-id bit, so each pair lands at
//                    chunk_base[e] + (earlier pairs of e in the chunk).
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace moe {

// Lanes of the warp whose value equals this lane's, among the lanes with
// ok set, for values in [0, 2^nbits): one ballot per value bit (nbits
// uniform across the warp).  Used in place of the match instruction, whose
// cost grows with the number of distinct values in the warp.
__device__ __forceinline__ unsigned same_value_lanes(int v, bool ok, int nbits) {
    unsigned m = __ballot_sync(0xffffffffu, ok);
    for (int b = 0; b < nbits; ++b) {
        const bool bit = (v >> b) & 1;
        const unsigned bb = __ballot_sync(0xffffffffu, bit);
        m &= bit ? bb : ~bb;
    }
    return m;
}

__host__ __device__ inline int value_bits(int E) {
    int n = 0;
    while ((1 << n) < E) ++n;
    return n;
}

__global__ void __launch_bounds__(256) route_hist(const int32_t* __restrict__ ids, int R, int E,
                                                  int32_t* __restrict__ chunk_hist, int* status) {
    extern __shared__ int hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int base = blockIdx.x * kRouteChunk;
    const int end = min(R, base + kRouteChunk);
    int bad = 0;
    for (int p = base + threadIdx.x; p < end; p += blockDim.x) {
        const int e = ids[p];
        if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
        else ++bad;
    }
    if (bad) {
        atomicAdd(&status[2], bad);
        report_error(status, ST_BAD_EXPERT_ID, 0);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        chunk_hist[static_cast<long long>(blockIdx.x) * E + e] = hist[e];
}

// blockDim.x = 1024 >= E.  Each thread owns one expert; the per-chunk counts
// are read in batches of independent loads so the loop is not one memory
// latency per chunk.
__global__ void __launch_bounds__(1024) route_scan(int nchunks, int E, int32_t* __restrict__ chunk_hist,
                                                   int32_t* __restrict__ m_indptr) {
    __shared__ int warp_tot[32];
    constexpr int kBatch = 16;
    const int e = threadIdx.x;
    int count = 0;
    if (e < E) {
        for (int c0 = 0; c0 < nchunks; c0 += kBatch) {
            int h[kBatch];
#pragma unroll
            for (int i = 0; i < kBatch; ++i)
                h[i] = (c0 + i < nchunks) ? chunk_hist[static_cast<long long>(c0 + i) * E + e] : 0;
#pragma unroll
            for (int i = 0; i < kBatch; ++i) {
                if (c0 + i < nchunks) chunk_hist[static_cast<long long>(c0 + i) * E + e] = count;  // rows of e in earlier chunks
                count += h[i];
            }
        }
    }
    // exclusive scan of count over experts
    const int lane = e & 31, w = e >> 5;
    int incl = count;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_tot[w] = incl;
    __syncthreads();
    if (w == 0) {
        int t = warp_tot[lane];
        int ti = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, ti, o);
            if (lane >= o) ti += v;
        }
        warp_tot[lane] = ti - t;  // exclusive prefix of warp totals
    }
    __syncthreads();
    const int excl = warp_tot[w] + incl - count;
    if (e < E) {
        m_indptr[e] = excl;
        for (int c = 0; c < nchunks; ++c) chunk_hist[static_cast<long long>(c) * E + e] += excl;
    }
    if (e == E - 1) m_indptr[E] = excl + count;
}

// blockDim.x = 32: one warp per chunk.  The chunk's expert ids are read up
// front (one batch of independent loads), then ranked 32 at a time.
__global__ void __launch_bounds__(32) route_scatter(const int32_t* __restrict__ ids, int R, int E,
                                                    const int32_t* __restrict__ chunk_base,
                                                    int32_t* __restrict__ perm,
                                                    int32_t* __restrict__ inv_perm) {
    extern __shared__ int cursor[];
    constexpr int kSteps = kRouteChunk / 32;
    const int lane = threadIdx.x;
    const int base = blockIdx.x * kRouteChunk;
    const int end = min(R, base + kRouteChunk);
    int my_ids[kSteps];
#pragma unroll
    for (int i = 0; i < kSteps; ++i) {
        const int p = base + i * 32 + lane;
        my_ids[i] = p < end ? ids[p] : -1;
    }
    for (int e = lane; e < E; e += 32)
        cursor[e] = chunk_base[static_cast<long long>(blockIdx.x) * E + e];
    __syncwarp();
#pragma unroll
    for (int i = 0; i < kSteps; ++i) {
        const int p = base + i * 32 + lane;
        if (base + i * 32 >= end) break;
        const bool live = p < end;
        const int e = my_ids[i];
        const bool ok = live && e >= 0 && e < E;
        const unsigned peers = same_value_lanes(e, ok, value_bits(E));
        const int rank = __popc(peers & ((1u << lane) - 1u));
        const int first = cursor[ok ? e : 0];
        __syncwarp();
        if (ok) {
            const int row = first + rank;
            perm[row] = p;
            if (inv_perm) inv_perm[p] = row;
            if (rank == 0) cursor[e] = first + __popc(peers);
        } else if (live && inv_perm) {
            inv_perm[p] = -1;
        }
        __syncwarp();
    }
}

// Small inputs (at most kSmallChunks chunks of 1024 pairs): the same three
// phases in one CTA of 1024 threads, so routing costs one launch.  The pairs
// are cut into up to 32 consecutive blocks, one per warp (as many as keep the
// per-block histograms within the default shared-memory limit), so the
// serial ranking steps of phase 3 are spread over the warps.  Phase 2 scans
// each expert's column of block counts with one warp (lane = block; rows of
// the table padded to E + 1 ints so a column read is conflict-free), then
// the experts' totals with one thread per expert.
constexpr int kSmallChunks = 8;
// 43 KB of table; with the static per-expert totals (4 KB) within 48 KB
constexpr int kSmallTabInts = 11008;

__host__ __device__ constexpr int small_route_warps(int E) {
    return (E + 1) * 32 <= kSmallTabInts ? 32 : kSmallTabInts / (E + 1);
}
static_assert(small_route_warps(kMaxRouteExperts) >= kSmallChunks,
              "route_small's pair blocks must stay within kRouteChunk pairs");

// Dynamic shared memory of route_small: the table, then the R entries of
// perm, which phase 3 writes in shared memory (scattered) and the CTA then
// copies out in order: scattered 4-byte global stores from one SM go out at
// about one sector per clock (4096 of them cost ~4 µs).
__host__ __device__ inline size_t small_route_smem(int R, int E) {
    return (static_cast<size_t>(small_route_warps(E)) * (E + 1) + R) * sizeof(int);
}
constexpr size_t kSmallRouteSmemMax = (kSmallTabInts + kSmallChunks * kRouteChunk) * sizeof(int);

// The three phases of route_small for a CTA of 1024 threads; tab is
// [small_route_warps(E)][E + 1] ints of shared memory followed by R ints.
__device__ __forceinline__ void route_small_body(const int32_t* __restrict__ ids, int R, int E,
                                                 int32_t* __restrict__ m_indptr,
                                                 int32_t* __restrict__ perm,
                                                 int32_t* __restrict__ inv_perm, int* status,
                                                 int* tab, bool clear_status) {
    __shared__ int warp_tot[32];
    __shared__ int cnt_s[kMaxRouteExperts];   // per-expert totals, then first rows
    __shared__ int valid_s;                   // pairs with a valid expert id
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int W = small_route_warps(E);
    const int Ep = E + 1;
    int* perm_s = tab + W * Ep;               // [R]: perm, staged
    // pairs per block: a multiple of 32, at most kRouteChunk (R <= 8 chunks, W >= 8)
    const int B = ((R + W - 1) / W + 31) & ~31;
    const int nchunks = B > 0 ? (R + B - 1) / B : 0;
    constexpr int kSteps = kRouteChunk / 32;
    // the caller's status words start clean before any error is reported
    if (clear_status && threadIdx.x < kStatusInts) status[threadIdx.x] = 0;
    for (int i = threadIdx.x; i < nchunks * Ep; i += blockDim.x) tab[i] = 0;
    __syncthreads();
    // phase 1: per-block histograms
    int my_ids[kSteps];
    const int base = warp * B;
    if (warp < nchunks) {
        const int end = min(R, base + B);
        int bad = 0;
#pragma unroll
        for (int i = 0; i < kSteps; ++i) {
            const int p = base + i * 32 + lane;
            my_ids[i] = p < end ? ids[p] : -1;
        }
#pragma unroll
        for (int i = 0; i < kSteps; ++i) {
            const int p = base + i * 32 + lane;
            if (p < end) {
                const int e = my_ids[i];
                if (e >= 0 && e < E) atomicAdd(&tab[warp * Ep + e], 1);
                else ++bad;
            }
        }
        if (bad) {
            atomicAdd(&status[2], bad);
            report_error(status, ST_BAD_EXPERT_ID, 0);
        }
    }
    __syncthreads();
    // phase 2a: per expert, exclusive scan over the blocks (warp per expert, lane = block)
    for (int ex = warp; ex < E; ex += 32) {
        const int h = lane < nchunks ? tab[lane * Ep + ex] : 0;
        int run = h;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, run, o);
            if (lane >= o) run += v;
        }
        if (lane < nchunks) tab[lane * Ep + ex] = run - h;
        if (lane == 31) cnt_s[ex] = run;
    }
    __syncthreads();
    // phase 2b: exclusive scan over the experts' totals (thread e)
    const int e = threadIdx.x;
    const int count = e < E ? cnt_s[e] : 0;
    int incl = count;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int t = warp_tot[lane];
        int ti = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, ti, o);
            if (lane >= o) ti += v;
        }
        warp_tot[lane] = ti - t;
    }
    __syncthreads();
    const int excl = warp_tot[warp] + incl - count;
    if (e < E) {
        m_indptr[e] = excl;
        cnt_s[e] = excl;   // only thread e read cnt_s[e] above
    }
    if (e == E - 1) {
        m_indptr[E] = excl + count;
        valid_s = excl + count;
    }
    __syncthreads();
    // phase 2c: first output row of every (block, expert)
    for (int ex = warp; ex < E; ex += 32)
        if (lane < nchunks) tab[lane * Ep + ex] += cnt_s[ex];
    __syncthreads();
    // phase 3: stable scatter, 32 pairs at a time per block
    const int nbits = value_bits(E);
    if (warp < nchunks) {
        const int end = min(R, base + B);
        int* cursor = tab + warp * Ep;
#pragma unroll
        for (int i = 0; i < kSteps; ++i) {
            const int p = base + i * 32 + lane;
            if (base + i * 32 >= end) break;
            const bool live = p < end;
            const int ex = my_ids[i];
            const bool ok = live && ex >= 0 && ex < E;
            const unsigned peers = same_value_lanes(ex, ok, nbits);
            const int rank = __popc(peers & ((1u << lane) - 1u));
            const int first = cursor[ok ? ex : 0];
            __syncwarp();
            if (ok) {
                const int row = first + rank;
                perm_s[row] = p;
                if (inv_perm) inv_perm[p] = row;
                if (rank == 0) cursor[ex] = first + __popc(peers);
            } else if (live && inv_perm) {
                inv_perm[p] = -1;
            }
            __syncwarp();
        }
    }
    __syncthreads();
    // perm out in order (rows of dropped pairs do not exist: only [0, valid) is written)
    const int valid = valid_s;
    for (int i = threadIdx.x; i < valid; i += blockDim.x) perm[i] = perm_s[i];
}

__global__ void __launch_bounds__(1024) route_small(const int32_t* __restrict__ ids, int R, int E,
                                                    int32_t* __restrict__ m_indptr,
                                                    int32_t* __restrict__ perm,
                                                    int32_t* __restrict__ inv_perm, int* status,
                                                    int clear_status) {
    extern __shared__ int tab[];  // [blocks][E + 1]: histograms, then first rows
    route_small_body(ids, R, E, m_indptr, perm, inv_perm, status, tab, clear_status != 0);
}

// Router (the step before the expert computation): one warp per token.
// Lane l holds logits l + 32 i; the k winners are taken one at a time by a
// warp-wide argmax (larger logit first, then the lower expert index), so the
// ids come out in descending logit order.  Lane j keeps the j-th winner's
// logit; the softmax subtracts the largest, takes expf per slot and sums the
// slots in order (every lane runs the same sequential sum), w_j = e_j / sum.
template <int PER>
__device__ __forceinline__ void router_token(const float* __restrict__ logits, int t, int E, int k,
                                             int32_t* __restrict__ ids, float* __restrict__ w) {
    const int lane = threadIdx.x & 31;
    const float* l = logits + static_cast<long long>(t) * E;
    float v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int e = lane + 32 * i;
        v[i] = e < E ? l[e] : 0.0f;
    }
    uint32_t taken = 0;
    float mine = 0.0f;  // logit of slot `lane`
    for (int j = 0; j < k; ++j) {
        float bv = 0.0f;
        int be = E;  // E = none
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !((taken >> i) & 1u) && (be == E || v[i] > bv)) {
                bv = v[i];
                be = e;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (oe != E && (be == E || ov > bv || (ov == bv && oe < be))) {
                bv = ov;
                be = oe;
            }
        }
        if (lane == (be & 31)) taken |= 1u << (be >> 5);
        if (lane == j) mine = bv;
        if (lane == 0) ids[static_cast<long long>(t) * k + j] = be;
    }
    const float m = __shfl_sync(0xffffffffu, mine, 0);
    const float ex = lane < k ? expf(mine - m) : 0.0f;
    float sum = 0.0f;
    for (int j = 0; j < k; ++j) sum += __shfl_sync(0xffffffffu, ex, j);
    if (lane < k) w[static_cast<long long>(t) * k + lane] = __fdiv_rn(ex, sum);
}

template <int PER>
__global__ void __launch_bounds__(256) router_topk_kernel(const float* __restrict__ logits, int T,
                                                          int E, int k, int32_t* __restrict__ ids,
                                                          float* __restrict__ w) {
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= T) return;
    router_token<PER>(logits, t, E, k, ids, w);
}

// Router and routing in one CTA of 1024 threads, for at most kSmallChunks
// chunks of pairs: each warp routes tokens warp, warp + 32, ..., then the
// CTA groups the pairs it just wrote (global writes made visible to the
// whole CTA by the barrier) with route_small's three phases.
template <int PER>
__global__ void __launch_bounds__(1024) router_route_small(const float* __restrict__ logits, int T,
                                                           int E, int k, int32_t* __restrict__ ids,
                                                           float* __restrict__ w,
                                                           int32_t* __restrict__ m_indptr,
                                                           int32_t* __restrict__ perm,
                                                           int32_t* __restrict__ inv_perm,
                                                           int* status) {
    extern __shared__ int tab[];
    for (int t = threadIdx.x >> 5; t < T; t += 32) router_token<PER>(logits, t, E, k, ids, w);
    __syncthreads();
    route_small_body(ids, T * k, E, m_indptr, perm, inv_perm, status, tab, false);
}

int launch_router_topk(const float* logits, int T, int E, int k, int32_t* ids, float* w,
                       cudaStream_t stream) {
    if (T == 0) return ST_OK;
    const unsigned blocks = static_cast<unsigned>((T + 7) / 8);
    if (E <= 256)
        router_topk_kernel<8><<<blocks, 256, 0, stream>>>(logits, T, E, k, ids, w);
    else
        router_topk_kernel<32><<<blocks, 256, 0, stream>>>(logits, T, E, k, ids, w);
    return cudaGetLastError() == cudaSuccess ? ST_OK : ST_CUDA;
}

// Opt-in of the single-CTA routing kernels to kSmallRouteSmemMax bytes of
// dynamic shared memory, once per device.
bool small_route_smem_ready() {
    static std::atomic<int> ready_dev{-1};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (ready_dev.load() == dev) return true;
    const int n = static_cast<int>(kSmallRouteSmemMax);
    if (cudaFuncSetAttribute(route_small, cudaFuncAttributeMaxDynamicSharedMemorySize, n) != cudaSuccess ||
        cudaFuncSetAttribute(router_route_small<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, n) !=
            cudaSuccess ||
        cudaFuncSetAttribute(router_route_small<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, n) !=
            cudaSuccess)
        return false;
    ready_dev.store(dev);
    return true;
}

int launch_router_route(const float* logits, const RouteArgs& r, float* w, cudaStream_t stream) {
    const int R = r.T * r.k;
    if (R == 0) return launch_route_permute(r, stream);
    const int nchunks = (R + kRouteChunk - 1) / kRouteChunk;
    if (nchunks <= kSmallChunks) {
        int32_t* ids = const_cast<int32_t*>(r.topk_ids);
        const size_t smem = small_route_smem(R, r.E);
        if (!small_route_smem_ready()) return ST_CUDA;
        if (r.E <= 256)
            router_route_small<8><<<1, 1024, smem, stream>>>(logits, r.T, r.E, r.k, ids, w,
                                                             r.m_indptr, r.perm, r.inv_perm, r.status);
        else
            router_route_small<32><<<1, 1024, smem, stream>>>(logits, r.T, r.E, r.k, ids, w,
                                                              r.m_indptr, r.perm, r.inv_perm, r.status);
        return cudaGetLastError() == cudaSuccess ? ST_OK : ST_CUDA;
    }
    int st = launch_router_topk(logits, r.T, r.E, r.k, const_cast<int32_t*>(r.topk_ids), w, stream);
    if (st) return st;
    return launch_route_permute(r, stream);
}

bool route_single_launch(int R) { return (R + kRouteChunk - 1) / kRouteChunk <= kSmallChunks; }

int launch_route_permute(const RouteArgs& r, cudaStream_t stream) {
    const int R = r.T * r.k;
    const int nchunks = (R + kRouteChunk - 1) / kRouteChunk;
    const size_t hist_smem = static_cast<size_t>(r.E) * sizeof(int);
    if (nchunks <= kSmallChunks) {
        const size_t smem = small_route_smem(R, r.E);
        if (!small_route_smem_ready()) return ST_CUDA;
        route_small<<<1, 1024, smem, stream>>>(r.topk_ids, R, r.E, r.m_indptr, r.perm, r.inv_perm,
                                               r.status, r.clear_status);
        return cudaGetLastError() == cudaSuccess ? ST_OK : ST_CUDA;
    }
    {
        route_hist<<<nchunks, 256, hist_smem, stream>>>(r.topk_ids, R, r.E, r.chunk_hist, r.status);
        if (cudaGetLastError() != cudaSuccess) return ST_CUDA;
    }
    route_scan<<<1, 1024, 0, stream>>>(nchunks, r.E, r.chunk_hist, r.m_indptr);
    if (cudaGetLastError() != cudaSuccess) return ST_CUDA;
    if (nchunks > 0) {
        route_scatter<<<nchunks, 32, hist_smem, stream>>>(r.topk_ids, R, r.E, r.chunk_hist, r.perm,
                                                          r.inv_perm);
        if (cudaGetLastError() != cudaSuccess) return ST_CUDA;
    }
    return ST_OK;
}

}  // namespace moe
