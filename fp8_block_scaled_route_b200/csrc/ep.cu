// Kernels of the expert-parallel data plane: the layer of the page
// "FlashInfer: Blackwell W8A8 AlphaMoE Expert 계산 커널 퓨전으로 성능 비약적
// 향상" (flashinfer PR #4287, section "문제점: MoE Expert 계산의 병목") with the
// experts split over G GPUs, each GPU owning a contiguous range of E/G
// experts.  A rank sends each (token, slot) pair's quantised activation row
// to the rank that owns the pair's expert, that rank runs the expert FFN on
// the rows it received, and the fp32 rows travel back for the combine.
//  * ep_owner_kernel: owner rank of every pair (-1 for an id outside
//    [0, E)), the key the routing kernels then sort the pairs by;
//  * gather_rows_kernel: received rows (any order) into expert-grouped order
//    for 128-token GEMM tiles (FP8 codes row by row, block scales from
//    row-major [n, H/128] to column-block-major [H/128, n]); smaller token
//    tiles read the received rows in place through the GEMM's row map.
#include "common.cuh"
#include "kernels.h"

namespace moe {

__global__ void __launch_bounds__(256) ep_owner_kernel(const int32_t* __restrict__ ids, long long R,
                                                       int E, int experts_per_rank,
                                                       int32_t* __restrict__ owner) {
    for (long long p = blockIdx.x * 256ll + threadIdx.x; p < R; p += gridDim.x * 256ll) {
        const int e = ids[p];
        owner[p] = (e >= 0 && e < E) ? e / experts_per_rank : -1;
    }
}

int launch_ep_owner(const int32_t* ids, long long R, int E, int experts_per_rank, int32_t* owner,
                    int num_sms, cudaStream_t stream) {
    if (R == 0) return ST_OK;
    long long blocks = (R + 255) / 256;
    if (blocks > num_sms * 8ll) blocks = num_sms * 8ll;
    ep_owner_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(ids, R, E, experts_per_rank,
                                                                        owner);
    return cudaGetLastError() == cudaSuccess ? ST_OK : ST_CUDA;
}

// One warp per grouped row r: copies row src_of[r] of xq (H bytes, 16 per
// lane per step) and scatters its H/128 scales into column-block-major order.
// Rows at or past *rows_dev (the grouped rows that exist) are skipped.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint8_t* __restrict__ xq,
                                                          const float* __restrict__ xs, int n,
                                                          int H, const int32_t* __restrict__ src_of,
                                                          int rows, const int32_t* __restrict__ rows_dev,
                                                          uint8_t* __restrict__ xq_g,
                                                          float* __restrict__ xs_g) {
    const long long r = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (r >= rows || (rows_dev && r >= *rows_dev)) return;
    const int lane = threadIdx.x & 31;
    const long long src = src_of[r];
    const uint4* s = reinterpret_cast<const uint4*>(xq + src * H);
    uint4* d = reinterpret_cast<uint4*>(xq_g + r * H);
    for (int c = lane; c < H / 16; c += 32) d[c] = s[c];
    const int nkb = H >> 7;
    for (int kb = lane; kb < nkb; kb += 32) xs_g[static_cast<long long>(kb) * n + r] = xs[src * nkb + kb];
}

int launch_gather_rows(const uint8_t* xq, const float* xs, int n, int H, const int32_t* src_of,
                       int rows, const int32_t* rows_dev, uint8_t* xq_g, float* xs_g,
                       cudaStream_t stream) {
    if (rows == 0) return ST_OK;
    const long long blocks = (rows + 7) / 8;
    gather_rows_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(xq, xs, n, H, src_of, rows,
                                                                          rows_dev, xq_g, xs_g);
    return cudaGetLastError() == cudaSuccess ? ST_OK : ST_CUDA;
}

}  // namespace moe
