// Internal host-side interface between the C ABI layer and the kernels.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace moe {

// Epilogue of the grouped GEMM.
enum Epilogue : int {
    EPI_BF16 = 0,          // plain: out[r, n] = bf16(G)
    EPI_SWIGLU_BF16 = 1,   // gated: out[r, i] = bf16(silu(G_gate) * G_up)
    EPI_SWIGLU_QUANT = 2,  // gated: h = silu(G_gate) * G_up, FP8 per row per 128 cols
    EPI_Y32 = 4,           // plain: y[r, n] = G (fp32, grouped row order, each row written once)
};

struct GemmArgs {
    // A [R, K] FP8 (grouped rows), B [E, N, K] FP8
    const void* a;
    const void* b;
    int R, N, K, E;
    // a_scale(r, kb) = a_scale[r * as_row + kb * as_kb]; b_scale [E, N/128, K/128]
    const float* a_scale;
    long long as_row, as_kb;
    const float* b_scale;
    const int32_t* m_indptr;  // [E+1]
    int epi;
    int tile_m;  // 16, 32, 64 (weights as the MMA M operand) or 128 (tokens as M)
    // EPI_SWIGLU_QUANT: hq [R, N/2] codes, hs [(N/2)/128, R]
    uint8_t* hq;
    float* hs;
    // When set, grouped row r reads row a_rowmap[r] / a_rowdiv of A (a_rows
    // rows) and of its scales, through TMA gather4 loads; null: row r of A.
    const int32_t* a_rowmap;
    int a_rowdiv;
    int a_rows;
    // EPI_Y32: y[r * ldy + n], or y[rowmap[r] * ldy + n] when rowmap is set
    float* y;
    int ldy;
    const int32_t* rowmap;
    // EPI_BF16 / EPI_SWIGLU_BF16
    void* out_bf16;
    int* status;
    uint64_t timeout_ns;
    int num_sms;
};

// Returns a moe_status_t value.
int launch_grouped_gemm(const GemmArgs& g, cudaStream_t stream);

// Largest K the swapped (tile_m < 128) kernels accept for a token tile.
int swap_max_k(int tile_m);

// Both expert GEMMs in one launch with the FP8 intermediate in shared
// memory (fused_expert.cu).  Reads the grouped token rows xq [R, H] with
// their scales xs [H/128, R] (the quantiser's k-copy layout).  Writes the
// fp32 rows y [R, H] in grouped order, and the intermediate to hq [R, I] /
// hs [I/128, R] when those are set.
struct FusedExpertArgs {
    const void* xq;
    const float* xs;
    int R, H, I, E;
    const void* w13;          // [E, 2I, H]
    const float* w13_scale;   // [E, 2I/128, H/128]
    const void* w2;           // [E, H, I]
    const float* w2_scale;    // [E, H/128, I/128]
    const int32_t* m_indptr;  // [E+1]
    float* y;
    uint8_t* hq;
    float* hs;
    int* status;
    uint64_t timeout_ns;
    int num_sms;
};

// Whether the fused expert kernel can hold the intermediate of a 64-token
// tile for this H, I, E (and enough pipeline stages) in shared memory.
bool fused_expert_fits(int H, int I, int E);
int launch_fused_expert(const FusedExpertArgs& g, cudaStream_t stream);

struct RouteArgs {
    const int32_t* topk_ids;
    int T, k, E;
    int32_t* m_indptr;
    int32_t* perm;
    int32_t* inv_perm;
    int32_t* chunk_hist;  // [nchunks, E]
    int* status;
    // single-launch routing only: the kernel zeroes status[0, kStatusInts)
    // before it reports anything (the caller then needs no clearing memset)
    int clear_status;
};
constexpr int kRouteChunk = 1024;
// Whether routing R pairs takes the single-launch (one CTA) path.
bool route_single_launch(int R);
// Largest expert count the routing kernels accept (MOE_MAX_EXPERTS of the C ABI).
constexpr int kMaxRouteExperts = 1024;
int launch_route_permute(const RouteArgs& r, cudaStream_t stream);

// logits fp32 [T, E] -> ids int32 [T, k] (descending logit, ties to the lower
// expert), w fp32 [T, k] = softmax of the selected logits.  E <= 1024, k <= 32.
int launch_router_topk(const float* logits, int T, int E, int k, int32_t* ids, float* w,
                       cudaStream_t stream);

// Router then routing: ids r.topk_ids [T, k] (written) and w [T, k] from
// logits [T, E] as launch_router_topk, then the tables as
// launch_route_permute; one launch for at most 8 chunks of pairs.
int launch_router_route(const float* logits, const RouteArgs& r, float* w, cudaStream_t stream);

// x [T, H] bf16 -> xq rows inv_perm[t*k + j] of [R, H] (row t*k + j when
// inv_perm is null), xs [H/128, R];
// also zeroes out_acc [T, H] when not null.
int launch_quant_scatter(const void* x, int T, int H, int k, int R, const int32_t* inv_perm,
                         uint8_t* xq, float* xs, float* out_acc, cudaStream_t stream);

// Expert-parallel dispatch: quantise x per token per 128 columns and write
// pair p = t*k + j's row to send slot slot_of_pair[p] (skipped when < 0):
// xq [S, H] codes, xs [S, H/128] fp32 (row-major), eid [S] = the pair's
// expert id modulo experts_per_rank (its index on the owning rank).
int launch_ep_pack(const void* x, const int32_t* ids, int T, int H, int k, int S,
                   const int32_t* slot_of_pair, int experts_per_rank, uint8_t* xq, float* xs,
                   int32_t* eid, cudaStream_t stream);

// owner[p] = ids[p] / experts_per_rank for ids in [0, E), else -1.
int launch_ep_owner(const int32_t* ids, long long R, int E, int experts_per_rank, int32_t* owner,
                    int num_sms, cudaStream_t stream);

// xq_g[r] = xq[src_of[r]] (rows of H bytes), xs_g[kb * n + r] =
// xs[src_of[r] * H/128 + kb], for r < rows and r < *rows_dev (when set; n =
// rows of the source and the column-block stride of xs_g).
int launch_gather_rows(const uint8_t* xq, const float* xs, int n, int H, const int32_t* src_of,
                       int rows, const int32_t* rows_dev, uint8_t* xq_g, float* xs_g,
                       cudaStream_t stream);

// MXFP8 variant: xq as above, xsf [H/128, R, 4] E8M0 codes (one per 32 columns).
int launch_mx_quant_scatter(const void* x, int T, int H, int k, int R, const int32_t* inv_perm,
                            uint8_t* xq, uint8_t* xsf, float* out_acc, cudaStream_t stream);

// Top-k weighted combine of per-pair rows: out[t, c] = bf16(sum_j
// fp32(topk_w[t, j] * y[inv_perm[t*k + j], c])) in ascending j (pairs with
// inv_perm < 0 skipped; inv_perm null = identity).  y [*, H] fp32, out [T, H]
// bf16, H % 8 == 0.
int launch_combine(const float* y, const int32_t* inv_perm, const float* topk_w, int T, int k,
                   int H, void* out, cudaStream_t stream);

// out [n] bf16 = in [n] fp32
int launch_f32_to_bf16(const float* in, void* out, long long n, int num_sms, cudaStream_t stream);

// Also clears the status word `status` (when set) from inside the kernel.
int launch_swiglu_mxfp8(const void* in, void* out, uint8_t* scale, int M, int K, int num_sms,
                        int* status, cudaStream_t stream);

// Grouped MXFP8 GEMM on the block-scaled tensor core path: E4M3 operands with
// one E8M0 scale per 32 K elements of every row of A and of B.
enum MxEpilogue : int {
    MX_EPI_BF16 = 0,            // plain bf16 G, or gated bf16 silu(gate) * up
    MX_EPI_SWIGLU_MXQUANT = 1,  // gated: h to MXFP8 (hq [R, N/2], hsf [N/256, R, 4])
    MX_EPI_COMBINE = 2,         // plain: out_acc[token, n] += topk_w * G (fp32 reduction)
};

struct MxGemmArgs {
    const void* a;            // [R, K] E4M3, grouped rows
    const void* b;            // [E, N, K] E4M3
    const uint8_t* a_sf;      // E8M0: [R, K/32] row-major (a_sf_mn = 0) or [K/128, R, 4] (1)
    int a_sf_mn;
    const uint8_t* b_sf;      // [E*N/128, K/128, 512] E8M0, tiled (launch_mx_tile_scales)
    const int32_t* m_indptr;  // [E+1]
    int R, N, K, E;
    int gated;                // out [R, N/2] = bf16(silu(G_gate) * G_up), else [R, N] = bf16(G)
    int epi;                  // MxEpilogue
    int tile_m;               // 32 (swapped) or 128; <= 0: by group size
    void* out;
    uint8_t* hq;
    uint8_t* hsf;
    const int32_t* perm;
    const float* topk_w;
    int topk;
    float* out_acc;
    int out_ld;
    int* status;
    uint64_t timeout_ns;
    int num_sms;
};
int launch_mx_gemm(const MxGemmArgs& g, cudaStream_t stream);

// Row-major E8M0 scales [rows, K/32] -> the tiled layout the MXFP8 GEMM reads
// for weights: [rows/128, K/128, 512], byte (r % 32) * 16 + ((r / 32) % 4) * 4 + j
// of atom (r / 128, kb) = scale j of row r in K block kb.  rows % 128 == 0.
int launch_mx_tile_scales(const uint8_t* rm, uint8_t* tiled, int rows, int K, int num_sms,
                          cudaStream_t stream);

// Grouped NVFP4 GEMM on the block-scaled tensor core path: E2M1 operands
// packed two per byte, one E4M3 scale per 16 K elements of every row of A and
// of B, G = alpha[e] * (block-scaled product).
enum NvEpilogue : int {
    NV_EPI_BF16 = 0,            // plain bf16 G, or gated bf16 silu(gate) * up
    NV_EPI_SWIGLU_NVQUANT = 1,  // gated: h to NVFP4 (hq [R, N/4] packed, hsf [N/128, R, 4])
    NV_EPI_COMBINE = 2,         // plain: out_acc[token, n] += topk_w * G (fp32 reduction)
};

struct NvGemmArgs {
    const void* a;            // [R, K/2] packed E2M1, grouped rows
    const void* b;            // [E, N, K/2] packed E2M1
    const uint8_t* a_sf;      // E4M3: [R, K/16] row-major (a_sf_mn = 0) or [K/64, R, 4] (1)
    int a_sf_mn;
    const uint8_t* b_sf;      // [E*N/128, K/64, 512] E4M3, tiled (launch_mx_tile_scales of 2K)
    const float* alpha;       // [E] 1 / (global scale of A * global scale of expert e)
    const int32_t* m_indptr;  // [E+1]
    int R, N, K, E;
    int gated;                // out [R, N/2] = bf16(silu(G_gate) * G_up), else [R, N] = bf16(G)
    int epi;                  // NvEpilogue
    void* out;
    uint8_t* hq;
    uint8_t* hsf;
    float h_gscale;           // NV_EPI_SWIGLU_NVQUANT: global scale of h
    const int32_t* perm;
    const float* topk_w;
    int topk;
    float* out_acc;
    int out_ld;
    int* status;
    uint64_t timeout_ns;
    int num_sms;
};
int launch_nvfp4_gemm(const NvGemmArgs& g, cudaStream_t stream);

// NVFP4 variant of launch_quant_scatter: xq [R, H/2] packed E2M1 codes and
// E4M3 scales with global scale g, at rows inv_perm[t*k + j] (row t when
// inv_perm is null and k = 1); xsf [R, H/16] row-major, or [H/64, R, 4] when
// sf_mn.
int launch_nv_quant_scatter(const void* x, int T, int H, int k, float g, const int32_t* inv_perm,
                            uint8_t* xq, uint8_t* xsf, int R, int sf_mn, float* out_acc,
                            cudaStream_t stream);

// Row-major E4M3 scales [R, K/16] -> K-block-major [K/64, R, 4] (4-byte
// aligned buffers; (R, K/64) up to (2^21, any)).
int launch_nv_sf_kblock_major(const uint8_t* rm, uint8_t* mn, int R, int K, cudaStream_t stream);

}  // namespace moe
