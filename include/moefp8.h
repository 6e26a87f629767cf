/*
 * moefp8.h - C ABI of the sm_100a (B200) fused W8A8 block-scaled MoE library.
 *
 * The operation is the Mixture-of-Experts expert computation described on
 * the page "FlashInfer: Blackwell W8A8 AlphaMoE Expert 계산 커널 퓨전으로 성능
 * 비약적 향상" (flashinfer PR #4287), section "문제점: MoE Expert 계산의 병목":
 *   (1) GEMM1 gate/up projection, (2) SwiGLU, (3) FP8 requantisation of the
 *   intermediate, (4) GEMM2 down projection, (5) combine,
 * preceded by grouping the (token, slot) pairs by expert.  The grouped GEMM
 * interface (m_indptr, per-block fp32 scales with explicit granularities,
 * scale_major_mode, is_gated, tactic tile sizes with -1 = automatic) follows
 * the page "FlashInfer SM120 MoE GEMM 최적화: 웨이브+잔여물 비용 모델 도입"
 * (flashinfer PR #4318), "코드 분석 1." and "2.".
 *
 * Conventions for every entry point:
 *  - Pointers named as device buffers are device pointers owned by the
 *    caller; the library never allocates, frees or keeps them.  Buffers must
 *    be 16-byte aligned; row pitches are the dense row lengths given.
 *  - Every call is asynchronous on `stream` (NULL = legacy default stream)
 *    and returns a moe_status_t that reflects host-side validation and
 *    launch errors only.  Errors detected on the device (a bounded wait that
 *    ran out, an expert id outside [0,E)) are written to a status word and
 *    read back with moe_get_device_status().
 *  - FP8 means OCP E4M3 "FN" (bias 7, max 448, no infinities), one byte per
 *    value.  bf16 is passed as 2-byte words.  Matrices are row-major.
 *  - Block scales are fp32.  Activation scales cover 1 row x 128 columns;
 *    weight scales cover 128 rows x 128 columns.  H, I, K and N must be
 *    multiples of 128.
 *  - Device requirement: compute capability 10.0 (sm_100a).
 */
#ifndef MOEFP8_H
#define MOEFP8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* moe_stream_t;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,     /* null pointer, bad size, misaligned pointer, k > E */
    MOE_ERR_UNSUPPORTED = 2,     /* granularity other than (1,128,128), device not sm_100, size limits */
    MOE_ERR_CUDA = 3,            /* a CUDA runtime call or launch failed */
    MOE_ERR_NO_TILE_CONFIG = 4,  /* requested tile sizes not in the kernel menu (mirrors the
                                    explicit error when shape filtering leaves no candidate,
                                    cuTile backend page, flashinfer PR #4646, review section) */
    MOE_ERR_DEVICE_TIMEOUT = 5,  /* device: a bounded pipeline wait ran out; outputs undefined */
    MOE_ERR_BAD_EXPERT_ID = 6    /* device: a topk id outside [0, E); that pair was dropped */
} moe_status_t;

/* Maximum number of experts. */
#define MOE_MAX_EXPERTS 1024
#define MOE_ROUTER_MAX_K 32

/* Human-readable name of a status code (static string). */
MOE_API const char* moe_status_string(int status);

/* ------------------------------------------------------------------ */
/* Routing and permutation (stage before GEMM1)                         */
/* ------------------------------------------------------------------ */

/* Workspace bytes moe_route_permute needs for T tokens, top-k, E experts. */
MOE_API size_t moe_route_workspace_size(int T, int k, int E);

/* Groups the R = T*k (token, slot) pairs by expert with a stable counting
 * sort (pair id p = t*k + j, ascending inside each expert).
 *  topk_ids  device int32 [T, k]  expert of each pair
 *  m_indptr  device int32 [E+1]   out: exclusive prefix of per-expert counts
 *  perm      device int32 [R]     out: grouped row -> pair id
 *  inv_perm  device int32 [R]     out: pair id -> grouped row (-1 if dropped);
 *                                  may be NULL
 *  ws        device, >= moe_route_workspace_size(T, k, E) bytes; its first
 *            bytes hold the device status word
 * Ids outside [0, E) are dropped and reported as MOE_ERR_BAD_EXPERT_ID by
 * moe_get_device_status(ws); m_indptr[E] then counts only valid pairs.
 * Returns MOE_ERR_INVALID_ARG for T < 0, k < 1, E < 1, E > MOE_MAX_EXPERTS,
 * null pointers or a workspace that is too small. */
MOE_API int moe_route_permute(const int32_t* topk_ids, int T, int k, int E,
                      int32_t* m_indptr, int32_t* perm, int32_t* inv_perm,
                      void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_route_permute for callers that cannot allocate device memory or
 * hand the library a workspace (for example code running inside a host
 * runtime that owns every device allocation through a fixed memory plan).
 * The method's pages have no counterpart of this entry point.
 * Same arguments and results as moe_route_permute without ws/ws_bytes; the
 * scratch lives in one device array inside the library (about 256 KB per
 * GPU, held until the process exits).  Limits: T*k <= 65536 pairs and
 * E <= MOE_MAX_EXPERTS, else MOE_ERR_INVALID_ARG.  All calls share that
 * array: calls whose kernels overlap on the GPU race and give undefined
 * results.  The first call on a device, and the first after a
 * cudaDeviceReset of it, looks up the array's address in that device's
 * context; make that call before any stream capture.  Ids outside [0, E) are
 * dropped (m_indptr[E] then counts only valid pairs) and not reported
 * through moe_get_device_status.  Allocates nothing. */
MOE_API int moe_route_permute_noalloc(const int32_t* topk_ids, int T, int k, int E,
                                      int32_t* m_indptr, int32_t* perm, int32_t* inv_perm,
                                      moe_stream_t stream);

/* Router: the step before the expert computation (the AlphaMoE page's
 * five-stage pipeline, section "문제점: MoE Expert 계산의 병목", starts from
 * each token's experts and weights; the pages do not define the router, so
 * this is the plainest reading): for each token the k largest logits in
 * descending order, ties to the lower expert index, and their softmax in
 * fp32 with the largest subtracted (expf per slot, slots summed in order,
 * w_j = e_j / sum).  Its outputs feed moe_route_permute / moe_fp8_fused.
 *  logits    device fp32 [T, E] (finite)
 *  topk_ids  device int32 [T, k] out;  topk_w device fp32 [T, k] out
 * 1 <= k <= min(E, MOE_ROUTER_MAX_K); E <= MOE_MAX_EXPERTS; T = 0 is a
 * no-op.  Caller owns all memory; asynchronous on `stream`; argument errors
 * are returned before any launch. */
MOE_API int moe_router_topk(const float* logits, int T, int E, int k, int32_t* topk_ids,
                            float* topk_w, moe_stream_t stream);

/* moe_router_topk and moe_route_permute in one call: from the router
 * logits to the expert grouping, with the same outputs as the two calls
 * (topk_ids [T, k], topk_w [T, k], m_indptr [E+1], perm [T*k], inv_perm
 * [T*k] or NULL, all device buffers owned by the caller) and ws of at least
 * moe_route_workspace_size(T, k, E) bytes.  Up to 8192 pairs (T*k) it is a
 * single kernel launch: one CTA selects every token's experts and then
 * groups the pairs it wrote; above that, the router kernel and then the
 * routing kernels.  Same argument rules as moe_router_topk. */
MOE_API int moe_router_route(const float* logits, int T, int E, int k, int32_t* topk_ids,
                             float* topk_w, int32_t* m_indptr, int32_t* perm, int32_t* inv_perm,
                             void* ws, size_t ws_bytes, moe_stream_t stream);

/* ------------------------------------------------------------------ */
/* The fused layer                                                      */
/* ------------------------------------------------------------------ */

/* Workspace bytes moe_fp8_fused needs (routing tables, quantised
 * activations, FP8 intermediate, the fp32 down-projection rows of every
 * (token, slot) pair [T*k, H], status word). */
MOE_API size_t moe_workspace_size(int T, int H, int I, int E, int k);

/* out[t, :] = bf16( sum_j topk_w[t,j] * Down_e( requant( SwiGLU( GateUp_e(
 *             quant(x[t, :]) ) ) ) ) ),  e = topk_ids[t, j].
 *  x          device bf16 [T, H]
 *  topk_ids   device int32 [T, k], distinct experts per token expected
 *  topk_w     device fp32  [T, k]
 *  w13        device FP8  [E, 2I, H]   rows [0,I) gate, rows [I,2I) up
 *  w13_scale  device fp32 [E, 2I/128, H/128]
 *  w2         device FP8  [E, H, I]
 *  w2_scale   device fp32 [E, H/128, I/128]
 *  out        device bf16 [T, H]
 *  ws         device, >= moe_workspace_size(T, H, I, E, k) bytes
 * Activations are quantised per token per 128 columns (scale = amax/448,
 * round-to-nearest-even, saturating); the intermediate is requantised the
 * same way per row per 128 columns; the router weight is applied after the
 * down projection: each pair's fp32 down-projection row is written once and
 * the combine sums a token's k weighted rows in ascending slot order (fp32,
 * each product rounded, then bf16), so the output does not depend on the
 * order in which the GEMM's tiles run.  The two expert GEMMs run as two
 * grouped-GEMM launches, or as one fused-expert launch that keeps each token
 * group's FP8 intermediate in shared memory (moe_fp8_fused_plan tells which;
 * moe_set_expert_fusion chooses); both give the same intermediate and
 * output.  T = 0 is a no-op.  Returns MOE_ERR_INVALID_ARG for
 * sizes that are not multiples of 128, k > E, null pointers, misaligned
 * pointers or a small workspace; MOE_ERR_UNSUPPORTED for E > 1024. */
MOE_API int moe_fp8_fused(const void* x, const int32_t* topk_ids, const float* topk_w,
                  const void* w13, const float* w13_scale,
                  const void* w2, const float* w2_scale,
                  void* out, int T, int H, int I, int E, int k,
                  void* ws, size_t ws_bytes, moe_stream_t stream);

/* Same as moe_fp8_fused, and also copies the routing tables and the FP8
 * intermediate out of the workspace (all device buffers, grouped-row order):
 *  m_indptr [E+1], perm [T*k], h_fp8 [T*k, I] codes, h_scale fp32
 *  [I/128, T*k] (column-block major).  Any of the four may be NULL. */
MOE_API int moe_fp8_fused_debug(const void* x, const int32_t* topk_ids, const float* topk_w,
                        const void* w13, const float* w13_scale,
                        const void* w2, const float* w2_scale,
                        void* out, int T, int H, int I, int E, int k,
                        void* ws, size_t ws_bytes, moe_stream_t stream,
                        int32_t* m_indptr, int32_t* perm, uint8_t* h_fp8, float* h_scale);

/* ------------------------------------------------------------------ */
/* Standalone grouped FP8 GEMM ("nt": both operands K-major)            */
/* ------------------------------------------------------------------ */

/* For every expert e and grouped row r in [m_indptr[e], m_indptr[e+1]):
 *   G[r, n] = sum_kb a_scale(r,kb) * b_scale[e, n/128, kb] * sum_{k in kb} a[r,k] * b[e,n,k]
 *   plain  (is_gated = 0): out[r, n] = bf16(G[r, n]),            out [R, N]
 *   gated  (is_gated = 1): out[r, i] = bf16(silu(G[r,i]) * G[r, N/2+i]), out [R, N/2]
 *  a        device FP8 [R, K]
 *  b        device FP8 [E, N, K]
 *  a_scale  device fp32; scale_major_mode 0: [R, K/128] (K-major),
 *           1: [K/128, R] (MN-major)
 *  b_scale  device fp32 [E, N/128, K/128]
 *  m_indptr device int32 [E+1], m_indptr[0] = 0, non-decreasing, m_indptr[E] <= R
 *  sg_m, sg_n, sg_k  scale granularities; only (1, 128, 128) is supported
 *  tile_m   -1 = automatic (wave+residue model), else one of 16, 32, 64, 128
 *  tile_n   -1 = automatic, else 128 (gated) / 256 (plain): output columns per tile
 * Rows of out outside [0, m_indptr[E]) are not written.  Gated needs an
 * even N with N/2 a multiple of 128.  Device-side errors go to the
 * library's own status word: read it with moe_get_device_status(NULL, ...). */
MOE_API int fp8_groupwise_moe_gemm(const void* a, const void* b,
                           const float* a_scale, const float* b_scale,
                           const int32_t* m_indptr, void* out,
                           int R, int N, int K, int E, int scale_major_mode,
                           int sg_m, int sg_n, int sg_k, int is_gated,
                           int tile_m, int tile_n, moe_stream_t stream);

/* Host-only tile selection used when tile_m = -1 (no device access).
 * total_rows = rows over all experts, n = weight rows per expert (2I when
 * gated), k = reduction size.  Writes tile_m (16, 32, 64 or 128) and tile_n
 * (output columns per tile).  Follows the wave+residue description of the
 * page "FlashInfer SM120 MoE GEMM 최적화: 웨이브+잔여물 비용 모델 도입", "코드
 * 분석 2." and "리뷰 피드백 반영", on the sm_100a tile menu. */
MOE_API int moe_select_tile_m(int total_rows, int n, int k, int E, int num_sms, int is_gated,
                      int* tile_m, int* tile_n);

/* ------------------------------------------------------------------ */
/* Tactic table (measured tile choice)                                  */
/* ------------------------------------------------------------------ */

/* The staged GEMM-pair autotuning of the cuTile page ("2. cuTile NVFP4 양자화
 * 지원": each GEMM of the pair tuned per architecture and shape): a
 * process-wide table maps a GEMM shape class to the token tile (tile_m) that
 * ran fastest on this GPU.  Class = (N, K, E, is_gated, bucket of ceil(R/E)),
 * the bucket being the power of two at or above the balanced rows per expert
 * (8 or fewer share one bucket).  fp8_groupwise_moe_gemm with tile_m = -1 and
 * both GEMMs of moe_fp8_fused use the class's entry when it exists, else the
 * wave + residue model of moe_select_tile_m.
 *
 * moe_tactic_tune_gemm: runs fp8_groupwise_moe_gemm on the caller's buffers
 * (arguments as there; `out` is overwritten) once per tile_m valid for K
 * (16, 32, 64, 128), one warm-up call and `iters` timed calls each (CUDA
 * events on `stream`; synchronises it), stores the fastest in the table and
 * writes it to *tile_m.  Errors of the GEMM are returned unchanged; nothing
 * is stored then.
 * moe_tactic_lookup: host only; MOE_OK and *tile_m for a stored class, else
 * MOE_ERR_NO_TILE_CONFIG.
 * moe_tactic_store: host only; sets a class's entry (e.g. restored from a
 * file); MOE_ERR_NO_TILE_CONFIG for a tile_m that is not 16/32/64/128 or that
 * cannot hold K.
 * moe_tactic_clear: host only; empties the table. */
MOE_API int moe_tactic_tune_gemm(const void* a, const void* b, const float* a_scale,
                                 const float* b_scale, const int32_t* m_indptr, void* out, int R,
                                 int N, int K, int E, int scale_major_mode, int is_gated, int iters,
                                 moe_stream_t stream, int* tile_m);
MOE_API int moe_tactic_lookup(int R, int N, int K, int E, int is_gated, int* tile_m);
MOE_API int moe_tactic_store(int R, int N, int K, int E, int is_gated, int tile_m);
MOE_API void moe_tactic_clear(void);

/* ------------------------------------------------------------------ */
/* Grouped MXFP8 GEMM (block-scaled tensor core path)                   */
/* ------------------------------------------------------------------ */

/* The MXFP8 grouped MoE GEMM that the page "FlashInfer SM120 MoE GEMM 최적화:
 * 웨이브+잔여물 비용 모델 도입" names beside FP8 (section "들어가며"; "mxfp8
 * grouped MoE" in "왜 이게 좋은가?"): E4M3 operands with one E8M0 scale per 32
 * consecutive K elements of every row of A and of B, in the grouped layout of
 * fp8_groupwise_moe_gemm:
 *   G[r, n] = sum over 32-wide K blocks b of
 *             2^(a_sf[r,b]-127) * 2^(b_sf[e,n,b]-127) * sum_k a[r,k] * b[e,n,k],
 *   e = the expert with m_indptr[e] <= r < m_indptr[e+1];
 * accumulated in fp32 by the tensor core (the scales are applied inside it).
 *  a       device FP8  [R, K] grouped rows
 *  b       device FP8  [E, N, K]
 *  a_sf    device uint8 E8M0 codes of the activations (4-byte aligned):
 *          a_sf_major = 0: [R, K/32] row-major; 1: [K/128, R, 4], the four
 *          scales of a 128-wide K block of each row together, rows
 *          consecutive (the rows of a tile are then read contiguously)
 *  b_sf    device uint8 E8M0 codes of the weights in the tiled layout that
 *          mxfp8_tile_scales produces from [E, N, K/32] row-major
 *          (16-byte aligned; weights are tiled once, not per call)
 *  m_indptr device int32 [E+1]
 *  out     device bf16: plain [R, N] = bf16(G); gated [R, N/2] =
 *          bf16(silu(G[:, :N/2]) * G[:, N/2:]) (gate rows then up rows of b)
 * Rows outside [m_indptr[0], m_indptr[E]) are not written.  K and N must be
 * multiples of 128 (gated: N/2 too); a, b, out 16-byte aligned.  Returns
 * MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED on bad arguments before any
 * launch; device timeouts are read with moe_get_device_status(NULL, stream).
 * Caller owns all memory; asynchronous on `stream`. */
MOE_API int mxfp8_moe_gemm(const void* a, const void* b, const uint8_t* a_sf,
                           const uint8_t* b_sf, const int32_t* m_indptr, void* out,
                           int R, int N, int K, int E, int a_sf_major, int is_gated,
                           moe_stream_t stream);

/* The fused layer of moe_fp8_fused in the MXFP8 variant: every FP8 operand
 * carries one E8M0 scale per 32 K elements (the Wave page's MXFP8 grouped
 * MoE GEMM format; the intermediate is requantised with the SwiGLU + MXFP8
 * rule of the page "NVIDIA R200(SM107)을 위한 SwiGLU + MXFP8 커널 최적화").
 * Stages: routing, x quantised per token per 32 columns and scattered into
 * the k grouped rows, GEMM1 gate/up (block-scaled tensor cores) with
 * SwiGLU and MXFP8 requantisation in its epilogue, GEMM2 down with the
 * top-k weighted fp32 combine in its epilogue, bf16 output.
 *  w13     device FP8 [E, 2I, H] (gate rows then up rows)
 *  w13_sf  device uint8: E8M0 scales of w13 ([E*2I, H/32] row-major)
 *          tiled by mxfp8_tile_scales (16-byte aligned)
 *  w2      device FP8 [E, H, I];  w2_sf: [E*H, I/32] tiled the same way
 *  x, topk_ids, topk_w, out, T, H, I, E, k, ws, ws_bytes, stream: as for
 *  moe_fp8_fused; the workspace size is moe_workspace_size(T, H, I, E, k).
 * Errors as for moe_fp8_fused. */
MOE_API int moe_mxfp8_fused(const void* x, const int32_t* topk_ids, const float* topk_w,
                            const void* w13, const uint8_t* w13_sf, const void* w2,
                            const uint8_t* w2_sf, void* out, int T, int H, int I, int E, int k,
                            void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_mxfp8_fused plus copies of m_indptr [E+1], perm [T*k], the FP8
 * intermediate h_fp8 [T*k, I] and its E8M0 scales h_sf [I/128, T*k, 4]
 * (any may be NULL). */
MOE_API int moe_mxfp8_fused_debug(const void* x, const int32_t* topk_ids, const float* topk_w,
                                  const void* w13, const uint8_t* w13_sf, const void* w2,
                                  const uint8_t* w2_sf, void* out, int T, int H, int I, int E,
                                  int k, void* ws, size_t ws_bytes, moe_stream_t stream,
                                  int32_t* m_indptr, int32_t* perm, uint8_t* h_fp8,
                                  uint8_t* h_sf);

/* Rearranges row-major E8M0 scales [rows, K/32] into the tiled layout that
 * mxfp8_moe_gemm reads for the weights: [rows/128, K/128, 512] bytes, where
 * byte (r % 32) * 16 + ((r / 32) % 4) * 4 + j of block (r / 128, kb) holds
 * scale j (of the four 32-wide steps) of row r in K block kb -- 128 rows x
 * 4 scales in the order the tensor core's scale-factor copy reads them.
 * No counterpart on the pages: it is the storage format of this library's
 * block-scaled GEMM.  rows and K must be multiples of 128; pointers 4-byte
 * aligned (16 for use by mxfp8_moe_gemm); asynchronous on `stream`. */
MOE_API int mxfp8_tile_scales(const uint8_t* sf_rowmajor, uint8_t* sf_tiled, int rows, int K,
                              moe_stream_t stream);

/* ------------------------------------------------------------------ */
/* Grouped NVFP4 GEMM (block-scaled tensor core path)                   */
/* ------------------------------------------------------------------ */

/* The NVFP4 (W4A4) expert GEMM of the page "FlashInfer에 cuTile 기반 Fused
 * MoE 백엔드 도입" (section "2. cuTile NVFP4 양자화 지원": fp4_quantize with a
 * per-expert global scale, sf_vec_size=16), in the grouped layout of
 * fp8_groupwise_moe_gemm.  E2M1 values (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6)
 * with one E4M3 scale per 16 consecutive K elements of every row and a global
 * scale per tensor; a real value is e2m1(q) * e4m3(s) / g:
 *   G[r, n] = alpha[e] * sum over 16-wide K blocks b of
 *             e4m3(a_sf[r,b]) * e4m3(b_sf[e,n,b]) * sum_k e2m1(a[r,k]) * e2m1(b[e,n,k]),
 *   alpha[e] = 1 / (g_a * g_b[e]),  e = the expert with m_indptr[e] <= r < m_indptr[e+1];
 * the block scales are applied inside the tensor core, fp32 accumulation.
 *  a       device uint8 [R, K/2]: E2M1 codes packed two per byte, element
 *          2i in the low nibble (sign bit 3 of each nibble)
 *  b       device uint8 [E, N, K/2], packed the same way
 *  a_sf    device uint8 E4M3 codes of the activations (4-byte aligned):
 *          a_sf_major = 0: [R, K/16] row-major; 1: [K/64, R, 4], the four
 *          scales of a 64-wide K block of each row together, rows
 *          consecutive (the rows of a tile are then read contiguously)
 *  b_sf    device uint8 E4M3 codes of the weights in the tiled layout that
 *          nvfp4_tile_scales produces from [E, N, K/16] row-major (16-byte
 *          aligned; weights are tiled once, not per call)
 *  alpha   device fp32 [E]
 *  m_indptr device int32 [E+1]
 *  out     device bf16: plain [R, N] = bf16(G); gated [R, N/2] =
 *          bf16(silu(G[:, :N/2]) * G[:, N/2:]) (gate rows then up rows of b)
 * Rows outside [m_indptr[0], m_indptr[E]) are not written.  K must be a
 * multiple of 256, N of 128 (gated: N/2 too); a, b, out 16-byte aligned.
 * Errors and ownership as for mxfp8_moe_gemm. */
MOE_API int nvfp4_moe_gemm(const void* a, const void* b, const uint8_t* a_sf,
                           const uint8_t* b_sf, const float* alpha, const int32_t* m_indptr,
                           void* out, int R, int N, int K, int E, int a_sf_major, int is_gated,
                           moe_stream_t stream);

/* The fused layer of moe_fp8_fused in the NVFP4 (W4A4) variant of the cuTile
 * page ("2. cuTile NVFP4 양자화 지원"): activations and weights in NVFP4 (E2M1,
 * an E4M3 scale per 16 elements, a global scale per tensor).  Stages: routing,
 * x quantised per token per 16 columns with the global scale a1_gscale and
 * scattered into the k grouped rows, GEMM1 gate/up on the block-scaled tensor
 * cores with SwiGLU (fp32) and NVFP4 requantisation of the intermediate
 * (global scale a2_gscale) in its epilogue, GEMM2 down with the top-k
 * weighted fp32 combine in its epilogue, bf16 output.
 *  w13       device uint8 [E, 2I, H/2] packed E2M1 (gate rows then up rows)
 *  w13_sf    device uint8 E4M3 scales of w13 ([E*2I, H/16] row-major) tiled
 *            by nvfp4_tile_scales (16-byte aligned)
 *  w13_alpha device fp32 [E] = 1 / (a1_gscale * global scale of w13[e])
 *  w2, w2_sf, w2_alpha: the same for the down weights [E, H, I/2], with
 *            w2_alpha[e] = 1 / (a2_gscale * global scale of w2[e])
 *  a1_gscale, a2_gscale  host fp32 > 0: global scales of x and of the
 *            intermediate (calibrated; values beyond 6 * 448 / g saturate)
 *  x, topk_ids, topk_w, out, T, E, k, ws, ws_bytes, stream: as for
 *  moe_fp8_fused; the workspace size is moe_workspace_size(T, H, I, E, k).
 * H and I must be multiples of 256.  Errors as for moe_fp8_fused. */
MOE_API int moe_nvfp4_fused(const void* x, const int32_t* topk_ids, const float* topk_w,
                            const void* w13, const uint8_t* w13_sf, const float* w13_alpha,
                            const void* w2, const uint8_t* w2_sf, const float* w2_alpha,
                            float a1_gscale, float a2_gscale, void* out, int T, int H, int I,
                            int E, int k, void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_nvfp4_fused plus copies of m_indptr [E+1], perm [T*k], the packed
 * NVFP4 intermediate h_fp4 [T*k, I/2] and its E4M3 scales h_sf
 * [I/64, T*k, 4] (K-block-major, as GEMM2 reads them; any may be NULL). */
MOE_API int moe_nvfp4_fused_debug(const void* x, const int32_t* topk_ids, const float* topk_w,
                                  const void* w13, const uint8_t* w13_sf, const float* w13_alpha,
                                  const void* w2, const uint8_t* w2_sf, const float* w2_alpha,
                                  float a1_gscale, float a2_gscale, void* out, int T, int H, int I,
                                  int E, int k, void* ws, size_t ws_bytes, moe_stream_t stream,
                                  int32_t* m_indptr, int32_t* perm, uint8_t* h_fp4,
                                  uint8_t* h_sf);

/* NVFP4 quantisation of bf16 rows, as the cuTile page's fp4_quantize(x,
 * global_scale, sf_vec_size=16, is_sf_swizzled_layout=False): per 16
 * consecutive values of a row, scale code c = E4M3_RNE_sat(amax * g / 6) and
 * codes E2M1_RNE_sat(v * g / e4m3(c)) (0 where the scale decodes to 0), each
 * step rounded in fp32 in that order.
 *  x   device bf16 [M, K]
 *  q   device uint8 [M, K/2] packed codes (element 2i in the low nibble)
 *  sf  device uint8 [M, K/16] E4M3 scale codes, row-major
 * K must be a multiple of 128, gscale > 0; x 16-byte aligned, q 8-byte
 * aligned.  Asynchronous on `stream`. */
MOE_API int nvfp4_quantize(const void* x, float gscale, uint8_t* q, uint8_t* sf, int M, int K,
                           moe_stream_t stream);

/* Rearranges row-major E4M3 block scales [rows, K/16] into the tiled layout
 * that nvfp4_moe_gemm reads for the weights: [rows/128, K/64, 512] bytes,
 * where byte (r % 32) * 16 + ((r / 32) % 4) * 4 + j of block (r / 128, kb)
 * holds scale j (of the four 16-wide blocks) of row r in K block kb -- the
 * scales one K = 64 tensor core step reads.  No counterpart on the pages: it
 * is this library's storage format.  rows a multiple of 128, K of 64;
 * pointers 4-byte aligned (16 for use by nvfp4_moe_gemm); asynchronous on
 * `stream`. */
MOE_API int nvfp4_tile_scales(const uint8_t* sf_rowmajor, uint8_t* sf_tiled, int rows, int K,
                              moe_stream_t stream);

/* ------------------------------------------------------------------ */
/* Standalone SwiGLU + MXFP8 quantisation                               */
/* ------------------------------------------------------------------ */

/* Page "NVIDIA R200(SM107)을 위한 SwiGLU + MXFP8 커널 최적화" (flashinfer
 * PR #8023): v = silu(gate) * up in fp32, then per 32 consecutive outputs an
 * E8M0 scale X = 2^s with s the smallest integer such that amax <= 448*2^s
 * (code s+127 clamped to [0,254]; an all-zero block gets code 0) and
 * codes RNE_sat(v / X).  Launch shape is chosen by size band: M*K < 2^20
 * uses small 256-thread CTAs, larger sizes a grid-stride streaming launch.
 *  in     device bf16 [M, 2K]: columns [0,K) gate, [K,2K) up
 *  out    device FP8  [M, K]
 *  scale  device uint8 [M, K/32] row-major E8M0 codes (not swizzled)
 * K must be a multiple of 32; M = 0 is a no-op. */
MOE_API int swiglu_mxfp8_quant(const void* in, void* out, uint8_t* scale, int M, int K,
                       moe_stream_t stream);

/* ------------------------------------------------------------------ */
/* Expert parallelism: the layer with its experts split over G GPUs      */
/* ------------------------------------------------------------------ */
/* The AlphaMoE page's five stages ("문제점: MoE Expert 계산의 병목") with rank g
 * of G owning experts [g*E/G, (g+1)*E/G) and keeping its own tokens.  The
 * pages do not describe expert parallelism; this follows the plainest
 * reading: every (token, slot) pair's quantised activation row travels to
 * the rank that owns its expert, that rank runs the expert FFN on the rows
 * it received, and the fp32 rows travel back for the combine (the
 * AG-matmul page, "1. 커널 최적화" and "왜 이게 좋은가", pairs the tensor cores
 * with NVLink transfers; its "2. API 개선" binds the group and buffers once).
 * The all-to-all exchanges between the steps are the caller's (for example
 * NCCL through torch.distributed); each step below is asynchronous on
 * `stream`.  The output equals the single-GPU moe_fp8_fused output up to the
 * GEMMs' accumulation order (each row is computed by the same kernels; the
 * combine order is the same). */

/* Workspace bytes of moe_ep_plan. */
MOE_API size_t moe_ep_workspace_size(int T, int k, int G);

/* Step 1, on every rank: where each of this rank's T*k pairs goes.
 *  topk_ids      device int32 [T, k], ids in [0, E); others are dropped and
 *                reported as MOE_ERR_BAD_EXPERT_ID through
 *                moe_get_device_status(ws)
 *  send_indptr   device int32 [G+1] out: pairs for rank g occupy send slots
 *                [send_indptr[g], send_indptr[g+1]); send_indptr[G] = S, the
 *                number of valid pairs
 *  send_pair     device int32 [T*k] out: send slot -> pair id t*k + j,
 *                ascending pair id within each rank's range
 *  slot_of_pair  device int32 [T*k] out: pair id -> send slot, -1 if dropped
 * Requires E % G == 0, E and G <= MOE_MAX_EXPERTS (else
 * MOE_ERR_INVALID_ARG).  Caller owns all memory. */
MOE_API int moe_ep_plan(const int32_t* topk_ids, int T, int k, int E, int G,
                        int32_t* send_indptr, int32_t* send_pair, int32_t* slot_of_pair,
                        void* ws, size_t ws_bytes, moe_stream_t stream);

/* Step 2, on every rank: quantise x per token per 128 columns (scale =
 * amax/448, round-to-nearest-even, as moe_fp8_fused) and write each pair's
 * row into its send slot s = slot_of_pair[p]:
 *  xq_send   device FP8 [S, H]; xs_send device fp32 [S, H/128] (row-major);
 *  eid_send  device int32 [S]: the pair's expert id minus the first expert
 *            of its owning rank (its local id there).
 * S = send_indptr[G] from step 1 (read back by the caller to size the
 * exchange).  H % 128 == 0, E % G == 0. */
MOE_API int moe_ep_pack(const void* x, const int32_t* topk_ids, const int32_t* slot_of_pair,
                        int T, int H, int k, int E, int G, int S, uint8_t* xq_send,
                        float* xs_send, int32_t* eid_send, moe_stream_t stream);

/* Workspace bytes of moe_fp8_expert_rows. */
MOE_API size_t moe_fp8_expert_rows_workspace_size(int n, int H, int I, int E);

/* Step 3, on the owning rank, after the exchange: the expert FFN on n
 * received rows in any order,
 *   y[i, :] = Down_e( requant( SwiGLU( GateUp_e( xq[i, :] * xs[i] ) ) ) ),
 * e = eid[i] in [0, E) (E = the rank's own experts; w13/w2 and their
 * scales are those E experts, laid out as for moe_fp8_fused).
 *  xq device FP8 [n, H], xs device fp32 [n, H/128], eid device int32 [n],
 *  y  device fp32 [n, H] out, row i for received row i.
 * Rows are grouped by expert on the device (stable), then run through the
 * same GEMM1 (SwiGLU + FP8 requant epilogue) and GEMM2 as moe_fp8_fused.
 * Rows with an eid outside [0, E) are not written; moe_get_device_status(ws)
 * then reports MOE_ERR_BAD_EXPERT_ID. */
MOE_API int moe_fp8_expert_rows(const uint8_t* xq, const float* xs, const int32_t* eid, int n,
                                const void* w13, const float* w13_scale, const void* w2,
                                const float* w2_scale, float* y, int H, int I, int E,
                                void* ws, size_t ws_bytes, moe_stream_t stream);

/* Step 4, on every rank, after the return exchange (and the last stage of
 * moe_fp8_fused on its own): out[t, :] = bf16( sum_j fp32( topk_w[t, j] *
 * y[row_of_pair[t*k + j], :] ) ), products rounded on their own and added in
 * ascending j; pairs with row_of_pair < 0 are skipped; row_of_pair = NULL
 * means row t*k + j.  y device fp32 [*, H], out device bf16 [T, H], H % 8 == 0. */
MOE_API int moe_combine(const float* y, const int32_t* row_of_pair, const float* topk_w, int T,
                        int k, int H, void* out, moe_stream_t stream);

/* ------------------------------------------------------------------ */
/* Device status                                                        */
/* ------------------------------------------------------------------ */

/* Synchronises `stream`, then returns the device status word written by the
 * last calls that used `ws` (a moe_fp8_fused / moe_route_permute workspace),
 * or, with ws = NULL, the library's own word used by fp8_groupwise_moe_gemm
 * and swiglu_mxfp8_quant.  Each entry point clears its word when it starts.
 * Returns MOE_OK, MOE_ERR_DEVICE_TIMEOUT, MOE_ERR_BAD_EXPERT_ID or
 * MOE_ERR_CUDA (the synchronise or the read failed). */
MOE_API int moe_get_device_status(const void* ws, moe_stream_t stream);

/* Stage timing for profiling.  When `events` is non-NULL, moe_fp8_fused and
 * moe_fp8_fused_debug record events[i] (cudaEvent_t handles created by the
 * caller) on the call's stream: 0 before routing, 1 after routing, 2 after
 * activation quantisation, 3 after GEMM1 (gate/up + SwiGLU + requant), 4
 * after GEMM2 (down projection), 5 after the combine and bf16 output.  n must be 6;
 * a NULL entry is not recorded (at least one must be set: each record costs
 * 2-3 µs of GPU time, so a caller timing one stage passes only its two);
 * events = NULL switches it off.  Process-wide setting. */
MOE_API int moe_set_stage_events(void* const* events, int n);

/* How moe_fp8_fused and moe_fp8_fused_debug run the two expert GEMMs.
 *   MOE_FUSION_AUTO (default): one fused-expert launch when the FP8
 *     intermediate of a 64-token group (I bytes per token) fits in shared
 *     memory beside the weight pipeline, the groups are small (the tile
 *     model picks weight-stationary GEMM1 tiles), and either the layer is
 *     tiny (at most 16 MB of touched weights: one launch fewer) or, for a
 *     balanced routing, the active experts make about one round over the
 *     SMs and fill at least half of them, their 64-token groups at most
 *     about two rounds, and an expert holds at most 6 MB of weights (3·H·I
 *     bytes); otherwise GEMM1 and GEMM2 as two launches.
 *   MOE_FUSION_ON: the fused launch whenever the intermediate fits.
 *   MOE_FUSION_OFF: always two launches.
 * The fused launch keeps each group's intermediate on chip: it is written
 * to the workspace only for moe_fp8_fused_debug's outputs.  Both paths give
 * the same quantised intermediate and sum each K block's partial products
 * in the same order.  With fusion, stage event 3 and 4 are recorded
 * back to back after the fused launch.  Process-wide; returns
 * MOE_ERR_INVALID_ARG for an unknown mode. */
/* The launch plan moe_fp8_fused would use on the calling thread's current
 * device for these sizes and the current fusion mode: the GEMM1 and GEMM2
 * token tiles (16, 32, 64: weight-stationary; 128: token-stationary) and
 * whether both GEMMs run as one fused-expert launch (*fused = 1).  Any
 * output pointer may be NULL.  Returns MOE_ERR_INVALID_ARG for sizes
 * moe_fp8_fused rejects, MOE_ERR_UNSUPPORTED off sm_100. */
MOE_API int moe_fp8_fused_plan(int T, int H, int I, int E, int k, int* tile_m1, int* tile_m2,
                               int* fused);

#define MOE_FUSION_AUTO 0
#define MOE_FUSION_ON 1
#define MOE_FUSION_OFF 2
MOE_API int moe_set_expert_fusion(int mode);

/* Upper bound, in nanoseconds of %globaltimer, on every spin-wait inside the
 * kernels launched by later calls from this process (default 2e9).  A wait
 * that runs out sets MOE_ERR_DEVICE_TIMEOUT and the kernel returns early. */
MOE_API void moe_set_wait_timeout_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif

#endif /* MOEFP8_H */
