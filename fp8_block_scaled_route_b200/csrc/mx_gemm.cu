// Grouped MXFP8 GEMM on the block-scaled tensor core path.
//
// Format: E4M3 operands with one E8M0 (power-of-two) scale per 32 consecutive
// K elements of every row of A and of B -- the MXFP8 format that the page
// "FlashInfer SM120 MoE GEMM 최적화: 웨이브+잔여물 비용 모델 도입" names beside
// FP8 for its grouped MoE GEMM (section "들어가며"; "mxfp8 grouped MoE" timings
// in "왜 이게 좋은가?"), with the scale rule of the SwiGLU + MXFP8 kernel of the
// page "NVIDIA R200(SM107)을 위한 SwiGLU + MXFP8 커널 최적화".
//
// Because the scales are powers of two, tcgen05.mma kind::mxf8f6f4.block_scale
// applies them inside the tensor core: the accumulator stays in TMEM for the
// whole K loop and the epilogue reads it once per tile (the FP8 kernel with
// fp32 block scales has to read and promote every 128-wide K block).
//
// Tile: 128 grouped rows (MMA M) x 256 weight rows (MMA N; gated: 128 gate +
// 128 up rows), persistent CTAs, 4-stage ring of 50 KB stages:
//   A  128 x 128 B  (TMA, 128-byte swizzle)        16 KB
//   B  256 x 128 B  (TMA, 128-byte swizzle)        32 KB
//   SF A 128 rows x 4 scales, B 256 rows x 4 scales, each 128-row group in
//      the 512-byte layout byte(r, j) = (r % 32) * 16 + (r / 32) * 4 + j
//      (j = 32-wide K step).  Weight scales come pre-tiled in that layout
//      ([E*N/128, K/128, 512], see mxfp8_tile_scales), one coalesced 16-byte
//      copy per lane per 128-row block; activation scales are row-major
//      [R, K/32] or K-block-major [K/128, R, 4] (a tile's rows start anywhere,
//      so four 4-byte copies per lane; coalesced in the second layout).
// Warps: 0 TMA producer, 1 MMA issuer (elected lane), 2 weight scale loader,
// 3 activation scale loader, 4-11 epilogue.  TMEM: accumulator columns [0, 256), A scale factors
// [256, 260), B scale factors [264, 272); one tcgen05.cp per 128 rows moves a
// stage's scale factors into TMEM ahead of its four MMAs (issued by the same
// thread, so they are ordered).
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

bool make_tma_map_fp8(CUtensorMap* out, const void* ptr, long long rows, long long cols,
                      int box_rows);

namespace {

constexpr int kMxStages = 4;
constexpr int kMxEpiWarps = 8;
constexpr int kMxA = 128 * 128;
constexpr int kMxB = 256 * 128;
constexpr int kMxSfOff = kMxA + kMxB;
constexpr int kMxStage = kMxA + kMxB + 2048;  // scale factors: 512 (A) + 1024 (B), padded
constexpr int kMxMaxE = 1024;
constexpr int kMxTable = ((2 * (kMxMaxE + 1) * 4) + 15) / 16 * 16;
constexpr int kMxCst = kMxEpiWarps * 32 * 16 * 4;  // combine: per-warp 32 x 16 fp32 transpose tile
constexpr int kMxSmem = 1024 + kMxStages * kMxStage + kMxTable + kMxCst + 256;
constexpr int kMxThreads = 384;
constexpr int kMxBoxes = 6;  // TMA boxes per stage: 2 x 64 token rows, 4 x 64 weight rows
constexpr uint32_t kMxTmemCols = 512;
constexpr uint32_t kMxSfaCol = 256;
constexpr uint32_t kMxSfbCol = 264;
static_assert(kMxStage % 1024 == 0, "stages must stay 1024-byte aligned for the swizzle");
static_assert(kMxSmem <= 232448, "shared memory budget");

struct MxParams {
    int R, N, K, E, nkb, gated, a_sf_mn;
    const uint8_t* a_sf;
    const uint8_t* b_sf;
    const int32_t* m_indptr;
    __nv_bfloat16* out;        // MX_EPI_BF16
    uint8_t* hq;               // MX_EPI_SWIGLU_MXQUANT: [R, N/2] codes
    uint8_t* hsf;              //   and [N/256, R, 4] E8M0 scales
    const int32_t* perm;       // MX_EPI_COMBINE: out_acc[perm[r] / topk] += topk_w[perm[r]] * G[r]
    const float* topk_w;
    int topk;
    float* out_acc;
    int out_ld;
    int* status;
    unsigned long long timeout_ns;
};

struct MxSmem {
    uint8_t* stages;
    float* cstage;
    int* tstart;  // [E+1] first tile of each expert
    int* mind;    // [E+1] clamped m_indptr
    uint64_t* full;
    uint64_t* empty;
    uint64_t* tfull;
    uint64_t* tempty;
    uint64_t* drain;
    uint32_t* tmem;
    volatile int* abort;
};

__device__ __forceinline__ MxSmem mx_carve(uint8_t* base) {
    MxSmem s;
    s.stages = base;
    uint8_t* p = base + kMxStages * kMxStage;
    s.tstart = reinterpret_cast<int*>(p);
    s.mind = s.tstart + (kMxMaxE + 1);
    p += kMxTable;
    s.cstage = reinterpret_cast<float*>(p);
    p += kMxCst;
    uint64_t* bars = reinterpret_cast<uint64_t*>(p);
    s.full = bars;
    s.empty = bars + kMxStages;
    s.tfull = bars + 2 * kMxStages;
    s.tempty = bars + 2 * kMxStages + 1;
    s.drain = bars + 2 * kMxStages + 2;
    s.tmem = reinterpret_cast<uint32_t*>(bars + 2 * kMxStages + 3);
    s.abort = reinterpret_cast<volatile int*>(bars + 2 * kMxStages + 4);
    return s;
}

struct MxTile {
    int e, nt, row0, rows;
};

// Tile t -> (expert, column tile, 128-row tile); column tiles outer within an
// expert so that consecutive CTAs share the weight tile.
__device__ __forceinline__ MxTile mx_decode(int t, const MxSmem& s, int E) {
    int lo = 0, hi = E;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s.tstart[mid] <= t) lo = mid; else hi = mid;
    }
    MxTile r;
    r.e = lo;
    const int local = t - s.tstart[lo];
    const int me = max(0, s.mind[lo + 1] - s.mind[lo]);
    const int mtiles = (me + 127) / 128;
    r.nt = local / mtiles;
    const int mt = local - r.nt * mtiles;
    r.row0 = s.mind[lo] + mt * 128;
    r.rows = min(128, me - mt * 128);
    return r;
}

// Global weight rows of the tile's two 128-row blocks.
__device__ __forceinline__ void mx_weight_rows(const MxTile& t, const MxParams& p, int& w0, int& w1) {
    if (p.gated) {
        w0 = t.e * p.N + t.nt * 128;
        w1 = t.e * p.N + (p.N >> 1) + t.nt * 128;
    } else {
        w0 = t.e * p.N + t.nt * 256;
        w1 = w0 + 128;
    }
}

__device__ __forceinline__ bool mx_warp_wait_spin(uint64_t* bar, uint32_t parity, const WaitCtl& wc,
                                                  int where) {
    return __all_sync(0xffffffffu, wait_bar_spin(bar, parity, wc, where)) != 0;
}
__device__ __forceinline__ bool mx_warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& wc,
                                             int where) {
    return __all_sync(0xffffffffu, wait_bar(bar, parity, wc, where)) != 0;
}

// Warp 0: lane l < 6 issues TMA box l of every stage.
__device__ void mx_producer(const CUtensorMap* tmA, const CUtensorMap* tmB, const MxParams& p,
                            const MxSmem& s, const WaitCtl& wc, int total) {
    const int l = threadIdx.x & 31;
    const bool issuer = l < kMxBoxes;
    const bool is_a = l < 2;
    const int b = l - 2;  // weight box 0..3: block b/2, half b%2
    const uint32_t off = is_a ? l * 64 * 128 : kMxA + b * 64 * 128;
    uint32_t stage = 0, phase = 0, armed = 0, armed_par = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const MxTile tl = mx_decode(t, s, p.E);
        int w0, w1;
        mx_weight_rows(tl, p, w0, w1);
        const int row = is_a ? tl.row0 + l * 64 : ((b >> 1) ? w1 : w0) + (b & 1) * 64;
        for (int kb = 0; kb < p.nkb; ++kb) {
            if (!mx_warp_wait_spin(&s.empty[stage], phase ^ 1, wc, 1)) { ok = false; break; }
            if (issuer) {
                mbar_arrive_expect_tx(&s.full[stage], 64 * 128);
                tma_load_2d(s.stages + stage * kMxStage + off, is_a ? tmA : tmB, &s.full[stage],
                            kb * 128, row);
            }
            __syncwarp();
            armed |= 1u << stage;
            armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
            if (++stage == kMxStages) { stage = 0; phase ^= 1; }
        }
    }
    for (int st = 0; st < kMxStages; ++st)
        if ((armed >> st) & 1u) wait_bar(&s.full[st], (armed_par >> st) & 1u, wc, 2, /*drain=*/true);
    __syncwarp();
}

// Warps 2 (weights) and 3 (activations): per stage, the 4 E8M0 scales of
// each of the tile's 256 weight rows or 128 token rows, in the 512-byte
// tcgen05.cp layout; completion arrives on the stage's full barrier.  Rows
// past the ends read as 0 (scale 2^-127; those outputs are not stored).
template <bool WEIGHTS>
__device__ void mx_sf_loader(const MxParams& p, const MxSmem& s, const WaitCtl& wc, int total) {
    const int lane = threadIdx.x & 31;
    const int nsf = p.K >> 5;  // row-major activation scale bytes per row
    const long long wblocks = static_cast<long long>(p.E) * p.N / 128;
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const MxTile tl = mx_decode(t, s, p.E);
        int w0, w1;
        mx_weight_rows(tl, p, w0, w1);
        for (int kb = 0; kb < p.nkb; ++kb) {
            if (!mx_warp_wait(&s.empty[stage], phase ^ 1, wc, 8)) { ok = false; break; }
            uint8_t* sf = s.stages + stage * kMxStage + kMxSfOff;
            if constexpr (WEIGHTS) {
#pragma unroll
                for (int blk = 0; blk < 2; ++blk) {
                    const long long wb = (blk ? w1 : w0) >> 7;
                    const bool v = wb < wblocks;
                    const uint8_t* src = v ? p.b_sf + (wb * p.nkb + kb) * 512 + lane * 16 : p.b_sf;
                    cp_async_16(sf + 512 + blk * 512 + lane * 16, src, v ? 16u : 0u);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) {  // token row lane + 32 i
                    const int r = tl.row0 + lane + 32 * i;
                    const bool v = r < p.R;
                    // [K/128, R, 4]: a warp's 32 rows are 128 contiguous bytes
                    const long long off = p.a_sf_mn ? (static_cast<long long>(kb) * p.R + r) * 4
                                                    : static_cast<long long>(r) * nsf + kb * 4;
                    cp_async_4(sf + lane * 16 + i * 4, v ? p.a_sf + off : p.a_sf, v ? 4u : 0u);
                }
            }
            cp_async_arrive_noinc(&s.full[stage]);
            if (++stage == kMxStages) { stage = 0; phase ^= 1; }
        }
    }
    cp_async_wait_all();
    __syncwarp();
}

// Warp 1: per stage, the scale factors into TMEM and four K=32 block-scaled
// MMAs (elected lane); the accumulator is released by the epilogue per tile.
__device__ void mx_mma(const MxParams& p, const MxSmem& s, const WaitCtl& wc, uint32_t tmem_base,
                       int total) {
    uint32_t stage = 0, phase = 0, it = 0;
    bool ok = true;
    const uint32_t sfa_t = tmem_base + kMxSfaCol;
    const uint32_t sfb_t = tmem_base + kMxSfbCol;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
        if (!mx_warp_wait_spin(s.tempty, (it & 1) ^ 1, wc, 3)) break;
        tc_fence_after();
        for (int kb = 0; kb < p.nkb; ++kb) {
            if (!mx_warp_wait_spin(&s.full[stage], phase, wc, 4)) { ok = false; break; }
            tc_fence_after();
            uint8_t* st = s.stages + stage * kMxStage;
            const uint32_t sa = smem_u32(st);
            const uint32_t sb = smem_u32(st + kMxA);
            const uint32_t ssf = smem_u32(st + kMxSfOff);
            if (elect_one()) {
                tmem_cp_32x128b_x4(sfa_t, smem_desc_k_noswizzle(ssf, 16, 128));
                tmem_cp_32x128b_x4(sfb_t, smem_desc_k_noswizzle(ssf + 512, 16, 128));
                tmem_cp_32x128b_x4(sfb_t + 4, smem_desc_k_noswizzle(ssf + 1024, 16, 128));
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_mx(tmem_base, smem_desc_k_sw128(sa + kk * 32), smem_desc_k_sw128(sb + kk * 32),
                            idesc_mx_e4m3(128, 256, kk, kk), sfa_t | (static_cast<uint32_t>(kk) << 30),
                            sfb_t | (static_cast<uint32_t>(kk) << 30), (kb | kk) != 0);
                umma_commit(&s.empty[stage]);
                if (kb == p.nkb - 1) umma_commit(s.tfull);
            }
            __syncwarp();
            if (++stage == kMxStages) { stage = 0; phase ^= 1; }
        }
    }
    if (elect_one()) umma_commit(s.drain);
    __syncwarp();
    wait_bar(s.drain, 0, wc, 5, /*drain=*/true);
    __syncwarp();
}

__device__ __forceinline__ float mx_silu(float z) { return z * rcp_approx(1.0f + __expf(-z)); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    uint32_t u;
    memcpy(&u, &h, 4);
    return u;
}

// Warps 4-11: thread = one row of the tile, 64 columns of each weight block
// (warp w: rows 32 (w % 4) .. +31, column half (w - 4) / 4).  The
// accumulator leaves TMEM once per tile; then, by mode:
//  MX_EPI_BF16           bf16 G (plain) or bf16 silu(gate) * up (gated)
//  MX_EPI_SWIGLU_MXQUANT h = silu(gate) * up requantised to MXFP8: the
//                        thread's 64 columns are two 32-column blocks, each
//                        with its own E8M0 scale (no exchange needed)
//  MX_EPI_COMBINE        out_acc[token] += w * G through a shared-memory
//                        transpose (8 rows x 64 contiguous bytes per reduction)
template <int MODE>
__device__ void mx_epilogue(const MxParams& p, const MxSmem& s, const WaitCtl& wc,
                            uint32_t tmem_base, int total) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3;
    const int g = (warp - 4) >> 2;
    const int rl = q * 32 + lane;
    const int colg = g * 64;
    const uint32_t tl_addr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + colg;
    uint32_t it = 0;
    uint32_t v[4][32];
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
        const MxTile tl = mx_decode(t, s, p.E);
        const bool row_ok = rl < tl.rows;
        const long long row = tl.row0 + rl;
        // combine: the row's pair id and weight, fetched while the tile computes
        int c_tok = -1;
        float c_w = 0.0f;
        if constexpr (MODE == MX_EPI_COMBINE) {
            if (row_ok) {
                const int pair = __ldg(p.perm + row);
                c_tok = pair / p.topk;
                c_w = __ldg(p.topk_w + pair);
            }
        }
        if (!mx_warp_wait(s.tfull, it & 1, wc, 6)) return;
        tc_fence_after();
        tmem_ld32_async(tl_addr, v[0]);
        tmem_ld32_async(tl_addr + 32, v[1]);
        tmem_ld32_async(tl_addr + 128, v[2]);
        tmem_ld32_async(tl_addr + 160, v[3]);
        tmem_wait_ld(v[0]);
        tmem_wait_ld(v[1]);
        tmem_wait_ld(v[2]);
        tmem_wait_ld(v[3]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s.tempty);
        if constexpr (MODE == MX_EPI_COMBINE) {
            float* stg = s.cstage + (warp - 4) * 512;
            const int rr = lane >> 2, cc = lane & 3;
            float* const obase = p.out_acc + tl.nt * 256 + colg;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                if (tl.nt * 256 + half * 128 >= p.N) break;
#pragma unroll
                for (int c16 = 0; c16 < 4; ++c16) {
                    const uint32_t* a = v[2 * half + (c16 >> 1)] + (c16 & 1) * 16;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int slot = (lane & 1) * 4 + ((q4 + (lane >> 1)) & 3);
                        *reinterpret_cast<float4*>(stg + (lane >> 1) * 32 + slot * 4) =
                            make_float4(c_w * __uint_as_float(a[4 * q4]),
                                        c_w * __uint_as_float(a[4 * q4 + 1]),
                                        c_w * __uint_as_float(a[4 * q4 + 2]),
                                        c_w * __uint_as_float(a[4 * q4 + 3]));
                    }
                    __syncwarp();
#pragma unroll
                    for (int rg = 0; rg < 4; ++rg) {
                        const int r = rg * 8 + rr;
                        const int slot = (r & 1) * 4 + ((cc + (r >> 1)) & 3);
                        const float4 x4 = *reinterpret_cast<const float4*>(stg + (r >> 1) * 32 + slot * 4);
                        const int t_r = __shfl_sync(0xffffffffu, c_tok, r);
                        if (t_r >= 0)
                            red_add_v4(obase + static_cast<long long>(t_r) * p.out_ld + half * 128 +
                                           c16 * 16 + cc * 4,
                                       x4.x, x4.y, x4.z, x4.w);
                    }
                    __syncwarp();
                }
            }
            continue;
        }
        if (!row_ok) continue;
        if constexpr (MODE == MX_EPI_SWIGLU_MXQUANT) {
            const int I = p.N >> 1;
            uint4* dst = reinterpret_cast<uint4*>(p.hq + row * I + tl.nt * 128 + colg);
            uint32_t sf2 = 0;
#pragma unroll
            for (int blk = 0; blk < 2; ++blk) {
                float h[32];
                float amax = 0.0f;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    h[i] = mx_silu(__uint_as_float(v[blk][i])) * __uint_as_float(v[2 + blk][i]);
                    amax = fmaxf(amax, fabsf(h[i]));
                }
                const uint32_t code = e8m0_code(amax);
                const float inv = e8m0_reciprocal(code);
                sf2 |= code << (8 * blk);
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint4 w;
                    w.x = cvt_e4m3x4(h[16 * c + 0] * inv, h[16 * c + 1] * inv, h[16 * c + 2] * inv, h[16 * c + 3] * inv);
                    w.y = cvt_e4m3x4(h[16 * c + 4] * inv, h[16 * c + 5] * inv, h[16 * c + 6] * inv, h[16 * c + 7] * inv);
                    w.z = cvt_e4m3x4(h[16 * c + 8] * inv, h[16 * c + 9] * inv, h[16 * c + 10] * inv, h[16 * c + 11] * inv);
                    w.w = cvt_e4m3x4(h[16 * c + 12] * inv, h[16 * c + 13] * inv, h[16 * c + 14] * inv, h[16 * c + 15] * inv);
                    dst[2 * blk + c] = w;
                }
            }
            // scales of h columns nt*128 + colg + [0, 64): bytes 2g, 2g + 1 of
            // the row's 4-byte entry for K block nt of the next GEMM
            *reinterpret_cast<uint16_t*>(p.hsf + (static_cast<long long>(tl.nt) * p.R + row) * 4 + 2 * g) =
                static_cast<uint16_t>(sf2);
        } else if (p.gated) {
            // h = silu(gate) * up, 64 bf16 values per row
            uint4* dst = reinterpret_cast<uint4*>(p.out + row * (p.N >> 1) + tl.nt * 128 + colg);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                float h[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int j = 8 * c + i;
                    h[i] = mx_silu(__uint_as_float(v[j >> 5][j & 31])) *
                           __uint_as_float(v[2 + (j >> 5)][j & 31]);
                }
                dst[c] = make_uint4(pack_bf16(h[0], h[1]), pack_bf16(h[2], h[3]),
                                    pack_bf16(h[4], h[5]), pack_bf16(h[6], h[7]));
            }
        } else {
            const int n0 = tl.nt * 256;
            __nv_bfloat16* rowp = p.out + row * p.N + n0 + colg;
#pragma unroll
            for (int blk = 0; blk < 2; ++blk) {
                if (n0 + blk * 128 >= p.N) break;
                uint4* dst = reinterpret_cast<uint4*>(rowp + blk * 128);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint32_t* a = v[2 * blk + (c >> 2)] + (c & 3) * 8;
                    dst[c] = make_uint4(pack_bf16(__uint_as_float(a[0]), __uint_as_float(a[1])),
                                        pack_bf16(__uint_as_float(a[2]), __uint_as_float(a[3])),
                                        pack_bf16(__uint_as_float(a[4]), __uint_as_float(a[5])),
                                        pack_bf16(__uint_as_float(a[6]), __uint_as_float(a[7])));
                }
            }
        }
    }
}

template <int MODE>
__global__ void __launch_bounds__(kMxThreads, 1)
    mx_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const MxParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const MxSmem s = mx_carve(base);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kMxStages; ++i) {
            mbar_init(&s.full[i], kMxBoxes + 64);  // TMA lanes + two scale-loader warps
            mbar_init(&s.empty[i], 1);
        }
        mbar_init(s.tfull, 1);
        mbar_init(s.tempty, kMxEpiWarps);
        mbar_init(s.drain, 1);
        *s.abort = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(s.tmem, kMxTmemCols);
        tmem_relinquish();
    }
    if (warp == 2) {
        // per-expert tile table: tiles of expert e = ceil(rows_e / 128) * column tiles
        const int E = p.E;
        const int ntn = p.gated ? (p.N >> 8) : ((p.N + 255) >> 8);
        const int per = (E + 31) >> 5;
        const int lo = min(E, lane * per), hi = min(E, lo + per);
        int sum = 0;
        for (int e = lo; e < hi; ++e) {
            const int m0 = min(max(p.m_indptr[e], 0), p.R);
            const int m1 = min(max(p.m_indptr[e + 1], 0), p.R);
            s.mind[e] = m0;
            sum += ((max(0, m1 - m0) + 127) / 128) * ntn;
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += x;
        }
        int run = incl - sum;
        for (int e = lo; e < hi; ++e) {
            s.tstart[e] = run;
            const int m0 = s.mind[e];
            const int m1 = min(max(p.m_indptr[e + 1], 0), p.R);
            run += ((max(0, m1 - m0) + 127) / 128) * ntn;
        }
        if (lane == 31) {
            s.tstart[E] = incl;
            s.mind[E] = min(max(p.m_indptr[E], 0), p.R);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s.tmem;
    const WaitCtl wc{s.abort, p.status, p.timeout_ns};
    const int total = s.tstart[p.E];
    if (warp == 0) mx_producer(&tmA, &tmB, p, s, wc, total);
    else if (warp == 1) mx_mma(p, s, wc, tmem_base, total);
    else if (warp == 2) mx_sf_loader<true>(p, s, wc, total);
    else if (warp == 3) mx_sf_loader<false>(p, s, wc, total);
    else if (warp >= 4) mx_epilogue<MODE>(p, s, wc, tmem_base, total);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kMxTmemCols);
}

// ---------------------------------------------------------------- swapped tile
// Small groups (decode-sized): the weights are the MMA M operand (two
// 128-row weight blocks per tile, one MMA each) and 32 token rows are N, so a
// tile streams 32 KB of weights and only 4 KB of tokens per K block instead
// of a 128-row token tile that is mostly padding.  The block scales swap
// sides too: the weights' pre-tiled scales are the MMA's A scale factors, the
// tokens' 32 rows its B scale factors (one TMEM column).  Accumulators stay in
// TMEM for the whole K loop, in 7 slots of 2 x 32 columns, so the weight
// stream continues through tile epilogues.  Warps: 0 TMA, 1 MMA, 2 weight
// scales, 3 token scales, 4-7 epilogue (thread = one weight row x 32 tokens).
constexpr int kSwBT = 32;
constexpr int kSwStages = 5;
constexpr int kSwW = 256 * 128;
constexpr int kSwT = kSwBT * 128;
constexpr int kSwSfOff = kSwW + kSwT;
constexpr int kSwStage = kSwW + kSwT + 2048;
constexpr int kSwSlots = 7;
constexpr uint32_t kSwSfCol = 448;  // weight block 0 [448,452), block 1 [452,456), tokens [456,460)
constexpr int kSwThreads = 256;
constexpr int kSwBoxes = 5;         // 1 token box (32 rows) + 4 weight boxes (64 rows)
constexpr int kSwSmem = 1024 + kSwStages * kSwStage + kMxTable + 512;
static_assert(kSwStage % 1024 == 0, "stages must stay 1024-byte aligned for the swizzle");
static_assert(kSwSmem <= 232448, "shared memory budget");
static_assert(kSwSlots * 2 * kSwBT <= static_cast<int>(kSwSfCol), "TMEM columns");

struct SwSmem {
    uint8_t* stages;
    int* tstart;
    int* mind;
    uint64_t* full;
    uint64_t* empty;
    uint64_t* tfull;
    uint64_t* tempty;
    uint64_t* drain;
    uint32_t* tmem;
    volatile int* abort;
};

__device__ __forceinline__ SwSmem sw_carve(uint8_t* base) {
    SwSmem s;
    s.stages = base;
    uint8_t* p = base + kSwStages * kSwStage;
    s.tstart = reinterpret_cast<int*>(p);
    s.mind = s.tstart + (kMxMaxE + 1);
    p += kMxTable;
    uint64_t* bars = reinterpret_cast<uint64_t*>(p);
    s.full = bars;
    s.empty = bars + kSwStages;
    s.tfull = bars + 2 * kSwStages;
    s.tempty = bars + 2 * kSwStages + kSwSlots;
    s.drain = bars + 2 * kSwStages + 2 * kSwSlots;
    s.tmem = reinterpret_cast<uint32_t*>(bars + 2 * kSwStages + 2 * kSwSlots + 1);
    s.abort = reinterpret_cast<volatile int*>(bars + 2 * kSwStages + 2 * kSwSlots + 2);
    return s;
}

__device__ __forceinline__ MxTile sw_decode(int t, const SwSmem& s, int E) {
    int lo = 0, hi = E;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s.tstart[mid] <= t) lo = mid; else hi = mid;
    }
    MxTile r;
    r.e = lo;
    const int local = t - s.tstart[lo];
    const int me = max(0, s.mind[lo + 1] - s.mind[lo]);
    const int mtiles = (me + kSwBT - 1) / kSwBT;
    r.nt = local / mtiles;
    const int mt = local - r.nt * mtiles;
    r.row0 = s.mind[lo] + mt * kSwBT;
    r.rows = min(kSwBT, me - mt * kSwBT);
    return r;
}

__device__ void sw_producer(const CUtensorMap* tmA, const CUtensorMap* tmB, const MxParams& p,
                            const SwSmem& s, const WaitCtl& wc, int total) {
    const int l = threadIdx.x & 31;
    const bool issuer = l < kSwBoxes;
    const bool is_tok = l == 0;
    const int b = l - 1;  // weight box 0..3: block b/2, half b%2
    const uint32_t off = is_tok ? kSwW : b * 64 * 128;
    const uint32_t bytes = is_tok ? kSwT : 64 * 128;
    uint32_t stage = 0, phase = 0, armed = 0, armed_par = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const MxTile tl = sw_decode(t, s, p.E);
        int w0, w1;
        mx_weight_rows(tl, p, w0, w1);
        const int row = is_tok ? tl.row0 : ((b >> 1) ? w1 : w0) + (b & 1) * 64;
        for (int kb = 0; kb < p.nkb; ++kb) {
            if (!mx_warp_wait_spin(&s.empty[stage], phase ^ 1, wc, 1)) { ok = false; break; }
            if (issuer) {
                mbar_arrive_expect_tx(&s.full[stage], bytes);
                tma_load_2d(s.stages + stage * kSwStage + off, is_tok ? tmA : tmB, &s.full[stage],
                            kb * 128, row);
            }
            __syncwarp();
            armed |= 1u << stage;
            armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
            if (++stage == kSwStages) { stage = 0; phase ^= 1; }
        }
    }
    for (int st = 0; st < kSwStages; ++st)
        if ((armed >> st) & 1u) wait_bar(&s.full[st], (armed_par >> st) & 1u, wc, 2, /*drain=*/true);
    __syncwarp();
}

// Warp 2: the two weight blocks' pre-tiled scales; warp 3: the 32 token rows'
// scales (byte lane * 16 + j of a 512-byte block, i.e. TMEM column 0).
template <bool WEIGHTS>
__device__ void sw_sf_loader(const MxParams& p, const SwSmem& s, const WaitCtl& wc, int total) {
    const int lane = threadIdx.x & 31;
    const int nsf = p.K >> 5;
    const long long wblocks = static_cast<long long>(p.E) * p.N / 128;
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const MxTile tl = sw_decode(t, s, p.E);
        int w0, w1;
        mx_weight_rows(tl, p, w0, w1);
        for (int kb = 0; kb < p.nkb; ++kb) {
            if (!mx_warp_wait(&s.empty[stage], phase ^ 1, wc, 8)) { ok = false; break; }
            uint8_t* sf = s.stages + stage * kSwStage + kSwSfOff;
            if constexpr (WEIGHTS) {
#pragma unroll
                for (int blk = 0; blk < 2; ++blk) {
                    const long long wb = (blk ? w1 : w0) >> 7;
                    const bool v = wb < wblocks;
                    const uint8_t* src = v ? p.b_sf + (wb * p.nkb + kb) * 512 + lane * 16 : p.b_sf;
                    cp_async_16(sf + blk * 512 + lane * 16, src, v ? 16u : 0u);
                }
            } else {
                const int r = tl.row0 + lane;
                const bool v = r < p.R;
                const long long off = p.a_sf_mn ? (static_cast<long long>(kb) * p.R + r) * 4
                                                : static_cast<long long>(r) * nsf + kb * 4;
                cp_async_4(sf + 1024 + lane * 16, v ? p.a_sf + off : p.a_sf, v ? 4u : 0u);
            }
            cp_async_arrive_noinc(&s.full[stage]);
            if (++stage == kSwStages) { stage = 0; phase ^= 1; }
        }
    }
    cp_async_wait_all();
    __syncwarp();
}

__device__ void sw_mma(const MxParams& p, const SwSmem& s, const WaitCtl& wc, uint32_t tmem_base,
                       int total) {
    uint32_t stage = 0, phase = 0, j = 0, jphase = 0;
    bool ok = true;
    const uint32_t sfw0 = tmem_base + kSwSfCol, sfw1 = sfw0 + 4, sft = sfw0 + 8;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        if (!mx_warp_wait_spin(&s.tempty[j], jphase ^ 1, wc, 3)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + j * (2 * kSwBT), d1 = d0 + kSwBT;
        for (int kb = 0; kb < p.nkb; ++kb) {
            if (!mx_warp_wait_spin(&s.full[stage], phase, wc, 4)) { ok = false; break; }
            tc_fence_after();
            uint8_t* st = s.stages + stage * kSwStage;
            const uint32_t sw = smem_u32(st);
            const uint32_t stok = smem_u32(st + kSwW);
            const uint32_t ssf = smem_u32(st + kSwSfOff);
            if (elect_one()) {
                tmem_cp_32x128b_x4(sfw0, smem_desc_k_noswizzle(ssf, 16, 128));
                tmem_cp_32x128b_x4(sfw1, smem_desc_k_noswizzle(ssf + 512, 16, 128));
                tmem_cp_32x128b_x4(sft, smem_desc_k_noswizzle(ssf + 1024, 16, 128));
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint32_t idesc = idesc_mx_e4m3(128, kSwBT, kk, kk);
                    const uint32_t acc = (kb | kk) != 0;
                    const uint32_t id = static_cast<uint32_t>(kk) << 30;
                    umma_mx(d0, smem_desc_k_sw128(sw + kk * 32), smem_desc_k_sw128(stok + kk * 32),
                            idesc, sfw0 | id, sft | id, acc);
                    umma_mx(d1, smem_desc_k_sw128(sw + 16384 + kk * 32),
                            smem_desc_k_sw128(stok + kk * 32), idesc, sfw1 | id, sft | id, acc);
                }
                umma_commit(&s.empty[stage]);
                if (kb == p.nkb - 1) umma_commit(&s.tfull[j]);
            }
            __syncwarp();
            if (++stage == kSwStages) { stage = 0; phase ^= 1; }
        }
        if (++j == kSwSlots) { j = 0; jphase ^= 1; }
    }
    if (elect_one()) umma_commit(s.drain);
    __syncwarp();
    wait_bar(s.drain, 0, wc, 5, /*drain=*/true);
    __syncwarp();
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Warps 4-7: lane = weight row q*32 + lane of each block (an output column),
// 32 tokens per thread.
template <int MODE>
__device__ void sw_epilogue(const MxParams& p, const SwSmem& s, const WaitCtl& wc,
                            uint32_t tmem_base, int total) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3;
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t j = 0, jphase = 0;
    uint32_t v0[32], v1[32];
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
        const MxTile tl = sw_decode(t, s, p.E);
        int c_tok = -1;
        float c_w = 0.0f;
        if constexpr (MODE == MX_EPI_COMBINE) {
            if (lane < tl.rows) {
                const int pair = __ldg(p.perm + tl.row0 + lane);
                c_tok = pair / p.topk;
                c_w = __ldg(p.topk_w + pair);
            }
        }
        if (!mx_warp_wait(&s.tfull[j], jphase, wc, 6)) return;
        tc_fence_after();
        tmem_ld32_async(lane_addr + j * (2 * kSwBT), v0);
        tmem_ld32_async(lane_addr + j * (2 * kSwBT) + kSwBT, v1);
        tmem_wait_ld(v0);
        tmem_wait_ld(v1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.tempty[j]);
        if (++j == kSwSlots) { j = 0; jphase ^= 1; }
        const int col = q * 32 + lane;  // row of each weight block
        if constexpr (MODE == MX_EPI_COMBINE) {
            const int n0 = tl.nt * 256 + col;
            const bool v1ok = tl.nt * 256 + 128 < p.N;
#pragma unroll
            for (int tok = 0; tok < kSwBT; ++tok) {
                const int tk = __shfl_sync(0xffffffffu, c_tok, tok);
                const float w = __shfl_sync(0xffffffffu, c_w, tok);
                if (tok >= tl.rows) continue;
                float* dst = p.out_acc + static_cast<long long>(tk) * p.out_ld + n0;
                red_add(dst, w * __uint_as_float(v0[tok]));
                if (v1ok) red_add(dst + 128, w * __uint_as_float(v1[tok]));
            }
        } else if constexpr (MODE == MX_EPI_SWIGLU_MXQUANT) {
            const int I = p.N >> 1;
#pragma unroll
            for (int tok = 0; tok < kSwBT; ++tok) {
                // the warp max runs for every token (a collective); rows past
                // the tile compute on zeros and store nothing
                const float h = mx_silu(__uint_as_float(v0[tok])) * __uint_as_float(v1[tok]);
                const uint32_t code = e8m0_code(warp_max(fabsf(h)));
                const float inv = e8m0_reciprocal(code);
                if (tok >= tl.rows) continue;
                const long long row = tl.row0 + tok;
                p.hq[row * I + tl.nt * 128 + col] =
                    static_cast<uint8_t>(cvt_e4m3x4(h * inv, 0.0f, 0.0f, 0.0f) & 0xFFu);
                if (lane == 0) p.hsf[(static_cast<long long>(tl.nt) * p.R + row) * 4 + q] =
                    static_cast<uint8_t>(code);
            }
        } else if (p.gated) {
#pragma unroll
            for (int tok = 0; tok < kSwBT; ++tok) {
                if (tok >= tl.rows) continue;
                const float h = mx_silu(__uint_as_float(v0[tok])) * __uint_as_float(v1[tok]);
                p.out[static_cast<long long>(tl.row0 + tok) * (p.N >> 1) + tl.nt * 128 + col] =
                    __float2bfloat16_rn(h);
            }
        } else {
            const bool v1ok = tl.nt * 256 + 128 < p.N;
#pragma unroll
            for (int tok = 0; tok < kSwBT; ++tok) {
                if (tok >= tl.rows) continue;
                __nv_bfloat16* o = p.out + static_cast<long long>(tl.row0 + tok) * p.N + tl.nt * 256 + col;
                o[0] = __float2bfloat16_rn(__uint_as_float(v0[tok]));
                if (v1ok) o[128] = __float2bfloat16_rn(__uint_as_float(v1[tok]));
            }
        }
    }
}

template <int MODE>
__global__ void __launch_bounds__(kSwThreads, 1)
    mx_gemm_swap_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, const MxParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const SwSmem s = sw_carve(base);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kSwStages; ++i) {
            mbar_init(&s.full[i], kSwBoxes + 64);  // TMA lanes + two scale-loader warps
            mbar_init(&s.empty[i], 1);
        }
        for (int i = 0; i < kSwSlots; ++i) {
            mbar_init(&s.tfull[i], 1);
            mbar_init(&s.tempty[i], 4);
        }
        mbar_init(s.drain, 1);
        *s.abort = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(s.tmem, kMxTmemCols);
        tmem_relinquish();
    }
    if (warp == 2) {
        const int E = p.E;
        const int ntn = p.gated ? (p.N >> 8) : ((p.N + 255) >> 8);
        const int per = (E + 31) >> 5;
        const int lo = min(E, lane * per), hi = min(E, lo + per);
        int sum = 0;
        for (int e = lo; e < hi; ++e) {
            const int m0 = min(max(p.m_indptr[e], 0), p.R);
            const int m1 = min(max(p.m_indptr[e + 1], 0), p.R);
            s.mind[e] = m0;
            sum += ((max(0, m1 - m0) + kSwBT - 1) / kSwBT) * ntn;
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += x;
        }
        int run = incl - sum;
        for (int e = lo; e < hi; ++e) {
            s.tstart[e] = run;
            const int m0 = s.mind[e];
            const int m1 = min(max(p.m_indptr[e + 1], 0), p.R);
            run += ((max(0, m1 - m0) + kSwBT - 1) / kSwBT) * ntn;
        }
        if (lane == 31) {
            s.tstart[E] = incl;
            s.mind[E] = min(max(p.m_indptr[E], 0), p.R);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s.tmem;
    const WaitCtl wc{s.abort, p.status, p.timeout_ns};
    const int total = s.tstart[p.E];
    if (warp == 0) sw_producer(&tmA, &tmB, p, s, wc, total);
    else if (warp == 1) sw_mma(p, s, wc, tmem_base, total);
    else if (warp == 2) sw_sf_loader<true>(p, s, wc, total);
    else if (warp == 3) sw_sf_loader<false>(p, s, wc, total);
    else sw_epilogue<MODE>(p, s, wc, tmem_base, total);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kMxTmemCols);
}

// Row-major E8M0 scales [rows, K/32] -> tiled [rows/128, K/128, 512]: one
// thread per 4-byte word (the 4 scales of one row in one 128-wide K block).
__global__ void __launch_bounds__(256) mx_tile_scales_kernel(const uint32_t* __restrict__ rm,
                                                             uint32_t* __restrict__ tiled,
                                                             long long words, int nkb) {
    for (long long w = blockIdx.x * 256ll + threadIdx.x; w < words; w += gridDim.x * 256ll) {
        const long long atom = w >> 7;  // (128-row block, K block)
        const int pos = static_cast<int>(w & 127);
        const long long blk = atom / nkb;
        const int kb = static_cast<int>(atom - blk * nkb);
        const int l = pos >> 2, g = pos & 3;
        const long long row = blk * 128 + g * 32 + l;
        tiled[w] = rm[row * nkb + kb];
    }
}

}  // namespace

int launch_mx_tile_scales(const uint8_t* rm, uint8_t* tiled, int rows, int K, int num_sms,
                          cudaStream_t stream) {
    const int nkb = K / 128;
    const long long words = static_cast<long long>(rows) * nkb;
    if (words == 0) return ST_OK;
    const long long blocks = (words + 255) / 256;
    const int grid = static_cast<int>(blocks < num_sms * 8ll ? blocks : num_sms * 8ll);
    mx_tile_scales_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint32_t*>(rm),
                                                    reinterpret_cast<uint32_t*>(tiled), words, nkb);
    return cudaGetLastError() == cudaSuccess ? ST_OK : ST_CUDA;
}

namespace {
template <int MODE>
int launch_mx_inst(const CUtensorMap& ma, const CUtensorMap& mb, const MxParams& p, int num_sms,
                   bool swap, cudaStream_t stream) {
    static int configured_dev[2] = {-1, -1};
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev[swap] != dev) {
        const cudaError_t e =
            swap ? cudaFuncSetAttribute(mx_gemm_swap_kernel<MODE>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, kSwSmem)
                 : cudaFuncSetAttribute(mx_gemm_kernel<MODE>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, kMxSmem);
        if (e != cudaSuccess) return ST_CUDA;
        configured_dev[swap] = dev;
    }
    if (swap)
        mx_gemm_swap_kernel<MODE><<<num_sms, kSwThreads, kSwSmem, stream>>>(ma, mb, p);
    else
        mx_gemm_kernel<MODE><<<num_sms, kMxThreads, kMxSmem, stream>>>(ma, mb, p);
    return cudaGetLastError() == cudaSuccess ? ST_OK : ST_CUDA;
}
}  // namespace

int launch_mx_gemm(const MxGemmArgs& g, cudaStream_t stream) {
    if (g.R <= 0 || g.E <= 0) return ST_OK;
    if (g.E > kMxMaxE) return ST_INVALID_ARG;
    // tile choice: 32-token swapped tiles when the groups are small (balanced
    // rows per expert below 32; measured: decode, ~2 rows per expert, 1.50 vs
    // 1.64 ms per layer; 32 rows per expert, 182 vs 170 µs the other way)
    const bool swap = g.tile_m == 32 || (g.tile_m <= 0 && (g.R + g.E - 1) / g.E < kSwBT);
    CUtensorMap ma, mb;
    if (!make_tma_map_fp8(&ma, g.a, g.R, g.K, swap ? kSwBT : 64)) return ST_CUDA;
    if (!make_tma_map_fp8(&mb, g.b, static_cast<long long>(g.E) * g.N, g.K, 64)) return ST_CUDA;
    MxParams p{};
    p.R = g.R; p.N = g.N; p.K = g.K; p.E = g.E; p.nkb = g.K / 128; p.gated = g.gated ? 1 : 0;
    p.a_sf_mn = g.a_sf_mn ? 1 : 0;
    p.a_sf = g.a_sf; p.b_sf = g.b_sf; p.m_indptr = g.m_indptr;
    p.out = static_cast<__nv_bfloat16*>(g.out);
    p.hq = g.hq; p.hsf = g.hsf;
    p.perm = g.perm; p.topk_w = g.topk_w; p.topk = g.topk > 0 ? g.topk : 1;
    p.out_acc = g.out_acc; p.out_ld = g.out_ld;
    p.status = g.status;
    p.timeout_ns = g.timeout_ns;
    switch (g.epi) {
        case MX_EPI_SWIGLU_MXQUANT:
            return launch_mx_inst<MX_EPI_SWIGLU_MXQUANT>(ma, mb, p, g.num_sms, swap, stream);
        case MX_EPI_COMBINE:
            return launch_mx_inst<MX_EPI_COMBINE>(ma, mb, p, g.num_sms, swap, stream);
        default:
            return launch_mx_inst<MX_EPI_BF16>(ma, mb, p, g.num_sms, swap, stream);
    }
}

}  // namespace moe
