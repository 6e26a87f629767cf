// Grouped NVFP4 GEMM on the block-scaled tensor core path.
//
// Format: E2M1 operands packed two per byte (element 2i in the low nibble),
// one E4M3 scale per 16 consecutive K elements of every row of A and of B,
// and an fp32 global scale per tensor -- the NVFP4 (W4A4) quantisation of the
// page "FlashInfer에 cuTile 기반 Fused MoE 백엔드 도입" (section "2. cuTile NVFP4
// 양자화 지원": fp4_quantize with a per-expert global scale and
// sf_vec_size=16).  The real value of an element is e2m1(q) * e4m3(s) / g.
//
// tcgen05.mma kind::mxf4nvf4 with 16-element scale vectors applies the block
// scales inside the tensor core (K = 64 per instruction: the four E4M3 scales
// of a row are the four bytes of one TMEM column), so the accumulator stays in
// TMEM for the whole K loop; the epilogue applies alpha_e = 1 / (g_a g_b[e]).
//
// Tile: 128 grouped rows (MMA M) x 256 weight rows (MMA N; gated: 128 gate +
// 128 up rows), persistent CTAs, 4-stage ring of 54 KB stages covering 256 K
// elements (128 bytes per row):
//   A  128 x 128 B  (TMA, 128-byte swizzle)        16 KB
//   B  256 x 128 B  (TMA, 128-byte swizzle)        32 KB
//   SF per K = 64 step kk (4 per stage), 512-byte atoms in the layout
//      byte(r, j) = (r % 32) * 16 + (r / 32) * 4 + j (j = 16-wide K block):
//      A atoms at kk * 512, B atoms at 2048 + blk * 2048 + kk * 512.
//      Weight scales come pre-tiled in that layout ([E*N/128, K/64, 512]),
//      activation scales row-major [R, K/16] or K-block-major [K/64, R, 4]
//      (the four scales of a 64-wide K block of each row together, rows
//      consecutive: a warp's 32 rows are 128 contiguous bytes); four 4-byte
//      copies per row per step.
// Warps: 0 TMA producer, 1 MMA issuer (elected lane), 2 weight scale loader,
// 3 activation scale loader, 4-11 epilogue.  TMEM: accumulator columns
// [0, 256), A scale factors [256, 272) (4 per step), B scale factors
// [272, 304) (8 per step: two 128-row blocks).  Epilogues: bf16 G (plain or
// gated), SwiGLU + NVFP4 requantisation of the intermediate (GEMM1 of the
// fused layer), top-k weighted fp32 combine (GEMM2; one stage fewer to make
// room for its transpose buffer).
//
// Also here: the NVFP4 quantise-and-scatter of x (the fused layer's first
// GEMM input), sharing the quantisation step (nv_quant16) with the
// requantising epilogue.
#include <cstdlib>

#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

bool make_tma_map_fp8(CUtensorMap* out, const void* ptr, long long rows, long long cols,
                      int box_rows);

namespace {

// tcgen05.mma kind::mxf4nvf4, 16-element E4M3 scale vectors.
__device__ __forceinline__ void umma_nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem),
        "r"(accumulate)
        : "memory");
}

// Instruction descriptor: E2M1 x E2M1 (packed), E4M3 scales, fp32
// accumulation, both operands K-major, dense K = 64, scale ids 0.
__host__ __device__ constexpr uint32_t idesc_nvf4(int M, int N) {
    return (1u << 7) | (1u << 10)                          // A, B format E2M1
           | (static_cast<uint32_t>(N >> 3) << 17)         // N / 8
           | (0u << 23)                                    // scale format E4M3
           | (static_cast<uint32_t>(M >> 4) << 24);        // M / 16
}

// NVFP4 quantisation of 16 values with global scale g (the cuTile page's
// fp4_quantize with sf_vec_size=16): scale code c = E4M3_RNE_sat(amax * g / 6),
// codes E2M1_RNE_sat(v * g / e4m3(c)) (all 0 when the scale decodes to 0), in
// the same fp32 operation order as the format's definition so that each
// rounding decision is reproducible.  Returns the scale code; codes[i/2]
// holds element i in its low nibble when i is even.
__device__ __forceinline__ uint32_t nv_e4m3_scale(float amax, float g, float& s) {
    const float t = __fdiv_rn(__fmul_rn(amax, g), 6.0f);
    const __nv_fp8_storage_t c = __nv_cvt_float_to_fp8(t, __NV_SATFINITE, __NV_E4M3);
    const __half_raw hr = __nv_cvt_fp8_to_halfraw(c, __NV_E4M3);
    s = __half2float(__half(hr));
    return static_cast<uint32_t>(c);
}

__device__ __forceinline__ uint32_t nv_e2m1(float v) {
    return static_cast<uint32_t>(__nv_cvt_float_to_fp4(v, __NV_E2M1, cudaRoundNearest)) & 0xFu;
}

// 16 values -> 8 packed bytes (uint2) and the scale code.
__device__ __forceinline__ uint32_t nv_quant16(const float (&v)[16], float g, uint2& packed) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    float s;
    const uint32_t c = nv_e4m3_scale(amax, g, s);
    uint32_t w[2] = {0u, 0u};
    if (s > 0.0f) {
#pragma unroll
        for (int i = 0; i < 16; ++i)
            w[i >> 3] |= nv_e2m1(__fdiv_rn(__fmul_rn(v[i], g), s)) << (4 * (i & 7));
    }
    packed = make_uint2(w[0], w[1]);
    return c;
}


constexpr int kNvEpiWarps = 8;
constexpr int kNvA = 128 * 128;
constexpr int kNvB = 256 * 128;
constexpr int kNvSfOff = kNvA + kNvB;
constexpr int kNvSfBytes = 4 * 512 + 2 * 4 * 512;  // A: 4 atoms, B: 2 blocks x 4 atoms
constexpr int kNvStage = kNvA + kNvB + kNvSfBytes;
constexpr int kNvMaxE = 1024;
constexpr int kNvTable = ((2 * (kNvMaxE + 1) * 4) + 15) / 16 * 16;
constexpr int kNvCst = kNvEpiWarps * 32 * 16 * 4;  // combine: per-warp 32 x 16 fp32 transpose tile
constexpr int kNvThreads = 384;
constexpr int kNvBoxes = 6;  // TMA boxes per stage: 2 x 64 token rows, 4 x 64 weight rows
constexpr uint32_t kNvTmemCols = 512;
constexpr uint32_t kNvSfaCol = 256;
constexpr uint32_t kNvSfbCol = 272;
static_assert(kNvStage % 1024 == 0, "stages must stay 1024-byte aligned for the swizzle");

// Per epilogue: ring depth and shared memory (the combine's transpose buffer
// costs one stage).
template <int MODE>
struct NvCfg {
    static constexpr int STAGES = MODE == NV_EPI_COMBINE ? 3 : 4;
    static constexpr int CST = MODE == NV_EPI_COMBINE ? kNvCst : 0;
    static constexpr int SMEM = 1024 + STAGES * kNvStage + kNvTable + CST + 256;
    static_assert(SMEM <= 232448, "shared memory budget");
};

struct NvParams {
    int R, N, K, E, nkb, gated;  // nkb: 256-element K blocks
    int a_sf_mn;                 // activation scales [K/64, R, 4] (1) or [R, K/16] (0)
    const uint8_t* a_sf;         // E4M3
    const uint8_t* b_sf;         // [E*N/128, K/64, 512] E4M3, tiled
    const float* alpha;          // [E]
    const int32_t* m_indptr;
    __nv_bfloat16* out;          // NV_EPI_BF16
    uint8_t* hq;                 // NV_EPI_SWIGLU_NVQUANT: [R, N/4] packed codes of h
    uint8_t* hsf;                //   and [N/128, R, 4] E4M3 scales (K-block-major for GEMM2)
    float h_gscale;              //   global scale of h
    const int32_t* perm;         // NV_EPI_COMBINE: out_acc[perm[r] / topk] += topk_w[perm[r]] * G[r]
    const float* topk_w;
    int topk;
    float* out_acc;
    int out_ld;
    int* status;
    unsigned long long timeout_ns;
};

struct NvSmem {
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

template <int MODE>
__device__ __forceinline__ NvSmem nv_carve(uint8_t* base) {
    constexpr int S = NvCfg<MODE>::STAGES;
    NvSmem s;
    s.stages = base;
    uint8_t* p = base + S * kNvStage;
    s.tstart = reinterpret_cast<int*>(p);
    s.mind = s.tstart + (kNvMaxE + 1);
    p += kNvTable;
    s.cstage = reinterpret_cast<float*>(p);
    p += NvCfg<MODE>::CST;
    uint64_t* bars = reinterpret_cast<uint64_t*>(p);
    s.full = bars;
    s.empty = bars + S;
    s.tfull = bars + 2 * S;
    s.tempty = bars + 2 * S + 1;
    s.drain = bars + 2 * S + 2;
    s.tmem = reinterpret_cast<uint32_t*>(bars + 2 * S + 3);
    s.abort = reinterpret_cast<volatile int*>(bars + 2 * S + 4);
    return s;
}

struct NvTile {
    int e, nt, row0, rows;
};

// Tile t -> (expert, column tile, 128-row tile); column tiles outer within an
// expert so that consecutive CTAs share the weight tile.
__device__ __forceinline__ NvTile nv_decode(int t, const NvSmem& s, int E) {
    int lo = 0, hi = E;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s.tstart[mid] <= t) lo = mid; else hi = mid;
    }
    NvTile r;
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
__device__ __forceinline__ void nv_weight_rows(const NvTile& t, const NvParams& p, int& w0, int& w1) {
    if (p.gated) {
        w0 = t.e * p.N + t.nt * 128;
        w1 = t.e * p.N + (p.N >> 1) + t.nt * 128;
    } else {
        w0 = t.e * p.N + t.nt * 256;
        w1 = w0 + 128;
    }
}

__device__ __forceinline__ bool nv_warp_wait_spin(uint64_t* bar, uint32_t parity, const WaitCtl& wc,
                                                  int where) {
    return __all_sync(0xffffffffu, wait_bar_spin(bar, parity, wc, where)) != 0;
}
__device__ __forceinline__ bool nv_warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& wc,
                                             int where) {
    return __all_sync(0xffffffffu, wait_bar(bar, parity, wc, where)) != 0;
}

// Warp 0: lane l < 6 issues TMA box l of every stage (x = byte offset of the
// stage's 256 K elements, a multiple of 128).
template <int S>
__device__ void nv_producer(const CUtensorMap* tmA, const CUtensorMap* tmB, const NvParams& p,
                            const NvSmem& s, const WaitCtl& wc, int total) {
    const int l = threadIdx.x & 31;
    const bool issuer = l < kNvBoxes;
    const bool is_a = l < 2;
    const int b = l - 2;  // weight box 0..3: block b/2, half b%2
    const uint32_t off = is_a ? l * 64 * 128 : kNvA + b * 64 * 128;
    uint32_t stage = 0, phase = 0, armed = 0, armed_par = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const NvTile tl = nv_decode(t, s, p.E);
        int w0, w1;
        nv_weight_rows(tl, p, w0, w1);
        const int row = is_a ? tl.row0 + l * 64 : ((b >> 1) ? w1 : w0) + (b & 1) * 64;
        for (int kb = 0; kb < p.nkb; ++kb) {
            if (!nv_warp_wait_spin(&s.empty[stage], phase ^ 1, wc, 1)) { ok = false; break; }
            if (issuer) {
                mbar_arrive_expect_tx(&s.full[stage], 64 * 128);
                tma_load_2d(s.stages + stage * kNvStage + off, is_a ? tmA : tmB, &s.full[stage],
                            kb * 128, row);
            }
            __syncwarp();
            armed |= 1u << stage;
            armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
            if (++stage == S) { stage = 0; phase ^= 1; }
        }
    }
    for (int st = 0; st < S; ++st)
        if ((armed >> st) & 1u) wait_bar(&s.full[st], (armed_par >> st) & 1u, wc, 2, /*drain=*/true);
    __syncwarp();
}

// Warps 2 (weights) and 3 (activations): per stage, the 16 E4M3 scales of
// each of the tile's 256 weight rows or 128 token rows, as four 512-byte
// atoms (one per K = 64 step); completion arrives on the stage's full
// barrier.  Rows past the ends read as 0 (those outputs are not stored).
template <bool WEIGHTS, int S>
__device__ void nv_sf_loader(const NvParams& p, const NvSmem& s, const WaitCtl& wc, int total) {
    const int lane = threadIdx.x & 31;
    const int nsf = p.K >> 4;  // activation scale bytes per row
    const int natoms = p.K >> 6;
    const long long wblocks = static_cast<long long>(p.E) * p.N / 128;
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const NvTile tl = nv_decode(t, s, p.E);
        int w0, w1;
        nv_weight_rows(tl, p, w0, w1);
        for (int kb = 0; kb < p.nkb; ++kb) {
            if (!nv_warp_wait(&s.empty[stage], phase ^ 1, wc, 8)) { ok = false; break; }
            uint8_t* sf = s.stages + stage * kNvStage + kNvSfOff;
            if constexpr (WEIGHTS) {
#pragma unroll
                for (int blk = 0; blk < 2; ++blk) {
                    const long long wb = (blk ? w1 : w0) >> 7;
                    const bool v = wb < wblocks;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint8_t* src =
                            v ? p.b_sf + (wb * natoms + kb * 4 + kk) * 512 + lane * 16 : p.b_sf;
                        cp_async_16(sf + 2048 + blk * 2048 + kk * 512 + lane * 16, src, v ? 16u : 0u);
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) {  // token row lane + 32 i
                    const int r = tl.row0 + lane + 32 * i;
                    const bool v = r < p.R;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const long long off =
                            p.a_sf_mn ? (static_cast<long long>(kb * 4 + kk) * p.R + r) * 4
                                      : static_cast<long long>(r) * nsf + kb * 16 + kk * 4;
                        cp_async_4(sf + kk * 512 + lane * 16 + i * 4, v ? p.a_sf + off : p.a_sf,
                                   v ? 4u : 0u);
                    }
                }
            }
            cp_async_arrive_noinc(&s.full[stage]);
            if (++stage == S) { stage = 0; phase ^= 1; }
        }
    }
    cp_async_wait_all();
    __syncwarp();
}

// Warp 1: per stage, the 12 scale-factor atoms into TMEM and four K = 64
// block-scaled MMAs (elected lane); the accumulator is released by the
// epilogue per tile.
template <int S>
__device__ void nv_mma(const NvParams& p, const NvSmem& s, const WaitCtl& wc, uint32_t tmem_base,
                       int total) {
    uint32_t stage = 0, phase = 0, it = 0;
    bool ok = true;
    const uint32_t sfa_t = tmem_base + kNvSfaCol;
    const uint32_t sfb_t = tmem_base + kNvSfbCol;
    constexpr uint32_t idesc = idesc_nvf4(128, 256);
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
        if (!nv_warp_wait_spin(s.tempty, (it & 1) ^ 1, wc, 3)) break;
        tc_fence_after();
        for (int kb = 0; kb < p.nkb; ++kb) {
            if (!nv_warp_wait_spin(&s.full[stage], phase, wc, 4)) { ok = false; break; }
            tc_fence_after();
            uint8_t* st = s.stages + stage * kNvStage;
            const uint32_t sa = smem_u32(st);
            const uint32_t sb = smem_u32(st + kNvA);
            const uint32_t ssf = smem_u32(st + kNvSfOff);
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    tmem_cp_32x128b_x4(sfa_t + 4 * kk, smem_desc_k_noswizzle(ssf + kk * 512, 16, 128));
                    tmem_cp_32x128b_x4(sfb_t + 8 * kk,
                                       smem_desc_k_noswizzle(ssf + 2048 + kk * 512, 16, 128));
                    tmem_cp_32x128b_x4(sfb_t + 8 * kk + 4,
                                       smem_desc_k_noswizzle(ssf + 4096 + kk * 512, 16, 128));
                }
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_nvf4(tmem_base, smem_desc_k_sw128(sa + kk * 32), smem_desc_k_sw128(sb + kk * 32),
                              idesc, sfa_t + 4 * kk, sfb_t + 8 * kk, (kb | kk) != 0);
                umma_commit(&s.empty[stage]);
                if (kb == p.nkb - 1) umma_commit(s.tfull);
            }
            __syncwarp();
            if (++stage == S) { stage = 0; phase ^= 1; }
        }
    }
    if (elect_one()) umma_commit(s.drain);
    __syncwarp();
    wait_bar(s.drain, 0, wc, 5, /*drain=*/true);
    __syncwarp();
}

__device__ __forceinline__ float nv_silu(float z) { return z * rcp_approx(1.0f + __expf(-z)); }

__device__ __forceinline__ uint32_t nv_pack_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    uint32_t u;
    memcpy(&u, &h, 4);
    return u;
}

// Warps 4-11: thread = one row of the tile, 64 columns of each weight block
// (warp w: rows 32 (w % 4) .. +31, column half (w - 4) / 4).  G = alpha_e *
// accumulator; then, by mode:
//  NV_EPI_BF16            bf16 G (plain) or bf16 silu(G_gate) * G_up (gated)
//  NV_EPI_SWIGLU_NVQUANT  h = silu(G_gate) * G_up requantised to NVFP4 with
//                         the global scale h_gscale: the thread's 64 columns
//                         are four 16-column blocks, each with its own scale
//  NV_EPI_COMBINE         out_acc[token] += w * G through a shared-memory
//                         transpose (8 rows x 64 contiguous bytes per reduction)
template <int MODE>
__device__ void nv_epilogue(const NvParams& p, const NvSmem& s, const WaitCtl& wc,
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
        const NvTile tl = nv_decode(t, s, p.E);
        const bool row_ok = rl < tl.rows;
        const long long row = tl.row0 + rl;
        const float al = __ldg(p.alpha + tl.e);
        // combine: the row's pair id and weight, fetched while the tile computes
        int c_tok = -1;
        float c_w = 0.0f;
        if constexpr (MODE == NV_EPI_COMBINE) {
            if (row_ok) {
                const int pair = __ldg(p.perm + row);
                c_tok = pair / p.topk;
                c_w = __ldg(p.topk_w + pair) * al;
            }
        }
        if (!nv_warp_wait(s.tfull, it & 1, wc, 6)) return;
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
        if constexpr (MODE == NV_EPI_COMBINE) {
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
        if constexpr (MODE == NV_EPI_SWIGLU_NVQUANT) {
            const int I = p.N >> 1;
            const long long col0 = static_cast<long long>(tl.nt) * 128 + colg;  // first h column
            uint2 packed[4];
            uint32_t sf4 = 0;
#pragma unroll
            for (int b16 = 0; b16 < 4; ++b16) {
                float h[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int j = 16 * b16 + i;
                    h[i] = nv_silu(al * __uint_as_float(v[j >> 5][j & 31])) *
                           (al * __uint_as_float(v[2 + (j >> 5)][j & 31]));
                }
                sf4 |= nv_quant16(h, p.h_gscale, packed[b16]) << (8 * b16);
            }
            uint4* dst = reinterpret_cast<uint4*>(p.hq + row * (I >> 1) + (col0 >> 1));
            dst[0] = make_uint4(packed[0].x, packed[0].y, packed[1].x, packed[1].y);
            dst[1] = make_uint4(packed[2].x, packed[2].y, packed[3].x, packed[3].y);
            // the thread's 64 columns are one 64-wide K block of GEMM2
            *reinterpret_cast<uint32_t*>(p.hsf + ((col0 >> 6) * p.R + row) * 4) = sf4;
        } else if (p.gated) {
            uint4* dst = reinterpret_cast<uint4*>(p.out + row * (p.N >> 1) + tl.nt * 128 + colg);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                float h[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int j = 8 * c + i;
                    h[i] = nv_silu(al * __uint_as_float(v[j >> 5][j & 31])) *
                           (al * __uint_as_float(v[2 + (j >> 5)][j & 31]));
                }
                dst[c] = make_uint4(nv_pack_bf16(h[0], h[1]), nv_pack_bf16(h[2], h[3]),
                                    nv_pack_bf16(h[4], h[5]), nv_pack_bf16(h[6], h[7]));
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
                    dst[c] = make_uint4(
                        nv_pack_bf16(al * __uint_as_float(a[0]), al * __uint_as_float(a[1])),
                        nv_pack_bf16(al * __uint_as_float(a[2]), al * __uint_as_float(a[3])),
                        nv_pack_bf16(al * __uint_as_float(a[4]), al * __uint_as_float(a[5])),
                        nv_pack_bf16(al * __uint_as_float(a[6]), al * __uint_as_float(a[7])));
                }
            }
        }
    }
}

template <int MODE>
__global__ void __launch_bounds__(kNvThreads, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const NvParams p) {
    constexpr int S = NvCfg<MODE>::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const NvSmem s = nv_carve<MODE>(base);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&s.full[i], kNvBoxes + 64);  // TMA lanes + two scale-loader warps
            mbar_init(&s.empty[i], 1);
        }
        mbar_init(s.tfull, 1);
        mbar_init(s.tempty, kNvEpiWarps);
        mbar_init(s.drain, 1);
        *s.abort = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(s.tmem, kNvTmemCols);
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
    if (warp == 0) nv_producer<S>(&tmA, &tmB, p, s, wc, total);
    else if (warp == 1) nv_mma<S>(p, s, wc, tmem_base, total);
    else if (warp == 2) nv_sf_loader<true, S>(p, s, wc, total);
    else if (warp == 3) nv_sf_loader<false, S>(p, s, wc, total);
    else nv_epilogue<MODE>(p, s, wc, tmem_base, total);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kNvTmemCols);
}

// x [T, H] bf16 -> NVFP4 codes xq [R, H/2] and scales xsf at rows
// inv_perm[t*k + j] (row t when inv_perm is null and k = 1; global scale g),
// xsf row-major [R, H/16] or, when sf_mn, K-block-major [H/64, R, 4];
// also zeroes out_acc [T, H] when not null.  Warp per (token, 512 columns),
// lane = one 16-column block: one 32-byte load, one 8-byte code store and
// one scale byte per destination row (a warp writes 256 + 32 contiguous
// bytes per row).
__global__ void __launch_bounds__(256) nv_quant_scatter_kernel(
    const __nv_bfloat16* __restrict__ x, int T, int H, int k, float g,
    const int32_t* __restrict__ inv_perm, uint8_t* __restrict__ xq, uint8_t* __restrict__ xsf,
    int R, int sf_mn, float* __restrict__ out_acc) {
    const int nch = (H + 511) >> 9;
    const long long item = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const long long items = static_cast<long long>(T) * nch;
    if (item >= items) return;
    const int lane = threadIdx.x & 31;
    const int t = items <= 0x7fffffffll ? static_cast<int>(item) / nch : static_cast<int>(item / nch);
    const int col = static_cast<int>(item - static_cast<long long>(t) * nch) * 512 + lane * 16;
    if (col >= H) return;
    const long long off = static_cast<long long>(t) * H + col;
    const uint4* src = reinterpret_cast<const uint4*>(x + off);
    const uint4 r0 = src[0], r1 = src[1];
    const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
    float v[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        __nv_bfloat162 b2;
        memcpy(&b2, &w[i], 4);
        const float2 f = __bfloat1622float2(b2);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
    uint2 packed;
    const uint32_t code = nv_quant16(v, g, packed);
    for (int j = 0; j < k; ++j) {
        const int row = inv_perm ? inv_perm[t * k + j] : t;
        if (row < 0) continue;
        *reinterpret_cast<uint2*>(xq + static_cast<long long>(row) * (H >> 1) + (col >> 1)) = packed;
        const long long so = sf_mn ? (static_cast<long long>(col >> 6) * R + row) * 4 + ((col >> 4) & 3)
                                   : static_cast<long long>(row) * (H >> 4) + (col >> 4);
        xsf[so] = static_cast<uint8_t>(code);
    }
    if (out_acc) {
        float4* o = reinterpret_cast<float4*>(out_acc + off);
#pragma unroll
        for (int i = 0; i < 4; ++i) o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// Row-major activation scales [R, A] 4-byte words (A = K/64: the four scales
// of a 64-wide K block) -> K-block-major [A, R] words, through a 32 x 32
// shared-memory tile (reads and writes 128 contiguous bytes per warp).
__global__ void __launch_bounds__(256) nv_sf_kblock_major_kernel(const uint32_t* __restrict__ rm,
                                                                 uint32_t* __restrict__ mn, int R,
                                                                 int A) {
    __shared__ uint32_t tile[32][33];
    const int a0 = blockIdx.x * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    const int ntiles = (R + 31) / 32;
    for (int rt = blockIdx.y; rt < ntiles; rt += gridDim.y) {  // row tiles, grid-stride
        const int r0 = rt * 32;
        for (int i = ty; i < 32; i += 8) {
            const int r = r0 + i, a = a0 + tx;
            if (r < R && a < A) tile[i][tx] = rm[static_cast<long long>(r) * A + a];
        }
        __syncthreads();
        for (int i = ty; i < 32; i += 8) {
            const int a = a0 + i, r = r0 + tx;
            if (r < R && a < A) mn[static_cast<long long>(a) * R + r] = tile[tx][i];
        }
        __syncthreads();
    }
}

template <int MODE>
int launch_nv_inst(const CUtensorMap& ma, const CUtensorMap& mb, const NvParams& p, int num_sms,
                   cudaStream_t stream) {
    static int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        if (cudaFuncSetAttribute(nvfp4_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 NvCfg<MODE>::SMEM) != cudaSuccess)
            return ST_CUDA;
        configured_dev = dev;
    }
    nvfp4_gemm_kernel<MODE><<<num_sms, kNvThreads, NvCfg<MODE>::SMEM, stream>>>(ma, mb, p);
    return cudaGetLastError() == cudaSuccess ? ST_OK : ST_CUDA;
}

}  // namespace

int launch_nvfp4_gemm(const NvGemmArgs& g, cudaStream_t stream) {
    if (g.R <= 0 || g.E <= 0) return ST_OK;
    if (g.E > kNvMaxE) return ST_INVALID_ARG;
    CUtensorMap ma, mb;
    // packed rows: K / 2 bytes; a TMA box is 64 rows x 128 bytes (256 elements)
    if (!make_tma_map_fp8(&ma, g.a, g.R, g.K / 2, 64)) return ST_CUDA;
    if (!make_tma_map_fp8(&mb, g.b, static_cast<long long>(g.E) * g.N, g.K / 2, 64)) return ST_CUDA;
    NvParams p{};
    p.R = g.R; p.N = g.N; p.K = g.K; p.E = g.E; p.nkb = g.K / 256; p.gated = g.gated ? 1 : 0;
    p.a_sf_mn = g.a_sf_mn ? 1 : 0;
    p.a_sf = g.a_sf; p.b_sf = g.b_sf; p.alpha = g.alpha; p.m_indptr = g.m_indptr;
    p.out = static_cast<__nv_bfloat16*>(g.out);
    p.hq = g.hq; p.hsf = g.hsf; p.h_gscale = g.h_gscale;
    p.perm = g.perm; p.topk_w = g.topk_w; p.topk = g.topk > 0 ? g.topk : 1;
    p.out_acc = g.out_acc; p.out_ld = g.out_ld;
    p.status = g.status;
    p.timeout_ns = g.timeout_ns;
    switch (g.epi) {
        case NV_EPI_SWIGLU_NVQUANT:
            return launch_nv_inst<NV_EPI_SWIGLU_NVQUANT>(ma, mb, p, g.num_sms, stream);
        case NV_EPI_COMBINE:
            return launch_nv_inst<NV_EPI_COMBINE>(ma, mb, p, g.num_sms, stream);
        default:
            return launch_nv_inst<NV_EPI_BF16>(ma, mb, p, g.num_sms, stream);
    }
}

int launch_nv_quant_scatter(const void* x, int T, int H, int k, float g, const int32_t* inv_perm,
                            uint8_t* xq, uint8_t* xsf, int R, int sf_mn, float* out_acc,
                            cudaStream_t stream) {
    const long long items = static_cast<long long>(T) * ((H + 511) / 512);
    if (items == 0) return ST_OK;
    const long long blocks = (items + 7) / 8;
    nv_quant_scatter_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(x), T, H, k, g, inv_perm, xq, xsf, R, sf_mn, out_acc);
    return cudaGetLastError() == cudaSuccess ? ST_OK : ST_CUDA;
}

int launch_nv_sf_kblock_major(const uint8_t* rm, uint8_t* mn, int R, int K, cudaStream_t stream) {
    const int A = K / 64;
    if (R == 0 || A == 0) return ST_OK;
    const int row_tiles = (R + 31) / 32;
    const dim3 grid((A + 31) / 32, row_tiles < 65535 ? row_tiles : 65535);
    nv_sf_kblock_major_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint32_t*>(rm),
                                                        reinterpret_cast<uint32_t*>(mn), R, A);
    return cudaGetLastError() == cudaSuccess ? ST_OK : ST_CUDA;
}

}  // namespace moe
