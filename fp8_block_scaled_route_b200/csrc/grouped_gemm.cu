// Grouped FP8 GEMM with 128x128 block scales on sm_100a (tcgen05 + TMEM + TMA).
//
// Computes, for every expert e and grouped row r of that expert (rows
// [m_indptr[e], m_indptr[e+1]) of A):
//   G[r, n] = sum_kb a_scale(r, kb) * b_scale[e, n/128, kb] * sum_{k in kb} A[r, k] * B[e, n, k]
// which is stage 1 (gate/up projection) and stage 4 (down projection) of the
// expert pipeline on the page "FlashInfer: Blackwell W8A8 AlphaMoE Expert
// 계산 커널 퓨전으로 성능 비약적 향상" (flashinfer PR #4287, section
// "문제점: MoE Expert 계산의 병목"), with the grouped "nt" interface of the page
// "FlashInfer SM120 MoE GEMM 최적화: 웨이브+잔여물 비용 모델 도입" (flashinfer
// PR #4318, "코드 분석 1.").  The epilogue fuses the next stages: SwiGLU and
// FP8 requantisation of the intermediate (stages 2-3), or the router-weighted
// combine (stage 5), or a bf16 store for the standalone GEMM.
//
// Design (one persistent CTA per SM, warp-specialised):
//  * warp 0 lane 0 - producer: TMA loads of a token tile [BT x 128] and a
//    weight tile [256 x 128] (two 128-row boxes) per 128-wide K block into
//    a multi-stage shared-memory ring (128-byte swizzle).
//  * warp 1 - allocates TMEM; lane 0 issues tcgen05.mma kind::f8f6f4 (K=32
//    per instruction, four per K block).  Each K block is accumulated into a
//    fresh TMEM buffer (two buffers, ping-pong) because the fp32 block scales
//    are not powers of two and must be applied per K block.
//  * epilogue warps - read each K-block partial out of TMEM, multiply by
//    a_scale * b_scale and accumulate in fp32 registers; after the last K
//    block they run the fused epilogue.
//  Two orientations:
//  * BT = 128 ("direct"): tokens are the MMA M operand (M=128), the 256
//    weight rows are N.  8 epilogue warps; each thread owns one token row and
//    128 of the 256 columns.  Register split via setmaxnreg.
//  * BT = 16/32/64 ("swapped", the small-M path): the weights are the MMA M
//    operand (two M=128 MMAs, one per 128-row weight block) and the tokens
//    are N = BT.  4 epilogue warps; each thread owns one weight row.
//  Every wait is bounded by %globaltimer; on expiry the CTA records
//  ST_DEVICE_TIMEOUT, drains its in-flight copies and MMAs, frees TMEM and
//  returns.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "gemm_common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kSmemLimit = 232448;  // 227 KB of opt-in dynamic shared memory per CTA
constexpr int kMaxE = 1024;
constexpr int kTableBytes = ((2 * (kMaxE + 1) * 4) + 15) / 16 * 16;
constexpr int kScaleSlots = 8;        // depth of the direct kernel's scale ring
constexpr int kScaleSlotFloats = 132;  // a_scale of 128 rows, then b_scale of the two blocks
// Register split of the direct kernel (384 threads x 168 registers at launch):
// the producer/MMA warpgroup drops to 56, the two epilogue warpgroups rise to
// 224:  128*56 + 256*224 = 64512 = 384*168.
constexpr int kDirectLaunchRegs = 168;
constexpr int kDirectLowRegs = 56;
constexpr int kDirectHighRegs = 224;
static_assert(128 * kDirectLowRegs + 256 * kDirectHighRegs <= 384 * kDirectLaunchRegs,
              "register split exceeds the launch allocation");

template <int BT>
struct Cfg {
    static constexpr bool SWAP = BT < 128;
    static constexpr int EPI_WARPS = SWAP ? 4 : 8;
    static constexpr int EPI_THREADS = EPI_WARPS * 32;
    static constexpr int THREADS = 128 + EPI_THREADS;
    static constexpr int A_BYTES = BT * 128;       // token tile per stage
    static constexpr int B_BYTES = 256 * 128;      // weight tile per stage
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int A_OFF = SWAP ? B_BYTES : 0;
    static constexpr int B_OFF = SWAP ? 0 : A_BYTES;
    static constexpr int AS_TILE_BYTES = SWAP ? 32768 : 0;  // a_scale staging [nkb][BT]
    static constexpr int XCH_BYTES = SWAP ? ((4 * BT + 2 * BT) * 4 + 15) / 16 * 16 : 2 * 128 * 4;
    static constexpr int SCALE_BYTES = SWAP ? 0 : kScaleSlots * kScaleSlotFloats * 4;
    // direct: area after the last pipeline stage that, with that stage, stages
    // the EPI_Y32 output boxes (16 KB)
    static constexpr int CST_BYTES = SWAP ? 0 : EPI_WARPS * 32 * 16 * 4;
    static constexpr int BAR_BYTES = 1024;
    static constexpr int FIXED =
        1024 + AS_TILE_BYTES + SCALE_BYTES + CST_BYTES + kTableBytes + XCH_BYTES + BAR_BYTES;
    static constexpr int STAGES_FIT = (kSmemLimit - FIXED) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
    static constexpr int SMEM_BYTES = FIXED + STAGES * STAGE_BYTES;
    static constexpr uint32_t TMEM_COLS = 512;
    // TMEM accumulator slots, each holding both 128-row weight blocks of one
    // K block: direct = 2 slots of 256 columns (one N = 256 MMA per K step);
    // swapped = up to 16 slots of 2 x BT columns, so the weight stream keeps
    // going while the epilogue finishes a tile.  (Four 128-column slots with
    // two N = 128 MMA groups per K block, each with its own commit and
    // release, measured 15% slower for GEMM1: twice the handshakes per K
    // block and the token tile read twice by the tensor core.)
    static constexpr int TSLOTS = SWAP ? (512 / (2 * BT) > 16 ? 16 : 512 / (2 * BT)) : 2;
    static constexpr int TBUF_COLS = SWAP ? 2 * BT : 256;
    static constexpr int MAX_NKB = SWAP ? AS_TILE_BYTES / (4 * BT) : 1 << 20;
    // TMA boxes per stage, one per issuing producer lane: the token tile in
    // boxes of at most 64 rows, and the 256 weight rows in four 64-row boxes.
    // A single thread's TMA issue rate (about 40 B/clk) cannot feed the MMA;
    // several lanes issuing in parallel can.
    static constexpr int A_BOX_ROWS = BT < 64 ? BT : 64;
    static constexpr int A_BOXES = BT / A_BOX_ROWS;
    static constexpr int NBOX = A_BOXES + 4;
    static_assert(STAGES >= 3, "pipeline too shallow");
    static_assert(SMEM_BYTES <= kSmemLimit, "shared memory budget");
    static_assert(STAGE_BYTES % 1024 == 0 && A_OFF % 1024 == 0 && B_OFF % 1024 == 0,
                  "operand tiles must be 1024-byte aligned for the 128-byte swizzle");
    // EPI_Y32 (direct): the last pipeline stage and the combine transpose
    // area, contiguous, become the staging buffers of the output stores: two
    // 4 KB boxes (32 rows x 32 fp32, 128-byte swizzle) per epilogue warp.
    static constexpr int Y_STAGE_BYTES = SWAP ? 0 : EPI_WARPS * 2 * 4096;
    static_assert(SWAP || STAGE_BYTES + CST_BYTES >= Y_STAGE_BYTES, "output staging does not fit");
};

struct KParams {
    int R, N, K, E, nkb;
    // Tiles are ordered by expert, then column tile, then row tile; ntn
    // column tiles per expert.
    int ntn;
    const float* a_scale;
    long long as_row, as_kb;
    const float* b_scale;
    const int32_t* m_indptr;
    uint8_t* hq;
    float* hs;
    float* y;
    int ldy;
    const int32_t* rowmap;
    // A row map: grouped row r reads row a_rowmap[r] / a_rowdiv of A and of
    // its scales (null: row r); a_rows = rows of A
    const int32_t* a_rowmap;
    int a_rowdiv;
    int a_rows;
    __nv_bfloat16* out_bf16;
    int* status;
    unsigned long long timeout_ns;
    int nstages;  // pipeline stages in use (EPI_Y32 direct: one less, its space stages the output)
};

struct Smem {
    uint8_t* stages;
    float* as_tile;
    int* tstart;  // [E+1] first tile of each expert
    int* mind;    // [E+1] clamped m_indptr
    float* xch;   // epilogue exchange area
    float* scales;  // direct kernel: kScaleSlots x {a_scale[128], b_scale[2], pad[2]}
    uint8_t* ystage;  // direct EPI_Y32 output staging (the last stage and the area after it)
    uint64_t* full;
    uint64_t* empty;
    uint64_t* tfull;
    uint64_t* tempty;
    uint64_t* drain;
    uint64_t* epi;
    uint64_t* sfull;
    uint64_t* sempty;
    uint32_t* tmem;
    volatile int* abort;
};

template <int BT>
__device__ __forceinline__ Smem carve(uint8_t* base) {
    using C = Cfg<BT>;
    Smem s;
    uint8_t* p = base;
    s.stages = p;
    p += C::STAGES * C::STAGE_BYTES;
    s.ystage = base + (C::STAGES - 1) * C::STAGE_BYTES;
    p += C::CST_BYTES;
    s.as_tile = reinterpret_cast<float*>(p);
    p += C::AS_TILE_BYTES;
    s.tstart = reinterpret_cast<int*>(p);
    s.mind = s.tstart + (kMaxE + 1);
    p += kTableBytes;
    s.xch = reinterpret_cast<float*>(p);
    p += C::XCH_BYTES;
    s.scales = reinterpret_cast<float*>(p);
    p += C::SCALE_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(p);
    s.full = bars;
    s.empty = bars + 8;
    s.tfull = bars + 16;
    s.tempty = bars + 32;
    s.drain = bars + 48;
    s.epi = bars + 49;
    s.sfull = bars + 50;
    s.sempty = bars + 50 + kScaleSlots;
    s.tmem = reinterpret_cast<uint32_t*>(bars + 50 + 2 * kScaleSlots);
    s.abort = reinterpret_cast<volatile int*>(bars + 51 + 2 * kScaleSlots);
    return s;
}

struct Tile {
    int e, mt, nt, row0, rows;
};

// Total tiles of the launch.
__device__ __forceinline__ int total_tiles(const Smem& s, const KParams& p) {
    return s.tstart[p.E];
}

template <int BT>
__device__ __forceinline__ Tile decode_tile(int t, const Smem& s, const KParams& p) {
    const int E = p.E;
    int lo = 0, hi = E;  // tstart[lo] <= t < tstart[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s.tstart[mid] <= t) lo = mid; else hi = mid;
    }
    Tile r;
    r.e = lo;
    const int local = t - s.tstart[lo];
    const int me = max(0, s.mind[lo + 1] - s.mind[lo]);
    const int mtiles = (me + BT - 1) / BT;
    r.nt = local / mtiles;
    r.mt = local - r.nt * mtiles;
    r.row0 = s.mind[lo] + r.mt * BT;
    r.rows = min(BT, me - r.mt * BT);
    return r;
}

// Weight-tile geometry of a tile: global B rows of the two 128-row boxes and
// the scale-block indices (into b_scale viewed as [E * N/128, nkb]).
struct WTile {
    int wrow0, wrow1;
    int sb0, sb1;
    bool v1;  // second block exists (plain tiles may end on an odd block)
};

template <bool GATED>
__device__ __forceinline__ WTile weight_tile(const Tile& t, int N) {
    WTile w;
    const int nblk = N >> 7;
    if (GATED) {
        w.wrow0 = t.e * N + t.nt * 128;
        w.wrow1 = t.e * N + (N >> 1) + t.nt * 128;
        w.sb0 = t.e * nblk + t.nt;
        w.sb1 = t.e * nblk + (nblk >> 1) + t.nt;
        w.v1 = true;
    } else {
        w.wrow0 = t.e * N + t.nt * 256;
        w.wrow1 = w.wrow0 + 128;
        w.sb0 = t.e * nblk + 2 * t.nt;
        w.v1 = (2 * t.nt + 1) < nblk;
        w.sb1 = w.v1 ? w.sb0 + 1 : w.sb0;
    }
    return w;
}

// Row of A (and of its scales) that grouped row `row` reads.
__device__ __forceinline__ int a_src_row(const KParams& p, int row) {
    if (!p.a_rowmap) return row;
    const int r = min(max(row, 0), p.R - 1);
    const int src = __ldg(p.a_rowmap + r) / p.a_rowdiv;
    return min(max(src, 0), p.a_rows - 1);
}

__device__ __forceinline__ float a_scale_at(const KParams& p, int row, int kb) {
    return p.a_scale[static_cast<long long>(row) * p.as_row + static_cast<long long>(kb) * p.as_kb];
}

__device__ __forceinline__ bool epi_sync(const Smem& s, uint32_t& phase, const WaitCtl& wc) {
    mbar_arrive(s.epi);
    const bool ok = warp_wait(s.epi, phase, wc, 7);
    phase ^= 1;
    return ok;
}

// ---------------------------------------------------------------- roles
// Producer (all of warp 0, converged): lane l < NBOX issues box l of every
// stage.
template <int BT, bool GATED>
__device__ void producer_role(const CUtensorMap* tmA, const CUtensorMap* tmB, const KParams& p,
                              const Smem& s, const WaitCtl& wc) {
    using C = Cfg<BT>;
    const int l = threadIdx.x & 31;
    // Tiled A (no row map): lane l < NBOX issues box l: A boxes first, then
    // the four 64-row weight boxes; each lane arms the barrier with its own
    // bytes.  Gathered A (row map): lane l < BT/4 loads token rows 4l..4l+3
    // with one gather4, lanes 0-3 also issue the weight boxes, and lane 0
    // arms the barrier with the whole stage.
    const bool gather = p.a_rowmap != nullptr;
    const bool issuer = l < C::NBOX;
    const bool is_a = l < C::A_BOXES;
    const int b = gather ? l : l - C::A_BOXES;  // weight box 0..3: block b/2, half b%2
    const bool b_lane = gather ? l < 4 : (issuer && !is_a);
    const bool g_lane = gather && l < BT / 4;
    const uint32_t off = is_a ? C::A_OFF + l * C::A_BOX_ROWS * 128 : C::B_OFF + b * 64 * 128;
    const uint32_t bytes = is_a ? C::A_BOX_ROWS * 128 : 64 * 128;
    uint32_t stage = 0, phase = 0, armed = 0, armed_par = 0;
    const int total = total_tiles(s, p);
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const Tile tl = decode_tile<BT>(t, s, p);
        const WTile wt = weight_tile<GATED>(tl, p.N);
        const int wrow = ((b >> 1) ? wt.wrow1 : wt.wrow0) + (b & 1) * 64;
        const int row = is_a ? tl.row0 + l * C::A_BOX_ROWS : wrow;
        // gathered rows of this lane (rows past the tile's end read its first row)
        int g0 = 0, g1 = 0, g2 = 0, g3 = 0;
        if (g_lane) {
            const int r = tl.row0 + 4 * l;
            g0 = a_src_row(p, 4 * l + 0 < tl.rows ? r + 0 : tl.row0);
            g1 = a_src_row(p, 4 * l + 1 < tl.rows ? r + 1 : tl.row0);
            g2 = a_src_row(p, 4 * l + 2 < tl.rows ? r + 2 : tl.row0);
            g3 = a_src_row(p, 4 * l + 3 < tl.rows ? r + 3 : tl.row0);
        }
        for (int kb = 0; kb < p.nkb; ++kb) {
            if (!warp_wait_spin(&s.empty[stage], phase ^ 1, wc, 1)) { ok = false; break; }
            uint8_t* st = s.stages + stage * C::STAGE_BYTES;
            if (gather) {
                if (l == 0) mbar_arrive_expect_tx(&s.full[stage], C::STAGE_BYTES);
                __syncwarp();
                if (g_lane)
                    tma_gather4_2d(st + C::A_OFF + l * 4 * 128, tmA, &s.full[stage], kb * 128, g0,
                                   g1, g2, g3);
                if (b_lane)
                    tma_load_2d(st + C::B_OFF + b * 64 * 128, tmB, &s.full[stage], kb * 128, wrow);
            } else if (issuer) {
                mbar_arrive_expect_tx(&s.full[stage], bytes);
                tma_load_2d(st + off, is_a ? tmA : tmB, &s.full[stage], kb * 128, row);
            }
            __syncwarp();
            armed |= 1u << stage;
            armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
            if (++stage == static_cast<uint32_t>(p.nstages)) { stage = 0; phase ^= 1; }
        }
    }
    // make sure no copy is still writing into shared memory when the CTA exits
    for (int st = 0; st < C::STAGES; ++st)
        if ((armed >> st) & 1u) wait_bar(&s.full[st], (armed_par >> st) & 1u, wc, 2, /*drain=*/true);
    __syncwarp();
}

// MMA issue (all of warp 1, converged; one elected lane issues).  Each K
// block goes into TMEM slot j: direct = one 128 x 256 MMA per K step (both
// weight blocks); swapped = one 128 x BT MMA per weight block per K step.
template <int BT>
__device__ void mma_role(const KParams& p, const Smem& s, const WaitCtl& wc, uint32_t tmem_base) {
    using C = Cfg<BT>;
    constexpr uint32_t idesc = C::SWAP ? idesc_e4m3_f32(128, BT) : idesc_e4m3_f32(128, 256);
    uint32_t stage = 0, phase = 0, j = 0, jphase = 0;
    const int total = total_tiles(s, p);
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        for (int kb = 0; kb < p.nkb; ++kb) {
            if (!warp_wait_spin(&s.tempty[j], jphase ^ 1, wc, 3)) { ok = false; break; }
            if (!warp_wait_spin(&s.full[stage], phase, wc, 4)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sa = smem_u32(s.stages + stage * C::STAGE_BYTES + C::A_OFF);
            const uint32_t sb = smem_u32(s.stages + stage * C::STAGE_BYTES + C::B_OFF);
            const uint32_t d = tmem_base + j * C::TBUF_COLS;
            if (!elect_one()) {
                // lanes that do not issue
            } else if constexpr (C::SWAP) {
                // weight block 0 into columns [0, BT), block 1 into [BT, 2BT)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    umma_f8(d, smem_desc_k_sw128(sb + kk * 32), smem_desc_k_sw128(sa + kk * 32),
                            idesc, kk);
                    umma_f8(d + BT, smem_desc_k_sw128(sb + 16384 + kk * 32),
                            smem_desc_k_sw128(sa + kk * 32), idesc, kk);
                }
                umma_commit(&s.empty[stage]);
                umma_commit(&s.tfull[j]);
            } else {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f8(d, smem_desc_k_sw128(sa + kk * 32), smem_desc_k_sw128(sb + kk * 32),
                            idesc, kk);
                umma_commit(&s.empty[stage]);
                umma_commit(&s.tfull[j]);
            }
            __syncwarp();
            if (++j == C::TSLOTS) { j = 0; jphase ^= 1; }
            if (++stage == static_cast<uint32_t>(p.nstages)) { stage = 0; phase ^= 1; }
        }
    }
    // every MMA this warp issued must be complete before TMEM is freed; the
    // drain commit comes from the lane that issued (elect.sync picks the same
    // lane of a converged warp every time)
    if (elect_one()) umma_commit(s.drain);
    __syncwarp();
    wait_bar(s.drain, 0, wc, 5, /*drain=*/true);
    __syncwarp();
}

// Scale stager of the direct kernel (warp 2): for every K block of every
// tile, in the pipeline's order, copies the tile's 128 activation scales of
// that K block and the two weight-block scales into a ring of shared-memory
// slots with cp.async; each lane's copies complete on the slot's mbarrier, so
// the stager never waits for global memory and runs up to kScaleSlots K
// blocks ahead of the epilogue.
template <bool GATED>
__device__ void scale_role(const KParams& p, const Smem& s, const WaitCtl& wc) {
    const int lane = threadIdx.x & 31;
    const int total = total_tiles(s, p);
    const int nkb = p.nkb;
    uint32_t slot = 0, sphase = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
        const Tile tl = decode_tile<128>(t, s, p);
        const WTile wt = weight_tile<GATED>(tl, p.N);
        const float* bs0 = p.b_scale + static_cast<long long>(wt.sb0) * nkb;
        const float* bs1 = p.b_scale + static_cast<long long>(wt.sb1) * nkb;
        int srow[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            srow[i] = lane + 32 * i < tl.rows ? a_src_row(p, tl.row0 + lane + 32 * i) : 0;
        for (int kb = 0; kb < nkb; ++kb) {
            if (!wait_bar(&s.sempty[slot], sphase ^ 1, wc, 8)) return;
            float* f = s.scales + slot * kScaleSlotFloats;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = lane + 32 * i;
                const bool ok = r < tl.rows;
                const float* src = ok ? p.a_scale + static_cast<long long>(srow[i]) * p.as_row +
                                            static_cast<long long>(kb) * p.as_kb
                                      : p.b_scale;
                cp_async_4(f + r, src, ok ? 4u : 0u);
            }
            if (lane == 0) cp_async_4(f + 128, bs0 + kb, 4u);
            if (lane == 1) cp_async_4(f + 129, bs1 + kb, 4u);
            cp_async_arrive_noinc(&s.sfull[slot]);
            if (++slot == kScaleSlots) { slot = 0; sphase ^= 1; }
        }
    }
    // copies still in flight land before the CTA exits
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// Direct orientation epilogue: thread = one token row, 128 of 256 columns.
template <int EPI>
__device__ void epilogue_direct(const KParams& p, const Smem& s, const WaitCtl& wc,
                                uint32_t tmem_base, const CUtensorMap* tmY) {
    constexpr bool GATED = (EPI == EPI_SWIGLU_BF16 || EPI == EPI_SWIGLU_QUANT);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3;          // TMEM lane quarter this warp may access
    const int g = (warp - 4) >> 2;   // column half
    const int rl = q * 32 + lane;    // row inside the tile
    // Each thread accumulates 64 columns of each of the tile's two 128-row
    // weight blocks: acc[0..63] = block 0 columns g*64.., acc[64..127] =
    // block 1 columns g*64.. (gated: gate and up; plain: the tile's first and
    // second 128 output columns).
    const int colg = g * 64;
    uint32_t tj = 0, tjphase = 0, ephase = 0, slot = 0, sphase = 0;
    uint32_t ybuf = 0;  // EPI_Y32: output boxes staged so far by this warp
    const int total = total_tiles(s, p);
    const int nkb = p.nkb;
    float2 acc[64];
    uint32_t va[32], vb[32];
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
        const Tile tl = decode_tile<128>(t, s, p);
        const WTile wt = weight_tile<GATED>(tl, p.N);
        const bool row_ok = rl < tl.rows;
        const int row = tl.row0 + rl;
        const bool v1 = GATED ? true : wt.v1;   // plain tiles may lack the second block
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.0f, 0.0f);
        const uint32_t tlane = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + colg;
        for (int kb = 0; kb < nkb; ++kb) {
            if (!warp_wait(&s.tfull[tj], tjphase, wc, 6)) return;
            tc_fence_after();
            const uint32_t tb = tlane + tj * 256;
            // weight block 0 columns: two 32-column loads, one wait
            tmem_ld32_async(tb, va);
            tmem_ld32_async(tb + 32, vb);
            if (!warp_wait(&s.sfull[slot], sphase, wc, 9)) return;
            const float* sl = s.scales + slot * kScaleSlotFloats;
            const float a_s = sl[rl];
            const float fA = a_s * sl[128];
            const float fB = a_s * sl[129];
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.sempty[slot]);
            if (++slot == kScaleSlots) { slot = 0; sphase ^= 1; }
            tmem_wait_ld(va);
            tmem_wait_ld(vb);
            // block 1 loads reuse each staging buffer as soon as its FMAs are issued
            ffma_chunk(acc, va, fA);
            tmem_ld32_async(tb + 128, va);
            ffma_chunk(acc + 16, vb, fA);
            tmem_ld32_async(tb + 160, vb);
            tmem_wait_ld(va);
            tmem_wait_ld(vb);
            // the TMEM slot is no longer read: hand it back before the last FMAs
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.tempty[tj]);
            tj ^= 1;
            if (tj == 0) tjphase ^= 1;
            ffma_chunk(acc + 32, va, fB);
            ffma_chunk(acc + 48, vb, fB);
        }
        const float* accf = reinterpret_cast<const float*>(acc);

        if constexpr (EPI == EPI_SWIGLU_QUANT) {
            float h[64];
            float amax = 0.0f;
#pragma unroll
            for (int j = 0; j < 64; ++j) {
                h[j] = silu_fast(accf[j]) * accf[64 + j];
                amax = fmaxf(amax, fabsf(h[j]));
            }
            s.xch[g * 128 + rl] = amax;
            if (!epi_sync(s, ephase, wc)) return;
            amax = fmaxf(s.xch[rl], s.xch[128 + rl]);
            const float sc = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
            const float inv = __frcp_rn(sc);
            if (row_ok) {
                const int ldh = p.N >> 1;
                uint4* dst = reinterpret_cast<uint4*>(p.hq + static_cast<long long>(row) * ldh +
                                                      tl.nt * 128 + g * 64);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint4 w;
                    w.x = cvt_e4m3x4(h[16 * c + 0] * inv, h[16 * c + 1] * inv, h[16 * c + 2] * inv,
                                     h[16 * c + 3] * inv);
                    w.y = cvt_e4m3x4(h[16 * c + 4] * inv, h[16 * c + 5] * inv, h[16 * c + 6] * inv,
                                     h[16 * c + 7] * inv);
                    w.z = cvt_e4m3x4(h[16 * c + 8] * inv, h[16 * c + 9] * inv, h[16 * c + 10] * inv,
                                     h[16 * c + 11] * inv);
                    w.w = cvt_e4m3x4(h[16 * c + 12] * inv, h[16 * c + 13] * inv,
                                     h[16 * c + 14] * inv, h[16 * c + 15] * inv);
                    dst[c] = w;
                }
                if (g == 0) p.hs[static_cast<long long>(tl.nt) * p.R + row] = sc;
            }
            if (!epi_sync(s, ephase, wc)) return;
        } else if constexpr (EPI == EPI_Y32) {
            // The warp's 32 rows x 128 columns leave as four 32 x 32 fp32
            // boxes through two 4 KB shared-memory buffers and TMA stores,
            // which the TMA unit drains while the warp goes on with the next
            // tile.  Buffer layout = the 128-byte swizzle of the tensor map:
            // 16-byte chunk c of row r sits at chunk c ^ (r % 8), so the eight
            // lanes of each store phase hit eight different bank groups.  A
            // quarter with fewer than 32 valid rows (the tile's last rows
            // belong to the next expert) is written with plain stores.
            uint8_t* const wbuf = s.ystage + (warp - 4) * 8192;
            const int rows_here = tl.rows - q * 32;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int blk = c >> 1;
                if (blk == 1 && !v1) break;
                const float* a = accf + blk * 64 + (c & 1) * 32;
                const int col = tl.nt * 256 + blk * 128 + colg + (c & 1) * 32;
                if (p.rowmap) {
                    // rows go to scattered places: plain stores of the thread's own row
                    if (row_ok) {
                        float4* dst = reinterpret_cast<float4*>(
                            p.y + static_cast<long long>(__ldg(p.rowmap + row)) * p.ldy + col);
#pragma unroll
                        for (int c4 = 0; c4 < 8; ++c4)
                            dst[c4] = make_float4(a[4 * c4], a[4 * c4 + 1], a[4 * c4 + 2], a[4 * c4 + 3]);
                    }
                } else if (rows_here >= 32) {
                    uint8_t* buf = wbuf + (ybuf & 1u) * 4096;
                    if (lane == 0) bulk_wait_group_read<1>();  // the box staged two boxes ago is read
                    __syncwarp();
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4)
                        *reinterpret_cast<float4*>(buf + lane * 128 + ((c4 ^ (lane & 7)) << 4)) =
                            make_float4(a[4 * c4], a[4 * c4 + 1], a[4 * c4 + 2], a[4 * c4 + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(tmY, buf, col, tl.row0 + q * 32);
                        bulk_commit_group();
                    }
                    ++ybuf;
                } else if (lane < rows_here) {
                    float4* dst = reinterpret_cast<float4*>(p.y + static_cast<long long>(row) * p.ldy + col);
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4)
                        dst[c4] = make_float4(a[4 * c4], a[4 * c4 + 1], a[4 * c4 + 2], a[4 * c4 + 3]);
                }
            }
        } else if constexpr (EPI == EPI_BF16) {
            if (row_ok) {
                __nv_bfloat16* rowp = p.out_bf16 + static_cast<long long>(row) * p.N + tl.nt * 256 + colg;
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    if (c >= 8 && !v1) break;
                    uint4* dst = reinterpret_cast<uint4*>(rowp + (c < 8 ? 8 * c : 128 + 8 * (c - 8)));
                    uint4 w;
                    __nv_bfloat162 b0 = __floats2bfloat162_rn(accf[8 * c + 0], accf[8 * c + 1]);
                    __nv_bfloat162 b1 = __floats2bfloat162_rn(accf[8 * c + 2], accf[8 * c + 3]);
                    __nv_bfloat162 b2 = __floats2bfloat162_rn(accf[8 * c + 4], accf[8 * c + 5]);
                    __nv_bfloat162 b3 = __floats2bfloat162_rn(accf[8 * c + 6], accf[8 * c + 7]);
                    memcpy(&w.x, &b0, 4); memcpy(&w.y, &b1, 4);
                    memcpy(&w.z, &b2, 4); memcpy(&w.w, &b3, 4);
                    *dst = w;
                }
            }
        } else {  // EPI_SWIGLU_BF16
            if (row_ok) {
                const int ldo = p.N >> 1;
                uint4* dst = reinterpret_cast<uint4*>(p.out_bf16 + static_cast<long long>(row) * ldo +
                                                      tl.nt * 128 + g * 64);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    float h[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) h[i] = silu_fast(accf[8 * c + i]) * accf[64 + 8 * c + i];
                    uint4 w;
                    __nv_bfloat162 b0 = __floats2bfloat162_rn(h[0], h[1]);
                    __nv_bfloat162 b1 = __floats2bfloat162_rn(h[2], h[3]);
                    __nv_bfloat162 b2 = __floats2bfloat162_rn(h[4], h[5]);
                    __nv_bfloat162 b3 = __floats2bfloat162_rn(h[6], h[7]);
                    memcpy(&w.x, &b0, 4); memcpy(&w.y, &b1, 4);
                    memcpy(&w.z, &b2, 4); memcpy(&w.w, &b3, 4);
                    dst[c] = w;
                }
            }
        }
    }
}

// Swapped orientation epilogue: thread = one weight row of each 128-row
// block, BT token columns per block.
template <int BT, int EPI>
__device__ void epilogue_swap(const KParams& p, const Smem& s, const WaitCtl& wc,
                              uint32_t tmem_base) {
    using C = Cfg<BT>;
    constexpr bool GATED = (EPI == EPI_SWIGLU_BF16 || EPI == EPI_SWIGLU_QUANT);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3;
    const int w = q * 32 + lane;          // weight row inside each block
    const int et = threadIdx.x - 128;     // epilogue thread index 0..127
    uint32_t buf = 0, bphase = 0, ephase = 0;
    const int total = total_tiles(s, p);
    const int nkb = p.nkb;
    float acc0[BT], acc1[BT];
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
        const Tile tl = decode_tile<BT>(t, s, p);
        const WTile wt = weight_tile<GATED>(tl, p.N);
        // stage this tile's activation scales
        if (!epi_sync(s, ephase, wc)) return;
        for (int idx = et; idx < nkb * BT; idx += 128) {
            const int kb = idx / BT, j = idx - kb * BT;
            s.as_tile[idx] = (j < tl.rows) ? a_scale_at(p, a_src_row(p, tl.row0 + j), kb) : 0.0f;
        }
        if (!epi_sync(s, ephase, wc)) return;
        const float* bs0 = p.b_scale + static_cast<long long>(wt.sb0) * nkb;
        const float* bs1 = p.b_scale + static_cast<long long>(wt.sb1) * nkb;
#pragma unroll
        for (int j = 0; j < BT; ++j) { acc0[j] = 0.0f; acc1[j] = 0.0f; }
        float b0n = bs0[0], b1n = bs1[0];
        for (int kb = 0; kb < nkb; ++kb) {
            const float b0 = b0n, b1 = b1n;
            if (kb + 1 < nkb) { b0n = bs0[kb + 1]; b1n = bs1[kb + 1]; }
            if (!warp_wait(&s.tfull[buf], bphase, wc, 6)) return;
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * (2 * BT);
            const float4* asv = reinterpret_cast<const float4*>(s.as_tile + kb * BT);
            if constexpr (BT <= 32) {
                // both blocks' partials in flight before one wait; the slot is
                // free again before the promotion arithmetic
                float v0[BT], v1[BT];
                tmem_load_pair<BT>(taddr, taddr + BT, v0, v1);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.tempty[buf]);
                promote2<BT>(acc0, acc1, v0, v1, asv, b0, b1);
            } else {
                float v[BT];
                tmem_load_cols<BT>(taddr, v);
#pragma unroll
                for (int j4 = 0; j4 < BT / 4; ++j4) {
                    const float4 a4 = asv[j4];
                    acc0[4 * j4 + 0] = fmaf(v[4 * j4 + 0], a4.x * b0, acc0[4 * j4 + 0]);
                    acc0[4 * j4 + 1] = fmaf(v[4 * j4 + 1], a4.y * b0, acc0[4 * j4 + 1]);
                    acc0[4 * j4 + 2] = fmaf(v[4 * j4 + 2], a4.z * b0, acc0[4 * j4 + 2]);
                    acc0[4 * j4 + 3] = fmaf(v[4 * j4 + 3], a4.w * b0, acc0[4 * j4 + 3]);
                }
                tmem_load_cols<BT>(taddr + BT, v);
#pragma unroll
                for (int j4 = 0; j4 < BT / 4; ++j4) {
                    const float4 a4 = asv[j4];
                    acc1[4 * j4 + 0] = fmaf(v[4 * j4 + 0], a4.x * b1, acc1[4 * j4 + 0]);
                    acc1[4 * j4 + 1] = fmaf(v[4 * j4 + 1], a4.y * b1, acc1[4 * j4 + 1]);
                    acc1[4 * j4 + 2] = fmaf(v[4 * j4 + 2], a4.z * b1, acc1[4 * j4 + 2]);
                    acc1[4 * j4 + 3] = fmaf(v[4 * j4 + 3], a4.w * b1, acc1[4 * j4 + 3]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.tempty[buf]);
            }
            if (++buf == C::TSLOTS) { buf = 0; bphase ^= 1; }
        }

        if constexpr (EPI == EPI_SWIGLU_QUANT) {
            float* red = s.xch;             // [4 warps][BT] per-token partial amax
            float* s_sc = s.xch + 4 * BT;   // [BT] scale of each token's 128-column block
            float* s_inv = s.xch + 5 * BT;  // [BT] its reciprocal
            constexpr int G = BT < 32 ? BT : 32;   // tokens per transpose group
#pragma unroll
            for (int g0 = 0; g0 < BT; g0 += G) {
                float m[G];
#pragma unroll
                for (int i = 0; i < G; ++i) {
                    const float h = silu_fast(acc0[g0 + i]) * acc1[g0 + i];
                    acc0[g0 + i] = h;
                    m[i] = fabsf(h);
                }
                // after this lane L holds the warp's max for token g0 + (L mod G)
                warp_transpose_max<G>(m);
                if (lane < G) red[q * BT + g0 + lane] = m[0];
            }
            if (!epi_sync(s, ephase, wc)) return;
            if (et < BT) {
                const float amax = fmaxf(fmaxf(red[et], red[BT + et]), fmaxf(red[2 * BT + et], red[3 * BT + et]));
                const float sc = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
                s_sc[et] = sc;
                s_inv[et] = __frcp_rn(sc);
                if (et < tl.rows) p.hs[static_cast<long long>(tl.nt) * p.R + tl.row0 + et] = sc;
            }
            if (!epi_sync(s, ephase, wc)) return;
            const int ldh = p.N >> 1;
            const int col = tl.nt * 128 + w;
#pragma unroll
            for (int j = 0; j < BT; ++j) {
                if (j < tl.rows)
                    p.hq[static_cast<long long>(tl.row0 + j) * ldh + col] =
                        static_cast<uint8_t>(cvt_e4m3x2(acc0[j] * s_inv[j], 0.0f) & 0xFF);
            }
        } else if constexpr (EPI == EPI_Y32) {
            const int colA = tl.nt * 256 + w;
#pragma unroll
            for (int j = 0; j < BT; ++j) {
                if (j < tl.rows) {
                    const int r = tl.row0 + j;
                    float* rowp = p.y + static_cast<long long>(p.rowmap ? __ldg(p.rowmap + r) : r) * p.ldy;
                    rowp[colA] = acc0[j];
                    if (wt.v1) rowp[colA + 128] = acc1[j];
                }
            }
        } else if constexpr (EPI == EPI_BF16) {
            const int colA = tl.nt * 256 + w;
#pragma unroll
            for (int j = 0; j < BT; ++j) {
                if (j < tl.rows) {
                    __nv_bfloat16* rowp = p.out_bf16 + static_cast<long long>(tl.row0 + j) * p.N;
                    rowp[colA] = __float2bfloat16_rn(acc0[j]);
                    if (wt.v1) rowp[colA + 128] = __float2bfloat16_rn(acc1[j]);
                }
            }
        } else {  // EPI_SWIGLU_BF16
            const int ldo = p.N >> 1;
            const int col = tl.nt * 128 + w;
#pragma unroll
            for (int j = 0; j < BT; ++j) {
                if (j < tl.rows)
                    p.out_bf16[static_cast<long long>(tl.row0 + j) * ldo + col] =
                        __float2bfloat16_rn(silu_fast(acc0[j]) * acc1[j]);
            }
        }
    }
}

// ---------------------------------------------------------------- kernel
template <int BT, int EPI>
__global__ void __launch_bounds__(Cfg<BT>::THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmY, const KParams p) {
    using C = Cfg<BT>;
    constexpr bool GATED = (EPI == EPI_SWIGLU_BF16 || EPI == EPI_SWIGLU_QUANT);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const Smem s = carve<BT>(base);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::STAGES; ++i) {
            mbar_init(&s.full[i], p.a_rowmap ? 1 : C::NBOX);
            mbar_init(&s.empty[i], 1);
        }
        for (int i = 0; i < C::TSLOTS; ++i) {
            mbar_init(&s.tfull[i], 1);
            mbar_init(&s.tempty[i], C::EPI_WARPS);
        }
        mbar_init(s.drain, 1);
        mbar_init(s.epi, C::EPI_THREADS);
        for (int i = 0; i < kScaleSlots; ++i) {
            mbar_init(&s.sfull[i], 32);
            mbar_init(&s.sempty[i], C::EPI_WARPS);
        }
        *s.abort = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if constexpr (EPI == EPI_Y32 && !C::SWAP) tma_prefetch_desc(&tmY);
    }
    if (warp == 1) {
        tmem_alloc(s.tmem, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 2) {
        // per-expert tile table: tiles of expert e = ceil(rows_e / BT) * n_tiles
        const int E = p.E;
        const int ntn = p.ntn;
        const int per = (E + 31) >> 5;
        const int lo = min(E, lane * per), hi = min(E, lo + per);
        int sum = 0;
        for (int e = lo; e < hi; ++e) {
            const int m0 = min(max(p.m_indptr[e], 0), p.R);
            const int m1 = min(max(p.m_indptr[e + 1], 0), p.R);
            s.mind[e] = m0;
            sum += ((max(0, m1 - m0) + BT - 1) / BT) * ntn;
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - sum;
        for (int e = lo; e < hi; ++e) {
            s.tstart[e] = run;
            const int m0 = s.mind[e];
            const int m1 = min(max(p.m_indptr[e + 1], 0), p.R);
            run += ((max(0, m1 - m0) + BT - 1) / BT) * ntn;
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

    if (warp < 4) {
        if constexpr (!C::SWAP) setmaxnreg_dec<kDirectLowRegs>();
        if (warp == 0) producer_role<BT, GATED>(&tmA, &tmB, p, s, wc);
        else if (warp == 1) mma_role<BT>(p, s, wc, tmem_base);
        else if (warp == 2) { if constexpr (!C::SWAP) scale_role<GATED>(p, s, wc); }
    } else {
        if constexpr (!C::SWAP) {
            setmaxnreg_inc<kDirectHighRegs>();
            epilogue_direct<EPI>(p, s, wc, tmem_base, &tmY);
            // output boxes still being stored read this CTA's shared memory
            if constexpr (EPI == EPI_Y32) {
                if (lane == 0) bulk_wait_group<0>();
                __syncwarp();
            }
        } else {
            epilogue_swap<BT, EPI>(p, s, wc, tmem_base);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

// ---------------------------------------------------------------- host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// Descriptor cache keyed by (address, rows, row bytes, box rows): repeated
// calls on the same weights reuse the encoded TMA descriptor.
struct MapKey {
    const void* ptr;
    long long rows, cols;
    int box_rows;
    bool operator==(const MapKey& o) const {
        return ptr == o.ptr && rows == o.rows && cols == o.cols && box_rows == o.box_rows;
    }
};
struct MapEntry {
    MapKey key;
    CUtensorMap map;
    bool used;
};
constexpr int kMapCache = 64;
MapEntry g_maps[kMapCache];
int g_map_next = 0;
std::mutex g_map_mu;

// 2-D map over a row-major FP8 matrix [rows, cols] with boxes of
// [box_rows x 128] bytes and the 128-byte swizzle; rows past the end read 0.
bool make_map(CUtensorMap* out, const void* ptr, long long rows, long long cols, int box_rows) {
    const MapKey key{ptr, rows, cols, box_rows};
    std::lock_guard<std::mutex> lk(g_map_mu);
    for (auto& e : g_maps)
        if (e.used && e.key == key) { *out = e.map; return true; }
    auto fn = encode_fn();
    if (!fn) return false;
    CUtensorMap m;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
    cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t es[2] = {1u, 1u};
    CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box,
                    es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    g_maps[g_map_next] = MapEntry{key, m, true};
    g_map_next = (g_map_next + 1) % kMapCache;
    *out = m;
    return true;
}

// 2-D map over a row-major fp32 matrix [rows, cols] (cols % 4 == 0, 16-byte
// aligned rows) with boxes of 32 rows x 32 columns (128 bytes) and the
// 128-byte swizzle, for the output stores of EPI_Y32.  Not cached: the
// output buffer changes from call to call more often than the weights.
bool make_map_f32_out(CUtensorMap* out, const void* ptr, long long rows, long long cols) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 4};
    cuuint32_t box[2] = {32u, 32u};
    cuuint32_t es[2] = {1u, 1u};
    return fn(out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool make_tma_map_fp8(CUtensorMap* out, const void* ptr, long long rows, long long cols,
                      int box_rows) {
    return make_map(out, ptr, rows, cols, box_rows);
}

namespace {

template <int BT, int EPI>
int launch_inst(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& my,
                const KParams& kp, int num_sms, cudaStream_t stream) {
    using C = Cfg<BT>;
    auto kern = grouped_gemm_kernel<BT, EPI>;
    static int configured_dev = -1;  // per-instance one-time set-up (device 0 assumed shared)
    static int checked = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
            cudaSuccess)
            return ST_CUDA;
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return ST_CUDA;
        // the direct kernel's setmaxnreg split assumes exactly this launch size
        checked = C::SWAP ? 1 : (fa.numRegs == kDirectLaunchRegs ? 1 : 0);
        if (!checked)
            fprintf(stderr, "moefp8: direct GEMM kernel has %d registers, expected %d\n", fa.numRegs,
                    kDirectLaunchRegs);
        configured_dev = dev;
    }
    if (!checked) return ST_UNSUPPORTED;
    kern<<<num_sms, C::THREADS, C::SMEM_BYTES, stream>>>(ma, mb, my, kp);
    return cudaGetLastError() == cudaSuccess ? ST_OK : ST_CUDA;
}

template <int BT>
int launch_bt(int epi, const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& my,
              KParams kp, int num_sms, cudaStream_t stream) {
    // direct EPI_Y32 gives its last pipeline stage to the output staging
    kp.nstages = (!Cfg<BT>::SWAP && epi == EPI_Y32) ? Cfg<BT>::STAGES - 1 : Cfg<BT>::STAGES;
    switch (epi) {
        case EPI_BF16: return launch_inst<BT, EPI_BF16>(ma, mb, my, kp, num_sms, stream);
        case EPI_SWIGLU_BF16:
            return launch_inst<BT, EPI_SWIGLU_BF16>(ma, mb, my, kp, num_sms, stream);
        case EPI_SWIGLU_QUANT:
            return launch_inst<BT, EPI_SWIGLU_QUANT>(ma, mb, my, kp, num_sms, stream);
        case EPI_Y32: return launch_inst<BT, EPI_Y32>(ma, mb, my, kp, num_sms, stream);
        default: return ST_INVALID_ARG;
    }
}

}  // namespace

int swap_max_k(int tile_m) {
    switch (tile_m) {
        case 16: return Cfg<16>::MAX_NKB * 128;
        case 32: return Cfg<32>::MAX_NKB * 128;
        case 64: return Cfg<64>::MAX_NKB * 128;
        default: return 1 << 30;
    }
}

int launch_grouped_gemm(const GemmArgs& g, cudaStream_t stream) {
    if (g.R <= 0 || g.E <= 0) return ST_OK;
    if (g.tile_m != 128 && g.K > swap_max_k(g.tile_m)) return ST_UNSUPPORTED;
    CUtensorMap ma, mb;
    // gathered A: one-row boxes over the A source rows; tiled A: boxes of up to 64 rows
    const long long a_rows = g.a_rowmap ? (g.a_rows > 0 ? g.a_rows : 1) : g.R;
    if (!make_map(&ma, g.a, a_rows, g.K, g.a_rowmap ? 1 : (g.tile_m < 64 ? g.tile_m : 64)))
        return ST_CUDA;
    if (!make_map(&mb, g.b, static_cast<long long>(g.E) * g.N, g.K, 64)) return ST_CUDA;
    KParams kp;
    kp.R = g.R; kp.N = g.N; kp.K = g.K; kp.E = g.E; kp.nkb = g.K / 128;
    kp.a_scale = g.a_scale; kp.as_row = g.as_row; kp.as_kb = g.as_kb;
    kp.b_scale = g.b_scale; kp.m_indptr = g.m_indptr;
    kp.hq = g.hq; kp.hs = g.hs;
    kp.y = g.y; kp.ldy = g.ldy; kp.rowmap = g.rowmap;
    kp.a_rowmap = g.a_rowmap; kp.a_rowdiv = g.a_rowdiv > 0 ? g.a_rowdiv : 1;
    kp.a_rows = static_cast<int>(a_rows);
    kp.out_bf16 = static_cast<__nv_bfloat16*>(g.out_bf16);
    kp.status = g.status;
    kp.timeout_ns = g.timeout_ns;
    const bool gated = g.epi == EPI_SWIGLU_BF16 || g.epi == EPI_SWIGLU_QUANT;
    kp.ntn = gated ? (g.N >> 8) : ((g.N + 255) >> 8);
    CUtensorMap my = mb;  // unused unless EPI_Y32
    if (g.epi == EPI_Y32) {
        if (!g.y || g.ldy < g.N || g.ldy % 4 || (reinterpret_cast<uintptr_t>(g.y) & 15))
            return ST_INVALID_ARG;
        if (!make_map_f32_out(&my, g.y, g.R, g.ldy)) return ST_CUDA;
    }
    switch (g.tile_m) {
        case 16: return launch_bt<16>(g.epi, ma, mb, my, kp, g.num_sms, stream);
        case 32: return launch_bt<32>(g.epi, ma, mb, my, kp, g.num_sms, stream);
        case 64: return launch_bt<64>(g.epi, ma, mb, my, kp, g.num_sms, stream);
        case 128: return launch_bt<128>(g.epi, ma, mb, my, kp, g.num_sms, stream);
        default: return ST_NO_TILE_CONFIG;
    }
}

}  // namespace moe
