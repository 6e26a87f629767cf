// Fused expert kernel: for one expert and up to 64 of its routed tokens per
// work item, GEMM1 (gate/up) + SwiGLU + FP8 requantisation of the
// intermediate + GEMM2 (down), with the FP8 intermediate kept in shared
// memory and read from there by the tensor core.
//
// This is the fusion the page "FlashInfer: Blackwell W8A8 AlphaMoE Expert
// 계산 커널 퓨전으로 성능 비약적 향상" (flashinfer PR #4287) is about (section
// "핵심 최적화: 5개 커널을 하나로" and "1. 커널 퓨전": the expert stages in one
// kernel, the intermediate staying on chip), for the shapes where one CTA can
// hold a token group's whole intermediate row: the per-expert groups are
// small (decode-like), so the weights are the MMA M operand (two 128-row
// blocks per K block) and the tokens the N operand (64), as in the swapped
// grouped GEMM.  One persistent CTA per SM walks the work items
// (expert, 64-token tile); an item streams its expert's gate/up weights once
// (phase 1, K = H) and its down weights once (phase 2, K = I).
//
//  * warp 0 - producer: phase 1 stages the tile's 64 grouped token rows (one
//    tiled TMA box) and two 128-row gate / up weight blocks per K block;
//    phase 2 stages two 128-row down-weight blocks per K block (the tokens
//    are already on chip).
//  * warp 1 - MMA issue (one elected lane): per K block two M=128, N=64
//    tcgen05.mma groups (one per weight block) into a TMEM slot; phase 2
//    reads its N operand (the intermediate codes) from shared memory, once
//    the epilogue has written all of them for the item.
//  * warp 3 - scale loader: stages every item's activation scales and its
//    expert's gate/up and down weight-block scales in shared memory (two
//    buffers, one item ahead), so no promotion waits on a global load.
//  * warps 4-11 - epilogue, thread = one weight row of each block and one
//    half of the 64 tokens (two warps per TMEM lane quadrant): promotes
//    every K block (acc += partial * a_scale * b_scale); after phase 1's K
//    loop of a 128-column block: h = silu(gate) * up, per-token amax over the
//    block's 128 columns (warp transposing max + shared memory), scale =
//    amax / 448, codes written into shared memory in the 128-byte-swizzled
//    K-major layout the MMA reads (and to global memory when a debug copy is
//    asked for); after phase 2: the fp32 rows y (grouped order), summed per
//    token by the combine kernel.
// Every wait is bounded by %globaltimer; on expiry the CTA records
// ST_DEVICE_TIMEOUT, drains its copies and MMAs, frees TMEM and returns.
#include <atomic>

#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "gemm_common.cuh"
#include "kernels.h"

namespace moe {

bool make_tma_map_fp8(CUtensorMap* out, const void* ptr, long long rows, long long cols,
                      int box_rows);

namespace fx {

constexpr int BT = 64;                        // tokens per work item (MMA N)
constexpr int EPI_WARPS = 8;                  // two per TMEM lane quadrant
constexpr int HT = BT / 2;                    // tokens per epilogue warp
constexpr int THREADS = 128 + 32 * EPI_WARPS;
constexpr int A_BYTES = BT * 128;             // token rows of one K block
constexpr int B_BYTES = 256 * 128;            // two 128-row weight blocks
constexpr int STAGE_BYTES = B_BYTES + A_BYTES;
constexpr int A_OFF = B_BYTES;                // weights first: both 1024-aligned
constexpr int TSLOTS = 512 / (2 * BT);        // 4 TMEM slots of 2 x 64 columns
constexpr int kSmemLimit = 232448;
constexpr int kMaxE = 1024;
constexpr int XCH_BYTES = 6 * BT * 4;
constexpr int BAR_BYTES = 512;
constexpr int MAX_STAGES = 6;
constexpr int MIN_STAGES = 3;

// One item's scales: activations [H/128][BT], gate/up weight blocks
// [2I/128][H/128], down weight blocks [H/128][I/128]; 16-byte multiple.
__host__ __device__ inline int scale_buf_floats(int H, int I) {
    return ((H / 128) * BT + 3 * (I / 128) * (H / 128) + 3) / 4 * 4;
}
__host__ __device__ inline int table_bytes(int E) { return (2 * (E + 1) * 4 + 15) / 16 * 16; }

// Shared memory: 1024 (alignment) + stages + intermediate codes
// [I/128][64 rows x 128 B] + two scale buffers + intermediate scales
// [I/128][64] + exchange + item tables + barriers.
__host__ __device__ inline int fixed_bytes(int H, int I, int E) {
    return 1024 + I * BT + 2 * scale_buf_floats(H, I) * 4 + (I / 128) * BT * 4 + XCH_BYTES +
           table_bytes(E) + BAR_BYTES;
}
__host__ __device__ inline int stages_for(int H, int I, int E) {
    const int n = (kSmemLimit - fixed_bytes(H, I, E)) / STAGE_BYTES;
    return n > MAX_STAGES ? MAX_STAGES : n;
}

struct Params {
    int R, H, I, E;
    int nstages;
    const float* xs;          // [H/128, R] activation scales of the grouped rows
    const float* w13_scale;   // [E, 2I/128, H/128]
    const float* w2_scale;    // [E, H/128, I/128]
    const int32_t* m_indptr;  // [E+1]
    float* y;                 // [R, H] fp32, grouped rows
    uint8_t* hq;              // debug copy of the intermediate [R, I] (or null)
    float* hs;                // debug copy of its scales [I/128, R] (or null)
    int* status;
    unsigned long long timeout_ns;
};

struct Smem {
    uint8_t* stages;
    uint8_t* hq;      // [I/128][BT x 128 B], swizzled
    float* sc;        // two scale buffers of scale_buf_floats
    float* hs;        // [I/128][BT]
    float* xch;
    int* tstart;
    int* mind;
    uint64_t* full;
    uint64_t* empty;
    uint64_t* tfull;
    uint64_t* tempty;
    uint64_t* sfull;
    uint64_t* sempty;
    uint64_t* hready;
    uint64_t* drain;
    uint64_t* epi;
    uint32_t* tmem;
    volatile int* abort;
};

__device__ __forceinline__ Smem carve(uint8_t* base, const Params& p) {
    Smem s;
    uint8_t* q = base;
    s.stages = q;
    q += p.nstages * STAGE_BYTES;
    s.hq = q;
    q += p.I * BT;
    s.sc = reinterpret_cast<float*>(q);
    q += 2 * scale_buf_floats(p.H, p.I) * 4;
    s.hs = reinterpret_cast<float*>(q);
    q += (p.I / 128) * BT * 4;
    s.xch = reinterpret_cast<float*>(q);
    q += XCH_BYTES;
    s.tstart = reinterpret_cast<int*>(q);
    s.mind = s.tstart + (p.E + 1);
    q += table_bytes(p.E);
    uint64_t* bars = reinterpret_cast<uint64_t*>(q);
    s.full = bars;
    s.empty = bars + MAX_STAGES;
    s.tfull = bars + 2 * MAX_STAGES;
    s.tempty = s.tfull + TSLOTS;
    s.sfull = s.tempty + TSLOTS;
    s.sempty = s.sfull + 2;
    s.hready = s.sempty + 2;
    s.drain = s.hready + 1;
    s.epi = s.hready + 2;
    s.tmem = reinterpret_cast<uint32_t*>(s.hready + 3);
    s.abort = reinterpret_cast<volatile int*>(s.hready + 4);
    return s;
}

struct Item {
    int e, row0, rows;
};

__device__ __forceinline__ Item decode(int t, const Smem& s, const Params& p) {
    int lo = 0, hi = p.E;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s.tstart[mid] <= t) lo = mid; else hi = mid;
    }
    Item it;
    it.e = lo;
    const int mt = t - s.tstart[lo];
    const int me = max(0, s.mind[lo + 1] - s.mind[lo]);
    it.row0 = s.mind[lo] + mt * BT;
    it.rows = min(BT, me - mt * BT);
    return it;
}

// Phase-2 column tiles (256 weight rows each).
__device__ __forceinline__ int ntiles2(const Params& p) { return (p.H + 255) >> 8; }

__device__ void producer(const CUtensorMap* tmA, const CUtensorMap* tmW13, const CUtensorMap* tmW2,
                         const Params& p, const Smem& s, const WaitCtl& wc, int total) {
    const int l = threadIdx.x & 31;
    const bool b_lane = l < 4;        // one 64-row weight box
    const bool a_lane = l == 4;       // the 64 token rows
    const int nkb1 = p.H >> 7, nkb2 = p.I >> 7, nt1s = p.I >> 7, nt2s = ntiles2(p);
    uint32_t stage = 0, phase = 0, armed = 0, armed_par = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const Item it = decode(t, s, p);
        // phase 1: gate block nt, up block nt (rows e*2I + nt*128 and e*2I + I + nt*128);
        // token rows past the item's own (the next expert's, or past R:
        // zero-filled) are loaded but carry a zero scale
        for (int nt = 0; nt < nt1s && ok; ++nt) {
            const int wrow = it.e * 2 * p.I + (l >> 1) * p.I + nt * 128 + (l & 1) * 64;
            for (int kb = 0; kb < nkb1; ++kb) {
                if (!warp_wait_spin(&s.empty[stage], phase ^ 1, wc, 1)) { ok = false; break; }
                uint8_t* st = s.stages + stage * STAGE_BYTES;
                if (l == 0) mbar_arrive_expect_tx(&s.full[stage], STAGE_BYTES);
                __syncwarp();
                if (b_lane) tma_load_2d(st + l * 64 * 128, tmW13, &s.full[stage], kb * 128, wrow);
                if (a_lane) tma_load_2d(st + A_OFF, tmA, &s.full[stage], kb * 128, it.row0);
                __syncwarp();
                armed |= 1u << stage;
                armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                if (++stage == static_cast<uint32_t>(p.nstages)) { stage = 0; phase ^= 1; }
            }
        }
        // phase 2: down blocks 2*nt and 2*nt+1 (rows e*H + nt*256 ...)
        for (int nt = 0; nt < nt2s && ok; ++nt) {
            const int wrow = it.e * p.H + nt * 256 + l * 64;
            for (int kb = 0; kb < nkb2; ++kb) {
                if (!warp_wait_spin(&s.empty[stage], phase ^ 1, wc, 1)) { ok = false; break; }
                uint8_t* st = s.stages + stage * STAGE_BYTES;
                if (l == 0) mbar_arrive_expect_tx(&s.full[stage], B_BYTES);
                __syncwarp();
                if (b_lane) tma_load_2d(st + l * 64 * 128, tmW2, &s.full[stage], kb * 128, wrow);
                __syncwarp();
                armed |= 1u << stage;
                armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                if (++stage == static_cast<uint32_t>(p.nstages)) { stage = 0; phase ^= 1; }
            }
        }
    }
    // no copy may still be writing into shared memory when the CTA exits
    for (int st = 0; st < p.nstages; ++st)
        if ((armed >> st) & 1u) wait_bar(&s.full[st], (armed_par >> st) & 1u, wc, 2, /*drain=*/true);
    __syncwarp();
}

__device__ void mma(const Params& p, const Smem& s, const WaitCtl& wc, uint32_t tmem_base, int total) {
    constexpr uint32_t idesc = idesc_e4m3_f32(128, BT);
    const int nkb1 = p.H >> 7, nkb2 = p.I >> 7, nt1s = p.I >> 7, nt2s = ntiles2(p);
    uint32_t stage = 0, phase = 0, j = 0, jphase = 0, item = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++item) {
        for (int ph = 0; ph < 2 && ok; ++ph) {
            if (ph == 1) {
                // the item's intermediate codes are all in shared memory
                if (!warp_wait_spin(s.hready, item & 1u, wc, 10)) { ok = false; break; }
                tc_fence_after();
            }
            const int ntiles = ph == 0 ? nt1s : nt2s;
            const int nkb = ph == 0 ? nkb1 : nkb2;
            for (int nt = 0; nt < ntiles && ok; ++nt) {
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!warp_wait_spin(&s.tempty[j], jphase ^ 1, wc, 3)) { ok = false; break; }
                    if (!warp_wait_spin(&s.full[stage], phase, wc, 4)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sw = smem_u32(s.stages + stage * STAGE_BYTES);
                    const uint32_t sx = ph == 0 ? sw + A_OFF : smem_u32(s.hq + kb * A_BYTES);
                    const uint32_t d = tmem_base + j * (2 * BT);
                    if (elect_one()) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            umma_f8(d, smem_desc_k_sw128(sw + kk * 32), smem_desc_k_sw128(sx + kk * 32),
                                    idesc, kk);
                            umma_f8(d + BT, smem_desc_k_sw128(sw + 16384 + kk * 32),
                                    smem_desc_k_sw128(sx + kk * 32), idesc, kk);
                        }
                        umma_commit(&s.empty[stage]);
                        umma_commit(&s.tfull[j]);
                    }
                    __syncwarp();
                    if (++j == TSLOTS) { j = 0; jphase ^= 1; }
                    if (++stage == static_cast<uint32_t>(p.nstages)) { stage = 0; phase ^= 1; }
                }
            }
        }
    }
    if (elect_one()) umma_commit(s.drain);
    __syncwarp();
    wait_bar(s.drain, 0, wc, 5, /*drain=*/true);
    __syncwarp();
}

// Scale loader: item n of this CTA goes to buffer n % 2; every lane arrives
// on the buffer's full barrier after its own plain stores.
__device__ void scale_loader(const Params& p, const Smem& s, const WaitCtl& wc, int total) {
    const int lane = threadIdx.x & 31;
    const int nkb1 = p.H >> 7, nkb2 = p.I >> 7, nt1s = p.I >> 7, nblk2 = p.H >> 7;
    const int nbuf = scale_buf_floats(p.H, p.I);
    uint32_t n = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++n) {
        const uint32_t b = n & 1u, par = (n >> 1) & 1u;
        if (!warp_wait(&s.sempty[b], par ^ 1u, wc, 8)) return;
        const Item it = decode(t, s, p);
        float* as = s.sc + b * nbuf;
        float* w13s = as + nkb1 * BT;
        float* w2s = w13s + 2 * nt1s * nkb1;
        for (int idx = lane; idx < nkb1 * BT; idx += 32) {
            const int kb = idx / BT, j = idx - kb * BT;
            as[idx] = j < it.rows ? __ldg(p.xs + static_cast<long long>(kb) * p.R + it.row0 + j) : 0.0f;
        }
        const float* g13 = p.w13_scale + static_cast<long long>(it.e) * 2 * nt1s * nkb1;
        for (int idx = lane; idx < 2 * nt1s * nkb1; idx += 32) w13s[idx] = __ldg(g13 + idx);
        const float* g2 = p.w2_scale + static_cast<long long>(it.e) * nblk2 * nkb2;
        for (int idx = lane; idx < nblk2 * nkb2; idx += 32) w2s[idx] = __ldg(g2 + idx);
        mbar_arrive(&s.sfull[b]);
    }
}

__device__ __forceinline__ bool epi_sync(const Smem& s, uint32_t& phase, const WaitCtl& wc) {
    mbar_arrive(s.epi);
    const bool ok = warp_wait(s.epi, phase, wc, 7);
    phase ^= 1;
    return ok;
}

// Byte offset of (token row j, column c) in a 64-row x 128-byte K-major tile
// with the 128-byte swizzle (16-byte chunk c/16 of row j at chunk (c/16) ^ (j%8)).
__device__ __forceinline__ int sw128_off(int j, int c) {
    return (j >> 3) * 1024 + (j & 7) * 128 + ((((c >> 4) ^ j) & 7) << 4) + (c & 15);
}

__device__ void epilogue(const Params& p, const Smem& s, const WaitCtl& wc, uint32_t tmem_base,
                         int total) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3;                       // TMEM lane quadrant
    const int hb = ((warp - 4) >> 2) * HT;        // first token of this warp's half
    const int w = q * 32 + lane;                  // weight row inside each 128-row block
    const int et = threadIdx.x - 128;             // epilogue thread 0..255
    const int nkb1 = p.H >> 7, nkb2 = p.I >> 7, nt1s = p.I >> 7, nt2s = ntiles2(p);
    const int nblk2 = p.H >> 7;
    const int nbuf = scale_buf_floats(p.H, p.I);
    uint32_t buf = 0, bphase = 0, ephase = 0, n = 0;
    float* red = s.xch;                   // [4 quadrants][BT] partial amax
    float* s_inv = s.xch + 4 * BT;        // [BT] reciprocal of each token's block scale
    // accumulators as token pairs: acc0[i] = tokens hb + 2i, hb + 2i + 1 of block 0
    float2 acc0[HT / 2], acc1[HT / 2];
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++n) {
        const Item it = decode(t, s, p);
        const uint32_t sb = n & 1u;
        if (!warp_wait(&s.sfull[sb], (n >> 1) & 1u, wc, 9)) return;
        const float* as1 = s.sc + sb * nbuf;
        const float* w13s = as1 + nkb1 * BT;
        const float* w2s = w13s + 2 * nt1s * nkb1;
        for (int ph = 0; ph < 2; ++ph) {
            const int ntiles = ph == 0 ? nt1s : nt2s;
            const int nkb = ph == 0 ? nkb1 : nkb2;
            const float* ascale = ph == 0 ? as1 : s.hs;
            for (int nt = 0; nt < ntiles; ++nt) {
                // weight-block scales of this column tile: gate/up (phase 1) or down blocks 2nt, 2nt+1
                const bool v1 = ph == 0 || 2 * nt + 1 < nblk2;
                const float* bs0 = ph == 0 ? w13s + nt * nkb1 : w2s + 2 * nt * nkb2;
                const float* bs1 = ph == 0 ? w13s + (nt1s + nt) * nkb1 : (v1 ? bs0 + nkb2 : bs0);
#pragma unroll
                for (int i = 0; i < HT / 2; ++i) {
                    acc0[i] = make_float2(0.0f, 0.0f);
                    acc1[i] = make_float2(0.0f, 0.0f);
                }
                for (int kb = 0; kb < nkb; ++kb) {
                    const float2 b0 = make_float2(bs0[kb], bs0[kb]);
                    const float2 b1 = make_float2(bs1[kb], bs1[kb]);
                    if (!warp_wait(&s.tfull[buf], bphase, wc, 6)) return;
                    tc_fence_after();
                    const uint32_t taddr =
                        tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * (2 * BT) + hb;
                    // both blocks' partials in flight before one wait
                    uint32_t u0[HT], u1[HT];
                    tmem_ld32_async(taddr, u0);
                    tmem_ld32_async(taddr + BT, u1);
                    tmem_wait_ld(u0);
                    tmem_wait_ld(u1);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s.tempty[buf]);
                    if (++buf == TSLOTS) { buf = 0; bphase ^= 1; }
                    // acc += partial * (a_scale * b_scale), two tokens per instruction
                    const float4* asv = reinterpret_cast<const float4*>(ascale + kb * BT + hb);
#pragma unroll
                    for (int j4 = 0; j4 < HT / 4; ++j4) {
                        const float4 a4 = asv[j4];
                        const float2 alo = make_float2(a4.x, a4.y), ahi = make_float2(a4.z, a4.w);
                        const float2 p0lo = __fmul2_rn(alo, b0), p0hi = __fmul2_rn(ahi, b0);
                        const float2 p1lo = __fmul2_rn(alo, b1), p1hi = __fmul2_rn(ahi, b1);
                        acc0[2 * j4] = __ffma2_rn(
                            make_float2(__uint_as_float(u0[4 * j4]), __uint_as_float(u0[4 * j4 + 1])), p0lo,
                            acc0[2 * j4]);
                        acc0[2 * j4 + 1] = __ffma2_rn(
                            make_float2(__uint_as_float(u0[4 * j4 + 2]), __uint_as_float(u0[4 * j4 + 3])),
                            p0hi, acc0[2 * j4 + 1]);
                        acc1[2 * j4] = __ffma2_rn(
                            make_float2(__uint_as_float(u1[4 * j4]), __uint_as_float(u1[4 * j4 + 1])), p1lo,
                            acc1[2 * j4]);
                        acc1[2 * j4 + 1] = __ffma2_rn(
                            make_float2(__uint_as_float(u1[4 * j4 + 2]), __uint_as_float(u1[4 * j4 + 3])),
                            p1hi, acc1[2 * j4 + 1]);
                    }
                }
                if (ph == 0) {
                    // SwiGLU, per-token amax over the block's 128 columns, FP8 codes of column w
                    float m[HT], h[HT];
#pragma unroll
                    for (int i = 0; i < HT; ++i) {
                        const float g = (i & 1) ? acc0[i >> 1].y : acc0[i >> 1].x;
                        const float u = (i & 1) ? acc1[i >> 1].y : acc1[i >> 1].x;
                        h[i] = silu_fast(g) * u;
                        m[i] = fabsf(h[i]);
                    }
                    // afterwards lane L holds this warp's max for token hb + L
                    warp_transpose_max<HT>(m);
                    red[q * BT + hb + lane] = m[0];
                    if (!epi_sync(s, ephase, wc)) return;
                    if (et < BT) {
                        const float amax = fmaxf(fmaxf(red[et], red[BT + et]),
                                                 fmaxf(red[2 * BT + et], red[3 * BT + et]));
                        const float sc = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
                        s_inv[et] = __frcp_rn(sc);
                        s.hs[nt * BT + et] = sc;
                        if (p.hs && et < it.rows)
                            p.hs[static_cast<long long>(nt) * p.R + it.row0 + et] = sc;
                    }
                    if (!epi_sync(s, ephase, wc)) return;
                    uint8_t* tile = s.hq + nt * A_BYTES;
#pragma unroll
                    for (int i = 0; i < HT; ++i) {
                        const int j = hb + i;
                        const uint8_t c = static_cast<uint8_t>(cvt_e4m3x2(h[i] * s_inv[j], 0.0f) & 0xFF);
                        tile[sw128_off(j, w)] = c;
                        if (p.hq && j < it.rows)
                            p.hq[static_cast<long long>(it.row0 + j) * p.I + nt * 128 + w] = c;
                    }
                    if (nt + 1 == ntiles) {
                        // the codes are read next by the tensor core (async proxy)
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(s.hready);
                    }
                } else {
                    const int colA = nt * 256 + w;
#pragma unroll
                    for (int i = 0; i < HT; ++i) {
                        const int j = hb + i;
                        if (j < it.rows) {
                            float* rowp = p.y + static_cast<long long>(it.row0 + j) * p.H;
                            rowp[colA] = (i & 1) ? acc0[i >> 1].y : acc0[i >> 1].x;
                            if (v1) rowp[colA + 128] = (i & 1) ? acc1[i >> 1].y : acc1[i >> 1].x;
                        }
                    }
                }
            }
        }
        // this item's scale buffer may be refilled
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.sempty[sb]);
    }
}

__global__ void __launch_bounds__(THREADS, 1)
    fused_expert_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmW13,
                        const __grid_constant__ CUtensorMap tmW2, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const Smem s = carve(base, p);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < p.nstages; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1);
        }
        for (int i = 0; i < TSLOTS; ++i) {
            mbar_init(&s.tfull[i], 1);
            mbar_init(&s.tempty[i], EPI_WARPS);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.sfull[i], 32);
            mbar_init(&s.sempty[i], EPI_WARPS);
        }
        mbar_init(s.hready, EPI_WARPS);
        mbar_init(s.drain, 1);
        mbar_init(s.epi, 32 * EPI_WARPS);
        *s.abort = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmW13);
        tma_prefetch_desc(&tmW2);
    }
    if (warp == 1) {
        tmem_alloc(s.tmem, 512);
        tmem_relinquish();
    }
    if (warp == 2) {
        // work items of expert e: ceil(rows_e / 64)
        const int E = p.E;
        const int per = (E + 31) >> 5;
        const int lo = min(E, lane * per), hi = min(E, lo + per);
        int sum = 0;
        for (int e = lo; e < hi; ++e) {
            const int m0 = min(max(p.m_indptr[e], 0), p.R);
            const int m1 = min(max(p.m_indptr[e + 1], 0), p.R);
            s.mind[e] = m0;
            sum += (max(0, m1 - m0) + BT - 1) / BT;
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
            const int m1 = min(max(p.m_indptr[e + 1], 0), p.R);
            run += (max(0, m1 - s.mind[e]) + BT - 1) / BT;
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
    if (warp == 0) producer(&tmA, &tmW13, &tmW2, p, s, wc, total);
    else if (warp == 1) mma(p, s, wc, tmem_base, total);
    else if (warp == 3) scale_loader(p, s, wc, total);
    else if (warp >= 4) epilogue(p, s, wc, tmem_base, total);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, 512);
}

}  // namespace fx

bool fused_expert_fits(int H, int I, int E) {
    return H % 128 == 0 && I % 128 == 0 && E >= 1 && E <= fx::kMaxE &&
           fx::stages_for(H, I, E) >= fx::MIN_STAGES;
}

int launch_fused_expert(const FusedExpertArgs& g, cudaStream_t stream) {
    if (g.R <= 0 || g.E <= 0) return ST_OK;
    if (!fused_expert_fits(g.H, g.I, g.E)) return ST_UNSUPPORTED;
    CUtensorMap ma, m13, m2;
    if (!make_tma_map_fp8(&ma, g.xq, g.R, g.H, fx::BT)) return ST_CUDA;
    if (!make_tma_map_fp8(&m13, g.w13, static_cast<long long>(g.E) * 2 * g.I, g.H, 64)) return ST_CUDA;
    if (!make_tma_map_fp8(&m2, g.w2, static_cast<long long>(g.E) * g.H, g.I, 64)) return ST_CUDA;
    fx::Params p{};
    p.R = g.R; p.H = g.H; p.I = g.I; p.E = g.E;
    p.nstages = fx::stages_for(g.H, g.I, g.E);
    p.xs = g.xs; p.w13_scale = g.w13_scale; p.w2_scale = g.w2_scale;
    p.m_indptr = g.m_indptr; p.y = g.y; p.hq = g.hq; p.hs = g.hs;
    p.status = g.status; p.timeout_ns = g.timeout_ns;
    const int smem = fx::fixed_bytes(g.H, g.I, g.E) + p.nstages * fx::STAGE_BYTES;
    static std::atomic<int> configured_dev{-1};  // opt-in to the largest dynamic shared memory
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ST_CUDA;
    if (configured_dev.load() != dev) {
        if (cudaFuncSetAttribute(fx::fused_expert_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 fx::kSmemLimit) != cudaSuccess)
            return ST_CUDA;
        configured_dev.store(dev);
    }
    // at most one work item per 64 grouped rows plus one partial tile per expert
    const long long items = (static_cast<long long>(g.R) + fx::BT - 1) / fx::BT + g.E;
    const int grid = static_cast<int>(items < g.num_sms ? items : g.num_sms);
    fx::fused_expert_kernel<<<grid, fx::THREADS, smem, stream>>>(ma, m13, m2, p);
    return cudaGetLastError() == cudaSuccess ? ST_OK : ST_CUDA;
}

}  // namespace moe
