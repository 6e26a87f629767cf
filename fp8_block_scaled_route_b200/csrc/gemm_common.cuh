// Device helpers shared by the FP8 grouped GEMM and the fused expert kernel:
// whole-warp bounded waits, the SiLU used in the epilogues, a warp-wide
// transposing max, TMEM column loads and the packed promotion FMA.
#pragma once
#include "common.cuh"

namespace moe {

// silu with the hardware exp2 and reciprocal (about 2 ulp); its result feeds
// an FP8 requantisation or a bf16 rounding, whose steps are 2^19 times
// coarser than that error.
__device__ __forceinline__ float silu_fast(float z) {
    return z * rcp_approx(1.0f + __expf(-z));
}

// Wait of a whole epilogue warp: every lane waits, and the warp proceeds only
// if every lane succeeded, so warp-collective tcgen05.ld never diverges.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& wc,
                                          int where) {
    const bool ok = wait_bar(bar, parity, wc, where);
    return __all_sync(0xffffffffu, ok) != 0;
}

__device__ __forceinline__ bool warp_wait_spin(uint64_t* bar, uint32_t parity, const WaitCtl& wc,
                                               int where) {
    const bool ok = wait_bar_spin(bar, parity, wc, where);
    return __all_sync(0xffffffffu, ok) != 0;
}

// Max over the 32 lanes of each of G values per lane (G = 16 or 32), by a
// transposing butterfly: afterwards v[0] of lane L holds the maximum of
// value (L mod G) over all lanes.  G - 1 + (32 / G - 1) * G shuffles instead
// of 5 * G.
template <int G>
__device__ __forceinline__ void warp_transpose_max(float (&v)[G]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 16; o >= G; o >>= 1) {
#pragma unroll
        for (int i = 0; i < G; ++i) v[i] = fmaxf(v[i], __shfl_xor_sync(0xffffffffu, v[i], o));
    }
#pragma unroll
    for (int o = G / 2; o >= 1; o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < o; ++i) {
            const float send = up ? v[i] : v[i + o];
            const float keep = up ? v[i + o] : v[i];
            v[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, o));
        }
    }
}

template <int BT>
__device__ __forceinline__ void tmem_load_cols(uint32_t taddr, float (&v)[BT]) {
    if constexpr (BT == 16) {
        tmem_ld16(taddr, v);
    } else if constexpr (BT == 32) {
        tmem_ld32(taddr, v);
    } else {
        float* lo = v;
        float* hi = v + 32;
        tmem_ld32(taddr, *reinterpret_cast<float(*)[32]>(lo));
        tmem_ld32(taddr + 32, *reinterpret_cast<float(*)[32]>(hi));
    }
}

// Two TMEM column groups of BT (16 or 32) columns each, both loads in flight
// before one wait.
template <int BT>
__device__ __forceinline__ void tmem_load_pair(uint32_t ta, uint32_t tb, float (&v0)[BT],
                                               float (&v1)[BT]) {
    uint32_t* r0 = reinterpret_cast<uint32_t*>(v0);
    uint32_t* r1 = reinterpret_cast<uint32_t*>(v1);
    if constexpr (BT == 16) {
        tmem_ld16_async(ta, *reinterpret_cast<uint32_t(*)[16]>(r0));
        tmem_ld16_async(tb, *reinterpret_cast<uint32_t(*)[16]>(r1));
        tmem_wait_ld(*reinterpret_cast<uint32_t(*)[16]>(r0));
        tmem_wait_ld(*reinterpret_cast<uint32_t(*)[16]>(r1));
    } else {
        static_assert(BT == 32, "tmem_load_pair: 16 or 32 columns");
        tmem_ld32_async(ta, *reinterpret_cast<uint32_t(*)[32]>(r0));
        tmem_ld32_async(tb, *reinterpret_cast<uint32_t(*)[32]>(r1));
        tmem_wait_ld(*reinterpret_cast<uint32_t(*)[32]>(r0));
        tmem_wait_ld(*reinterpret_cast<uint32_t(*)[32]>(r1));
    }
}

// acc0[j] += v0[j] * (a[j] * b0), acc1[j] += v1[j] * (a[j] * b1) for BT
// tokens, two per packed instruction (each product and sum rounded as the
// scalar fmul / fmaf would round it).
template <int BT>
__device__ __forceinline__ void promote2(float (&acc0)[BT], float (&acc1)[BT], const float (&v0)[BT],
                                         const float (&v1)[BT], const float4* asv, float b0f,
                                         float b1f) {
    const float2 b0 = make_float2(b0f, b0f), b1 = make_float2(b1f, b1f);
#pragma unroll
    for (int j4 = 0; j4 < BT / 4; ++j4) {
        const float4 a4 = asv[j4];
        const float2 alo = make_float2(a4.x, a4.y), ahi = make_float2(a4.z, a4.w);
        const float2 p0lo = __fmul2_rn(alo, b0), p0hi = __fmul2_rn(ahi, b0);
        const float2 p1lo = __fmul2_rn(alo, b1), p1hi = __fmul2_rn(ahi, b1);
        float2 r;
        r = __ffma2_rn(make_float2(v0[4 * j4], v0[4 * j4 + 1]), p0lo,
                       make_float2(acc0[4 * j4], acc0[4 * j4 + 1]));
        acc0[4 * j4] = r.x; acc0[4 * j4 + 1] = r.y;
        r = __ffma2_rn(make_float2(v0[4 * j4 + 2], v0[4 * j4 + 3]), p0hi,
                       make_float2(acc0[4 * j4 + 2], acc0[4 * j4 + 3]));
        acc0[4 * j4 + 2] = r.x; acc0[4 * j4 + 3] = r.y;
        r = __ffma2_rn(make_float2(v1[4 * j4], v1[4 * j4 + 1]), p1lo,
                       make_float2(acc1[4 * j4], acc1[4 * j4 + 1]));
        acc1[4 * j4] = r.x; acc1[4 * j4 + 1] = r.y;
        r = __ffma2_rn(make_float2(v1[4 * j4 + 2], v1[4 * j4 + 3]), p1hi,
                       make_float2(acc1[4 * j4 + 2], acc1[4 * j4 + 3]));
        acc1[4 * j4 + 2] = r.x; acc1[4 * j4 + 3] = r.y;
    }
}

__device__ __forceinline__ void ffma_chunk(float2* acc, const uint32_t (&v)[32], float f) {
    const float2 f2 = make_float2(f, f);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float2 x = make_float2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
        acc[i] = __ffma2_rn(x, f2, acc[i]);
    }
}

}  // namespace moe
