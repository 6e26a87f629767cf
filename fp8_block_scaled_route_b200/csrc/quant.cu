// Memory-bound element-wise kernels of the layer:
//  * quant_scatter: activation quantisation (W8A8 "A8", one fp32 scale per
//    token per 128 columns: scale = amax/448, codes = RNE_sat(x/scale)),
//    written straight into the k grouped rows of the token so GEMM1 reads a
//    dense [R, H] operand; also zeroes the token's fp32 combine row.
//  * f32_to_bf16: the combine buffer to the bf16 output (round to nearest even).
//  * swiglu_mxfp8: standalone SwiGLU + MXFP8 quantisation (E8M0 scale per 32).
// Page references: "FlashInfer: Blackwell W8A8 AlphaMoE Expert ..." (flashinfer
// PR #4287) for the W8A8 setting; "NVIDIA R200(SM107)을 위한 SwiGLU + MXFP8 커널
// 최적화" (flashinfer PR #8023) for SwiGLU + MXFP8 and its size-band launch.
#include <cuda_bf16.h>

#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace moe {

// One warp per (token, 128-column block): lane i owns columns 4i..4i+3.
__global__ void __launch_bounds__(256) quant_scatter_kernel(
    const __nv_bfloat16* __restrict__ x, int T, int H, int k, int R,
    const int32_t* __restrict__ inv_perm, uint8_t* __restrict__ xq, float* __restrict__ xs,
    float* __restrict__ out_acc) {
    const int nkb = H >> 7;
    const long long item = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (item >= static_cast<long long>(T) * nkb) return;
    const int lane = threadIdx.x & 31;
    const int t = static_cast<int>(item / nkb);
    const int kb = static_cast<int>(item - static_cast<long long>(t) * nkb);
    const long long off = static_cast<long long>(t) * H + kb * 128 + lane * 4;
    uint2 raw = *reinterpret_cast<const uint2*>(x + off);
    __nv_bfloat162 b01, b23;
    memcpy(&b01, &raw.x, 4);
    memcpy(&b23, &raw.y, 4);
    const float2 f01 = __bfloat1622float2(b01);
    const float2 f23 = __bfloat1622float2(b23);
    float amax = fmaxf(fmaxf(fabsf(f01.x), fabsf(f01.y)), fmaxf(fabsf(f23.x), fabsf(f23.y)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    const uint32_t codes = cvt_e4m3x4(__fdiv_rn(f01.x, s), __fdiv_rn(f01.y, s),
                                      __fdiv_rn(f23.x, s), __fdiv_rn(f23.y, s));
    for (int j = 0; j < k; ++j) {
        const int row = inv_perm[t * k + j];
        if (row < 0) continue;
        *reinterpret_cast<uint32_t*>(xq + static_cast<long long>(row) * H + kb * 128 + lane * 4) = codes;
        if (lane == 0) xs[static_cast<long long>(kb) * R + row] = s;
    }
    if (out_acc) *reinterpret_cast<float4*>(out_acc + off) = make_float4(0.f, 0.f, 0.f, 0.f);
}

int launch_quant_scatter(const void* x, int T, int H, int k, int R, const int32_t* inv_perm,
                         uint8_t* xq, float* xs, float* out_acc, cudaStream_t stream) {
    const long long items = static_cast<long long>(T) * (H / 128);
    if (items == 0) return ST_OK;
    const long long blocks = (items + 7) / 8;
    quant_scatter_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(x), T, H, k, R, inv_perm, xq, xs, out_acc);
    return cudaGetLastError() == cudaSuccess ? ST_OK : ST_CUDA;
}

__global__ void __launch_bounds__(256) f32_to_bf16_kernel(const float* __restrict__ in,
                                                          __nv_bfloat16* __restrict__ out,
                                                          long long n4) {
    for (long long i = blockIdx.x * 256ll + threadIdx.x; i < n4; i += static_cast<long long>(gridDim.x) * 256) {
        const float4 v = reinterpret_cast<const float4*>(in)[i];
        __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
        __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
        uint2 o;
        memcpy(&o.x, &a, 4);
        memcpy(&o.y, &b, 4);
        reinterpret_cast<uint2*>(out)[i] = o;
    }
}

int launch_f32_to_bf16(const float* in, void* out, long long n, int num_sms, cudaStream_t stream) {
    if (n == 0) return ST_OK;
    const long long n4 = n / 4;  // n is a multiple of 128
    long long blocks = (n4 + 255) / 256;
    const long long cap = static_cast<long long>(num_sms) * 8;
    if (blocks > cap) blocks = cap;
    f32_to_bf16_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        in, static_cast<__nv_bfloat16*>(out), n4);
    return cudaGetLastError() == cudaSuccess ? ST_OK : ST_CUDA;
}

// ------------------------------------------------------------ SwiGLU + MXFP8
// E8M0 code of the smallest power of two X = 2^s with amax <= 448 * X.
// With amax = m * 2^e, m in [1, 2): 448 = 1.75 * 2^8, so s = e - 8 when
// m <= 1.75 and s = e - 7 otherwise; computed exactly from the fp32 bits.
__device__ __forceinline__ uint32_t e8m0_code(float amax) {
    if (!(amax > 0.0f)) return 0u;
    uint32_t u = __float_as_uint(amax);
    int e;
    uint32_t mant;
    if ((u >> 23) == 0) {  // subnormal: normalise
        const int lz = __clz(u) - 8;  // leading zeros within the 24-bit significand
        mant = (u << lz) & 0x7FFFFFu;
        e = -126 - lz;
    } else {
        e = static_cast<int>(u >> 23) - 127;
        mant = u & 0x7FFFFFu;
    }
    const int s = e - 8 + (mant > 0x600000u ? 1 : 0);
    int c = s + 127;
    c = c < 0 ? 0 : (c > 254 ? 254 : c);
    return static_cast<uint32_t>(c);
}

__device__ __forceinline__ float e8m0_value(uint32_t c) {
    // 2^(c-127); c = 0 is the fp32 subnormal 2^-127
    return c == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(c << 23);
}

__device__ __forceinline__ float silu_q(float z) { return __fdiv_rn(z, 1.0f + expf(-z)); }

// Four threads per 32-element block, eight outputs each (16-byte loads).  The
// loop bound is uniform per warp so every lane reaches the shuffles.
__global__ void __launch_bounds__(256) swiglu_mxfp8_kernel(const __nv_bfloat16* __restrict__ in,
                                                           uint8_t* __restrict__ out,
                                                           uint8_t* __restrict__ scale, int M, int K) {
    const long long groups = static_cast<long long>(M) * (K / 8);
    const int kg = K / 8;
    for (long long gi = blockIdx.x * 256ll + threadIdx.x; gi - (threadIdx.x & 31) < groups;
         gi += static_cast<long long>(gridDim.x) * 256) {
        const bool live = gi < groups;
        float v[8];
        float amax = 0.0f;
        long long m = 0;
        int c0 = 0;
        if (live) {
            m = gi / kg;
            c0 = static_cast<int>(gi - m * kg) * 8;
            const uint4 gr = *reinterpret_cast<const uint4*>(in + m * 2 * K + c0);
            const uint4 ur = *reinterpret_cast<const uint4*>(in + m * 2 * K + K + c0);
            const uint32_t gw[4] = {gr.x, gr.y, gr.z, gr.w};
            const uint32_t uw[4] = {ur.x, ur.y, ur.z, ur.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                __nv_bfloat162 gb, ub;
                memcpy(&gb, &gw[i], 4);
                memcpy(&ub, &uw[i], 4);
                const float2 gf = __bfloat1622float2(gb);
                const float2 uf = __bfloat1622float2(ub);
                v[2 * i] = silu_q(gf.x) * uf.x;
                v[2 * i + 1] = silu_q(gf.y) * uf.y;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
        }
        // the four threads of a 32-block are lanes 4j..4j+3 of the warp
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        if (live) {
            const uint32_t code = e8m0_code(amax);
            const float X = e8m0_value(code);
            uint2 o;
            o.x = cvt_e4m3x4(__fdiv_rn(v[0], X), __fdiv_rn(v[1], X), __fdiv_rn(v[2], X), __fdiv_rn(v[3], X));
            o.y = cvt_e4m3x4(__fdiv_rn(v[4], X), __fdiv_rn(v[5], X), __fdiv_rn(v[6], X), __fdiv_rn(v[7], X));
            *reinterpret_cast<uint2*>(out + m * K + c0) = o;
            if ((c0 & 31) == 0) scale[m * (K / 32) + c0 / 32] = static_cast<uint8_t>(code);
        }
    }
}

int launch_swiglu_mxfp8(const void* in, void* out, uint8_t* scale, int M, int K, int num_sms,
                        cudaStream_t stream) {
    const long long groups = static_cast<long long>(M) * (K / 8);
    if (groups == 0) return ST_OK;
    long long blocks = (groups + 255) / 256;
    // size band: small problems (M*K < 2^20) use one 256-thread CTA per 2048
    // outputs so that several CTAs share an SM; larger ones stream with a
    // grid of a few waves of CTAs per SM.
    if (static_cast<long long>(M) * K >= (1ll << 20)) {
        const long long cap = static_cast<long long>(num_sms) * 8;
        if (blocks > cap) blocks = cap;
    }
    swiglu_mxfp8_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(in), static_cast<uint8_t*>(out), scale, M, K);
    return cudaGetLastError() == cudaSuccess ? ST_OK : ST_CUDA;
}

}  // namespace moe
