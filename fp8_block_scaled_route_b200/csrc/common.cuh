// Shared device-side definitions: status codes, the device status word and
// bounded waits.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace moe {

enum : int {
    ST_OK = 0,
    ST_INVALID_ARG = 1,
    ST_UNSUPPORTED = 2,
    ST_CUDA = 3,
    ST_NO_TILE_CONFIG = 4,
    ST_DEVICE_TIMEOUT = 5,
    ST_BAD_EXPERT_ID = 6,
};

// Layout of a device status word (4 ints, 16 bytes):
//   [0] first error code recorded (0 = none)
//   [1] where a timeout happened (role id), for diagnostics
//   [2] number of dropped pairs (bad expert ids)
//   [3] reserved
constexpr int kStatusInts = 4;

__device__ __forceinline__ void report_error(int* status, int code, int where) {
    if (status == nullptr) return;
    if (atomicCAS(status, 0, code) == 0) status[1] = where;
}

// Control block for bounded waits inside one CTA.  `abort` lives in shared
// memory: once any thread of the CTA gives up, the others stop waiting too.
struct WaitCtl {
    volatile int* abort;
    int* status;
    uint64_t timeout_ns;
};

// Bound of the waits that drain in-flight copies and MMAs before a CTA
// exits; independent of the caller's timeout so that an early abort still
// lets every outstanding copy land.
constexpr uint64_t kDrainTimeoutNs = 2000000000ull;

// Waits until the mbarrier phase with the given parity has completed.
// Returns false when the CTA is aborting or the wait ran out of time (the
// first thread to run out records ST_DEVICE_TIMEOUT).  With `drain = true`
// the wait ignores the abort flag and is bounded by kDrainTimeoutNs.
// The thread sleeps in the barrier (hardware suspend, woken by the phase
// completing) instead of spinning, and reads the clock only every 8th round,
// so waiting warps take almost no issue slots from working ones.
constexpr uint32_t kWaitSuspendNs = 20000;

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const WaitCtl& c,
                                         int where, bool drain = false) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    const uint64_t limit = drain ? kDrainTimeoutNs : c.timeout_ns;
#pragma unroll 1
    for (uint32_t round = 1;; ++round) {
        if (mbar_try_wait_sleep(bar, parity, kWaitSuspendNs)) return true;
        if (!drain && *c.abort) return false;
        if ((round & 7) == 0 || limit < 1000000ull) {
            if (globaltimer() - t0 > limit) {
                *c.abort = 1;
                report_error(c.status, ST_DEVICE_TIMEOUT, where);
                return false;
            }
        }
    }
}

// Spinning variant for the single producer and MMA threads: no hardware
// suspend, so a completed phase is seen within a few cycles; the clock is
// read every 256th poll.
__device__ __forceinline__ bool wait_bar_spin(uint64_t* bar, uint32_t parity, const WaitCtl& c,
                                              int where) {
    if (mbar_test_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    const bool short_limit = c.timeout_ns < 1000000ull;
#pragma unroll 1
    for (uint32_t round = 1;; ++round) {
        if (mbar_test_wait(bar, parity)) return true;
        if ((round & 255) == 0 || short_limit) {
            if (*c.abort) return false;
            if (globaltimer() - t0 > c.timeout_ns) {
                *c.abort = 1;
                report_error(c.status, ST_DEVICE_TIMEOUT, where);
                return false;
            }
        }
    }
}

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

// 2^(127 - c): the exact reciprocal of the E8M0 value 2^(c - 127).  x * 2^-s
// and x / 2^s round the same exact value once, so the product is bit-identical
// to the IEEE quotient for every x (subnormal results included).
__device__ __forceinline__ float e8m0_reciprocal(uint32_t c) {
    // c = 0 -> 2^127, c = 254 -> 2^-127 (an fp32 subnormal, exactly representable)
    return c == 254 ? __uint_as_float(0x00400000u) : __uint_as_float((254u - c) << 23);
}

}  // namespace moe
