// kernel_common.cuh -- device helpers shared by the tcgen05 kernels: bounded
// mbarrier waits and tile geometry.
#pragma once

#include "../../include/veda.h"
#include "ptx.cuh"

namespace veda {

// Suspend-time hint of one barrier test in the drains on the way out: the
// waiting warp sleeps in hardware (woken when the phase completes).
constexpr uint32_t kSuspendNs = 20000;

// Bounded wait: false when the time limit expired (VEDA_ERR_TIMEOUT is then
// recorded and the CTA's abort flag raised) or another role aborted.  P is a
// kernel parameter struct with `status` and `wait_limit_ns` fields.  The wait
// spins on the non-blocking test (the clock is read every 64 tests): the
// pipelines hand off every few hundred cycles, and waking a suspended thread
// costs more than the spin takes from the warps sharing its sub-partition
// (measured: 2-4% faster attention than suspending between tests).
template <class P>
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const P& p,
                                         volatile int* abort_flag) {
    for (int i = 0; i < 64; ++i)
        if (mbar_test_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        for (int i = 0; i < 64; ++i)
            if (mbar_test_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > p.wait_limit_ns) {
            *abort_flag = 1;
            atomicCAS(p.status, 0, (int)VEDA_ERR_TIMEOUT);
            return false;
        }
    }
}

// Bounded wait that ignores the abort flag (drain on the way out).
template <class P>
__device__ __forceinline__ void drain_bar(uint64_t* bar, uint32_t parity, const P& p) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait_sleep(bar, parity, kSuspendNs)) {
        if (global_timer_ns() - t0 > p.wait_limit_ns) {
            atomicCAS(p.status, 0, (int)VEDA_ERR_TIMEOUT);
            return;
        }
    }
}

// Warp-uniform bounded wait: lane 0 polls, the outcome is broadcast and the
// warp re-converges (the thread sync orders the other lanes after the wait).
template <class P>
__device__ __forceinline__ bool warp_wait_bar(uint64_t* bar, uint32_t parity, const P& p,
                                              volatile int* abort_flag) {
    int ok = 0;
    if ((threadIdx.x & 31) == 0) ok = wait_bar(bar, parity, p, abort_flag) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// Order-preserving 32-bit key of a finite fp32 score: a larger score gives a
// larger key; -0.0 and +0.0 give the same key.
__device__ __forceinline__ uint32_t order_key(float v) {
    uint32_t u = __float_as_uint(v);
    if ((u << 1) == 0) u = 0;  // -0.0 -> +0.0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Grid origin (t0, y0, x0) of tile t for tile shape (pt, ph, pw).
__device__ __forceinline__ void tile_origin(int t, int pt, int ph, int pw, int Hs, int Ws,
                                            int& t0, int& y0, int& x0) {
    const int nh = Hs / ph, nw = Ws / pw;
    t0 = (t / (nh * nw)) * pt;
    y0 = ((t / nw) % nh) * ph;
    x0 = (t % nw) * pw;
}

}  // namespace veda
