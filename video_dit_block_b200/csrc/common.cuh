// common.cuh -- device-side error word and bounded waits shared by the kernels.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace sba {

enum DeviceError : int { kErrNone = 0, kErrTimeout = 5, kErrBadRouting = 6 };

// One error word per device (the whole library is one translation unit).  The
// first error recorded wins; sba_get_device_status reads and clears it.
__device__ int g_device_error;

__device__ __forceinline__ void raise_device_error(int code) {
    atomicCAS(&g_device_error, 0, code);
}

// Limits below this are for tests of the timeout path: those waits only poll (a
// try_wait may suspend the thread for tens of microseconds, longer than such a limit).
constexpr uint64_t kPollOnlyLimit = 1ull << 20;

// Wait for phase `parity` of mbarrier `bar`, giving up when another thread of
// the CTA has set *abort, or after `limit` clock cycles (then the error word is
// set and *abort raised so every role of the CTA unwinds).  Returns true when
// the phase completed.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity,
                                             volatile uint32_t* abort, uint64_t limit) {
    if (limit < kPollOnlyLimit) {
        const long long t0 = clock64();
        while (!mbar_test_wait(bar, parity)) {
            if (*abort) return false;
            if ((uint64_t)(clock64() - t0) > limit) {
                raise_device_error(kErrTimeout);
                *abort = 1u;
                return false;
            }
        }
        return true;
    }
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if ((uint64_t)(clock64() - t0) > limit) {
            raise_device_error(kErrTimeout);
            *abort = 1u;
            return false;
        }
    }
}

// Bounded wait by polling (the thread is never suspended, so it resumes as soon as the
// phase completes).  For the MMA thread, whose every stall idles the tensor pipe.
__device__ __forceinline__ bool poll_bounded(uint32_t bar, uint32_t parity, volatile uint32_t* abort,
                                             uint64_t limit) {
    if (mbar_test_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_test_wait(bar, parity)) return true;
        if (*abort) return false;
        if ((uint64_t)(clock64() - t0) > limit) {
            raise_device_error(kErrTimeout);
            *abort = 1u;
            return false;
        }
    }
}

// Warp-collective form: every lane waits, and all lanes agree on the outcome,
// so warp-synchronous tcgen05 loads that follow are never reached by part of a warp.
__device__ __forceinline__ bool warp_wait_bounded(uint32_t bar, uint32_t parity,
                                                  volatile uint32_t* abort, uint64_t limit) {
    const bool ok = wait_bounded(bar, parity, abort, limit);
    return __all_sync(0xffffffffu, ok);
}

}  // namespace sba
