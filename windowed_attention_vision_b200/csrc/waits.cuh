// Bounded waits shared by the persistent kernels: each gives up after
// kWaitLimitNs, sets the CTA's abort flag and the device status word, and
// returns false, so every role can drain and return instead of hanging.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace winattn {

// Bounded wait that also gives up as soon as another role has aborted.  A
// try_wait blocks in hardware until the phase completes or a system-dependent
// time passes (thousands of cycles), so a waiting warp takes almost no issue
// slots from the warps doing the work.  Without a suspend-time hint it wakes
// sooner after the phase completes (measured per tile on the pipelined kernel).
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile uint32_t *abort_flag)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag)
            return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            *abort_flag = 1u;
            atomicOr(&g_status_word, 1u);
            return false;
        }
    }
    return true;
}

// The same, with one verdict for the whole warp (its tcgen05 loads and stores
// are warp-collective, so the warp must leave a loop together).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile uint32_t *abort_flag)
{
    return __all_sync(0xffffffffu, wait_or_abort(bar, parity, abort_flag));
}

}  // namespace winattn
