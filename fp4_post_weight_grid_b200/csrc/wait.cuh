// wait.cuh -- the one spin-wait of the library, bounded.
//
// A thread block that has to wait for other thread blocks of the same launch
// (the batch kernel's NVFP4 tiles for the maximum of their weight, the
// one-launch sweep's grid barrier) polls a counter in global memory through
// this function.  It gives up after `limit` polls about 128 ns apart (the
// hardware sleeps between 0 and twice the requested time), so no wait can
// hang: its caller reports a wait that ran out as FP4Q_FLAG_TIMEOUT and
// skips the work that depended on it.
#pragma once

#include <cstdint>

namespace fp4q {

// Default limit of the library's waits: 2^24 polls, about 2 to 4 seconds.
constexpr unsigned kWaitLimit = 1u << 24;

// True once *p >= target; false if it is still below after `limit` polls.
__device__ __forceinline__ bool wait_geq(const unsigned* p, unsigned target, unsigned limit)
{
    const volatile unsigned* v = p;
    for (unsigned it = 0; it < limit; ++it) {
        if (*v >= target) return true;
        __nanosleep(128);
    }
    return *v >= target;
}

}  // namespace fp4q
