// sscan_check.cuh -- index checks of the debug build (compiled with SSCAN_DEBUG_BOUNDS,
// which the build script sets for libsscan_debug.so together with relocatable device
// code, so that every kernel reports into the one device status word).
//
// The kernels guard each access to a workspace, parameter or state array whose index
// they compute (as opposed to the TMA tile copies, which the hardware bounds) with
// in_range(index, extent).  The release build compiles the guard away.  The debug
// build checks it: on an index outside [0, extent) it raises bit 3 of the device
// status word (read by sscan_device_status) and returns false, and the caller skips
// the access -- a stand-in for a memory checker that never faults or traps.
#pragma once

#include <cstdint>

namespace sscan {

constexpr unsigned int kErrBounds = 8u;

#ifdef SSCAN_DEBUG_BOUNDS
extern __device__ unsigned int g_device_error;
#endif

__device__ __forceinline__ bool in_range(int64_t i, int64_t n) {
#ifdef SSCAN_DEBUG_BOUNDS
    if (i >= 0 && i < n) return true;
    atomicOr(&g_device_error, kErrBounds);
    return false;
#else
    (void)i;
    (void)n;
    return true;
#endif
}

}  // namespace sscan
