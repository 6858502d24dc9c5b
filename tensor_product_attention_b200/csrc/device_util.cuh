// Small device helpers shared by the kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace tpa {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Record the first device-side error in the library's error word (never traps).
__device__ __forceinline__ void raise_error(int* err, int code) {
    if (err) atomicCAS(err, 0, code);
}

// Index checks of the bounds-checked build (-DTPA_DEBUG_BOUNDS, libtpa_debug.so): a
// plain global access is made only if in_bounds() holds; a failed check records
// TPA_DEVERR_BOUNDS (2) in the error word and the access is skipped, so a bad index
// shows up as an error code, never as a fault.  Release builds compile the checks away.
__device__ __forceinline__ bool in_bounds(bool ok, int* err) {
#ifdef TPA_DEBUG_BOUNDS
    if (!ok) raise_error(err, 2);
    return ok;
#else
    (void)ok;
    (void)err;
    return true;
#endif
}

}  // namespace tpa
