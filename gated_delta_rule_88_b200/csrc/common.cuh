// common.cuh -- small device helpers shared by the KDA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// Device error word: kernels that wait on barriers receive its address and
// set it (never trap) when a bounded wait runs out; kda_get_device_error()
// reads and clears it.  The word itself is defined in api.cu.
enum DeviceError : int {
    kErrNone = 0,
    kErrWaitTimeout = 1,     // an mbarrier wait exceeded its bound
};

__device__ __forceinline__ void set_device_error(int *word, int code) {
    if (word) atomicCAS(word, 0, code);
}

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Streaming 128-bit global load / store (evict-first: data touched once).
__device__ __forceinline__ float4 ld_stream(const float4 *p) { return __ldcs(p); }
__device__ __forceinline__ void st_stream(float4 *p, float4 v) { __stcs(p, v); }

}  // namespace kda
