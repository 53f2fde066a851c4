// Shared device helpers for the retention kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "ret.h"

namespace ret {

// Device error word. A kernel whose bounded wait runs out ORs a code in here;
// ret_last_device_error() reads and clears it. One per device (module scope).
__device__ unsigned int g_error_word;

enum : unsigned int {
    kErrWaitTimeout = 1u,  // an mbarrier / flag wait exceeded its iteration limit
};

__device__ __forceinline__ void raise_error(unsigned int code) { atomicOr(&g_error_word, code); }

// ---------------------------------------------------------------- element IO

template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float load(const float* p) { return *p; }
    static __device__ __forceinline__ void store(float* p, float x) { *p = x; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
};

template <typename T>
__device__ __forceinline__ float ld_elem(const T* p) { return Elem<T>::load(p); }
template <typename T>
__device__ __forceinline__ void st_elem(T* p, float x) { Elem<T>::store(p, x); }

// gamma^n for an integer n >= 0 given log2(gamma); gamma^0 = 1 even for gamma = 0
// (log2(0) = -inf and exp2(-inf) = 0 give the n > 0 cases).
__device__ __forceinline__ float pow_int_log2(float log2g, int n) {
    return n == 0 ? 1.0f : exp2f(log2g * (float)n);
}

constexpr float kLog2e = 1.4426950408889634f;

}  // namespace ret
