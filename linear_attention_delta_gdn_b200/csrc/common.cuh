// common.cuh -- small device helpers shared by the libgdn2 kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn2.h"

namespace gdn2 {

// Problem sizes of one call. Token tensors are [B, T, H, D]; states [B, H, Dk, Dv].
struct Dims {
    int B, T, H, Dk, Dv, chunk;
    int nchunks() const { return (T + chunk - 1) / chunk; }
};

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// offset of element (b, t, h, 0) of a [B, T, H, D] tensor
__host__ __device__ __forceinline__ size_t tok_off(int b, int t, int h, int T, int H, int D) {
    return (((size_t)b * T + t) * H + h) * (size_t)D;
}

__device__ __forceinline__ float fast_exp(float x) { return exp2f(x * 1.4426950408889634f); }

// Index checks of the debug build (compiled with -DGDN2_DEBUG into libgdn2_debug.so). GDN2_IN(word, cond) is
// true when cond holds; otherwise it sets GDN2_DBG_BIT in the kernel's error word and is false, and the caller
// skips the access it guards, so the kernel returns normally and gdn2_device_status reports the failure.
// Nothing traps. In release builds every check is the constant true and costs nothing.
constexpr unsigned int GDN2_DBG_BIT = 1u << 30;
#ifdef GDN2_DEBUG
#define GDN2_IN(word, cond) ((cond) ? true : (atomicOr(&(word), ::gdn2::GDN2_DBG_BIT), false))
#else
#define GDN2_IN(word, cond) true
#endif

}  // namespace gdn2
