// common.cuh -- small device helpers shared by the libmuir kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace muir {

// Loads of one input element as float32, whatever its storage type.
__device__ __forceinline__ float ldf(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ldf(const __nv_bfloat16* p) {
    return __bfloat162float(__ldg(reinterpret_cast<const __nv_bfloat16*>(p)));
}

// Stores of a float32 value in the output storage type (round to nearest even).
__device__ __forceinline__ void stf(float* p, float x) { *p = x; }
__device__ __forceinline__ void stf(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// Lower clamp on the per-token log decay inside the chunk kernels: every
// pivoted exponential then stays below exp(4 * 20) = exp(80), inside float32.
constexpr float kLogDecayMin = -20.0f;

}  // namespace muir
