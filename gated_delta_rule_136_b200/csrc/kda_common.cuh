// kda_common.cuh -- small device helpers shared by the KDA kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// Per-device error word.  Kernels OR a status bit in and return instead of
// trapping; kda_get_device_status() reads and clears it.
__device__ unsigned int g_err_word;

enum : unsigned int { ERR_TIMEOUT = 1u, ERR_BOUNDS = 2u };

__device__ __forceinline__ void raise_error(unsigned int bit) { atomicOr(&g_err_word, bit); }

// Element loads/stores for the two I/O dtypes.
__device__ __forceinline__ float ld(const float *p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ld(const __nv_bfloat16 *p, int64_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ void st(float *p, int64_t i, float x) { p[i] = x; }
__device__ __forceinline__ void st(__nv_bfloat16 *p, int64_t i, float x) { p[i] = __float2bfloat16_rn(x); }

__device__ __forceinline__ float sigmoidf(float z) { return 1.0f / (1.0f + expf(-z)); }

}  // namespace kda
