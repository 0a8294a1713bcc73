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

// Device-side argument checks of the debug build (-DKDA_DEBUG, built as
// libkda_b200_debug.so): a kernel checks the token range, sequence and head
// of its unit before touching memory; a bad one records ERR_BOUNDS and the
// unit is skipped (never a trap: the error word is read by
// kda_get_device_status).  In the release build the checks compile away.
#ifdef KDA_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif

// Element loads/stores for the two I/O dtypes.
__device__ __forceinline__ float ld(const float *p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ld(const __nv_bfloat16 *p, int64_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ void st(float *p, int64_t i, float x) { p[i] = x; }
__device__ __forceinline__ void st(__nv_bfloat16 *p, int64_t i, float x) { p[i] = __float2bfloat16_rn(x); }

__device__ __forceinline__ float sigmoidf(float z) { return 1.0f / (1.0f + expf(-z)); }

// Snapshots of the state at token offsets that are multiples of `interval`
// (the prefix-cache hook): slot base[n] + m - 1 of `states` ([total][H][dk][dv]
// fp32) receives sequence n's state after its first m * interval tokens.
struct SnapOut {
    float *states;          // nullptr: no snapshots
    const int64_t *base;    // [num_seqs + 1], caller-provided first slot per sequence
    int64_t total;          // slots in `states`
    int32_t interval;       // a positive multiple of the chunk
};

// Slot for the state after `rel` tokens of sequence n, or -1 if none is due.
// A slot outside [0, total) records a bounds error and is skipped.
__device__ __forceinline__ int64_t snap_slot(const SnapOut &sn, int n, int64_t rel) {
    if (!sn.states || rel <= 0 || rel % sn.interval != 0) return -1;
    const int64_t slot = sn.base[n] + rel / sn.interval - 1;
    if (slot < 0 || slot >= sn.total) {
        if (threadIdx.x == 0) raise_error(ERR_BOUNDS);
        return -1;
    }
    return slot;
}

}  // namespace kda
