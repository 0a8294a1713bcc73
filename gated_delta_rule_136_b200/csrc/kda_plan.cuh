// kda_plan.cuh -- device-side work planning: sequences ordered longest-first
// (longest-processing-time-first), so the CTAs that carry the longest state
// chains start first and short sequences fill in behind them.
#pragma once

#include "kda_common.cuh"

namespace kda {

constexpr int32_t kPlanSortLimit = 8192;   // above this, keep the natural order

// order[rank(n)] = n with rank(n) = #{m : L_m > L_n or (L_m == L_n and m < n)}:
// a stable descending sort by length, one thread per sequence.
__global__ void plan_longest_first_kernel(const int32_t *__restrict__ cu, int32_t N,
                                          int32_t *__restrict__ order)
{
    __shared__ int32_t lens[1024];
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    const int32_t Ln = n < N ? cu[n + 1] - cu[n] : 0;
    int32_t rank = 0;
    for (int base = 0; base < N; base += 1024) {
        __syncthreads();
        for (int i = threadIdx.x; i < 1024 && base + i < N; i += blockDim.x)
            lens[i] = cu[base + i + 1] - cu[base + i];
        __syncthreads();
        const int lim = min(1024, N - base);
        for (int i = 0; i < lim; ++i) {
            const int32_t Lm = lens[i];
            const int m = base + i;
            rank += (Lm > Ln) || (Lm == Ln && m < n);
        }
    }
    if (n < N) order[rank] = n;
}

__global__ void plan_identity_kernel(int32_t N, int32_t *__restrict__ order)
{
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n < N) order[n] = n;
}

inline cudaError_t launch_plan_longest_first(const int32_t *cu, int32_t N, int32_t *order,
                                             cudaStream_t stream)
{
    const int threads = 256;
    const int blocks = (N + threads - 1) / threads;
    if (N <= kPlanSortLimit)
        plan_longest_first_kernel<<<blocks, threads, 0, stream>>>(cu, N, order);
    else
        plan_identity_kernel<<<blocks, threads, 0, stream>>>(N, order);
    return cudaGetLastError();
}

}  // namespace kda
