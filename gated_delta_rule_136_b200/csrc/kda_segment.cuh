// kda_segment.cuh -- prefix scan of the long-sequence segment split.
//
// A long sequence is cut into segments p = 0..P-1.  Every segment's effect on
// the state is affine: S_end = M_p S_in + S_loc,p, with M_p the product of the
// segment's transitions and S_loc,p the state the segment grows from zero
// (from S0 for p = 0).  A first prefill pass produces S_loc,p and M_p for every
// segment independently; this kernel then stitches them in order,
//   S_in(1) = S_loc,0,   S_in(p+1) = M_p S_in(p) + S_loc,p,
// and a second pass reruns every segment from its S_in (the context-parallel
// decomposition of the fupanwang.com Kimi K3 report digest, section 基础设施:
// own state plus the incoming state times the transition product, joined by a
// prefix scan).  Across GPUs the same fold runs on the summaries that every
// rank contributes to an all-gather (kda_state_combine): there only the last
// start state, S_last, is written.
#pragma once

#include "kda_common.cuh"

namespace kda {

struct ScanJob {
    const float *S_loc;   // [P][dk][dv] segment-local final states (stride job_stride)
    const float *M;       // [P][dk][dk] segment transition products
    float *S_in;          // [P][dk][dv] start states (entries 1..P-1 written), or null
    int64_t stride;       // floats between consecutive segments' matrices
    int32_t num_segments;
    float *S_last;        // if not null: S_in(P-1) is also written here
    int32_t product;      // 1: S_loc is read for segment 0 only, so S_in(P-1) = M_{P-2} ... M_1 S_loc,0
};

// One CTA (256 threads) per (sequence, head).  dk = dv = 128; thread (v, half)
// computes rows c in [64 half, 64 half + 64) of column v.
__device__ __forceinline__ void scan_one(const ScanJob &job)
{
    constexpr int D = 128;
    extern __shared__ float4 scan_smem[];
    float *Ms = reinterpret_cast<float *>(scan_smem);   // [D][D]
    float *Ss = Ms + D * D;                              // [D][D]
    const int tid = threadIdx.x, v = tid & 127, half = tid >> 7;

    for (int idx = tid; idx < D * D; idx += 256) {
        const float x = job.S_loc[idx];
        Ss[idx] = x;
        if (job.S_in) job.S_in[job.stride + idx] = x;     // S_in(1) = S_loc,0
        if (job.S_last && job.num_segments == 2) job.S_last[idx] = x;
    }
    __syncthreads();
    for (int seg = 1; seg + 1 < job.num_segments; ++seg) {
        const float *Mp = job.M + seg * job.stride;
        for (int idx = tid; idx < D * D / 4; idx += 256)
            reinterpret_cast<float4 *>(Ms)[idx] = reinterpret_cast<const float4 *>(Mp)[idx];
        __syncthreads();
        float acc[64];
        const float *Sl = job.S_loc + seg * job.stride;
#pragma unroll
        for (int r = 0; r < 64; ++r) acc[r] = job.product ? 0.0f : Sl[(half * 64 + r) * D + v];
        for (int c4 = 0; c4 < D; c4 += 4) {
            const float s0 = Ss[(c4 + 0) * D + v], s1 = Ss[(c4 + 1) * D + v];
            const float s2 = Ss[(c4 + 2) * D + v], s3 = Ss[(c4 + 3) * D + v];
#pragma unroll
            for (int r = 0; r < 64; ++r) {
                const float4 m = *reinterpret_cast<const float4 *>(Ms + (half * 64 + r) * D + c4);
                acc[r] = fmaf(m.x, s0, fmaf(m.y, s1, fmaf(m.z, s2, fmaf(m.w, s3, acc[r]))));
            }
        }
        __syncthreads();
        float *out = job.S_in ? job.S_in + (seg + 1) * job.stride
                              : (seg + 2 == job.num_segments ? job.S_last : nullptr);
        float *out2 = job.S_in && seg + 2 == job.num_segments ? job.S_last : nullptr;
#pragma unroll
        for (int r = 0; r < 64; ++r) {
            Ss[(half * 64 + r) * D + v] = acc[r];
            if (out) out[(half * 64 + r) * D + v] = acc[r];
            if (out2) out2[(half * 64 + r) * D + v] = acc[r];
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(256) segment_scan_kernel(const ScanJob *jobs)
{
    scan_one(jobs[blockIdx.x]);
}

// kda_state_combine: block u folds the summaries of (sequence, head) u, laid
// out [P][2][units][D][D] (S_loc, then M), into S_last[u].
__global__ void __launch_bounds__(256) state_combine_kernel(const float *summaries, float *S_in,
                                                            int64_t units, int32_t num_summaries)
{
    constexpr int64_t DD = 128 * 128;
    const int64_t u = blockIdx.x;
    scan_one(ScanJob{summaries + u * DD, summaries + (units + u) * DD, nullptr, 2 * units * DD,
                     num_summaries + 1, S_in + u * DD, 0});
}

}  // namespace kda
