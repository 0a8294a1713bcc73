// kda_lib.cu -- the C ABI of include/kda.h: argument validation, planning,
// kernel dispatch and device status.  All kernels are included here so the
// library is one translation unit (the device error word needs no
// relocatable device code).
#include "kda.h"

#include <cmath>
#include <cstdint>
#include <cstring>

#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>
#include <algorithm>
#include <cstdlib>
#include <mutex>
#include <initializer_list>
#include <vector>

#include "kda_common.cuh"
#include "kda_chunk_simt.cuh"
#include "kda_chunk_tc.cuh"
#include "kda_decode.cuh"
#include "kda_spec.cuh"
#include "kda_plan.cuh"
#include "kda_segment.cuh"
#include "kda_bwd.cuh"
#include "kda_bwd_chunk.cuh"

namespace {
// NVTX range over a host-side launch sequence (plan, chunk passes, scan, ...):
// a profiler attached to the process shows which kernels each range issued.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};
}  // namespace

namespace {

using kda::SimtParams;
using kda::DecodeParams;

constexpr float kMinFloor = -5.45f;   // 16 * floor must stay above ln(FLT_MIN)

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool supported_dim(int32_t d) { return d == 64 || d == 128; }

struct Range {
    uintptr_t lo, hi;   // [lo, hi)
};

inline Range range_of(const void *p, int64_t bytes) {
    uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return Range{a, a + static_cast<uintptr_t>(bytes)};
}

inline bool overlaps(Range a, Range b) {
    if (a.lo == a.hi || b.lo == b.hi || a.lo == 0 || b.lo == 0) return false;
    return a.lo < b.hi && b.lo < a.hi;
}

// element count a*b*c without int64 overflow; -1 on overflow
inline int64_t mul3(int64_t a, int64_t b, int64_t c) {
    if (a < 0 || b < 0 || c < 0) return -1;
    const int64_t lim = INT64_MAX / 16;
    if (a && b > lim / a) return -1;
    int64_t ab = a * b;
    if (ab && c > lim / ab) return -1;
    return ab * c;
}

kda_status validate_fwd_desc(const kda_fwd_desc *d) {
    if (!d) return KDA_ERR_INVALID_ARG;
    if (d->num_seqs < 1 || d->num_heads < 1 || d->total_tokens < 0) return KDA_ERR_INVALID_ARG;
    if (d->dk <= 0 || d->dv <= 0) return KDA_ERR_INVALID_ARG;
    if (!supported_dim(d->dk) || !supported_dim(d->dv)) return KDA_ERR_UNSUPPORTED;
    if (d->io_dtype != KDA_BF16 && d->io_dtype != KDA_FP32) return KDA_ERR_INVALID_ARG;
    if (!std::isfinite(d->scale)) return KDA_ERR_INVALID_ARG;
    if (!(d->g_floor >= kMinFloor && d->g_floor <= 0.0f)) return KDA_ERR_INVALID_ARG;
    if (d->chunk != 0 && d->chunk != 16 && d->chunk != 64) return KDA_ERR_INVALID_ARG;
    if (d->max_seqlen < 0) return KDA_ERR_INVALID_ARG;
    if (mul3(d->total_tokens, d->num_heads, 128) < 0) return KDA_ERR_INVALID_ARG;
    if (mul3(d->num_seqs, d->num_heads, (int64_t)d->dk * d->dv) < 0) return KDA_ERR_INVALID_ARG;
    return KDA_OK;
}

kda_status validate_host_seqlens(const kda_fwd_desc *d, const int32_t *cu) {
    if (!cu) return KDA_OK;
    if (cu[0] != 0) return KDA_ERR_INVALID_ARG;
    for (int32_t n = 0; n < d->num_seqs; ++n)
        if (cu[n + 1] < cu[n]) return KDA_ERR_INVALID_ARG;
    if ((int64_t)cu[d->num_seqs] != d->total_tokens) return KDA_ERR_INVALID_ARG;
    if (d->max_seqlen > 0) {
        for (int32_t n = 0; n < d->num_seqs; ++n)
            if (cu[n + 1] - cu[n] > d->max_seqlen) return KDA_ERR_INVALID_ARG;
    }
    return KDA_OK;
}

// ---------------------------------------------------------------- long-sequence split
// When there are fewer (sequence, head) units than SMs, long sequences are cut
// into segments so that the tensor-core prefill still fills the GPU (needs
// cu_seqlens_host).  KDA_SEGMENTS=<P> forces P segments per sequence, and
// KDA_SEGMENTS=1 disables the split (tuning and tests).
constexpr int64_t kMinSegTokens = 1024;

int device_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        (void)cudaGetLastError();
        return 148;
    }
    return n;
}

struct SegPlan {
    bool active = false;
    std::vector<int32_t> nseg;      // segments per sequence (1: not split)
    std::vector<int64_t> seglen;    // tokens per segment (multiple of 64)
    int64_t pass1_units = 0, pass2_units = 0, jobs = 0, mat_blocks = 0;
};

bool tc_shape(const kda_fwd_desc &d) {
    return d.io_dtype == KDA_BF16 && d.dk == 128 && d.dv == 128 && d.chunk != 16 &&
           d.total_tokens > 0 && d.total_tokens <= INT32_MAX - 64;
}

SegPlan plan_segments(const kda_fwd_desc &d, const int32_t *cu) {
    SegPlan pl;
    const int32_t N = d.num_seqs, H = d.num_heads;
    pl.nseg.assign(N, 1);
    pl.seglen.assign(N, 0);
    if (!cu || !tc_shape(d)) {
        pl.pass2_units = (int64_t)N * H;
        return pl;
    }
    const char *env = std::getenv("KDA_SEGMENTS");
    const int forced = env ? std::atoi(env) : 0;
    const int64_t units = (int64_t)N * H;
    const int sms = device_sm_count();
    // Wave model with the longest sequence's chunk count C: unsplit time ~
    // ceil(U / SMs) * C; with P segments pass 1 runs U (2P - 3) units and pass 2
    // U P units, each of ceil(C / P) chunks.  Take the best P, and split only
    // if it saves at least 10 %.
    int64_t best_p = 1;
    if (forced < 1 && units < sms) {          // KDA_SEGMENTS=1: no split
        int64_t cmax = 0;
        for (int32_t n = 0; n < N; ++n) cmax = std::max<int64_t>(cmax, ((int64_t)cu[n + 1] - cu[n] + 63) / 64);
        auto waves = [&](int64_t x) { return (x + sms - 1) / sms; };
        const int64_t t1 = waves(units) * cmax;
        int64_t best_t = t1;
        for (int64_t P = 2; P <= 64 && P * kMinSegTokens / 64 <= cmax; ++P) {
            const int64_t t = (waves(units * (2 * P - 3)) + waves(units * P)) * ((cmax + P - 1) / P);
            if (t < best_t) { best_t = t; best_p = P; }
        }
        if (best_t * 10 > t1 * 9) best_p = 1;
    }
    for (int32_t n = 0; n < N; ++n) {
        const int64_t L = (int64_t)cu[n + 1] - cu[n];
        int64_t P = 1;
        if (forced > 1)
            P = std::min<int64_t>(forced, L / 128);
        else if (best_p > 1)
            P = std::min<int64_t>(best_p, L / kMinSegTokens);
        if (P >= 2) {
            const int64_t seg = ((L + P - 1) / P + 63) / 64 * 64;
            P = (L + seg - 1) / seg;
        }
        if (P >= 2) {
            pl.active = true;
            pl.nseg[n] = (int32_t)P;
            pl.seglen[n] = ((L + P - 1) / P + 63) / 64 * 64;
            pl.pass1_units += (int64_t)H * ((P - 1) + (P - 2));
            pl.jobs += H;
            pl.mat_blocks += (int64_t)H * P;
        }
        pl.pass2_units += (int64_t)H * pl.nseg[n];
    }
    return pl;
}

// Workspace layout (each region 256-byte aligned):
//   int32 seq_order[N]                       sequences longest-first
//   with a segment split (cu_seqlens_host given, see plan_segments):
//   TcUnit pass1[...], TcUnit pass2[...], ScanJob jobs[...],
//   fp32 matrices: per split (sequence, head), per segment: S_loc, M, S_in
struct WsLayout {
    size_t order = 0, pass1 = 0, pass2 = 0, jobs = 0, mats = 0, total = 0;
};

WsLayout ws_layout(const kda_fwd_desc *d, const SegPlan &pl) {
    WsLayout w;
    size_t off = align256(sizeof(int32_t) * (size_t)d->num_seqs);
    if (pl.active) {
        w.pass1 = off; off += align256(sizeof(kda::tck::TcUnit) * (size_t)pl.pass1_units);
        w.pass2 = off; off += align256(sizeof(kda::tck::TcUnit) * (size_t)pl.pass2_units);
        w.jobs = off;  off += align256(sizeof(kda::ScanJob) * (size_t)pl.jobs);
        w.mats = off;  off += align256((size_t)pl.mat_blocks * 3u * 128u * 128u * sizeof(float));
    }
    w.total = off;
    return w;
}

size_t fwd_workspace_bytes(const kda_fwd_desc *d, const int32_t *cu_host) {
    return ws_layout(d, plan_segments(*d, cu_host)).total;
}

template <int DK, int DV, typename TIO>
cudaError_t launch_simt(const SimtParams &p, int32_t num_seqs, cudaStream_t stream) {
    const size_t smem = kda::simt_smem_bytes<DK, DV>();
    auto kern = kda::chunk_simt_kernel<DK, DV, TIO>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t blocks = (int64_t)num_seqs * p.num_heads;
    if (blocks > INT32_MAX) return cudaErrorInvalidConfiguration;
    kern<<<(unsigned)blocks, 2 * DV, smem, stream>>>(p);
    return cudaGetLastError();
}

template <typename TIO>
cudaError_t dispatch_simt(int dk, int dv, const SimtParams &p, int32_t n, cudaStream_t s) {
    if (dk == 128 && dv == 128) return launch_simt<128, 128, TIO>(p, n, s);
    if (dk == 128 && dv == 64) return launch_simt<128, 64, TIO>(p, n, s);
    if (dk == 64 && dv == 128) return launch_simt<64, 128, TIO>(p, n, s);
    return launch_simt<64, 64, TIO>(p, n, s);
}

// cuTensorMapEncodeTiled through the runtime, so the library needs no link
// against the driver library.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 2-D view [rows, cols] of a row-major bf16 tensor, 64 x 64 boxes, 128-byte swizzle.
bool encode_bf16_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The tensor-core prefill covers bf16 I/O with dk = dv = 128 and 16-byte
// aligned q, k, v, g and o (all moved by TMA); chunk = 16 and every other
// shape use the CUDA-core kernel.
bool tc_path_applies(const kda_fwd_desc &d, const void *q, const void *k, const void *v,
                     const void *g, const void *o) {
    if (!tc_shape(d)) return false;
    for (const void *ptr : {q, k, v, g, o})
        if (reinterpret_cast<uintptr_t>(ptr) % 16 != 0) return false;
    return true;
}

cudaError_t launch_tc_units(const kda_fwd_desc &d, const void *q, const void *k, const void *v,
                            const void *g, const kda::tck::TcParams &p, int64_t blocks,
                            cudaStream_t stream, bool no_out = false);

cudaError_t launch_tc(const kda_fwd_desc &d, const void *q, const void *k, const void *v,
                      const void *g, const kda::tck::TcParams &p, cudaStream_t stream) {
    return launch_tc_units(d, q, k, v, g, p, (int64_t)d.num_seqs * d.num_heads, stream);
}

// no_out: no unit of the launch stores outputs (the split's first pass, the
// context-parallel summaries): the kernel instance without the q side.
cudaError_t launch_tc_units(const kda_fwd_desc &d, const void *q, const void *k, const void *v,
                            const void *g, const kda::tck::TcParams &p, int64_t blocks,
                            cudaStream_t stream, bool no_out) {
    CUtensorMap tq, tk, tg, tv, to;
    const uint64_t rows = (uint64_t)d.total_tokens, cols = (uint64_t)d.num_heads * 128u;
    if (!encode_bf16_2d(&tq, q, rows, cols) || !encode_bf16_2d(&tk, k, rows, cols) ||
        !encode_bf16_2d(&tg, g, rows, cols) || !encode_bf16_2d(&tv, v, rows, cols) ||
        // no output buffer (summaries): the map is never stored through, since
        // no unit carries UNIT_STORE_O; q stands in for a valid address
        !encode_bf16_2d(&to, p.o ? p.o : q, rows, cols))
        return cudaErrorInvalidValue;
    auto kern = p.snap.states ? kda::tck::chunk_tc_kernel<true>
                              : no_out ? kda::tck::chunk_tc_kernel<false, true> : kda::tck::chunk_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kda::tck::SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    if (blocks > INT32_MAX) return cudaErrorInvalidConfiguration;
    if (blocks == 0) return cudaSuccess;
    kern<<<(unsigned)blocks, kda::tck::NT, kda::tck::SMEM_ALLOC, stream>>>(tq, tk, tg, tv, to, p);
    return cudaGetLastError();
}

// The prefill kernels after planning: the tensor-core kernel where it applies,
// else the CUDA-core kernel.  Shared by both prefill entry points.
cudaError_t launch_prefill(const kda_fwd_desc &d, const void *q, const void *k, const void *v,
                           const void *g, const void *beta, const float *S0,
                           const int32_t *cu_seqlens, const int32_t *seq_order, const void *gate,
                           void *o, float *S_T, const kda::SnapOut &sn, cudaStream_t stream) {
    if (tc_path_applies(d, q, k, v, g, o)) {
        kda::tck::TcParams tp{beta, gate, S0, cu_seqlens, seq_order, o, S_T, d.num_heads, d.scale,
                              d.g_floor, nullptr, sn, d.total_tokens, d.num_seqs};
        return launch_tc(d, q, k, v, g, tp, stream);
    }
    SimtParams p{q, k, v, g, beta, gate, S0, cu_seqlens, seq_order, o, S_T,
                 d.num_heads, d.scale, d.g_floor, sn, d.total_tokens, d.num_seqs};
    return d.io_dtype == KDA_BF16 ? dispatch_simt<__nv_bfloat16>(d.dk, d.dv, p, d.num_seqs, stream)
                                  : dispatch_simt<float>(d.dk, d.dv, p, d.num_seqs, stream);
}

// Segment split: pass 1 (S_loc and M per segment), scan, pass 2 (outputs).
cudaError_t launch_split(const kda_fwd_desc &d, const SegPlan &pl, const int32_t *cu,
                         const void *q, const void *k, const void *v, const void *g,
                         const void *beta, const float *S0, const void *gate, void *o, float *S_T,
                         const kda::SnapOut &sn, unsigned char *ws, cudaStream_t stream) {
    using kda::tck::TcUnit;
    const WsLayout w = ws_layout(&d, pl);
    const int32_t N = d.num_seqs, H = d.num_heads;
    const size_t DD = 128u * 128u;
    float *mats = reinterpret_cast<float *>(ws + w.mats);
    std::vector<TcUnit> p1, p2;
    std::vector<kda::ScanJob> jobs;
    p1.reserve((size_t)pl.pass1_units);
    p2.reserve((size_t)pl.pass2_units);
    size_t mat_off = 0;   // floats used so far: each split (sequence, head) takes P x 3 x D^2, P per sequence
    for (int32_t n = 0; n < N; ++n) {
        const int64_t t0 = cu[n], t1 = cu[n + 1];
        const int32_t P = pl.nseg[n];
        for (int32_t h = 0; h < H; ++h) {
            const size_t unit = (size_t)n * H + h;
            const float *s0 = S0 ? S0 + unit * DD : nullptr;
            float *st = S_T ? S_T + unit * DD : nullptr;
            if (P == 1) {
                p2.push_back(TcUnit{t0, t1, s0, st, h, kda::tck::UNIT_STORE_O, n, t0});
                continue;
            }
            float *base = mats + mat_off;
            mat_off += (size_t)P * 3u * DD;
            auto Sloc = [&](int32_t sp) { return base + ((size_t)sp * 3u + 0u) * DD; };
            auto Mp = [&](int32_t sp) { return base + ((size_t)sp * 3u + 1u) * DD; };
            auto Sin = [&](int32_t sp) { return base + ((size_t)sp * 3u + 2u) * DD; };
            for (int32_t sp = 0; sp < P; ++sp) {
                const int64_t a = t0 + (int64_t)sp * pl.seglen[n];
                const int64_t b = std::min<int64_t>(t1, a + pl.seglen[n]);
                if (sp + 1 < P) p1.push_back(TcUnit{a, b, sp == 0 ? s0 : nullptr, Sloc(sp), h, 0, n, t0});
                if (sp >= 1 && sp + 1 < P)
                    p1.push_back(TcUnit{a, b, nullptr, Mp(sp), h,
                                        kda::tck::UNIT_ZERO_V | kda::tck::UNIT_S0_IDENTITY, n, t0});
                p2.push_back(TcUnit{a, b, sp == 0 ? s0 : Sin(sp), sp + 1 == P ? st : nullptr, h,
                                    kda::tck::UNIT_STORE_O, n, t0});
            }
            jobs.push_back(kda::ScanJob{Sloc(0), Mp(0), Sin(0), (int64_t)(3u * DD), P, nullptr, 0});
        }
    }
    auto longest_first = [](const TcUnit &x, const TcUnit &y) {
        return (x.t_end - x.t_begin) > (y.t_end - y.t_begin);
    };
    std::stable_sort(p1.begin(), p1.end(), longest_first);
    std::stable_sort(p2.begin(), p2.end(), longest_first);
    TcUnit *d1 = reinterpret_cast<TcUnit *>(ws + w.pass1);
    TcUnit *d2 = reinterpret_cast<TcUnit *>(ws + w.pass2);
    kda::ScanJob *dj = reinterpret_cast<kda::ScanJob *>(ws + w.jobs);
    cudaError_t e;
    if (!p1.empty() &&
        (e = cudaMemcpyAsync(d1, p1.data(), p1.size() * sizeof(TcUnit), cudaMemcpyHostToDevice, stream)) != cudaSuccess)
        return e;
    if ((e = cudaMemcpyAsync(d2, p2.data(), p2.size() * sizeof(TcUnit), cudaMemcpyHostToDevice, stream)) != cudaSuccess)
        return e;
    if ((e = cudaMemcpyAsync(dj, jobs.data(), jobs.size() * sizeof(kda::ScanJob), cudaMemcpyHostToDevice,
                             stream)) != cudaSuccess)
        return e;
    kda::tck::TcParams tp{beta, gate, nullptr, nullptr, nullptr, o, nullptr, H, d.scale, d.g_floor, d1, sn,
                          d.total_tokens, d.num_seqs};
    if (!p1.empty()) {
        tp.units = d1;
        NvtxRange r("kda.split.pass1");
        if ((e = launch_tc_units(d, q, k, v, g, tp, (int64_t)p1.size(), stream, true)) != cudaSuccess) return e;
    }
    const size_t scan_smem = 2u * DD * sizeof(float);
    if ((e = cudaFuncSetAttribute(kda::segment_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)scan_smem)) != cudaSuccess)
        return e;
    {
        NvtxRange r("kda.split.scan");
        kda::segment_scan_kernel<<<(unsigned)jobs.size(), 256, scan_smem, stream>>>(dj);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    tp.units = d2;
    NvtxRange r("kda.split.pass2");
    return launch_tc_units(d, q, k, v, g, tp, (int64_t)p2.size(), stream);
}

template <int DK, int DV, typename TIO>
cudaError_t launch_decode(const DecodeParams &p, int64_t units, cudaStream_t stream) {
    if (units > INT32_MAX) return cudaErrorInvalidConfiguration;
    kda::decode_kernel<DK, DV, TIO><<<(unsigned)units, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

template <typename TIO>
cudaError_t dispatch_decode(int dk, int dv, const DecodeParams &p, int64_t u, cudaStream_t s) {
    if (dk == 128 && dv == 128) return launch_decode<128, 128, TIO>(p, u, s);
    if (dk == 128 && dv == 64) return launch_decode<128, 64, TIO>(p, u, s);
    if (dk == 64 && dv == 128) return launch_decode<64, 128, TIO>(p, u, s);
    return launch_decode<64, 64, TIO>(p, u, s);
}

template <int DK, int DV, typename TIO, bool COMMIT>
cudaError_t launch_spec(const kda::SpecParams &p, int64_t units, cudaStream_t stream) {
    if (units > INT32_MAX) return cudaErrorInvalidConfiguration;
    kda::spec_kernel<DK, DV, TIO, COMMIT><<<(unsigned)units, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

template <typename TIO, bool COMMIT>
cudaError_t dispatch_spec(int dk, int dv, const kda::SpecParams &p, int64_t u, cudaStream_t s) {
    if (dk == 128 && dv == 128) return launch_spec<128, 128, TIO, COMMIT>(p, u, s);
    if (dk == 128 && dv == 64) return launch_spec<128, 64, TIO, COMMIT>(p, u, s);
    if (dk == 64 && dv == 128) return launch_spec<64, 128, TIO, COMMIT>(p, u, s);
    return launch_spec<64, 64, TIO, COMMIT>(p, u, s);
}

// Checks shared by verify and commit: the descriptor, required pointers, and
// that the state (and, for verify, the outputs) overlap no input.
kda_status validate_spec(const kda_spec_desc *desc, const void *q, const void *k, const void *v,
                         const void *g, const void *beta, const float *S, const void *gate,
                         const void *o, const int32_t *accepted) {
    if (!desc) return KDA_ERR_INVALID_ARG;
    const kda_spec_desc &d = *desc;
    if (d.batch < 1 || d.num_heads < 1 || d.dk <= 0 || d.dv <= 0) return KDA_ERR_INVALID_ARG;
    if (d.draft < 1 || d.draft > KDA_SPEC_MAX_DRAFT) return KDA_ERR_INVALID_ARG;
    if (!supported_dim(d.dk) || !supported_dim(d.dv)) return KDA_ERR_UNSUPPORTED;
    if (d.io_dtype != KDA_BF16 && d.io_dtype != KDA_FP32) return KDA_ERR_INVALID_ARG;
    if (!std::isfinite(d.scale)) return KDA_ERR_INVALID_ARG;
    if (!(d.g_floor >= kMinFloor && d.g_floor <= 0.0f)) return KDA_ERR_INVALID_ARG;
    if (!q || !k || !v || !g || !beta || !S) return KDA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(S) % 16 != 0) return KDA_ERR_INVALID_ARG;
    const int64_t units = (int64_t)d.batch * d.num_heads, rows = units * d.draft;
    const size_t esz = d.io_dtype == KDA_BF16 ? 2 : 4;
    const int64_t nk = rows * d.dk * (int64_t)esz, nv = rows * d.dv * (int64_t)esz;
    const Range rS = range_of(S, units * d.dk * d.dv * 4), ro = range_of(o, o ? nv : 0);
    const Range ins[] = {range_of(q, nk), range_of(k, nk), range_of(g, nk), range_of(v, nv),
                         range_of(beta, rows * (int64_t)esz), range_of(gate, gate ? nv : 0),
                         range_of(accepted, accepted ? 4 * (int64_t)d.batch : 0)};
    for (const Range &r : ins)
        if (overlaps(rS, r) || overlaps(ro, r)) return KDA_ERR_INVALID_ARG;
    if (overlaps(rS, ro)) return KDA_ERR_INVALID_ARG;
    return KDA_OK;
}

}  // namespace

extern "C" {

size_t kda_chunk_fwd_workspace_size(const kda_fwd_desc *desc, const int32_t *cu_seqlens_host) {
    if (validate_fwd_desc(desc) != KDA_OK) return SIZE_MAX;
    if (validate_host_seqlens(desc, cu_seqlens_host) != KDA_OK) return SIZE_MAX;
    return fwd_workspace_bytes(desc, cu_seqlens_host);
}

namespace {
kda_status chunk_fwd_impl(const kda_fwd_desc *desc, const kda_snapshots *snap, const void *q,
                          const void *k, const void *v, const void *g, const void *beta,
                          const float *S0, const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                          const void *gate, void *o, float *S_T, void *workspace,
                          size_t workspace_bytes, cudaStream_t stream) {
    kda_status st = validate_fwd_desc(desc);
    if (st != KDA_OK) return st;
    st = validate_host_seqlens(desc, cu_seqlens_host);
    if (st != KDA_OK) return st;
    const kda_fwd_desc &d = *desc;
    if (!cu_seqlens) return KDA_ERR_INVALID_ARG;
    if (d.total_tokens > 0 && (!q || !k || !v || !g || !beta || !o)) return KDA_ERR_INVALID_ARG;

    const size_t esz = d.io_dtype == KDA_BF16 ? 2 : 4;
    const int64_t T = d.total_tokens, H = d.num_heads;
    const int64_t nk = T * H * d.dk * (int64_t)esz, nv = T * H * d.dv * (int64_t)esz;
    const int64_t nb = T * H * (int64_t)esz;
    const int64_t ns = (int64_t)d.num_seqs * H * d.dk * d.dv * 4;
    const Range ins[] = {range_of(q, nk), range_of(k, nk), range_of(g, nk), range_of(v, nv),
                         range_of(beta, nb), range_of(gate, gate ? nv : 0), range_of(S0, S0 ? ns : 0),
                         range_of(cu_seqlens, 4 * (int64_t)(d.num_seqs + 1))};
    const Range ro = range_of(o, nv), rs = range_of(S_T, S_T ? ns : 0);
    for (const Range &r : ins) {
        if (overlaps(ro, r) || overlaps(rs, r)) return KDA_ERR_INVALID_ARG;
    }
    if (overlaps(ro, rs)) return KDA_ERR_INVALID_ARG;

    kda::SnapOut sn{nullptr, nullptr, 0, 64};
    Range rsn{}, rsb{};
    if (snap) {
        if (snap->interval <= 0 || snap->interval % 64 != 0 || snap->total < 0) return KDA_ERR_INVALID_ARG;
        if (snap->total > 0) {
            if (!snap->states || !snap->base) return KDA_ERR_INVALID_ARG;
            if (cu_seqlens_host) {               // the slots the sequences need must exist
                int64_t need_slots = 0;
                for (int32_t n = 0; n < d.num_seqs; ++n)
                    need_slots += ((int64_t)cu_seqlens_host[n + 1] - cu_seqlens_host[n]) / snap->interval;
                if (need_slots > snap->total) return KDA_ERR_INVALID_ARG;
            }
            rsn = range_of(snap->states, snap->total * H * d.dk * d.dv * 4);
            rsb = range_of(snap->base, 8 * (int64_t)(d.num_seqs + 1));
            for (const Range &r : ins)
                if (overlaps(rsn, r)) return KDA_ERR_INVALID_ARG;
            if (overlaps(rsn, ro) || overlaps(rsn, rs) || overlaps(rsb, ro) || overlaps(rsb, rs) ||
                overlaps(rsb, rsn))
                return KDA_ERR_INVALID_ARG;
            sn = kda::SnapOut{snap->states, snap->base, snap->total, snap->interval};
        }
    }

    const size_t need = fwd_workspace_bytes(desc, cu_seqlens_host);
    if (need > 0) {
        if (!workspace || workspace_bytes < need) return KDA_ERR_WORKSPACE;
        if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return KDA_ERR_WORKSPACE;
        const Range rw = range_of(workspace, (int64_t)need);
        for (const Range &r : ins)
            if (overlaps(rw, r)) return KDA_ERR_INVALID_ARG;
        if (overlaps(rw, ro) || overlaps(rw, rs) || overlaps(rw, rsn) || overlaps(rw, rsb))
            return KDA_ERR_INVALID_ARG;
    }

    const SegPlan pl = plan_segments(d, cu_seqlens_host);
    if (pl.active && tc_path_applies(d, q, k, v, g, o)) {
        const cudaError_t e = launch_split(d, pl, cu_seqlens_host, q, k, v, g, beta, S0, gate, o, S_T,
                                           sn, static_cast<unsigned char *>(workspace), stream);
        return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }

    int32_t *seq_order = static_cast<int32_t *>(workspace);
    cudaError_t e;
    {
        NvtxRange r("kda.plan");
        e = kda::launch_plan_longest_first(cu_seqlens, d.num_seqs, seq_order, stream);
    }
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    NvtxRange r("kda.prefill");
    e = launch_prefill(d, q, k, v, g, beta, S0, cu_seqlens, seq_order, gate, o, S_T, sn, stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}
}  // namespace

kda_status kda_chunk_fwd(const kda_fwd_desc *desc, const void *q, const void *k, const void *v,
                         const void *g, const void *beta, const float *S0,
                         const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                         const void *gate, void *o, float *S_T, void *workspace,
                         size_t workspace_bytes, cudaStream_t stream) {
    return chunk_fwd_impl(desc, nullptr, q, k, v, g, beta, S0, cu_seqlens, cu_seqlens_host, gate, o,
                          S_T, workspace, workspace_bytes, stream);
}

kda_status kda_chunk_fwd_snapshots(const kda_fwd_desc *desc, const kda_snapshots *snap,
                                   const void *q, const void *k, const void *v, const void *g,
                                   const void *beta, const float *S0, const int32_t *cu_seqlens,
                                   const int32_t *cu_seqlens_host, const void *gate, void *o,
                                   float *S_T, void *workspace, size_t workspace_bytes,
                                   cudaStream_t stream) {
    if (!snap) return KDA_ERR_INVALID_ARG;
    return chunk_fwd_impl(desc, snap, q, k, v, g, beta, S0, cu_seqlens, cu_seqlens_host, gate, o,
                          S_T, workspace, workspace_bytes, stream);
}

kda_status kda_decode_step(const kda_decode_desc *desc, const void *q, const void *k,
                           const void *v, const void *g, const void *beta, float *S,
                           const void *gate, void *o, cudaStream_t stream) {
    if (!desc) return KDA_ERR_INVALID_ARG;
    const kda_decode_desc &d = *desc;
    if (d.batch < 1 || d.num_heads < 1 || d.dk <= 0 || d.dv <= 0) return KDA_ERR_INVALID_ARG;
    if (!supported_dim(d.dk) || !supported_dim(d.dv)) return KDA_ERR_UNSUPPORTED;
    if (d.io_dtype != KDA_BF16 && d.io_dtype != KDA_FP32) return KDA_ERR_INVALID_ARG;
    if (!std::isfinite(d.scale)) return KDA_ERR_INVALID_ARG;
    if (!(d.g_floor >= kMinFloor && d.g_floor <= 0.0f)) return KDA_ERR_INVALID_ARG;
    if (!q || !k || !v || !g || !beta || !S || !o) return KDA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(S) % 16 != 0) return KDA_ERR_INVALID_ARG;

    const int64_t units = (int64_t)d.batch * d.num_heads;
    const size_t esz = d.io_dtype == KDA_BF16 ? 2 : 4;
    const int64_t nk = units * d.dk * (int64_t)esz, nv = units * d.dv * (int64_t)esz;
    const Range rS = range_of(S, units * d.dk * d.dv * 4), ro = range_of(o, nv);
    const Range ins[] = {range_of(q, nk), range_of(k, nk), range_of(g, nk), range_of(v, nv),
                         range_of(beta, units * (int64_t)esz), range_of(gate, gate ? nv : 0)};
    for (const Range &r : ins)
        if (overlaps(rS, r) || overlaps(ro, r)) return KDA_ERR_INVALID_ARG;
    if (overlaps(rS, ro)) return KDA_ERR_INVALID_ARG;

    DecodeParams p{q, k, v, g, beta, gate, S, o, d.scale, d.g_floor};
    NvtxRange r("kda.decode");
    cudaError_t e = d.io_dtype == KDA_BF16 ? dispatch_decode<__nv_bfloat16>(d.dk, d.dv, p, units, stream)
                                           : dispatch_decode<float>(d.dk, d.dv, p, units, stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_spec_verify(const kda_spec_desc *desc, const void *q, const void *k, const void *v,
                           const void *g, const void *beta, const float *S, const void *gate,
                           void *o, cudaStream_t stream) {
    if (!o) return KDA_ERR_INVALID_ARG;
    const kda_status st = validate_spec(desc, q, k, v, g, beta, S, gate, o, nullptr);
    if (st != KDA_OK) return st;
    const kda_spec_desc &d = *desc;
    kda::SpecParams p{q, k, v, g, beta, gate, const_cast<float *>(S), o, nullptr, d.num_heads,
                      d.draft, d.scale, d.g_floor};
    const int64_t units = (int64_t)d.batch * d.num_heads;
    NvtxRange r("kda.spec.verify");
    cudaError_t e = d.io_dtype == KDA_BF16 ? dispatch_spec<__nv_bfloat16, false>(d.dk, d.dv, p, units, stream)
                                           : dispatch_spec<float, false>(d.dk, d.dv, p, units, stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_spec_commit(const kda_spec_desc *desc, const void *q, const void *k, const void *v,
                           const void *g, const void *beta, float *S, const int32_t *accepted,
                           cudaStream_t stream) {
    if (!accepted) return KDA_ERR_INVALID_ARG;
    const kda_status st = validate_spec(desc, q, k, v, g, beta, S, nullptr, nullptr, accepted);
    if (st != KDA_OK) return st;
    const kda_spec_desc &d = *desc;
    kda::SpecParams p{q, k, v, g, beta, nullptr, S, nullptr, accepted, d.num_heads, d.draft,
                      d.scale, d.g_floor};
    const int64_t units = (int64_t)d.batch * d.num_heads;
    NvtxRange r("kda.spec.commit");
    cudaError_t e = d.io_dtype == KDA_BF16 ? dispatch_spec<__nv_bfloat16, true>(d.dk, d.dv, p, units, stream)
                                           : dispatch_spec<float, true>(d.dk, d.dv, p, units, stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

// ---------------------------------------------------------------- backward
namespace {
// bf16 I/O at dk = dv = 128: the chunked backward (kda_bwd_chunk.cuh).  Other
// head sizes, and fp32 I/O: the per-token backward (kda_bwd.cuh), whose dg is
// formed per token; the chunked form's dg sums the chunk's pair terms, which
// cancel, and under strong decay (g near the floor) keeps about 3e-4 of
// relative accuracy in fp32 arithmetic, short of fp32 I/O's 1e-4.
// The chunked kernels also read q, k, g, dout and the gate in 16-byte pieces.
bool chunked_bwd(const kda_fwd_desc &d) { return d.dk == 128 && d.dv == 128 && d.io_dtype == KDA_BF16; }
bool chunked_bwd_applies(const kda_fwd_desc &d, std::initializer_list<const void *> ptrs) {
    if (!chunked_bwd(d)) return false;
    for (const void *ptr : ptrs)
        if (reinterpret_cast<uintptr_t>(ptr) % 16 != 0) return false;
    return true;
}

struct BwdLayout {
    size_t base = 0, states = 0, o = 0, fws = 0, scratch = 0, total = 0;
    size_t ctab = 0;               // chunked: chunk tables
    int64_t slots = 0, chunks = 0;
    size_t fws_bytes = 0;
};

BwdLayout bwd_layout(const kda_fwd_desc &d, const int32_t *cu) {
    BwdLayout w;
    for (int32_t n = 0; n < d.num_seqs; ++n) {
        const int64_t L = (int64_t)cu[n + 1] - cu[n];
        w.slots += L / kda::bwd::CH;
        w.chunks += (L + kda::bwdc::C - 1) / kda::bwdc::C;
    }
    const size_t esz = d.io_dtype == KDA_BF16 ? 2 : 4;
    const size_t DD = (size_t)d.dk * d.dv;
    const size_t NH = (size_t)d.num_seqs * d.num_heads;
    size_t off = 0;
    w.base = off;    off += align256(sizeof(int64_t) * (size_t)(d.num_seqs + 1));
    w.states = off;  off += align256((size_t)w.slots * d.num_heads * DD * sizeof(float));
    w.o = off;       off += align256((size_t)d.total_tokens * d.num_heads * d.dv * esz);
    w.fws_bytes = fwd_workspace_bytes(&d, cu);
    w.fws = off;     off += align256(w.fws_bytes);
    // the per-token kernel's scratch, or (chunked shape) the larger of it and the
    // chunked kernels' (the per-token kernel also runs the chunked shape when a
    // tensor is not 16-byte aligned)
    size_t scratch = NH * kda::bwd::scratch_floats(d.dk, d.dv) * sizeof(float);
    if (chunked_bwd(d)) {
        w.ctab = off;    off += align256(sizeof(int64_t) * (size_t)(d.num_seqs + 1) + 2 * sizeof(int32_t) * (size_t)w.chunks);
        scratch = std::max(scratch, (size_t)w.chunks * d.num_heads * kda::bwdc::Scratch::FLOATS * sizeof(float));
    }
    w.scratch = off; off += align256(scratch);
    w.total = off;
    return w;
}
extern "C++" {
template <int DK, int DV, typename TIO>
cudaError_t launch_bwd(const kda::bwd::BwdParams &bp, int64_t units, cudaStream_t stream) {
    using SM = kda::bwd::BwdSmem<DK, DV>;
    auto kern = kda::bwd::bwd_kernel<DK, DV, TIO>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SM::BYTES);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)units, kda::bwd::NT, SM::BYTES, stream>>>(bp);
    return cudaGetLastError();
}

cudaError_t launch_bwd_chunked(const kda::bwdc::ChunkBwdParams &bp, int64_t chunk_heads, int64_t units,
                               cudaStream_t stream) {
    using namespace kda::bwdc;
    auto prep = chain_prep_kernel<__nv_bfloat16, false>;
    auto chain = chain_kernel<false>;
    auto grad = chain_grad_kernel<__nv_bfloat16, false>;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PrepSmem::BYTES)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(chain, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ChainSmem::BYTES)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(grad, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)GradSmem::BYTES)) != cudaSuccess)
        return e;
    if (chunk_heads > 0) {
        NvtxRange r("kda.bwd.chain_prep");
        prep<<<(unsigned)chunk_heads, NT, PrepSmem::BYTES, stream>>>(bp);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        NvtxRange r("kda.bwd.chain");
        chain<<<(unsigned)(2 * units), CHAIN_NT, ChainSmem::BYTES, stream>>>(bp);   // two column halves
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (chunk_heads > 0) {
        NvtxRange r("kda.bwd.chain_grad");
        grad<<<(unsigned)chunk_heads, NT, GradSmem::BYTES, stream>>>(bp);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <typename TIO>
cudaError_t dispatch_bwd(int dk, int dv, const kda::bwd::BwdParams &bp, int64_t units, cudaStream_t stream) {
    if (dk == 128 && dv == 128) return launch_bwd<128, 128, TIO>(bp, units, stream);
    if (dk == 128 && dv == 64) return launch_bwd<128, 64, TIO>(bp, units, stream);
    if (dk == 64 && dv == 128) return launch_bwd<64, 128, TIO>(bp, units, stream);
    return launch_bwd<64, 64, TIO>(bp, units, stream);
}
}  // extern "C++"
}  // namespace

size_t kda_chunk_bwd_workspace_size(const kda_fwd_desc *desc, const int32_t *cu_seqlens_host) {
    if (validate_fwd_desc(desc) != KDA_OK || !cu_seqlens_host) return SIZE_MAX;
    if (validate_host_seqlens(desc, cu_seqlens_host) != KDA_OK) return SIZE_MAX;
    return bwd_layout(*desc, cu_seqlens_host).total;
}

kda_status kda_chunk_bwd(const kda_fwd_desc *desc, const void *q, const void *k, const void *v,
                         const void *g, const void *beta, const float *S0, const int32_t *cu_seqlens,
                         const int32_t *cu_seqlens_host, const void *gate, const void *dout,
                         const float *dS_T, void *dq, void *dk, void *dv, void *dg, void *dbeta,
                         void *dgate, float *dS0, void *workspace, size_t workspace_bytes,
                         cudaStream_t stream) {
    kda_status st = validate_fwd_desc(desc);
    if (st != KDA_OK) return st;
    const kda_fwd_desc &d = *desc;
    if (!cu_seqlens || !cu_seqlens_host) return KDA_ERR_INVALID_ARG;
    if ((st = validate_host_seqlens(desc, cu_seqlens_host)) != KDA_OK) return st;
    const bool any = d.total_tokens > 0;
    if (any && (!q || !k || !v || !g || !beta || !dout || !dq || !dk || !dv || !dg || !dbeta))
        return KDA_ERR_INVALID_ARG;
    if (any && gate && !dgate) return KDA_ERR_INVALID_ARG;
    const int32_t N = d.num_seqs, H = d.num_heads;
    if ((int64_t)N * H > INT32_MAX) return KDA_ERR_INVALID_ARG;
    for (const void *ptr : {static_cast<const void *>(S0), static_cast<const void *>(dS_T),
                            static_cast<const void *>(dS0)})   // moved as float4
        if (reinterpret_cast<uintptr_t>(ptr) % 16 != 0) return KDA_ERR_INVALID_ARG;
    const size_t esz = d.io_dtype == KDA_BF16 ? 2 : 4;
    const int64_t T = d.total_tokens, DD = (int64_t)d.dk * d.dv;
    const int64_t nk = T * H * d.dk * (int64_t)esz, nv = T * H * d.dv * (int64_t)esz;
    const int64_t nb = T * H * (int64_t)esz, ns = (int64_t)N * H * DD * 4;
    const Range ins[] = {range_of(q, nk), range_of(k, nk), range_of(g, nk), range_of(v, nv),
                         range_of(beta, nb), range_of(gate, gate ? nv : 0), range_of(dout, nv),
                         range_of(S0, S0 ? ns : 0), range_of(dS_T, dS_T ? ns : 0),
                         range_of(cu_seqlens, 4 * (int64_t)(N + 1))};
    const Range outs[] = {range_of(dq, nk), range_of(dk, nk), range_of(dv, nv), range_of(dg, nk),
                          range_of(dbeta, nb), range_of(dgate, gate ? nv : 0), range_of(dS0, dS0 ? ns : 0)};
    for (const Range &a : outs) {
        for (const Range &b : ins)
            if (overlaps(a, b)) return KDA_ERR_INVALID_ARG;
    }
    for (size_t i = 0; i < sizeof(outs) / sizeof(outs[0]); ++i)
        for (size_t j = i + 1; j < sizeof(outs) / sizeof(outs[0]); ++j)
            if (overlaps(outs[i], outs[j])) return KDA_ERR_INVALID_ARG;
    const BwdLayout w = bwd_layout(d, cu_seqlens_host);
    if (!workspace || workspace_bytes < w.total || reinterpret_cast<uintptr_t>(workspace) % 256 != 0)
        return KDA_ERR_WORKSPACE;
    const Range rw = range_of(workspace, (int64_t)w.total);
    for (const Range &r : ins)
        if (overlaps(rw, r)) return KDA_ERR_INVALID_ARG;
    for (const Range &r : outs)
        if (overlaps(rw, r)) return KDA_ERR_INVALID_ARG;
    if (!any) {
        // nothing to differentiate through: dS0 = dS_T (or zero)
        if (!dS0) return KDA_OK;
        const cudaError_t e = dS_T ? cudaMemcpyAsync(dS0, dS_T, (size_t)ns, cudaMemcpyDeviceToDevice, stream)
                                   : cudaMemsetAsync(dS0, 0, (size_t)ns, stream);
        return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }

    // the states at every 64-token chunk start: the forward with snapshots
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    std::vector<int64_t> base((size_t)N + 1, 0);
    for (int32_t n = 0; n < N; ++n)
        base[n + 1] = base[n] + ((int64_t)cu_seqlens_host[n + 1] - cu_seqlens_host[n]) / kda::bwd::CH;
    int64_t *base_dev = reinterpret_cast<int64_t *>(ws + w.base);
    if (cudaMemcpyAsync(base_dev, base.data(), base.size() * sizeof(int64_t), cudaMemcpyHostToDevice,
                        stream) != cudaSuccess)
        return KDA_ERR_CUDA;
    float *states = reinterpret_cast<float *>(ws + w.states);
    const kda_snapshots sn{kda::bwd::CH, w.slots, base_dev, states};
    const bool chunked = chunked_bwd_applies(d, {q, k, g, dout, gate});
    st = chunk_fwd_impl(desc, &sn, q, k, v, g, beta, S0, cu_seqlens, cu_seqlens_host, nullptr,
                        ws + w.o, nullptr, w.fws_bytes ? ws + w.fws : nullptr, w.fws_bytes, stream);
    if (st != KDA_OK) return st;

    if (chunked) {
        // chunk c of sequence n is chunk_base[n] + (its index in the sequence)
        std::vector<int64_t> cbase((size_t)N + 1, 0);
        std::vector<int32_t> cmap(2 * (size_t)w.chunks);
        for (int32_t n = 0; n < N; ++n) {
            const int64_t L = (int64_t)cu_seqlens_host[n + 1] - cu_seqlens_host[n];
            const int64_t nc = (L + kda::bwdc::C - 1) / kda::bwdc::C;
            for (int64_t ci = 0; ci < nc; ++ci) {
                cmap[(size_t)(cbase[n] + ci)] = n;
                cmap[(size_t)(w.chunks + cbase[n] + ci)] = (int32_t)ci;
            }
            cbase[n + 1] = cbase[n] + nc;
        }
        int64_t *cbase_dev = reinterpret_cast<int64_t *>(ws + w.ctab);
        int32_t *cmap_dev = reinterpret_cast<int32_t *>(cbase_dev + N + 1);
        if (cudaMemcpyAsync(cbase_dev, cbase.data(), cbase.size() * sizeof(int64_t), cudaMemcpyHostToDevice,
                            stream) != cudaSuccess ||
            (w.chunks > 0 && cudaMemcpyAsync(cmap_dev, cmap.data(), cmap.size() * sizeof(int32_t),
                                             cudaMemcpyHostToDevice, stream) != cudaSuccess))
            return KDA_ERR_CUDA;
        kda::bwdc::ChunkBwdParams cp{q, k, v, g, beta, gate, dout, S0, dS_T, cu_seqlens, states, base_dev,
                                     cmap_dev, cmap_dev + w.chunks, cbase_dev,
                                     reinterpret_cast<float *>(ws + w.scratch), dq, dk, dv, dg, dbeta, dgate, dS0,
                                     H, d.scale, d.g_floor, d.total_tokens, N};
        NvtxRange r("kda.bwd");
        const int64_t ch = w.chunks * H, units = (int64_t)N * H;
        const cudaError_t e = launch_bwd_chunked(cp, ch, units, stream);
        return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }

    kda::bwd::BwdParams bp{q, k, v, g, beta, gate, dout, S0, dS_T, cu_seqlens, states, base_dev,
                           reinterpret_cast<float *>(ws + w.scratch), dq, dk, dv, dg, dbeta, dgate, dS0,
                           H, d.scale, d.g_floor, d.total_tokens, w.slots};
    NvtxRange r("kda.bwd");
    const cudaError_t e = d.io_dtype == KDA_BF16 ? dispatch_bwd<__nv_bfloat16>(d.dk, d.dv, bp, (int64_t)N * H, stream)
                                                 : dispatch_bwd<float>(d.dk, d.dv, bp, (int64_t)N * H, stream);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

// ---------------------------------------------------------------- context parallel (KCP)
namespace {
// Sub-segments per piece for the summary: the chains (S_loc, and M where
// asked) of every (sequence, head) are cut like the prefill's long-sequence
// split when they are fewer than the SMs, then folded by the scan kernel.
struct SummaryPlan {
    std::vector<int32_t> nseg;      // sub-segments per sequence
    std::vector<int64_t> seglen;    // tokens per sub-segment (multiple of 64)
    int64_t mat_blocks = 0;         // (sequence, head, sub-segment) entries of the split buffers
    int64_t jobs = 0, units = 0;
};

SummaryPlan plan_summary(const kda_fwd_desc &d, const int32_t *cu, bool with_M) {
    SummaryPlan pl;
    const int32_t N = d.num_seqs, H = d.num_heads;
    pl.nseg.assign(N, 1);
    pl.seglen.assign(N, 0);
    const int64_t chains = (int64_t)N * H * (with_M ? 2 : 1);
    const char *env = std::getenv("KDA_SEGMENTS");
    const int forced = env ? std::atoi(env) : 0;
    const int sms = device_sm_count();
    int64_t best_p = 1;
    if (forced < 1 && chains < sms) {         // KDA_SEGMENTS=1: no split
        int64_t cmax = 0;
        for (int32_t n = 0; n < N; ++n) cmax = std::max<int64_t>(cmax, ((int64_t)cu[n + 1] - cu[n] + 63) / 64);
        auto waves = [&](int64_t x) { return (x + sms - 1) / sms; };
        const int64_t t1 = waves(chains) * cmax;
        int64_t best_t = t1;
        for (int64_t P = 2; P <= 64 && P * kMinSegTokens / 64 <= cmax; ++P) {
            // every sub-segment needs both chains (M for the fold), plus the folds
            const int64_t t = waves((int64_t)N * H * 2 * P) * ((cmax + P - 1) / P) + P;
            if (t < best_t) { best_t = t; best_p = P; }
        }
        if (best_t * 10 > t1 * 9) best_p = 1;
    }
    for (int32_t n = 0; n < N; ++n) {
        const int64_t L = (int64_t)cu[n + 1] - cu[n];
        int64_t P = forced > 1 ? std::min<int64_t>(forced, L / 128)
                               : (best_p > 1 ? std::min<int64_t>(best_p, L / kMinSegTokens) : 1);
        if (P >= 2) {
            const int64_t seg = ((L + P - 1) / P + 63) / 64 * 64;
            P = (L + seg - 1) / seg;
        }
        if (P >= 2) {
            pl.nseg[n] = (int32_t)P;
            pl.seglen[n] = ((L + P - 1) / P + 63) / 64 * 64;
            pl.mat_blocks += (int64_t)H * P;
            pl.jobs += (int64_t)H * (with_M ? 2 : 1);
            pl.units += (int64_t)H * 2 * P;
        } else {
            pl.units += (int64_t)H * (with_M ? 2 : 1);
        }
    }
    return pl;
}

struct SummaryLayout {
    size_t units = 0, jobs = 0, mats = 0, total = 0;
};

SummaryLayout summary_layout(const SummaryPlan &pl) {
    SummaryLayout w;
    size_t off = 0;
    w.units = off; off += align256(sizeof(kda::tck::TcUnit) * (size_t)std::max<int64_t>(pl.units, 1));
    w.jobs = off;  off += align256(sizeof(kda::ScanJob) * (size_t)std::max<int64_t>(pl.jobs, 1));
    w.mats = off;  off += align256((size_t)pl.mat_blocks * 2u * 128u * 128u * sizeof(float));
    w.total = off;
    return w;
}
}  // namespace

size_t kda_segment_summary_workspace_size(const kda_fwd_desc *desc, const int32_t *cu_seqlens_host,
                                          int32_t with_M) {
    if (validate_fwd_desc(desc) != KDA_OK || !cu_seqlens_host) return SIZE_MAX;
    if (validate_host_seqlens(desc, cu_seqlens_host) != KDA_OK) return SIZE_MAX;
    return summary_layout(plan_summary(*desc, cu_seqlens_host, with_M != 0)).total;
}

kda_status kda_segment_summary(const kda_fwd_desc *desc, const void *q, const void *k,
                               const void *v, const void *g, const void *beta, const float *S0,
                               const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                               float *S_loc, float *M, void *workspace, size_t workspace_bytes,
                               cudaStream_t stream) {
    using kda::tck::TcUnit;
    kda_status st = validate_fwd_desc(desc);
    if (st != KDA_OK) return st;
    const kda_fwd_desc &d = *desc;
    if (d.io_dtype != KDA_BF16 || d.dk != 128 || d.dv != 128 || d.chunk == 16) return KDA_ERR_UNSUPPORTED;
    if (d.total_tokens < 1 || d.total_tokens > INT32_MAX - 64) return KDA_ERR_INVALID_ARG;
    if (!cu_seqlens || !cu_seqlens_host || !S_loc || !q || !k || !v || !g || !beta) return KDA_ERR_INVALID_ARG;
    if ((st = validate_host_seqlens(desc, cu_seqlens_host)) != KDA_OK) return st;
    for (const void *ptr : {q, k, v, g})      // moved by TMA
        if (reinterpret_cast<uintptr_t>(ptr) % 16 != 0) return KDA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(S_loc) % 16 != 0 || reinterpret_cast<uintptr_t>(M) % 16 != 0)
        return KDA_ERR_INVALID_ARG;            // written by the scan kernel as float4

    const int32_t N = d.num_seqs, H = d.num_heads;
    const int64_t T = d.total_tokens, DD = 128 * 128;
    const int64_t nk = T * H * 128 * 2, nb = T * H * 2, ns = (int64_t)N * H * DD * 4;
    const Range ins[] = {range_of(q, nk), range_of(k, nk), range_of(g, nk), range_of(v, nk),
                         range_of(beta, nb), range_of(S0, S0 ? ns : 0),
                         range_of(cu_seqlens, 4 * (int64_t)(N + 1))};
    const Range rl = range_of(S_loc, ns), rm = range_of(M, M ? ns : 0);
    for (const Range &r : ins)
        if (overlaps(rl, r) || overlaps(rm, r)) return KDA_ERR_INVALID_ARG;
    if (overlaps(rl, rm)) return KDA_ERR_INVALID_ARG;
    const SummaryPlan pl = plan_summary(d, cu_seqlens_host, M != nullptr);
    const SummaryLayout w = summary_layout(pl);
    if (!workspace || workspace_bytes < w.total || reinterpret_cast<uintptr_t>(workspace) % 256 != 0)
        return KDA_ERR_WORKSPACE;
    const Range rw = range_of(workspace, (int64_t)w.total);
    for (const Range &r : ins)
        if (overlaps(rw, r)) return KDA_ERR_INVALID_ARG;
    if (overlaps(rw, rl) || overlaps(rw, rm)) return KDA_ERR_INVALID_ARG;

    // chains: unsplit pieces write S_loc (and M) directly; a split piece runs
    // both chains per sub-segment into the workspace, and the scan folds them
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    float *mats = reinterpret_cast<float *>(ws + w.mats);
    std::vector<TcUnit> units;
    std::vector<kda::ScanJob> jobs;
    units.reserve((size_t)pl.units);
    size_t mat_off = 0;   // floats used so far: each split (sequence, head) takes P x 2 x D^2, P per sequence
    for (int32_t n = 0; n < N; ++n) {
        const int64_t a0 = cu_seqlens_host[n], a1 = cu_seqlens_host[n + 1];
        const int32_t P = pl.nseg[n];
        for (int32_t h = 0; h < H; ++h) {
            const int64_t u = (int64_t)n * H + h;
            const float *s0 = S0 ? S0 + u * DD : nullptr;
            if (P == 1) {
                units.push_back(TcUnit{a0, a1, s0, S_loc + u * DD, h, 0, n, a0});
                if (M)
                    units.push_back(TcUnit{a0, a1, nullptr, M + u * DD, h,
                                           kda::tck::UNIT_ZERO_V | kda::tck::UNIT_S0_IDENTITY, n, a0});
                continue;
            }
            float *Lb = mats + mat_off;                        // [P] S_loc, then [P] M
            float *Mb = Lb + (size_t)P * DD;
            mat_off += (size_t)P * 2u * DD;
            for (int32_t sp = 0; sp < P; ++sp) {
                const int64_t b0 = a0 + (int64_t)sp * pl.seglen[n];
                const int64_t b1 = std::min<int64_t>(a1, b0 + pl.seglen[n]);
                units.push_back(TcUnit{b0, b1, sp == 0 ? s0 : nullptr, Lb + sp * DD, h, 0, n, a0});
                units.push_back(TcUnit{b0, b1, nullptr, Mb + sp * DD, h,
                                       kda::tck::UNIT_ZERO_V | kda::tck::UNIT_S0_IDENTITY, n, a0});
            }
            jobs.push_back(kda::ScanJob{Lb, Mb, nullptr, DD, P + 1, S_loc + u * DD, 0});
            if (M) jobs.push_back(kda::ScanJob{Mb, Mb, nullptr, DD, P + 1, M + u * DD, 1});
        }
    }
    std::stable_sort(units.begin(), units.end(), [](const TcUnit &x, const TcUnit &y) {
        return (x.t_end - x.t_begin) > (y.t_end - y.t_begin);
    });
    TcUnit *du = reinterpret_cast<TcUnit *>(ws + w.units);
    if (cudaMemcpyAsync(du, units.data(), units.size() * sizeof(TcUnit), cudaMemcpyHostToDevice,
                        stream) != cudaSuccess)
        return KDA_ERR_CUDA;
    kda::tck::TcParams tp{beta, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, H, d.scale,
                          d.g_floor, du, kda::SnapOut{nullptr, nullptr, 0, 64}, d.total_tokens, d.num_seqs};
    {
        NvtxRange r("kda.summary.chains");
        if (launch_tc_units(d, q, k, v, g, tp, (int64_t)units.size(), stream, true) != cudaSuccess) return KDA_ERR_CUDA;
    }
    if (jobs.empty()) return KDA_OK;
    kda::ScanJob *dj = reinterpret_cast<kda::ScanJob *>(ws + w.jobs);
    if (cudaMemcpyAsync(dj, jobs.data(), jobs.size() * sizeof(kda::ScanJob), cudaMemcpyHostToDevice,
                        stream) != cudaSuccess)
        return KDA_ERR_CUDA;
    const size_t scan_smem = 2u * (size_t)DD * sizeof(float);
    if (cudaFuncSetAttribute(kda::segment_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)scan_smem) != cudaSuccess)
        return KDA_ERR_CUDA;
    NvtxRange r("kda.summary.scan");
    kda::segment_scan_kernel<<<(unsigned)jobs.size(), 256, scan_smem, stream>>>(dj);
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_state_combine(const kda_combine_desc *desc, const float *summaries, float *S_in,
                             cudaStream_t stream) {
    if (!desc || !summaries || !S_in) return KDA_ERR_INVALID_ARG;
    const kda_combine_desc &c = *desc;
    if (c.num_seqs < 1 || c.num_heads < 1 || c.num_summaries < 1 || c.dk <= 0 || c.dv <= 0)
        return KDA_ERR_INVALID_ARG;
    if (c.dk != 128 || c.dv != 128) return KDA_ERR_UNSUPPORTED;
    if (reinterpret_cast<uintptr_t>(summaries) % 16 != 0 || reinterpret_cast<uintptr_t>(S_in) % 16 != 0)
        return KDA_ERR_INVALID_ARG;
    const int64_t DD = 128 * 128;
    const int64_t units = mul3(c.num_seqs, c.num_heads, 1);
    const int64_t per_piece = mul3(units, 2, DD);
    if (units < 0 || per_piece < 0 || units > INT32_MAX) return KDA_ERR_INVALID_ARG;
    const int64_t all = mul3(per_piece, c.num_summaries, 4);
    if (all < 0) return KDA_ERR_INVALID_ARG;
    if (overlaps(range_of(summaries, all), range_of(S_in, units * DD * 4))) return KDA_ERR_INVALID_ARG;
    const size_t smem = 2u * (size_t)DD * sizeof(float);
    if (cudaFuncSetAttribute(kda::state_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return KDA_ERR_CUDA;
    NvtxRange r("kda.combine");
    kda::state_combine_kernel<<<(unsigned)units, 256, smem, stream>>>(summaries, S_in, units,
                                                                      c.num_summaries);
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

namespace {
// One warp waits, bounded, on an mbarrier whose phase nothing completes.
__global__ void selftest_wait_kernel(uint32_t max_polls) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        kda::tc::mbar_init(&bar, 1);
        kda::tc::mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)kda::tc::mbar_wait(&bar, 0, max_polls);
    __syncthreads();
}
}  // namespace

kda_status kda_selftest_bounded_wait(int32_t max_polls, cudaStream_t stream) {
    if (max_polls < 1 || max_polls > 65536) return KDA_ERR_INVALID_ARG;
    selftest_wait_kernel<<<1, 32, 0, stream>>>((uint32_t)max_polls);
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_get_device_status(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return KDA_ERR_CUDA;
    unsigned int word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, kda::g_err_word, sizeof(word)) != cudaSuccess) return KDA_ERR_CUDA;
    if (word && cudaMemcpyToSymbol(kda::g_err_word, &zero, sizeof(zero)) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (word & kda::ERR_TIMEOUT) return KDA_ERR_TIMEOUT;
    if (word & kda::ERR_BOUNDS) return KDA_ERR_DEVICE_BOUNDS;
    return KDA_OK;
}

const char *kda_status_string(kda_status s) {
    switch (s) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
    case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT";
    case KDA_ERR_DEVICE_BOUNDS: return "KDA_ERR_DEVICE_BOUNDS";
    }
    return "KDA_UNKNOWN_STATUS";
}

int32_t kda_version(void) { return 100; }

}  // extern "C"

// ---------------------------------------------------------------------------
// kda_chunk_fwd_noalloc: the chunked prefill for callers that cannot give the
// library any device memory of its own -- for instance a host framework whose
// plugin interface passes only input and output buffers, or a serving runtime
// that lays out all device memory before it starts and forbids allocations
// (and the synchronisation they bring) afterwards.  Instead of a caller
// workspace, the per-call scratch (the longest-first sequence order) lives in
// a fixed array compiled into the library.
// ---------------------------------------------------------------------------
#include <mutex>

namespace {

// One slot per sequence; every device that loads the library holds this
// array (256 KiB) until the process exits.
static __device__ __align__(256) int32_t g_noalloc_seq_order[KDA_NOALLOC_MAX_SEQS];

constexpr int kMaxDevices = 128;
std::mutex g_noalloc_mutex;
struct NoallocSlot {
    CUcontext ctx;      // the context the address belongs to
    int32_t *ptr;
};
NoallocSlot g_noalloc_slot[kMaxDevices] = {};

// cuCtxGetCurrent through the runtime (no link against the driver library).
PFN_cuCtxGetCurrent_v4000 ctx_getter() {
    static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &ptr, 4000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(ptr);
    });
    return fn;
}

// Device address of the scratch array in the current context.  The address
// is cached per device together with the context it was looked up in; a new
// context on the device (after cudaDeviceReset, or after the primary context
// was released and created again) looks it up afresh.
cudaError_t noalloc_scratch(int32_t **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    PFN_cuCtxGetCurrent_v4000 get_ctx = ctx_getter();
    CUcontext ctx = nullptr;
    if (!get_ctx || get_ctx(&ctx) != CUDA_SUCCESS) return cudaErrorInitializationError;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    NoallocSlot &slot = g_noalloc_slot[dev];
    if (!slot.ptr || !ctx || slot.ctx != ctx) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_seq_order);   // (creates the context if none is current)
        if (e != cudaSuccess) return e;
        if (!ctx && (get_ctx(&ctx) != CUDA_SUCCESS || !ctx)) return cudaErrorInitializationError;
        slot.ctx = ctx;
        slot.ptr = static_cast<int32_t *>(p);
    }
    *out = slot.ptr;
    return cudaSuccess;
}

}  // namespace

extern "C" kda_status kda_chunk_fwd_noalloc(const kda_fwd_desc *desc, const void *q,
                                            const void *k, const void *v, const void *g,
                                            const void *beta, const float *S0,
                                            const int32_t *cu_seqlens, const void *gate, void *o,
                                            float *S_T, cudaStream_t stream) {
    kda_status st = validate_fwd_desc(desc);
    if (st != KDA_OK) return st;
    const kda_fwd_desc &d = *desc;
    if (d.num_seqs > KDA_NOALLOC_MAX_SEQS) return KDA_ERR_WORKSPACE;
    if (!cu_seqlens) return KDA_ERR_INVALID_ARG;
    if (d.total_tokens > 0 && (!q || !k || !v || !g || !beta || !o)) return KDA_ERR_INVALID_ARG;

    const size_t esz = d.io_dtype == KDA_BF16 ? 2 : 4;
    const int64_t T = d.total_tokens, H = d.num_heads;
    const int64_t nk = T * H * d.dk * (int64_t)esz, nv = T * H * d.dv * (int64_t)esz;
    const int64_t nb = T * H * (int64_t)esz;
    const int64_t ns = (int64_t)d.num_seqs * H * d.dk * d.dv * 4;
    const Range ins[] = {range_of(q, nk), range_of(k, nk), range_of(g, nk), range_of(v, nv),
                         range_of(beta, nb), range_of(gate, gate ? nv : 0), range_of(S0, S0 ? ns : 0),
                         range_of(cu_seqlens, 4 * (int64_t)(d.num_seqs + 1))};
    const Range ro = range_of(o, nv), rs = range_of(S_T, S_T ? ns : 0);
    for (const Range &r : ins)
        if (overlaps(ro, r) || overlaps(rs, r)) return KDA_ERR_INVALID_ARG;
    if (overlaps(ro, rs)) return KDA_ERR_INVALID_ARG;

    int32_t *seq_order = nullptr;
    if (noalloc_scratch(&seq_order) != cudaSuccess) return KDA_ERR_CUDA;
    // every entry [0, num_seqs) is rewritten by the plan kernel before use,
    // so the previous call's contents never need clearing
    NvtxRange r("kda.prefill.noalloc");
    cudaError_t e = kda::launch_plan_longest_first(cu_seqlens, d.num_seqs, seq_order, stream);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    e = launch_prefill(d, q, k, v, g, beta, S0, cu_seqlens, seq_order, gate, o, S_T, kda::SnapOut{nullptr, nullptr, 0, 64}, stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Prefill from and to host memory (kda_chunk_fwd_host).  The batch is cut
// into groups of whole sequences; the host-to-device copy of group i+1, the
// prefill of group i and the device-to-host copy of group i-1 run on three
// streams (the two copy engines and the SMs), with input and output slots
// double-buffered in the caller's device workspace.
// ---------------------------------------------------------------------------
namespace {

constexpr int kHostGroups = 8;

struct HostPipe {
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t entry = nullptr, in_ready[2] = {}, computed[2] = {}, out_free[2] = {};
};
std::mutex g_pipe_mutex;          // held while a call enqueues its work
HostPipe g_pipe[kMaxDevices];

cudaError_t host_pipe(HostPipe **out) {   // caller holds g_pipe_mutex
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    HostPipe &p = g_pipe[dev];
    if (!p.h2d) {
        HostPipe n;
        if ((e = cudaStreamCreateWithFlags(&n.h2d, cudaStreamNonBlocking)) != cudaSuccess) return e;
        if ((e = cudaStreamCreateWithFlags(&n.d2h, cudaStreamNonBlocking)) != cudaSuccess) return e;
        cudaEvent_t *evs[] = {&n.entry, &n.in_ready[0], &n.in_ready[1], &n.computed[0], &n.computed[1],
                              &n.out_free[0], &n.out_free[1]};
        for (cudaEvent_t *ev : evs)
            if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess) return e;
        p = n;
    }
    *out = &p;
    return cudaSuccess;
}

struct HostGroup {
    int32_t s0, s1;     // sequences [s0, s1)
    int64_t t0, t1;     // tokens [t0, t1)
    size_t cu_off;      // this group's relative cu_seqlens in the cu region (entries)
};

struct HostLayout {
    std::vector<HostGroup> groups;
    std::vector<int32_t> cu_rel;                 // every group's cu_seqlens, relative to its start
    int64_t tmax = 0, smax = 0;
    size_t cu = 0, in[2] = {}, out[2] = {}, fws = 0, fws_bytes = 0, total = 0;
    size_t off_q = 0, off_k = 0, off_g = 0, off_v = 0, off_b = 0, off_z = 0, off_s0 = 0, in_bytes = 0;
    size_t off_o = 0, off_st = 0, out_bytes = 0;
};

kda_fwd_desc group_desc(const kda_fwd_desc &d, const HostGroup &gr) {
    kda_fwd_desc g = d;
    g.total_tokens = gr.t1 - gr.t0;
    g.num_seqs = gr.s1 - gr.s0;
    return g;
}

HostLayout host_layout(const kda_fwd_desc &d, const int32_t *cu, bool gate, bool s0, bool st) {
    HostLayout w;
    const int32_t N = d.num_seqs;
    const int G = std::min<int32_t>(N, kHostGroups);
    const int64_t T = d.total_tokens;
    int32_t s = 0;
    for (int gi = 0; gi < G; ++gi) {
        int32_t e = s + 1;
        const int64_t target = T * (gi + 1) / G;
        while (e < N - (G - 1 - gi) && cu[e] < target) ++e;
        if (gi == G - 1) e = N;
        w.groups.push_back(HostGroup{s, e, cu[s], cu[e], w.cu_rel.size()});
        for (int32_t n = s; n <= e; ++n) w.cu_rel.push_back(cu[n] - cu[s]);
        w.tmax = std::max<int64_t>(w.tmax, (int64_t)cu[e] - cu[s]);
        w.smax = std::max<int64_t>(w.smax, e - s);
        s = e;
    }
    const size_t esz = d.io_dtype == KDA_BF16 ? 2 : 4, H = (size_t)d.num_heads;
    const size_t tm = (size_t)w.tmax, sm = (size_t)w.smax, DKV = (size_t)d.dk * d.dv * 4;
    size_t o = 0;
    w.off_q = o; o += align256(tm * H * d.dk * esz);
    w.off_k = o; o += align256(tm * H * d.dk * esz);
    w.off_g = o; o += align256(tm * H * d.dk * esz);
    w.off_v = o; o += align256(tm * H * d.dv * esz);
    w.off_b = o; o += align256(tm * H * esz);
    w.off_z = o; o += gate ? align256(tm * H * d.dv * esz) : 0;
    w.off_s0 = o; o += s0 ? align256(sm * H * DKV) : 0;
    w.in_bytes = o;
    o = 0;
    w.off_o = o; o += align256(tm * H * d.dv * esz);
    w.off_st = o; o += st ? align256(sm * H * DKV) : 0;
    w.out_bytes = o;
    for (const HostGroup &gr : w.groups) {
        const kda_fwd_desc gd = group_desc(d, gr);
        w.fws_bytes = std::max(w.fws_bytes, fwd_workspace_bytes(&gd, w.cu_rel.data() + gr.cu_off));
    }
    size_t off = 0;
    w.cu = off;     off += align256(sizeof(int32_t) * w.cu_rel.size());
    w.in[0] = off;  off += w.in_bytes;
    w.in[1] = off;  off += w.in_bytes;
    w.out[0] = off; off += w.out_bytes;
    w.out[1] = off; off += w.out_bytes;
    w.fws = off;    off += align256(w.fws_bytes);
    w.total = off;
    return w;
}

}  // namespace

extern "C" size_t kda_chunk_fwd_host_workspace_size(const kda_fwd_desc *desc, const int32_t *cu_seqlens_host,
                                                    int32_t with_gate, int32_t with_S0, int32_t with_S_T) {
    if (validate_fwd_desc(desc) != KDA_OK || !cu_seqlens_host) return SIZE_MAX;
    if (validate_host_seqlens(desc, cu_seqlens_host) != KDA_OK) return SIZE_MAX;
    return host_layout(*desc, cu_seqlens_host, with_gate != 0, with_S0 != 0, with_S_T != 0).total;
}

extern "C" kda_status kda_chunk_fwd_host(const kda_fwd_desc *desc, const void *q, const void *k,
                                         const void *v, const void *g, const void *beta, const float *S0,
                                         const int32_t *cu_seqlens_host, const void *gate, void *o,
                                         float *S_T, void *workspace, size_t workspace_bytes,
                                         cudaStream_t stream) {
    kda_status st = validate_fwd_desc(desc);
    if (st != KDA_OK) return st;
    const kda_fwd_desc &d = *desc;
    if (!cu_seqlens_host) return KDA_ERR_INVALID_ARG;
    if ((st = validate_host_seqlens(desc, cu_seqlens_host)) != KDA_OK) return st;
    if (d.total_tokens > 0 && (!q || !k || !v || !g || !beta || !o)) return KDA_ERR_INVALID_ARG;
    const HostLayout w = host_layout(d, cu_seqlens_host, gate != nullptr, S0 != nullptr, S_T != nullptr);
    if (!workspace || workspace_bytes < w.total || reinterpret_cast<uintptr_t>(workspace) % 256 != 0)
        return KDA_ERR_WORKSPACE;

    std::lock_guard<std::mutex> lock(g_pipe_mutex);
    HostPipe *pp = nullptr;
    if (host_pipe(&pp) != cudaSuccess) return KDA_ERR_CUDA;
    HostPipe &P = *pp;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    const size_t esz = d.io_dtype == KDA_BF16 ? 2 : 4, H = (size_t)d.num_heads;
    const size_t rk = H * d.dk * esz, rv = H * d.dv * esz, rb = H * esz;      // bytes per token row
    const size_t rs = H * (size_t)d.dk * d.dv * sizeof(float);               // bytes per sequence state
    int32_t *cu_dev = reinterpret_cast<int32_t *>(ws + w.cu);
    auto ok = [](cudaError_t e) { return e == cudaSuccess; };
    auto cp = [](void *dst, const void *src, size_t n, cudaMemcpyKind kind, cudaStream_t s) {
        return n == 0 ? cudaSuccess : cudaMemcpyAsync(dst, src, n, kind, s);
    };
    // every group's relative cu_seqlens, then the copy streams join the caller's stream
    if (!ok(cudaMemcpyAsync(cu_dev, w.cu_rel.data(), w.cu_rel.size() * sizeof(int32_t), cudaMemcpyHostToDevice,
                            stream)) ||
        !ok(cudaEventRecord(P.entry, stream)) || !ok(cudaStreamWaitEvent(P.h2d, P.entry, 0)) ||
        !ok(cudaStreamWaitEvent(P.d2h, P.entry, 0)))
        return KDA_ERR_CUDA;
    const char *cq = static_cast<const char *>(q), *ck = static_cast<const char *>(k);
    const char *cg = static_cast<const char *>(g), *cv = static_cast<const char *>(v);
    const char *cb = static_cast<const char *>(beta), *cz = static_cast<const char *>(gate);
    const char *cs0 = reinterpret_cast<const char *>(S0);
    char *co = static_cast<char *>(o), *cst = reinterpret_cast<char *>(S_T);
    const int G = (int)w.groups.size();
    for (int i = 0; i < G; ++i) {
        const HostGroup &gr = w.groups[i];
        NvtxRange r("kda.host.group");
        const int sl = i & 1;
        unsigned char *in = ws + w.in[sl], *out = ws + w.out[sl];
        const size_t nt = (size_t)(gr.t1 - gr.t0), ns = (size_t)(gr.s1 - gr.s0);
        const size_t t0 = (size_t)gr.t0, s0 = (size_t)gr.s0;
        // inputs of group i, once the prefill of group i-2 has consumed the slot
        if (i >= 2 && !ok(cudaStreamWaitEvent(P.h2d, P.computed[sl], 0))) return KDA_ERR_CUDA;
        if (!ok(cp(in + w.off_q, cq + t0 * rk, nt * rk, cudaMemcpyHostToDevice, P.h2d)) ||
            !ok(cp(in + w.off_k, ck + t0 * rk, nt * rk, cudaMemcpyHostToDevice, P.h2d)) ||
            !ok(cp(in + w.off_g, cg + t0 * rk, nt * rk, cudaMemcpyHostToDevice, P.h2d)) ||
            !ok(cp(in + w.off_v, cv + t0 * rv, nt * rv, cudaMemcpyHostToDevice, P.h2d)) ||
            !ok(cp(in + w.off_b, cb + t0 * rb, nt * rb, cudaMemcpyHostToDevice, P.h2d)) ||
            (gate && !ok(cp(in + w.off_z, cz + t0 * rv, nt * rv, cudaMemcpyHostToDevice, P.h2d))) ||
            (S0 && !ok(cp(in + w.off_s0, cs0 + s0 * rs, ns * rs, cudaMemcpyHostToDevice, P.h2d))) ||
            !ok(cudaEventRecord(P.in_ready[sl], P.h2d)))
            return KDA_ERR_CUDA;
        // the prefill of group i, once its inputs are in and group i-2's outputs are out
        if (!ok(cudaStreamWaitEvent(stream, P.in_ready[sl], 0)) ||
            (i >= 2 && !ok(cudaStreamWaitEvent(stream, P.out_free[sl], 0))))
            return KDA_ERR_CUDA;
        const kda_fwd_desc gd = group_desc(d, gr);
        st = chunk_fwd_impl(&gd, nullptr, in + w.off_q, in + w.off_k, in + w.off_v, in + w.off_g, in + w.off_b,
                            S0 ? reinterpret_cast<const float *>(in + w.off_s0) : nullptr, cu_dev + gr.cu_off,
                            w.cu_rel.data() + gr.cu_off, gate ? in + w.off_z : nullptr, out + w.off_o,
                            S_T ? reinterpret_cast<float *>(out + w.off_st) : nullptr, ws + w.fws, w.fws_bytes,
                            stream);
        if (st != KDA_OK) return st;
        if (!ok(cudaEventRecord(P.computed[sl], stream))) return KDA_ERR_CUDA;
        // the outputs of group i
        if (!ok(cudaStreamWaitEvent(P.d2h, P.computed[sl], 0)) ||
            !ok(cp(co + t0 * rv, out + w.off_o, nt * rv, cudaMemcpyDeviceToHost, P.d2h)) ||
            (S_T && !ok(cp(cst + s0 * rs, out + w.off_st, ns * rs, cudaMemcpyDeviceToHost, P.d2h))) ||
            !ok(cudaEventRecord(P.out_free[sl], P.d2h)))
            return KDA_ERR_CUDA;
    }
    // the caller's stream covers the last copies (the copy streams are in order)
    if (G > 0 && !ok(cudaStreamWaitEvent(stream, P.out_free[(G - 1) & 1], 0))) return KDA_ERR_CUDA;
    return KDA_OK;
}
