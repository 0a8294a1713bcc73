// kda_bwd.cuh -- KDA backward (gradients of the forward recurrence), dk, dv in {64, 128}.
//
// The forward, per head (Kimi K3 report digest, section "KDA": per-channel
// decay with a log-decay floor, delta-rule write, optional sigmoid output gate):
//   alpha_t = exp(max(g_t, floor)),  P = Diag(alpha_t) S_{t-1},  u_t = P^T k_t,
//   S_t = P + beta_t k_t (v_t - u_t)^T,  o_t = scale S_t^T q_t [* sigmoid(z_t)].
// Reverse mode, token t, with dS the gradient of S_t (dS_T at the end):
//   go = do_t [* sigmoid(z_t)];  dS += scale q_t go^T;  r = dS^T k_t;
//   dv_t = beta_t r;  dbeta_t = r . (v_t - u_t);
//   dq_t = scale (P go + beta_t k_t ((v_t - u_t) . go));
//   dk_t = beta_t (dS (v_t - u_t) - P r);
//   dP = dS - beta_t k_t r^T;  dalpha_t = rowsum(dP o S_{t-1});
//   dg_t = dalpha_t alpha_t where g_t >= floor (0 below it);
//   dz_t = go (1 - sigmoid(z_t)) (S_t^T q_t scale);  dS <- Diag(alpha_t) dP.
//
// One CTA of 512 threads per (sequence, head): warp w owns state columns
// CPW w .. CPW w + CPW-1 (CPW = dv / 16), lane l rows RPT l .. RPT l + RPT-1
// (RPT = dk / 32), so the reductions over rows (u, S^T q, r) are warp shuffles and only the per-row gradient sums (dq, dk, dalpha)
// cross warps, through shared memory once per token.  States come back by
// recomputation: the states at 64-token chunk starts are given (the forward
// with snapshots); a chunk is replayed once to keep its 16-token sub-block
// starts, then each sub-block, last first, is replayed keeping S_{t-1} of
// every token in a per-unit scratch (each thread rereads only what it wrote)
// and run backwards.
#pragma once

#include "kda_common.cuh"

namespace kda {
namespace bwd {

constexpr int NT = 512;
constexpr int NW = NT / 32;     // warps = column groups
constexpr int SB = 16;          // sub-block of tokens replayed at a time
constexpr int CH = 64;          // checkpoint interval (tokens)
constexpr int64_t scratch_floats(int dk, int dv) { return (int64_t)(CH / SB - 1 + SB) * dk * dv; }   // per unit

struct BwdParams {
    const void *q, *k, *v, *g, *beta, *gate, *dout;
    const float *S0, *dS_T;
    const int32_t *cu_seqlens;
    const float *ckpt;            // [slots][H][dk][dv]: state after 64 m tokens of a sequence
    const int64_t *ckpt_base;     // [N + 1]: sequence n's first slot
    float *scratch;               // [units][scratch_floats(dk, dv)]
    void *dq, *dk, *dv, *dg, *dbeta, *dgate;
    float *dS0;
    int32_t num_heads;
    float scale, g_floor;
    int64_t total_tokens;         // for the debug build's unit checks
    int64_t slots;                // snapshot slots (the same)
};

// shared memory, floats: key-side [SB][DK] x 4, value-side [SB][DV] x 5, beta,
// per-row partial sums [2][NW][3][DK], per-warp scalars [2][NW][2]
template <int DK, int DV>
struct BwdSmem {
    static constexpr int K = 0, Q = K + SB * DK, A = Q + SB * DK, AM = A + SB * DK;
    static constexpr int V = AM + SB * DK, GO = V + SB * DV, SG = GO + SB * DV;
    static constexpr int U = SG + SB * DV, OR = U + SB * DV, B = OR + SB * DV;
    static constexpr int RED = B + SB;
    static constexpr int SCAL = RED + 2 * NW * 3 * DK;
    static constexpr int FLOATS = SCAL + 2 * NW * 2;
    static constexpr size_t BYTES = (size_t)FLOATS * sizeof(float);
};

// Sums x[0..NV-1] (NV = 8 or 4) over the warp's 32 lanes by halving the vector
// at each of the first log2(NV) exchange steps (9 shuffles for 8 values, 6 for
// 4, instead of 5 per value).  On return lane l holds the total of value
// j(l): for 8 values j = 4 b4 + 2 b3 + b2, for 4 values j = 2 b4 + b3 (b = the
// bits of l); reduce_lane(j) is a lane that holds it.
template <int NV>
__device__ __forceinline__ float warp_reduce(const float (&x)[NV], int lane) {
    static_assert(NV == 8 || NV == 4, "eight or four values per lane");
    const bool h4 = lane & 16, h3 = lane & 8;
    float w;
    if constexpr (NV == 8) {
        const bool h2 = lane & 4;
        float y[4], z[2];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            y[i] = (h4 ? x[i + 4] : x[i]) + __shfl_xor_sync(0xffffffffu, h4 ? x[i] : x[i + 4], 16);
#pragma unroll
        for (int i = 0; i < 2; ++i)
            z[i] = (h3 ? y[i + 2] : y[i]) + __shfl_xor_sync(0xffffffffu, h3 ? y[i] : y[i + 2], 8);
        w = (h2 ? z[1] : z[0]) + __shfl_xor_sync(0xffffffffu, h2 ? z[0] : z[1], 4);
    } else {
        float y[2];
#pragma unroll
        for (int i = 0; i < 2; ++i)
            y[i] = (h4 ? x[i + 2] : x[i]) + __shfl_xor_sync(0xffffffffu, h4 ? x[i] : x[i + 2], 16);
        w = (h3 ? y[1] : y[0]) + __shfl_xor_sync(0xffffffffu, h3 ? y[0] : y[1], 8);
        w += __shfl_xor_sync(0xffffffffu, w, 4);
    }
    w += __shfl_xor_sync(0xffffffffu, w, 2);
    w += __shfl_xor_sync(0xffffffffu, w, 1);
    return w;
}
template <int NV>
__device__ __forceinline__ int reduce_lane(int j) {
    return NV == 8 ? ((j >> 2) << 4) | (((j >> 1) & 1) << 3) | ((j & 1) << 2) : ((j >> 1) << 4) | ((j & 1) << 3);
}
template <int NV>
__device__ __forceinline__ int reduce_index(int lane) {
    return NV == 8 ? ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1)
                   : ((lane >> 4) & 1) * 2 + ((lane >> 3) & 1);
}
template <int NV>
__device__ __forceinline__ bool reduce_holder(int lane) { return (lane & (NV == 8 ? 3 : 7)) == 0; }
// every lane gets all NV totals
template <int NV>
__device__ __forceinline__ void warp_allreduce(float (&x)[NV], int lane) {
    const float w = warp_reduce<NV>(x, lane);
#pragma unroll
    for (int j = 0; j < NV; ++j) x[j] = __shfl_sync(0xffffffffu, w, reduce_lane<NV>(j));
}

template <int DK, int DV, typename TIO>
__global__ void __launch_bounds__(NT, 1) bwd_kernel(BwdParams p)
{
    constexpr int CPW = DV / NW;     // state columns per warp: 8 or 4
    constexpr int RPT = DK / 32;     // state rows per lane: 4 or 2
    using SM = BwdSmem<DK, DV>;
    constexpr int64_t SCRATCH_FLOATS = scratch_floats(DK, DV);
    extern __shared__ float4 bwd_smem4[];
    float *sm = reinterpret_cast<float *>(bwd_smem4);
    const TIO *q = static_cast<const TIO *>(p.q);
    const TIO *k = static_cast<const TIO *>(p.k);
    const TIO *v = static_cast<const TIO *>(p.v);
    const TIO *g = static_cast<const TIO *>(p.g);
    const TIO *beta = static_cast<const TIO *>(p.beta);
    const TIO *gate = static_cast<const TIO *>(p.gate);
    const TIO *dout = static_cast<const TIO *>(p.dout);

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int c0 = w * CPW, r0 = lane * RPT;
    const int H = p.num_heads;
    const int64_t unit = blockIdx.x;
    const int64_t n = unit / H, h = unit % H;
    const int64_t tb = p.cu_seqlens[n];
    const int64_t L = (int64_t)p.cu_seqlens[n + 1] - tb;
    // debug build: the sequence's tokens and snapshots as the host validated them (uniform over the CTA)
    if (kDebugChecks && (tb < 0 || L < 0 || tb + L > p.total_tokens ||
                         p.ckpt_base[n] + L / CH != p.ckpt_base[n + 1] || p.ckpt_base[n + 1] > p.slots)) {
        if (tid == 0) raise_error(ERR_BOUNDS);
        return;
    }
    float *scr = p.scratch + unit * SCRATCH_FLOATS;      // [3][DK][DV] sub-block starts, [SB][DK][DV] states
    float *scr_st = scr + (int64_t)(CH / SB - 1) * DK * DV;

    auto load_state = [&](float (&s)[RPT][CPW], const float *src) {
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
#pragma unroll
            for (int c4 = 0; c4 < CPW / 4; ++c4) {
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                if (src) x = *reinterpret_cast<const float4 *>(src + (r0 + r) * DV + c0 + 4 * c4);
                s[r][4 * c4] = x.x; s[r][4 * c4 + 1] = x.y; s[r][4 * c4 + 2] = x.z; s[r][4 * c4 + 3] = x.w;
            }
        }
    };
    auto store_state = [&](const float (&s)[RPT][CPW], float *dst) {
#pragma unroll
        for (int r = 0; r < RPT; ++r)
#pragma unroll
            for (int c4 = 0; c4 < CPW / 4; ++c4)
                *reinterpret_cast<float4 *>(dst + (r0 + r) * DV + c0 + 4 * c4) =
                    make_float4(s[r][4 * c4], s[r][4 * c4 + 1], s[r][4 * c4 + 2], s[r][4 * c4 + 3]);
    };
    // tokens tok0 .. tok0 + cnt - 1 of the sequence into shared memory
    auto stage = [&](int64_t tok0, int cnt) {
        for (int i = tid; i < cnt * DK; i += NT) {
            const int t = i / DK, c = i % DK;
            const int64_t row = (tb + tok0 + t) * H + h;
            const float gr = ld(g, row * DK + c);
            const float a = expf(fmaxf(gr, p.g_floor));
            sm[SM::K + i] = ld(k, row * DK + c);
            sm[SM::Q + i] = ld(q, row * DK + c);
            sm[SM::A + i] = a;
            sm[SM::AM + i] = gr >= p.g_floor ? a : 0.0f;
        }
        for (int i = tid; i < cnt * DV; i += NT) {
            const int t = i / DV, c = i % DV;
            const int64_t row = (tb + tok0 + t) * H + h;
            const float sg = gate ? sigmoidf(ld(gate, row * DV + c)) : 1.0f;
            sm[SM::V + i] = ld(v, row * DV + c);
            sm[SM::SG + i] = sg;
            sm[SM::GO + i] = ld(dout, row * DV + c) * sg;
        }
        if (tid < cnt) sm[SM::B + tid] = ld(beta, (tb + tok0 + tid) * H + h);
    };
    // one forward token on the registers' state; with `keep`, u_t and S_t^T q_t
    // of this warp's columns go to the shared rings
    auto replay = [&](float (&s)[RPT][CPW], int t, bool keep) {
        float kk[RPT];
        float u[CPW];
#pragma unroll
        for (int c = 0; c < CPW; ++c) u[c] = 0.0f;
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const float a = sm[SM::A + t * DK + r0 + r];
            kk[r] = sm[SM::K + t * DK + r0 + r];
#pragma unroll
            for (int c = 0; c < CPW; ++c) {
                s[r][c] *= a;
                u[c] = fmaf(s[r][c], kk[r], u[c]);
            }
        }
        warp_allreduce<CPW>(u, lane);
        const float bt = sm[SM::B + t];
#pragma unroll
        for (int c = 0; c < CPW; ++c) {
            const float d = sm[SM::V + t * DV + c0 + c] - u[c];
#pragma unroll
            for (int r = 0; r < RPT; ++r) s[r][c] = fmaf(bt * kk[r], d, s[r][c]);
        }
        if (keep) {
            float o[CPW];
#pragma unroll
            for (int c = 0; c < CPW; ++c) o[c] = 0.0f;
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float qq = sm[SM::Q + t * DK + r0 + r];
#pragma unroll
                for (int c = 0; c < CPW; ++c) o[c] = fmaf(s[r][c], qq, o[c]);
            }
            const float ot = warp_reduce<CPW>(o, lane);
            if (reduce_holder<CPW>(lane)) {      // the lanes that hold a total
                const int c = reduce_index<CPW>(lane);
                sm[SM::OR + t * DV + c0 + c] = p.scale * ot;
            }
            if (lane < CPW) {
#pragma unroll
                for (int c = 0; c < CPW; ++c)
                    if (lane == c) sm[SM::U + t * DV + c0 + c] = u[c];
            }
        }
    };

    float dS[RPT][CPW];
    load_state(dS, p.dS_T ? p.dS_T + unit * DK * DV : nullptr);
    int par = 0;
    const int nch = (int)((L + CH - 1) / CH);
    for (int ci = nch - 1; ci >= 0; --ci) {
        const int64_t tc0 = (int64_t)ci * CH;
        const int clen = (int)(L - tc0 < CH ? L - tc0 : CH);
        const int nsb = (clen + SB - 1) / SB;
        const float *start = ci == 0 ? (p.S0 ? p.S0 + unit * DK * DV : nullptr)
                                     : p.ckpt + ((p.ckpt_base[n] + ci - 1) * H + h) * DK * DV;
        {   // the chunk's sub-block starts
            float s[RPT][CPW];
            load_state(s, start);
            for (int sb = 0; sb + 1 < nsb; ++sb) {
                __syncthreads();
                stage(tc0 + sb * SB, SB);
                __syncthreads();
                for (int t = 0; t < SB; ++t) replay(s, t, false);
                store_state(s, scr + (int64_t)sb * DK * DV);
            }
        }
        for (int sb = nsb - 1; sb >= 0; --sb) {
            const int cnt = clen - sb * SB < SB ? clen - sb * SB : SB;
            {
                float s[RPT][CPW];
                load_state(s, sb == 0 ? start : scr + (int64_t)(sb - 1) * DK * DV);
                __syncthreads();
                stage(tc0 + sb * SB, cnt);
                __syncthreads();
                for (int t = 0; t < cnt; ++t) {
                    store_state(s, scr_st + (int64_t)t * DK * DV);     // S_{t-1}
                    replay(s, t, true);
                }
                __syncwarp();
            }
            for (int t = cnt - 1; t >= 0; --t) {
                const int64_t row = (tb + tc0 + sb * SB + t) * H + h;
                const float bt = sm[SM::B + t];
                float go[CPW], rr[CPW], vu[CPW];
#pragma unroll
                for (int c = 0; c < CPW; ++c) {
                    go[c] = sm[SM::GO + t * DV + c0 + c];
                    vu[c] = sm[SM::V + t * DV + c0 + c] - sm[SM::U + t * DV + c0 + c];
                    rr[c] = 0.0f;
                }
                float kk[RPT], aa[RPT];
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const float qq = p.scale * sm[SM::Q + t * DK + r0 + r];
                    kk[r] = sm[SM::K + t * DK + r0 + r];
                    aa[r] = sm[SM::A + t * DK + r0 + r];
#pragma unroll
                    for (int c = 0; c < CPW; ++c) {
                        dS[r][c] = fmaf(qq, go[c], dS[r][c]);
                        rr[c] = fmaf(dS[r][c], kk[r], rr[c]);
                    }
                }
                warp_allreduce<CPW>(rr, lane);
                float *red = sm + SM::RED + par * (NW * 3 * DK) + w * 3 * DK;
                const float *Sprev = scr_st + (int64_t)t * DK * DV;
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    float sp[CPW];
#pragma unroll
                    for (int c4 = 0; c4 < CPW / 4; ++c4) {
                        const float4 x = *reinterpret_cast<const float4 *>(Sprev + (r0 + r) * DV + c0 + 4 * c4);
                        sp[4 * c4] = x.x; sp[4 * c4 + 1] = x.y; sp[4 * c4 + 2] = x.z; sp[4 * c4 + 3] = x.w;
                    }
                    float dqp = 0.0f, dkp = 0.0f, dap = 0.0f;
#pragma unroll
                    for (int c = 0; c < CPW; ++c) {
                        const float P = aa[r] * sp[c];
                        dqp = fmaf(P, go[c], dqp);
                        dkp = fmaf(dS[r][c], vu[c], dkp);
                        dkp = fmaf(-P, rr[c], dkp);
                        const float dP = fmaf(-bt * kk[r], rr[c], dS[r][c]);
                        dap = fmaf(dP, sp[c], dap);
                        dS[r][c] = aa[r] * dP;
                    }
                    red[0 * DK + r0 + r] = dqp;
                    red[1 * DK + r0 + r] = dkp;
                    red[2 * DK + r0 + r] = dap;
                }
                if (lane == 0) {
                    float cw = 0.0f, dbw = 0.0f;
#pragma unroll
                    for (int c = 0; c < CPW; ++c) {
                        cw = fmaf(vu[c], go[c], cw);
                        dbw = fmaf(rr[c], vu[c], dbw);
                    }
                    sm[SM::SCAL + (par * NW + w) * 2 + 0] = cw;
                    sm[SM::SCAL + (par * NW + w) * 2 + 1] = dbw;
                }
#pragma unroll
                for (int c = 0; c < CPW; ++c) {
                    if (lane == c) {
                        st(static_cast<TIO *>(p.dv), row * DV + c0 + c, bt * rr[c]);
                        if (gate) {
                            const float sg = sm[SM::SG + t * DV + c0 + c];
                            st(static_cast<TIO *>(p.dgate), row * DV + c0 + c,
                               go[c] * (1.0f - sg) * sm[SM::OR + t * DV + c0 + c]);
                        }
                    }
                }
                __syncthreads();
                if (tid < DK) {
                    const float *rp = sm + SM::RED + par * (NW * 3 * DK);
                    float sq = 0.0f, sk = 0.0f, sa = 0.0f, cw = 0.0f;
#pragma unroll
                    for (int ww = 0; ww < NW; ++ww) {
                        sq += rp[ww * 3 * DK + tid];
                        sk += rp[ww * 3 * DK + DK + tid];
                        sa += rp[ww * 3 * DK + 2 * DK + tid];
                        cw += sm[SM::SCAL + (par * NW + ww) * 2];
                    }
                    const float ki = sm[SM::K + t * DK + tid];
                    st(static_cast<TIO *>(p.dq), row * DK + tid, p.scale * fmaf(bt * ki, cw, sq));
                    st(static_cast<TIO *>(p.dk), row * DK + tid, bt * sk);
                    st(static_cast<TIO *>(p.dg), row * DK + tid, sa * sm[SM::AM + t * DK + tid]);
                } else if (tid == DK) {
                    float db = 0.0f;
#pragma unroll
                    for (int ww = 0; ww < NW; ++ww) db += sm[SM::SCAL + (par * NW + ww) * 2 + 1];
                    st(static_cast<TIO *>(p.dbeta), row, db);
                }
                par ^= 1;
            }
        }
    }
    if (p.dS0) store_state(dS, p.dS0 + unit * DK * DV);
}

}  // namespace bwd
}  // namespace kda
