// kda_bwd.cuh -- KDA backward (gradients of the forward recurrence), dk = dv = 128.
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
// 8w .. 8w+7, lane l rows 4l .. 4l+3, so the reductions over rows (u, S^T q,
// r) are warp shuffles and only the per-row gradient sums (dq, dk, dalpha)
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

constexpr int D = 128;          // dk = dv
constexpr int NT = 512;
constexpr int NW = NT / 32;     // warps = column groups
constexpr int CPW = D / NW;     // columns per warp: 8
constexpr int RPT = D / 32;     // rows per lane: 4
constexpr int SB = 16;          // sub-block of tokens replayed at a time
constexpr int CH = 64;          // checkpoint interval (tokens)
constexpr int64_t SCRATCH_FLOATS = (int64_t)(CH / SB - 1 + SB) * D * D;   // per unit

struct BwdParams {
    const void *q, *k, *v, *g, *beta, *gate, *dout;
    const float *S0, *dS_T;
    const int32_t *cu_seqlens;
    const float *ckpt;            // [slots][H][D][D]: state after 64 m tokens of a sequence
    const int64_t *ckpt_base;     // [N + 1]: sequence n's first slot
    float *scratch;               // [units][SCRATCH_FLOATS]
    void *dq, *dk, *dv, *dg, *dbeta, *dgate;
    float *dS0;
    int32_t num_heads;
    float scale, g_floor;
};

// shared memory, floats
constexpr int SM_K = 0, SM_Q = SM_K + SB * D, SM_A = SM_Q + SB * D, SM_AM = SM_A + SB * D;
constexpr int SM_V = SM_AM + SB * D, SM_GO = SM_V + SB * D, SM_SG = SM_GO + SB * D;
constexpr int SM_U = SM_SG + SB * D, SM_OR = SM_U + SB * D, SM_B = SM_OR + SB * D;
constexpr int SM_RED = SM_B + SB;                       // [2][NW][3][D]
constexpr int SM_SCAL = SM_RED + 2 * NW * 3 * D;        // [2][NW][2]
constexpr int SM_FLOATS = SM_SCAL + 2 * NW * 2;
constexpr size_t SMEM_BYTES = (size_t)SM_FLOATS * sizeof(float);

// Sums x[0..7] over the warp's 32 lanes by halving the vector at each of the
// first three exchange steps (9 shuffles instead of 40).  On return lane l
// holds the total of value j(l) = 4 b4 + 2 b3 + b2 (b = the bits of l).
__device__ __forceinline__ float warp_reduce8(const float (&x)[CPW], int lane) {
    static_assert(CPW == 8, "eight values per lane");
    const bool h4 = lane & 16, h3 = lane & 8, h2 = lane & 4;
    float y[4], z[2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        y[i] = (h4 ? x[i + 4] : x[i]) + __shfl_xor_sync(0xffffffffu, h4 ? x[i] : x[i + 4], 16);
#pragma unroll
    for (int i = 0; i < 2; ++i)
        z[i] = (h3 ? y[i + 2] : y[i]) + __shfl_xor_sync(0xffffffffu, h3 ? y[i] : y[i + 2], 8);
    float w = (h2 ? z[1] : z[0]) + __shfl_xor_sync(0xffffffffu, h2 ? z[0] : z[1], 4);
    w += __shfl_xor_sync(0xffffffffu, w, 2);
    w += __shfl_xor_sync(0xffffffffu, w, 1);
    return w;
}
__device__ __forceinline__ int reduce8_lane(int j) { return ((j >> 2) << 4) | (((j >> 1) & 1) << 3) | ((j & 1) << 2); }
__device__ __forceinline__ int reduce8_index(int lane) { return ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1); }
// every lane gets all eight totals
__device__ __forceinline__ void warp_allreduce8(float (&x)[CPW], int lane) {
    const float w = warp_reduce8(x, lane);
#pragma unroll
    for (int j = 0; j < CPW; ++j) x[j] = __shfl_sync(0xffffffffu, w, reduce8_lane(j));
}

template <typename TIO>
__global__ void __launch_bounds__(NT, 1) bwd_kernel(BwdParams p)
{
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
    float *scr = p.scratch + unit * SCRATCH_FLOATS;      // [3][D][D] sub-block starts, [SB][D][D] states
    float *scr_st = scr + (int64_t)(CH / SB - 1) * D * D;

    auto load_state = [&](float (&s)[RPT][CPW], const float *src) {
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
#pragma unroll
            for (int c4 = 0; c4 < CPW / 4; ++c4) {
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                if (src) x = *reinterpret_cast<const float4 *>(src + (r0 + r) * D + c0 + 4 * c4);
                s[r][4 * c4] = x.x; s[r][4 * c4 + 1] = x.y; s[r][4 * c4 + 2] = x.z; s[r][4 * c4 + 3] = x.w;
            }
        }
    };
    auto store_state = [&](const float (&s)[RPT][CPW], float *dst) {
#pragma unroll
        for (int r = 0; r < RPT; ++r)
#pragma unroll
            for (int c4 = 0; c4 < CPW / 4; ++c4)
                *reinterpret_cast<float4 *>(dst + (r0 + r) * D + c0 + 4 * c4) =
                    make_float4(s[r][4 * c4], s[r][4 * c4 + 1], s[r][4 * c4 + 2], s[r][4 * c4 + 3]);
    };
    // tokens tok0 .. tok0 + cnt - 1 of the sequence into shared memory
    auto stage = [&](int64_t tok0, int cnt) {
        for (int i = tid; i < cnt * D; i += NT) {
            const int t = i / D, c = i % D;
            const int64_t row = (tb + tok0 + t) * H + h;
            const float gr = ld(g, row * D + c);
            const float a = expf(fmaxf(gr, p.g_floor));
            sm[SM_K + i] = ld(k, row * D + c);
            sm[SM_Q + i] = ld(q, row * D + c);
            sm[SM_A + i] = a;
            sm[SM_AM + i] = gr >= p.g_floor ? a : 0.0f;
            const float sg = gate ? sigmoidf(ld(gate, row * D + c)) : 1.0f;
            sm[SM_V + i] = ld(v, row * D + c);
            sm[SM_SG + i] = sg;
            sm[SM_GO + i] = ld(dout, row * D + c) * sg;
        }
        if (tid < cnt) sm[SM_B + tid] = ld(beta, (tb + tok0 + tid) * H + h);
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
            const float a = sm[SM_A + t * D + r0 + r];
            kk[r] = sm[SM_K + t * D + r0 + r];
#pragma unroll
            for (int c = 0; c < CPW; ++c) {
                s[r][c] *= a;
                u[c] = fmaf(s[r][c], kk[r], u[c]);
            }
        }
        warp_allreduce8(u, lane);
        const float bt = sm[SM_B + t];
#pragma unroll
        for (int c = 0; c < CPW; ++c) {
            const float d = sm[SM_V + t * D + c0 + c] - u[c];
#pragma unroll
            for (int r = 0; r < RPT; ++r) s[r][c] = fmaf(bt * kk[r], d, s[r][c]);
        }
        if (keep) {
            float o[CPW];
#pragma unroll
            for (int c = 0; c < CPW; ++c) o[c] = 0.0f;
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float qq = sm[SM_Q + t * D + r0 + r];
#pragma unroll
                for (int c = 0; c < CPW; ++c) o[c] = fmaf(s[r][c], qq, o[c]);
            }
            const float ot = warp_reduce8(o, lane);
            if ((lane & 3) == 0) {               // the eight lanes that hold a total
                const int c = reduce8_index(lane);
                sm[SM_OR + t * D + c0 + c] = p.scale * ot;
            }
            if (lane < CPW) {
#pragma unroll
                for (int c = 0; c < CPW; ++c)
                    if (lane == c) sm[SM_U + t * D + c0 + c] = u[c];
            }
        }
    };

    float dS[RPT][CPW];
    load_state(dS, p.dS_T ? p.dS_T + unit * D * D : nullptr);
    int par = 0;
    const int nch = (int)((L + CH - 1) / CH);
    for (int ci = nch - 1; ci >= 0; --ci) {
        const int64_t tc0 = (int64_t)ci * CH;
        const int clen = (int)(L - tc0 < CH ? L - tc0 : CH);
        const int nsb = (clen + SB - 1) / SB;
        const float *start = ci == 0 ? (p.S0 ? p.S0 + unit * D * D : nullptr)
                                     : p.ckpt + ((p.ckpt_base[n] + ci - 1) * H + h) * D * D;
        {   // the chunk's sub-block starts
            float s[RPT][CPW];
            load_state(s, start);
            for (int sb = 0; sb + 1 < nsb; ++sb) {
                __syncthreads();
                stage(tc0 + sb * SB, SB);
                __syncthreads();
                for (int t = 0; t < SB; ++t) replay(s, t, false);
                store_state(s, scr + (int64_t)sb * D * D);
            }
        }
        for (int sb = nsb - 1; sb >= 0; --sb) {
            const int cnt = clen - sb * SB < SB ? clen - sb * SB : SB;
            {
                float s[RPT][CPW];
                load_state(s, sb == 0 ? start : scr + (int64_t)(sb - 1) * D * D);
                __syncthreads();
                stage(tc0 + sb * SB, cnt);
                __syncthreads();
                for (int t = 0; t < cnt; ++t) {
                    store_state(s, scr_st + (int64_t)t * D * D);     // S_{t-1}
                    replay(s, t, true);
                }
                __syncwarp();
            }
            for (int t = cnt - 1; t >= 0; --t) {
                const int64_t row = (tb + tc0 + sb * SB + t) * H + h;
                const float bt = sm[SM_B + t];
                float go[CPW], rr[CPW], vu[CPW];
#pragma unroll
                for (int c = 0; c < CPW; ++c) {
                    go[c] = sm[SM_GO + t * D + c0 + c];
                    vu[c] = sm[SM_V + t * D + c0 + c] - sm[SM_U + t * D + c0 + c];
                    rr[c] = 0.0f;
                }
                float kk[RPT], aa[RPT];
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const float qq = p.scale * sm[SM_Q + t * D + r0 + r];
                    kk[r] = sm[SM_K + t * D + r0 + r];
                    aa[r] = sm[SM_A + t * D + r0 + r];
#pragma unroll
                    for (int c = 0; c < CPW; ++c) {
                        dS[r][c] = fmaf(qq, go[c], dS[r][c]);
                        rr[c] = fmaf(dS[r][c], kk[r], rr[c]);
                    }
                }
                warp_allreduce8(rr, lane);
                float *red = sm + SM_RED + par * (NW * 3 * D) + w * 3 * D;
                const float *Sprev = scr_st + (int64_t)t * D * D;
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    float sp[CPW];
#pragma unroll
                    for (int c4 = 0; c4 < CPW / 4; ++c4) {
                        const float4 x = *reinterpret_cast<const float4 *>(Sprev + (r0 + r) * D + c0 + 4 * c4);
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
                    red[0 * D + r0 + r] = dqp;
                    red[1 * D + r0 + r] = dkp;
                    red[2 * D + r0 + r] = dap;
                }
                if (lane == 0) {
                    float cw = 0.0f, dbw = 0.0f;
#pragma unroll
                    for (int c = 0; c < CPW; ++c) {
                        cw = fmaf(vu[c], go[c], cw);
                        dbw = fmaf(rr[c], vu[c], dbw);
                    }
                    sm[SM_SCAL + (par * NW + w) * 2 + 0] = cw;
                    sm[SM_SCAL + (par * NW + w) * 2 + 1] = dbw;
                }
#pragma unroll
                for (int c = 0; c < CPW; ++c) {
                    if (lane == c) {
                        st(static_cast<TIO *>(p.dv), row * D + c0 + c, bt * rr[c]);
                        if (gate) {
                            const float sg = sm[SM_SG + t * D + c0 + c];
                            st(static_cast<TIO *>(p.dgate), row * D + c0 + c,
                               go[c] * (1.0f - sg) * sm[SM_OR + t * D + c0 + c]);
                        }
                    }
                }
                __syncthreads();
                if (tid < D) {
                    const float *rp = sm + SM_RED + par * (NW * 3 * D);
                    float sq = 0.0f, sk = 0.0f, sa = 0.0f, cw = 0.0f;
#pragma unroll
                    for (int ww = 0; ww < NW; ++ww) {
                        sq += rp[ww * 3 * D + tid];
                        sk += rp[ww * 3 * D + D + tid];
                        sa += rp[ww * 3 * D + 2 * D + tid];
                        cw += sm[SM_SCAL + (par * NW + ww) * 2];
                    }
                    const float ki = sm[SM_K + t * D + tid];
                    st(static_cast<TIO *>(p.dq), row * D + tid, p.scale * fmaf(bt * ki, cw, sq));
                    st(static_cast<TIO *>(p.dk), row * D + tid, bt * sk);
                    st(static_cast<TIO *>(p.dg), row * D + tid, sa * sm[SM_AM + t * D + tid]);
                } else if (tid == D) {
                    float db = 0.0f;
#pragma unroll
                    for (int ww = 0; ww < NW; ++ww) db += sm[SM_SCAL + (par * NW + ww) * 2 + 1];
                    st(static_cast<TIO *>(p.dbeta), row, db);
                }
                par ^= 1;
            }
        }
    }
    if (p.dS0) store_state(dS, p.dS0 + unit * D * D);
}

}  // namespace bwd
}  // namespace kda
