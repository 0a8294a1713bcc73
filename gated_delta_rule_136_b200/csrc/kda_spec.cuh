// kda_spec.cuh -- speculative-decode verify and commit over D draft tokens
// per (sequence, head): the replay of the fupanwang.com Kimi K3 report digest,
// section 基础设施 (verify the draft on chip, then commit only the accepted
// prefix in place).
//
// Verify runs the decode recurrence over all D draft tokens from S, with the
// state in registers, and writes every token's output; S is not written.
// Commit replays the first `accepted[b]` tokens from S and writes the state
// back once.  Per token, with alpha = exp(max(g, floor)):
//   S' = Diag(alpha) S,  u = S'^T k,  w = S'^T q,
//   S  = S' + beta k (v - u)^T,   o = scale (w + beta (k.q) (v - u)) [* sigmoid(z)]
// Inputs are token-major per sequence: q, k, g [B, D, H, dk]; v, gate, o
// [B, D, H, dv]; beta [B, D, H].  Each pass streams the 64 KiB state once
// (verify: read; commit: read + write), whatever D is.
#pragma once

#include "kda_common.cuh"

namespace kda {

struct SpecParams {
    const void *q, *k, *v, *g, *beta, *gate;
    float *S;
    void *o;                       // verify: outputs; commit: unused
    const int32_t *accepted;       // commit: tokens to apply per sequence (clamped to [0, D])
    int32_t num_heads, draft;
    float scale, g_floor;
};

template <int DK, int DV, typename TIO, bool COMMIT>
__global__ void __launch_bounds__(256) spec_kernel(SpecParams p)
{
    constexpr int NT = 256;
    constexpr int C4 = DV / 4;        // float4 per state row
    constexpr int RG = NT / C4;       // row groups
    constexpr int F = DK / RG;        // state rows per thread
    static_assert(DK % RG == 0, "row split");

    __shared__ float sq[DK], sk[DK], sa[DK], sv[DV];
    __shared__ float4 red_u[RG][C4], red_w[RG][C4];
    __shared__ float s_kq;

    const TIO *q = static_cast<const TIO *>(p.q);
    const TIO *k = static_cast<const TIO *>(p.k);
    const TIO *v = static_cast<const TIO *>(p.v);
    const TIO *g = static_cast<const TIO *>(p.g);
    const TIO *beta = static_cast<const TIO *>(p.beta);
    const TIO *gate = static_cast<const TIO *>(p.gate);
    TIO *o = static_cast<TIO *>(p.o);

    const int tid = threadIdx.x;
    const int col4 = tid % C4;
    const int rg = tid / C4;
    const int H = p.num_heads, D = p.draft;
    const int64_t unit = blockIdx.x;             // b * H + h
    const int64_t b = unit / H, h = unit % H;
    float4 *Sp = reinterpret_cast<float4 *>(p.S + unit * DK * DV);

    int ntok = D;
    if (COMMIT) {
        const int a = p.accepted[b];
        ntok = a < 0 ? 0 : (a > D ? D : a);
        if (ntok == 0) return;                   // nothing accepted: S stays as it is
    }

    float4 s[F];
#pragma unroll
    for (int f = 0; f < F; ++f) s[f] = __ldcs(&Sp[(rg + f * RG) * C4 + col4]);

    for (int t = 0; t < ntok; ++t) {
        const int64_t row = (b * D + t) * H + h;  // (token, head) row of the packed inputs
        for (int i = tid; i < DK; i += NT) {
            sq[i] = ld(q, row * DK + i);
            sk[i] = ld(k, row * DK + i);
            sa[i] = expf(fmaxf(ld(g, row * DK + i), p.g_floor));
        }
        for (int i = tid; i < DV; i += NT) sv[i] = ld(v, row * DV + i);
        __syncthreads();

        if (!COMMIT && tid < 32) {
            float acc = 0.0f;
            for (int i = tid; i < DK; i += 32) acc = fmaf(sk[i], sq[i], acc);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (tid == 0) s_kq = acc;
        }

        float4 u = make_float4(0.f, 0.f, 0.f, 0.f), w = u;
#pragma unroll
        for (int f = 0; f < F; ++f) {
            const int c = rg + f * RG;
            const float a = sa[c], kc = sk[c], qc = sq[c];
            s[f].x *= a; s[f].y *= a; s[f].z *= a; s[f].w *= a;
            u.x = fmaf(s[f].x, kc, u.x); u.y = fmaf(s[f].y, kc, u.y);
            u.z = fmaf(s[f].z, kc, u.z); u.w = fmaf(s[f].w, kc, u.w);
            if (!COMMIT) {
                w.x = fmaf(s[f].x, qc, w.x); w.y = fmaf(s[f].y, qc, w.y);
                w.z = fmaf(s[f].z, qc, w.z); w.w = fmaf(s[f].w, qc, w.w);
            }
        }
        red_u[rg][col4] = u;
        if (!COMMIT) red_w[rg][col4] = w;
        __syncthreads();

        float4 U = make_float4(0.f, 0.f, 0.f, 0.f), W = U;
#pragma unroll
        for (int r = 0; r < RG; ++r) {
            const float4 a = red_u[r][col4];
            U.x += a.x; U.y += a.y; U.z += a.z; U.w += a.w;
            if (!COMMIT) {
                const float4 c = red_w[r][col4];
                W.x += c.x; W.y += c.y; W.z += c.z; W.w += c.w;
            }
        }
        const float bt = ld(beta, row);
        const float4 d = make_float4(sv[4 * col4 + 0] - U.x, sv[4 * col4 + 1] - U.y,
                                     sv[4 * col4 + 2] - U.z, sv[4 * col4 + 3] - U.w);
#pragma unroll
        for (int f = 0; f < F; ++f) {
            const float bk = bt * sk[rg + f * RG];
            s[f].x = fmaf(bk, d.x, s[f].x); s[f].y = fmaf(bk, d.y, s[f].y);
            s[f].z = fmaf(bk, d.z, s[f].z); s[f].w = fmaf(bk, d.w, s[f].w);
        }
        if (!COMMIT && rg == 0) {
            const float bkq = bt * s_kq;
            const float oo[4] = {W.x + bkq * d.x, W.y + bkq * d.y, W.z + bkq * d.z, W.w + bkq * d.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int64_t off = row * DV + 4 * col4 + e;
                float x = p.scale * oo[e];
                if (gate) x *= sigmoidf(ld(gate, off));
                st(o, off, x);
            }
        }
        __syncthreads();                         // the token's shared values are consumed
    }

    if (COMMIT) {
#pragma unroll
        for (int f = 0; f < F; ++f) __stcs(&Sp[(rg + f * RG) * C4 + col4], s[f]);
    }
}

}  // namespace kda
