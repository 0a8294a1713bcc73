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
//
// One CTA of 256 threads per (sequence, head).  Tokens are staged 8 at a time
// in shared memory as {alpha, alpha k, alpha q, beta k} per state row; each
// thread keeps F rows x 4 columns of the state in registers and updates them
// with packed f32x2 arithmetic; u and w are summed over the row groups through
// shared memory, double-buffered by token parity, so each token costs one
// barrier.  The output of token j is written by row group j mod RG.
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
    constexpr int F = DK / RG;        // state rows per thread: rows rg * F .. rg * F + F - 1
    constexpr int G = 8;              // tokens staged in shared memory at a time
    static_assert(DK % RG == 0, "row split");

    // per staged token and state row: {alpha, alpha k, alpha q, beta k}
    __shared__ float4 srow[G][DK];
    __shared__ float sv[G][DV], sz[COMMIT ? 1 : G][DV], skq[G];
    __shared__ float4 red_u[2][RG][C4], red_w[2][RG][C4];   // by token parity

    const TIO *q = static_cast<const TIO *>(p.q);
    const TIO *k = static_cast<const TIO *>(p.k);
    const TIO *v = static_cast<const TIO *>(p.v);
    const TIO *g = static_cast<const TIO *>(p.g);
    const TIO *beta = static_cast<const TIO *>(p.beta);
    const TIO *gate = static_cast<const TIO *>(p.gate);
    TIO *o = static_cast<TIO *>(p.o);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
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

    // the state slice as column pairs: s[f][0] = columns 4 col4 + {0,1}, s[f][1] = + {2,3}
    float2 s[F][2];
#pragma unroll
    for (int f = 0; f < F; ++f) {
        const float4 x = __ldcs(&Sp[(rg * F + f) * C4 + col4]);
        s[f][0] = make_float2(x.x, x.y);
        s[f][1] = make_float2(x.z, x.w);
    }

    for (int t0 = 0; t0 < ntok; t0 += G) {
        const int nt = ntok - t0 < G ? ntok - t0 : G;
        __syncthreads();                         // the previous group's values are consumed
        // stage the group's tokens, row (b, t, h) of the packed inputs
        if (COMMIT) {
            // one element after another (measured faster for the commit than
            // issuing every load first); q is not needed
            for (int i = tid; i < nt * DK; i += NT) {
                const int j = i / DK, c = i % DK;
                const int64_t row = (b * D + t0 + j) * H + h;
                const float kk = ld(k, row * DK + c);
                const float a = expf(fmaxf(ld(g, row * DK + c), p.g_floor));
                srow[j][c] = make_float4(a, a * kk, 0.0f, ld(beta, row) * kk);
            }
            for (int i = tid; i < nt * DV; i += NT) {
                const int j = i / DV, c = i % DV;
                sv[j][c] = ld(v, ((b * D + t0 + j) * H + h) * DV + c);
            }
        } else {
            // every load issued before the first shared-memory store
            constexpr int EK = G * DK / NT, EV = G * DV / NT;
            float kk[EK], qq[EK], gg[EK], bb[EK], vv[EV], zz[EV];
#pragma unroll
            for (int e = 0; e < EK; ++e) {
                const int i = tid + e * NT, j = i / DK, c = i % DK;
                if (j < nt) {
                    const int64_t row = (b * D + t0 + j) * H + h;
                    kk[e] = ld(k, row * DK + c);
                    qq[e] = ld(q, row * DK + c);
                    gg[e] = ld(g, row * DK + c);
                    bb[e] = ld(beta, row);
                }
            }
#pragma unroll
            for (int e = 0; e < EV; ++e) {
                const int i = tid + e * NT, j = i / DV, c = i % DV;
                if (j < nt) {
                    const int64_t off = ((b * D + t0 + j) * H + h) * DV + c;
                    vv[e] = ld(v, off);
                    zz[e] = gate ? ld(gate, off) : 0.0f;
                }
            }
#pragma unroll
            for (int e = 0; e < EK; ++e) {
                const int i = tid + e * NT, j = i / DK, c = i % DK;
                if (j < nt) {
                    const float a = expf(fmaxf(gg[e], p.g_floor));
                    srow[j][c] = make_float4(a, a * kk[e], a * qq[e], bb[e] * kk[e]);
                }
            }
#pragma unroll
            for (int e = 0; e < EV; ++e) {
                const int i = tid + e * NT, j = i / DV, c = i % DV;
                if (j < nt) {
                    sv[j][c] = vv[e];
                    sz[COMMIT ? 0 : j][c] = gate ? sigmoidf(zz[e]) : 1.0f;
                }
            }
        }
        __syncthreads();
        if (!COMMIT && warp < nt) {              // beta (k.q) of token `warp`
            float acc = 0.0f;
            for (int i = lane; i < DK; i += 32) {
                const float4 r = srow[warp][i];
                acc = fmaf(r.w, r.z / r.x, acc);   // (beta k)(alpha q) / alpha
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (lane == 0) skq[warp] = acc;
        }

        for (int j = 0; j < nt; ++j) {
            const int par = j & 1;
            float2 u0 = make_float2(0.f, 0.f), u1 = u0, w0 = u0, w1 = u0;
#pragma unroll
            for (int f = 0; f < F; ++f) {
                const float4 r = srow[j][rg * F + f];
                const float2 ak = make_float2(r.y, r.y);
                u0 = __ffma2_rn(s[f][0], ak, u0);
                u1 = __ffma2_rn(s[f][1], ak, u1);
                if (!COMMIT) {
                    const float2 aq = make_float2(r.z, r.z);
                    w0 = __ffma2_rn(s[f][0], aq, w0);
                    w1 = __ffma2_rn(s[f][1], aq, w1);
                }
            }
            red_u[par][rg][col4] = make_float4(u0.x, u0.y, u1.x, u1.y);
            if (!COMMIT) red_w[par][rg][col4] = make_float4(w0.x, w0.y, w1.x, w1.y);
            // one barrier per token: the other parity's buffers were read before it
            __syncthreads();

            float2 U0 = make_float2(0.f, 0.f), U1 = U0;
#pragma unroll
            for (int r = 0; r < RG; ++r) {
                const float4 x = red_u[par][r][col4];
                U0 = __fadd2_rn(U0, make_float2(x.x, x.y));
                U1 = __fadd2_rn(U1, make_float2(x.z, x.w));
            }
            const float4 vj = *reinterpret_cast<const float4 *>(&sv[j][4 * col4]);
            const float2 d0 = make_float2(vj.x - U0.x, vj.y - U0.y);
            const float2 d1 = make_float2(vj.z - U1.x, vj.w - U1.y);
            // S = alpha S + (beta k) d^T
#pragma unroll
            for (int f = 0; f < F; ++f) {
                const float4 r = srow[j][rg * F + f];
                const float2 al = make_float2(r.x, r.x), bk = make_float2(r.w, r.w);
                s[f][0] = __ffma2_rn(s[f][0], al, __fmul2_rn(bk, d0));
                s[f][1] = __ffma2_rn(s[f][1], al, __fmul2_rn(bk, d1));
            }
            if (!COMMIT && rg == j % RG) {         // the output of token j, one row group
                float2 W0 = make_float2(0.f, 0.f), W1 = W0;
#pragma unroll
                for (int r = 0; r < RG; ++r) {
                    const float4 y = red_w[par][r][col4];
                    W0 = __fadd2_rn(W0, make_float2(y.x, y.y));
                    W1 = __fadd2_rn(W1, make_float2(y.z, y.w));
                }
                const int64_t off = ((b * D + t0 + j) * H + h) * DV + 4 * col4;
                const float bkq = skq[j];
                const float4 zg = *reinterpret_cast<const float4 *>(&sz[COMMIT ? 0 : j][4 * col4]);
                st(o, off + 0, p.scale * fmaf(bkq, d0.x, W0.x) * zg.x);
                st(o, off + 1, p.scale * fmaf(bkq, d0.y, W0.y) * zg.y);
                st(o, off + 2, p.scale * fmaf(bkq, d1.x, W1.x) * zg.z);
                st(o, off + 3, p.scale * fmaf(bkq, d1.y, W1.y) * zg.w);
            }
        }
    }

    if (COMMIT) {
#pragma unroll
        for (int f = 0; f < F; ++f)
            __stcs(&Sp[(rg * F + f) * C4 + col4],
                   make_float4(s[f][0].x, s[f][0].y, s[f][1].x, s[f][1].y));
    }
}

}  // namespace kda
