// kda_chunk_simt.cuh -- chunked KDA prefill on the CUDA cores in fp32,
// chunk length 16.  It is the fp32-I/O path (where tensor-core operand
// rounding would miss the fp32 bound) and the chunk-16 tiling of the bf16
// path.
//
// One CTA carries one (sequence, head) state through its chunks.  For a
// chunk of 16 tokens with G = inclusive cumulative max(g, floor) inside the
// chunk (the floor keeps exp(+-G) inside fp32 range over 16 tokens, the
// property the fupanwang.com Kimi K3 report digest, KDA section, Fig. 3,
// attributes to the decay lower bound):
//
//   A_qk[i,j] = sum_c q_ic k_jc e^{G_ic - G_jc}          (j <= i)
//   A_kk[i,j] = beta_i sum_c k_ic k_jc e^{G_ic - G_jc}   (j <  i)
//   T' = (I + A_kk)^-1 Diag(beta)
//   W  = T' (K * e^G),   U = T' V                       (WY / UT transform)
//   Vn = U - W S                                        (state-dependent part)
//   O  = scale ((Q * e^G) S + A_qk Vn)   [* sigmoid(z)]
//   S  = Diag(e^{G_last}) S + (K * e^{G_last - G})^T Vn
//
// This reproduces the token recurrence exactly in real arithmetic ("intra-
// chunk parallel, then cross-chunk state propagation": fupanwang.com digest,
// section 基础设施, FlashKDA).
//
// Thread layout: 2*DV threads; thread (v = tid % DV, half = tid / DV) keeps
// state rows [half*DK/2, (half+1)*DK/2) of value column v in registers.
#pragma once

#include "kda_common.cuh"

namespace kda {

constexpr int SC = 16;   // chunk length
constexpr int SP = 20;   // padded stride (floats) of the [channel][token] tiles

template <int DK, int DV>
struct SimtSmem {
    union {
        struct { float q[SC][DK]; float k[SC][DK]; } raw;   // loaded rows
        struct { float p[SC][DV]; float o[SC][DV]; } part;  // upper-half partials
    } u0;
    float g[SC][DK];
    float v[SC][DV];
    float U[SC][DV];          // U, then Vn in place
    float Qgt[DK][SP];        // q * e^G           [channel][token]
    float Kgt[DK][SP];        // k * e^G
    float Kinvt[DK][SP];      // k * e^-G
    float Khatt[DK][SP];      // k * e^{G_last - G}
    float Wt[DK][SP];         // W^T
    float gam[DK];            // e^{G_last}
    float Aqk[SC][SC + 1];
    float Akk[SC][SC + 1];
    float Tb[SC][SC + 1];     // T' = T Diag(beta)
    float beta[SC];
};

struct SimtParams {
    const void *q, *k, *v, *g, *beta, *gate;
    const float *S0;
    const int32_t *cu_seqlens;
    const int32_t *seq_order;   // sequences longest-first, or nullptr
    void *o;
    float *S_T;
    int32_t num_heads;
    float scale, g_floor;
    SnapOut snap;
    int64_t total_tokens;       // extents, for the debug build's unit checks
    int32_t num_seqs;
};

template <int DK, int DV, typename TIO>
__global__ void __launch_bounds__(2 * DV, 1) chunk_simt_kernel(SimtParams p)
{
    constexpr int NT = 2 * DV;
    constexpr int RH = DK / 2;
    extern __shared__ float4 smem_f4[];
    SimtSmem<DK, DV> &s = *reinterpret_cast<SimtSmem<DK, DV> *>(smem_f4);

    const TIO *q = static_cast<const TIO *>(p.q);
    const TIO *k = static_cast<const TIO *>(p.k);
    const TIO *v = static_cast<const TIO *>(p.v);
    const TIO *g = static_cast<const TIO *>(p.g);
    const TIO *beta = static_cast<const TIO *>(p.beta);
    const TIO *gate = static_cast<const TIO *>(p.gate);
    TIO *o = static_cast<TIO *>(p.o);

    const int tid = threadIdx.x;
    const int vcol = tid % DV;
    const int half = tid / DV;
    const int H = p.num_heads;
    const int n_slot = blockIdx.x / H;
    const int h = blockIdx.x % H;
    const int n = p.seq_order ? p.seq_order[n_slot] : n_slot;
    if (kDebugChecks && (n < 0 || n >= p.num_seqs)) {   // (uniform over the CTA)
        if (tid == 0) raise_error(ERR_BOUNDS);
        return;
    }
    const int64_t t_begin = p.cu_seqlens[n];
    const int64_t t_end = p.cu_seqlens[n + 1];
    if (kDebugChecks && (t_begin < 0 || t_end < t_begin || t_end > p.total_tokens)) {
        if (tid == 0) raise_error(ERR_BOUNDS);
        return;
    }
    const int64_t unit = (int64_t)n * H + h;

    float S[RH];
#pragma unroll
    for (int r = 0; r < RH; ++r)
        S[r] = p.S0 ? p.S0[(unit * DK + half * RH + r) * DV + vcol] : 0.0f;

    for (int64_t c0 = t_begin; c0 < t_end; c0 += SC) {
        const int L = (int)(t_end - c0 < SC ? t_end - c0 : SC);
        // 1. rows of the chunk (zero rows past the end make padded tokens identity steps)
        for (int idx = tid; idx < SC * DK; idx += NT) {
            const int i = idx / DK, c = idx % DK;
            const bool ok = i < L;
            const int64_t off = ((c0 + i) * H + h) * DK + c;
            s.u0.raw.q[i][c] = ok ? ld(q, off) : 0.0f;
            s.u0.raw.k[i][c] = ok ? ld(k, off) : 0.0f;
            s.g[i][c] = ok ? fmaxf(ld(g, off), p.g_floor) : 0.0f;
        }
        for (int idx = tid; idx < SC * DV; idx += NT) {
            const int i = idx / DV, c = idx % DV;
            s.v[i][c] = i < L ? ld(v, ((c0 + i) * H + h) * DV + c) : 0.0f;
        }
        if (tid < SC)
            s.beta[tid] = tid < L ? ld(beta, (c0 + tid) * H + h) : 0.0f;
        __syncthreads();

        // 2. per key channel: cumulative decay and the decayed operand tiles
        for (int c = tid; c < DK; c += NT) {
            float G[SC];
            float acc = 0.0f;
#pragma unroll
            for (int i = 0; i < SC; ++i) { acc += s.g[i][c]; G[i] = acc; }
            const float Gl = G[SC - 1];
#pragma unroll
            for (int i = 0; i < SC; ++i) {
                const float e = expf(G[i]);
                const float qq = s.u0.raw.q[i][c], kk = s.u0.raw.k[i][c];
                s.Qgt[c][i] = qq * e;
                s.Kgt[c][i] = kk * e;
                s.Kinvt[c][i] = kk * expf(-G[i]);
                s.Khatt[c][i] = kk * expf(Gl - G[i]);
            }
            s.gam[c] = expf(Gl);
        }
        __syncthreads();

        // 3. the two intra-chunk matrices
        for (int idx = tid; idx < SC * SC; idx += NT) {
            const int i = idx / SC, j = idx % SC;
            float aq = 0.0f, ak = 0.0f;
            if (j <= i) {
                for (int c = 0; c < DK; ++c) {
                    const float kv = s.Kinvt[c][j];
                    aq = fmaf(s.Qgt[c][i], kv, aq);
                    ak = fmaf(s.Kgt[c][i], kv, ak);
                }
            }
            s.Aqk[i][j] = j <= i ? aq : 0.0f;
            s.Akk[i][j] = j < i ? s.beta[i] * ak : 0.0f;
        }
        __syncthreads();

        // 4. T = (I + A_kk)^-1 by forward substitution, one column per thread
        if (tid < SC) {
            const int j = tid;
            float t[SC];
#pragma unroll
            for (int i = 0; i < SC; ++i) t[i] = (i == j) ? 1.0f : 0.0f;
#pragma unroll
            for (int i = 1; i < SC; ++i) {
                float acc = 0.0f;
#pragma unroll
                for (int m = 0; m < i; ++m) acc = fmaf(s.Akk[i][m], t[m], acc);
                if (i > j) t[i] = -acc;
            }
#pragma unroll
            for (int i = 0; i < SC; ++i) s.Tb[i][j] = t[i] * s.beta[j];
        }
        __syncthreads();

        // 5. W^T per key channel, U per value column
        for (int x = tid; x < DK + DV; x += NT) {
            if (x < DK) {
                float kg[SC];
#pragma unroll
                for (int j = 0; j < SC; ++j) kg[j] = s.Kgt[x][j];
#pragma unroll
                for (int i = 0; i < SC; ++i) {
                    float acc = 0.0f;
#pragma unroll
                    for (int j = 0; j <= i; ++j) acc = fmaf(s.Tb[i][j], kg[j], acc);
                    s.Wt[x][i] = acc;
                }
            } else {
                const int c = x - DK;
                float vv[SC];
#pragma unroll
                for (int j = 0; j < SC; ++j) vv[j] = s.v[j][c];
#pragma unroll
                for (int i = 0; i < SC; ++i) {
                    float acc = 0.0f;
#pragma unroll
                    for (int j = 0; j <= i; ++j) acc = fmaf(s.Tb[i][j], vv[j], acc);
                    s.U[i][c] = acc;
                }
            }
        }
        __syncthreads();

        // 6. W S and (Q e^G) S over this thread's half of the key channels
        float pp[SC], po[SC];
#pragma unroll
        for (int i = 0; i < SC; ++i) { pp[i] = 0.0f; po[i] = 0.0f; }
#pragma unroll
        for (int r = 0; r < RH; ++r) {
            const int c = half * RH + r;
            const float sv = S[r];
            const float4 *w4 = reinterpret_cast<const float4 *>(&s.Wt[c][0]);
            const float4 *q4 = reinterpret_cast<const float4 *>(&s.Qgt[c][0]);
#pragma unroll
            for (int b = 0; b < SC / 4; ++b) {
                const float4 w = w4[b], qg = q4[b];
                pp[4 * b + 0] = fmaf(w.x, sv, pp[4 * b + 0]);
                pp[4 * b + 1] = fmaf(w.y, sv, pp[4 * b + 1]);
                pp[4 * b + 2] = fmaf(w.z, sv, pp[4 * b + 2]);
                pp[4 * b + 3] = fmaf(w.w, sv, pp[4 * b + 3]);
                po[4 * b + 0] = fmaf(qg.x, sv, po[4 * b + 0]);
                po[4 * b + 1] = fmaf(qg.y, sv, po[4 * b + 1]);
                po[4 * b + 2] = fmaf(qg.z, sv, po[4 * b + 2]);
                po[4 * b + 3] = fmaf(qg.w, sv, po[4 * b + 3]);
            }
        }
        if (half == 1) {
#pragma unroll
            for (int i = 0; i < SC; ++i) { s.u0.part.p[i][vcol] = pp[i]; s.u0.part.o[i][vcol] = po[i]; }
        }
        __syncthreads();
        if (half == 0) {
#pragma unroll
            for (int i = 0; i < SC; ++i) {
                s.U[i][vcol] -= pp[i] + s.u0.part.p[i][vcol];   // Vn = U - W S
                po[i] += s.u0.part.o[i][vcol];
            }
        }
        __syncthreads();

        float vn[SC];
#pragma unroll
        for (int i = 0; i < SC; ++i) vn[i] = s.U[i][vcol];

        // 7. outputs of the chunk
        if (half == 0) {
#pragma unroll
            for (int i = 0; i < SC; ++i) {
                if (i < L) {
                    float acc = po[i];
#pragma unroll
                    for (int j = 0; j <= i; ++j) acc = fmaf(s.Aqk[i][j], vn[j], acc);
                    acc *= p.scale;
                    const int64_t off = ((c0 + i) * H + h) * DV + vcol;
                    if (gate) acc *= sigmoidf(ld(gate, off));
                    st(o, off, acc);
                }
            }
        }

        // 8. carry the state to the next chunk
#pragma unroll
        for (int r = 0; r < RH; ++r) {
            const int c = half * RH + r;
            float acc = s.gam[c] * S[r];
            const float4 *k4 = reinterpret_cast<const float4 *>(&s.Khatt[c][0]);
#pragma unroll
            for (int b = 0; b < SC / 4; ++b) {
                const float4 kh = k4[b];
                acc = fmaf(kh.x, vn[4 * b + 0], acc);
                acc = fmaf(kh.y, vn[4 * b + 1], acc);
                acc = fmaf(kh.z, vn[4 * b + 2], acc);
                acc = fmaf(kh.w, vn[4 * b + 3], acc);
            }
            S[r] = acc;
        }
        const int64_t slot = snap_slot(p.snap, n, c0 + L - t_begin);
        if (slot >= 0) {
#pragma unroll
            for (int r = 0; r < RH; ++r)
                p.snap.states[((slot * H + h) * DK + half * RH + r) * DV + vcol] = S[r];
        }
        __syncthreads();
    }

    if (p.S_T) {
#pragma unroll
        for (int r = 0; r < RH; ++r)
            p.S_T[(unit * DK + half * RH + r) * DV + vcol] = S[r];
    }
}

template <int DK, int DV>
constexpr size_t simt_smem_bytes() { return sizeof(SimtSmem<DK, DV>); }

}  // namespace kda
