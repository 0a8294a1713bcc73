// kda_bwd_chunk.cuh -- KDA backward in the chunked form (dk = dv = 128, bf16 I/O).
//
// The forward of one 64-token chunk with start state S0, in the chunk's frame
// (Kimi K3 report digest, section "KDA": per-channel decay with a floor,
// delta-rule write, sigmoid output gate):
//   lG_t = sum_{s<=t} max(g_s, floor),  lgam = lG_63
//   Qbar = q e^{lG}, Kbar = k e^{lG}, Khat = k e^{lgam - lG}
//   A_qk[i][j] = sum_c q_ic k_jc e^{lG_ic - lG_jc} (j <= i),  At the same with k_i (j < i)
//   T = (I + Diag(beta) At)^-1,  Z = V - Kbar S0,  nu = T Diag(beta) Z
//   Oraw = scale (Qbar S0 + A_qk nu),  o = Oraw sigmoid(z),  S_C = e^{lgam} S0 + Khat^T nu
// Every pair factor e^{lG_i - lG_j} (i >= j) is a_i m[b(i)][b(j)] bf_j over
// 16-token blocks (a = e^{lG - r_b}, bf = 1 / a, m = e^{r_bi - r_bj}, r_b the
// sum up to block b), so no factor leaves fp32's range for |floor| <= 5.45.
//
// Reverse mode in three kernels (dS_C: gradient of the chunk's end state):
//   chain_prep  (a CTA per chunk x head): the chain's per-chunk constants
//       Et = Diag(beta) T^T (scale A_qk^T go),  Wt = Diag(beta) T^T Khat,
//       F = scale Qbar^T go,  Kbar,  e^{lgam},  with go = do sigmoid(z);
//       and Z, nu, T, At, A_qk for the last kernel, dz of the output gate.
//   chain       (two CTAs per sequence x head, 64 value columns each; chunks last first):
//       dZ = Et + Wt dS_C,  dS0 = F + e^{lgam} dS_C - Kbar^T dZ  (dS_C of every chunk kept).
//   chain_grad  (a CTA per chunk x head): with dS_C,
//       dnu = scale A_qk^T go + Khat dS_C,  dY = T^T dnu,  dv = Diag(beta) dY,
//       dT = dnu (Diag(beta) Z)^T,  dA_kk = -T^T dT T^T (j < i),  dA_qk = scale go nu^T (j <= i),
//       dq  = a (e^{r} scale go S0^T + sum_j dA_qk m bf k_j),
//       dk1 = a (-e^{r} Diag(beta) dY S0^T + sum_j Diag(beta) dA_kk m bf k_j),
//       dk2 = bf (sum_i dA_qk m a q_i + sum_i Diag(beta) dA_kk m a k_i + e^{lgam - r} nu dS_C^T),
//       dk = dk1 + dk2,  dg_s = [g_s >= floor] (sum_{t>=s} (q dq + k (dk1 - dk2))_t + dlgam),
//       dlgam = e^{lgam} rowsum(dS_C o S0) + sum_t k_t dkh_t, dkh the Khat part of dk2
//       (the same rounded terms as in dk2, so the two sides of the cancellation
//       inside sum_t match; S_C from a forward's snapshot would not),
//       dbeta = rowsum(dY o Z) + rowsum(dA_kk o At).
// Every product runs on the warp-level tensor cores in tf32 with fp32
// accumulation; the four products (dq, dk1, dk2 and its Khat part) whose
// outputs hold the two sides of the pair terms that cancel inside dg's sum
// over the chunk run in 3xTF32 (leading and low parts), so that they cancel
// to fp32 accuracy.  SPLIT puts every other product in 3xTF32 as well.
#pragma once

#include <type_traits>

#include "kda_common.cuh"

namespace kda {
namespace bwdc {

constexpr int C = 64;           // chunk
constexpr int D = 128;          // dk = dv
constexpr int NB = 4;           // 16-token blocks per chunk
constexpr int NT = 512, NW = NT / 32;
constexpr int CD = C * D, CC = C * C, DD = D * D;

// per (chunk, head) scratch, floats
struct Scratch {
    static constexpr int64_t ET = 0, WT = ET + CD, KBAR = WT + CD, Z = KBAR + CD, NU = Z + CD,
                             DY = NU + CD, F = DY + CD, DSC = F + DD, T = DSC + DD, AT = T + CC,
                             AQK = AT + CC, GAM = AQK + CC, FLOATS = GAM + D;
};

struct ChunkBwdParams {
    const void *q, *k, *v, *g, *beta, *gate, *dout;   // I/O dtype
    const float *S0, *dS_T;                           // [N][H][D][D] or null
    const int32_t *cu_seqlens;                        // [N + 1]
    const float *ckpt;                                // state after 64 m tokens: slot ckpt_base[n] + m - 1
    const int64_t *ckpt_base;                         // [N + 1]
    const int32_t *chunk_seq, *chunk_idx;             // [chunks]: sequence, index in it
    const int64_t *chunk_base;                        // [N + 1]: first chunk of sequence n
    float *scratch;                                   // [chunks * H][Scratch::FLOATS]
    void *dq, *dk, *dv, *dg, *dbeta, *dgate;
    float *dS0;
    int32_t num_heads;
    float scale, g_floor;
    int64_t total_tokens;                             // for the debug build's unit checks
    int32_t num_seqs;                                 // (the same)
};

// XOR-swizzled element offsets of row-major fp32 tiles (128 or 64 columns):
// groups of 4 columns move with the row's low 3 bits, so the fragment loads
// below (8 rows x 4 columns, or 4 rows x 8 columns) touch distinct banks, or
// two-way at most, without padding.
__device__ __forceinline__ int xd(int r, int c) { return r * D + (c ^ ((r & 7) << 2)); }
__device__ __forceinline__ int xc(int r, int c) { return r * C + (c ^ ((r & 7) << 2)); }

__device__ __forceinline__ uint32_t tf32_rna(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// D[16x8] += A[16x8] B[8x8], tf32 inputs, fp32 accumulation; g = lane / 4, t = lane % 4:
//   a = {A[g][t], A[g+8][t], A[g][t+4], A[g+8][t+4]},  b = {B[t][g], B[t+4][g]},
//   d = {D[g][2t], D[g][2t+1], D[g+8][2t], D[g+8][2t+1]}.
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
                 "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// out[M x N] = sum_k A(i, k) B(k, j): warp tiles of 16 rows x 8 NT8 columns,
// dealt round-robin to warps w0 .. w0 + nw - 1.  krange(i0, j0, lo, hi) gives
// the tile's contraction range (multiples of 8); fa(i, k) and fb(i0, k, j) the
// operands (fb sees the tile's first row, for factors that depend on the output
// row block); epi(i, j, x) receives every result.  SPLIT: 3xTF32.
template <int M, int N, int NT8, bool SPLIT, class FK, class FA, class FB, class FE>
__device__ __forceinline__ void gemm(int warp, int w0, int nw, int lane, FK krange, FA fa, FB fb, FE epi) {
    static_assert(M % 16 == 0 && N % (8 * NT8) == 0, "tile shape");
    constexpr int TN = N / (8 * NT8), TILES = (M / 16) * TN;
    if (warp < w0 || warp >= w0 + nw) return;
    const int g = lane >> 2, t = lane & 3;
    for (int tile = warp - w0; tile < TILES; tile += nw) {
        const int i0 = (tile / TN) * 16, j0 = (tile % TN) * (8 * NT8);
        float acc[NT8][4];
#pragma unroll
        for (int n = 0; n < NT8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.0f;
        int lo, hi;
        krange(i0, j0, lo, hi);
        // fragments of the next k-step are read while the current one's MMAs issue
        float av[4], bv[NT8][2];
        auto fetch = [&](int k0) {
            av[0] = fa(i0 + g, k0 + t); av[1] = fa(i0 + g + 8, k0 + t);
            av[2] = fa(i0 + g, k0 + t + 4); av[3] = fa(i0 + g + 8, k0 + t + 4);
#pragma unroll
            for (int n = 0; n < NT8; ++n) {
                bv[n][0] = fb(i0, k0 + t, j0 + 8 * n + g);
                bv[n][1] = fb(i0, k0 + t + 4, j0 + 8 * n + g);
            }
        };
        if (lo < hi) fetch(lo);
#pragma unroll 1
        for (int k0 = lo; k0 < hi; k0 += 8) {
            uint32_t ah[4], al[4], bh[NT8][2], bl[NT8][2];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                ah[e] = tf32_rna(av[e]);
                if constexpr (SPLIT) al[e] = tf32_rna(av[e] - __uint_as_float(ah[e]));
            }
#pragma unroll
            for (int n = 0; n < NT8; ++n)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    bh[n][e] = tf32_rna(bv[n][e]);
                    if constexpr (SPLIT) bl[n][e] = tf32_rna(bv[n][e] - __uint_as_float(bh[n][e]));
                }
            if (k0 + 8 < hi) fetch(k0 + 8);
#pragma unroll
            for (int n = 0; n < NT8; ++n) {
                mma_tf32(acc[n], ah, bh[n][0], bh[n][1]);
                if constexpr (SPLIT) {
                    mma_tf32(acc[n], ah, bl[n][0], bl[n][1]);
                    mma_tf32(acc[n], al, bh[n][0], bh[n][1]);
                }
            }
        }
#pragma unroll
        for (int n = 0; n < NT8; ++n) {
            const int j = j0 + 8 * n + 2 * t;
            epi(i0 + g, j, acc[n][0]);
            epi(i0 + g, j + 1, acc[n][1]);
            epi(i0 + g + 8, j, acc[n][2]);
            epi(i0 + g + 8, j + 1, acc[n][3]);
        }
    }
}

// The chunk a CTA works on, and where its tokens are.
struct ChunkRef {
    int64_t u;          // chunk * H + head: scratch index
    int64_t n, h, ci;   // sequence, head, chunk index in the sequence
    int64_t tok0;       // first token (packed row) of the chunk
    int Lc;             // tokens in the chunk
    int64_t L;          // tokens in the sequence
    bool ok;            // debug build: the chunk lies where the host said (else it is skipped)
};

__device__ __forceinline__ ChunkRef chunk_ref(const ChunkBwdParams &p) {
    ChunkRef r;
    const int64_t H = p.num_heads;
    const int64_t c = blockIdx.x / H;
    r.h = blockIdx.x % H;
    r.u = blockIdx.x;
    r.n = p.chunk_seq[c];
    r.ci = p.chunk_idx[c];
    r.ok = true;
    if (kDebugChecks && (r.n < 0 || r.n >= p.num_seqs || r.ci < 0)) {
        r.ok = false;
        r.n = 0;
        r.ci = 0;
    }
    const int64_t tb = p.cu_seqlens[r.n];
    r.L = (int64_t)p.cu_seqlens[r.n + 1] - tb;
    r.tok0 = tb + r.ci * C;
    const int64_t left = r.L - r.ci * C;
    r.Lc = (int)(left < C ? left : C);
    // debug build: the device cu_seqlens agree with the host's chunk table (uniform over the CTA)
    if (kDebugChecks && (tb < 0 || r.L < 0 || tb + r.L > p.total_tokens || left <= 0 ||
                         p.chunk_base[r.n] + r.ci >= p.chunk_base[r.n + 1] ||
                         (r.ci > 0 && p.ckpt_base[r.n] + r.ci > p.ckpt_base[r.n + 1])))
        r.ok = false;
    return r;
}

// the chunk's start state (null: zero)
__device__ __forceinline__ const float *start_state(const ChunkBwdParams &p, const ChunkRef &r) {
    const int64_t H = p.num_heads;
    if (r.ci == 0) return p.S0 ? p.S0 + (r.n * H + r.h) * DD : nullptr;
    return p.ckpt + ((p.ckpt_base[r.n] + r.ci - 1) * H + r.h) * DD;
}

// Decay tables of a chunk from gc = max(g, floor) (zero past the chunk's end,
// swizzled [C][D] at gc): a = e^{lG - r_b} into `a_out` (may alias gc), and
// m[bi][bj] = e^{r_bi - r_bj} (bi >= bj, else 0), eR[b] = e^{r_b},
// eG[b] = e^{lgam - r_b}, gam = e^{lgam}.  Every exponent is a sum of at most
// 16 terms or of block totals, never a difference of long running sums.
// Thread (b, c) = (tid / D, tid % D) runs block b of channel c; the block
// totals meet in eG's rows.  Every thread of the CTA calls it (block barriers).
__device__ __forceinline__ void decay_tables(int tid, float *gc, float *a_out, float *m, float *eR,
                                             float *eG, float *gam) {
    static_assert(NT == NB * D, "one thread per (block, channel)");
    const int c = tid % D, b = tid / D;
    float x = 0.0f;
#pragma unroll
    for (int t = 16 * b; t < 16 * b + 16; ++t) {
        x += gc[xd(t, c)];
        a_out[xd(t, c)] = expf(x);
    }
    eG[b * D + c] = x;                   // block total, for a moment
    __syncthreads();
    float tot[NB];
#pragma unroll
    for (int bb = 0; bb < NB; ++bb) tot[bb] = eG[bb * D + c];
    __syncthreads();
    float r = 0.0f, rest = 0.0f;
#pragma unroll
    for (int bb = 0; bb < NB; ++bb) {
        if (bb < b) r += tot[bb];
        else rest += tot[bb];
    }
    eR[b * D + c] = expf(r);
    eG[b * D + c] = expf(rest);
#pragma unroll
    for (int bj = 0; bj < NB; ++bj) {
        float y = 0.0f;
#pragma unroll
        for (int bb = 0; bb < NB; ++bb)
            if (bb >= bj && bb < b) y += tot[bb];
        m[(b * NB + bj) * D + c] = bj <= b ? expf(y) : 0.0f;
    }
    if (b == 0) gam[c] = expf((tot[0] + tot[1]) + (tot[2] + tot[3]));
}

// T = (I + Diag(beta) At)^-1 (unit lower triangular, 64 x 64, swizzled [C][C]
// at Tm) from At (swizzled, at At) and beta: 16 x 16 diagonal blocks by forward
// substitution, then the merges [[T11, 0], [T21, T22]], T21 = -T22 (A21 T11),
// for 16 -> 32 and 32 -> 64.  xs: 2 x 16 x 16 + 32 x 32 floats of scratch.
// Every thread of the CTA calls it (it holds block barriers).
template <bool SPLIT>
__device__ void invert_T(int tid, int warp, int lane, const float *At, const float *beta, float *Tm, float *xs) {
    for (int i = tid; i < CC; i += NT) Tm[i] = 0.0f;
    __syncthreads();
    if (warp < 2) {
        const int d0 = 32 * warp + 16 * (lane >> 4), jj = lane & 15;
        float t[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) t[i] = i == jj ? 1.0f : 0.0f;
#pragma unroll
        for (int i = 1; i < 16; ++i) {
            const float b = beta[d0 + i];
            float acc = 0.0f;
#pragma unroll
            for (int m = 0; m < 15; ++m)
                if (m < i) acc = fmaf(b * At[xc(d0 + i, d0 + m)], t[m], acc);
            if (i > jj) t[i] = -acc;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) Tm[xc(d0 + i, d0 + jj)] = t[i];
    }
    __syncthreads();
    // 16 -> 32, pair p on warp p: X = A21 T11, T21 = -T22 X
    if (warp < 2) {
        const int p = warp, o = 32 * p;
        float *X = xs + p * 256;           // [16][16]
        auto kr = [](int, int, int &lo, int &hi) { lo = 0; hi = 16; };
        gemm<16, 16, 2, SPLIT>(warp, p, 1, lane, kr,
            [&](int i, int m) { return beta[o + 16 + i] * At[xc(o + 16 + i, o + m)]; },
            [&](int, int m, int j) { return Tm[xc(o + m, o + j)]; },
            [&](int i, int j, float x) { X[i * 16 + j] = x; });
        __syncwarp();
        gemm<16, 16, 2, SPLIT>(warp, p, 1, lane, kr,
            [&](int i, int m) { return Tm[xc(o + 16 + i, o + 16 + m)]; },
            [&](int, int m, int j) { return X[m * 16 + j]; },
            [&](int i, int j, float x) { Tm[xc(o + 16 + i, o + j)] = -x; });
    }
    __syncthreads();
    // 32 -> 64: X = A[32:64, 0:32] T[0:32, 0:32], T[32:64, 0:32] = -T[32:64, 32:64] X
    {
        float *X = xs + 512;               // [32][32]
        auto kr = [](int, int, int &lo, int &hi) { lo = 0; hi = 32; };
        gemm<32, 32, 4, SPLIT>(warp, 0, NW, lane, kr,
            [&](int i, int m) { return beta[32 + i] * At[xc(32 + i, m)]; },
            [&](int, int m, int j) { return Tm[xc(m, j)]; },
            [&](int i, int j, float x) { X[i * 32 + j] = x; });
        __syncthreads();
        gemm<32, 32, 4, SPLIT>(warp, 0, NW, lane, kr,
            [&](int i, int m) { return Tm[xc(32 + i, 32 + m)]; },
            [&](int, int m, int j) { return X[m * 32 + j]; },
            [&](int i, int j, float x) { Tm[xc(32 + i, j)] = -x; });
    }
    __syncthreads();
}

// shared memory of chain_prep: 3 [C][D] tiles, 3 [C][C] tiles, tables, and
// last kb's [C][D] tile with a second one after it: once kb is spent the two
// hold S0 [D][D] in the same swizzle.
struct PrepSmem {
    static constexpr int B0 = 0, B1 = B0 + CD, B3 = B1 + CD;
    static constexpr int AQ = B3 + CD, AT = AQ + CC, TT = AT + CC;
    static constexpr int M = TT + CC, ER = M + NB * NB * D, EG = ER + NB * D, GM = EG + NB * D;
    static constexpr int BT = GM + D, B2 = BT + C, FLOATS = B2 + DD;
    static constexpr size_t BYTES = (size_t)FLOATS * sizeof(float);
    static_assert(B2 % 4 == 0, "S0 is staged in 16-byte pieces");
    static_assert(BYTES <= 232448, "fits in 227 KB");
};

// Loads of data that no thread writes during the launch (inputs, and what
// earlier launches left in the scratch): the read-only path, which also lets
// the compiler issue them ahead of the stores that follow.
__device__ __forceinline__ float ldn(const float *p) { return __ldg(p); }
__device__ __forceinline__ float ldn(const __nv_bfloat16 *p) { return __bfloat162float(__ldg(p)); }
__device__ __forceinline__ float4 ldn4(const float *p) { return __ldg(reinterpret_cast<const float4 *>(p)); }

// A [C][D] bf16 tile of the chunk (rows past its end zero) as 16-byte pieces:
// thread tid holds pieces tid and tid + NT (row = piece / 16, 8 channels from
// (piece % 16) * 8).  The rows of a token are D = 128 bf16 = 256 bytes apart
// within a head, and the host sends only 16-byte aligned tensors here.
struct Tile8 {
    uint4 v[2];
};
__device__ __forceinline__ Tile8 load_tile8(const __nv_bfloat16 *base, const ChunkRef &r, int64_t H, int tid) {
    Tile8 x;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int piece = tid + u * NT, t = piece >> 4, c8 = (piece & 15) * 8;
        x.v[u] = t < r.Lc ? __ldg(reinterpret_cast<const uint4 *>(base + ((r.tok0 + t) * H + r.h) * D + c8))
                          : make_uint4(0u, 0u, 0u, 0u);
    }
    return x;
}
__device__ __forceinline__ void unpack8(uint4 w, float (&f)[8]) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        f[2 * e] = __uint_as_float(u[e] << 16);
        f[2 * e + 1] = __uint_as_float(u[e] & 0xFFFF0000u);
    }
}
// 8 floats at (t, c8) of a swizzled [C][D] tile: two 4-float groups
__device__ __forceinline__ void put8(float *tile, int t, int c8, const float (&f)[8]) {
    *reinterpret_cast<float4 *>(tile + xd(t, c8)) = make_float4(f[0], f[1], f[2], f[3]);
    *reinterpret_cast<float4 *>(tile + xd(t, c8 + 4)) = make_float4(f[4], f[5], f[6], f[7]);
}

// Stage the chunk's q, k (bf16 -> fp32) and gc = max(g, floor), zero past its end;
// with `mask`, bit c % 32 of mask[t * 4 + c / 32] = [g_tc >= floor].
__device__ __forceinline__ void stage_qkg(const ChunkBwdParams &p, const ChunkRef &r, int tid, float *sq,
                                          float *sk, float *sg, float *sb, uint32_t *mask) {
    const int64_t H = p.num_heads;
    const Tile8 tq = load_tile8(static_cast<const __nv_bfloat16 *>(p.q), r, H, tid);
    const Tile8 tk = load_tile8(static_cast<const __nv_bfloat16 *>(p.k), r, H, tid);
    const Tile8 tg = load_tile8(static_cast<const __nv_bfloat16 *>(p.g), r, H, tid);
    const float bt = tid < r.Lc ? ldn(static_cast<const __nv_bfloat16 *>(p.beta) + (r.tok0 + tid) * H + r.h) : 0.0f;
    if (mask && tid < C * D / 32) mask[tid] = 0u;
    if (mask) __syncthreads();
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int piece = tid + u * NT, t = piece >> 4, c8 = (piece & 15) * 8;
        float f[8];
        unpack8(tq.v[u], f);
        put8(sq, t, c8, f);
        unpack8(tk.v[u], f);
        put8(sk, t, c8, f);
        unpack8(tg.v[u], f);
        uint32_t bits = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (t < r.Lc && f[e] >= p.g_floor) bits |= 1u << e;
            f[e] = t < r.Lc ? fmaxf(f[e], p.g_floor) : 0.0f;
        }
        put8(sg, t, c8, f);
        if (mask) atomicOr(mask + t * (D / 32) + (c8 >> 5), bits << (c8 & 31));
    }
    if (tid < C) sb[tid] = bt;
}

template <typename TIO, bool SPLIT>
__global__ void __launch_bounds__(NT, 1) chain_prep_kernel(ChunkBwdParams p) {
    static_assert(std::is_same<TIO, __nv_bfloat16>::value, "the chunked backward reads bf16 in 16-byte pieces");
    using S = PrepSmem;
    extern __shared__ float4 bwdc_smem4[];
    float *sm = reinterpret_cast<float *>(bwdc_smem4);
    float *qa = sm + S::B0, *ka = sm + S::B1, *kb = sm + S::B2, *b3 = sm + S::B3;
    float *Aq = sm + S::AQ, *At = sm + S::AT, *Tm = sm + S::TT;
    float *m = sm + S::M, *eR = sm + S::ER, *eG = sm + S::EG, *gam = sm + S::GM, *sb = sm + S::BT;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const ChunkRef r = chunk_ref(p);
    if (kDebugChecks && !r.ok) {
        if (threadIdx.x == 0) raise_error(ERR_BOUNDS);
        return;
    }
    const int64_t H = p.num_heads;
    float *scr = p.scratch + r.u * Scratch::FLOATS;
    const float *S0p = start_state(p, r);
    const TIO *vin = static_cast<const TIO *>(p.v);
    const TIO *dout = static_cast<const TIO *>(p.dout);
    const TIO *gate = static_cast<const TIO *>(p.gate);
    const float scale = p.scale;

    // q -> qa, k -> ka (and kb), gc -> a (in b3)
    stage_qkg(p, r, tid, qa, ka, b3, sb, nullptr);
    __syncthreads();
    decay_tables(tid, b3, b3, m, eR, eG, gam);
    __syncthreads();
    for (int i = tid; i < CD; i += NT) {
        const int t = i / D, c = i % D, x = xd(t, c);
        const float a = b3[x], kv = ka[x];
        qa[x] *= a;
        ka[x] = kv * a;
        kb[x] = kv / a;
    }
    __syncthreads();

    // A_qk (warps 0-7) and At (warps 8-15): the pair factor's middle term rides on kb
    auto kr_tri = [](int i0, int j0, int &lo, int &hi) { lo = 0; hi = j0 > i0 + 15 ? 0 : D; };
    auto fb_mkb = [&](int i0, int c, int j) { return kb[xd(j, c)] * m[((i0 >> 4) * NB + (j >> 4)) * D + c]; };
    gemm<C, C, 4, SPLIT>(warp, 0, 8, lane, kr_tri, [&](int i, int c) { return qa[xd(i, c)]; }, fb_mkb,
                         [&](int i, int j, float x) { Aq[xc(i, j)] = j <= i ? x : 0.0f; });
    gemm<C, C, 4, SPLIT>(warp, 8, 8, lane, kr_tri, [&](int i, int c) { return ka[xd(i, c)]; }, fb_mkb,
                         [&](int i, int j, float x) { At[xc(i, j)] = j < i ? x : 0.0f; });
    __syncthreads();
    invert_T<SPLIT>(tid, warp, lane, At, sb, Tm, b3);   // b3 (a) is not needed any more

    // Wt = Diag(beta) T^T Khat (to scratch): kb's last use
    gemm<C, D, 4, SPLIT>(warp, 0, NW, lane, [](int i0, int, int &lo, int &hi) { lo = i0; hi = C; },
        [&](int i, int l) { return Tm[xc(l, i)]; },
        [&](int, int l, int c) { return kb[xd(l, c)] * eG[(l >> 4) * D + c]; },
        [&](int i, int c, float x) { scr[Scratch::WT + i * D + c] = sb[i] * x; });
    // S0 into kb's tile and the one after it, for the two products that read it
    constexpr int SU = DD / 4 / NT;
    float4 xs[SU];
    if (S0p) {
#pragma unroll
        for (int u = 0; u < SU; ++u) xs[u] = ldn4(S0p + 4 * (tid + u * NT));
    }
    __syncthreads();
    float *s0s = kb;
    if (S0p) {
#pragma unroll
        for (int u = 0; u < SU; ++u) {
            const int piece = tid + u * NT, row = piece / (D / 4), c4 = (piece % (D / 4)) * 4;
            *reinterpret_cast<float4 *>(s0s + xd(row, c4)) = xs[u];
        }
    }
    __syncthreads();

    // Z = V - Kbar S0 (into b3), Kbar and the small tiles to scratch
    gemm<C, D, 4, SPLIT>(warp, 0, NW, lane,
        [&](int, int, int &lo, int &hi) { lo = 0; hi = S0p ? D : 0; },
        [&](int i, int c) { return ka[xd(i, c)] * eR[(i >> 4) * D + c]; },
        [&](int, int c, int v) { return s0s[xd(c, v)]; },
        [&](int i, int v, float x) {
            const float vi = i < r.Lc ? ldn(vin + ((r.tok0 + i) * H + r.h) * D + v) : 0.0f;
            const float z = vi - x;
            b3[xd(i, v)] = z;
            scr[Scratch::Z + i * D + v] = z;
        });
    for (int i = tid; i < CD; i += NT) {
        const int t = i / D, c = i % D;
        scr[Scratch::KBAR + i] = ka[xd(t, c)] * eR[(t >> 4) * D + c];
    }
    for (int i = tid; i < CC; i += NT) {
        const int a = i / C, b = i % C;
        scr[Scratch::T + i] = Tm[xc(a, b)];
        scr[Scratch::AT + i] = At[xc(a, b)];
        scr[Scratch::AQK + i] = Aq[xc(a, b)];
    }
    if (tid < D) scr[Scratch::GAM + tid] = gam[tid];
    __syncthreads();
    // nu = T Diag(beta) Z (into ka)
    gemm<C, D, 4, SPLIT>(warp, 0, NW, lane,
        [&](int i0, int, int &lo, int &hi) { lo = 0; hi = i0 + 16; },
        [&](int i, int l) { return Tm[xc(i, l)]; },
        [&](int, int l, int v) { return sb[l] * b3[xd(l, v)]; },
        [&](int i, int v, float x) {
            ka[xd(i, v)] = x;
            scr[Scratch::NU + i * D + v] = x;
        });
    __syncthreads();
    // Oraw = scale (Qbar S0 + A_qk nu): dz of the gate, and go = do sigmoid(z) (into b3)
    float *nu = ka;
    gemm<C, D, 4, SPLIT>(warp, 0, NW, lane,
        [&](int i0, int, int &lo, int &hi) { lo = S0p ? 0 : D; hi = D + i0 + 16; },
        [&](int i, int k) { return k < D ? qa[xd(i, k)] * eR[(i >> 4) * D + k] : Aq[xc(i, k - D)]; },
        [&](int, int k, int v) { return k < D ? s0s[xd(k, v)] : nu[xd(k - D, v)]; },
        [&](int i, int v, float x) {
            float go = 0.0f;
            if (i < r.Lc) {
                const int64_t e = ((r.tok0 + i) * H + r.h) * D + v;
                const float dov = ldn(dout + e);
                if (gate) {
                    const float sg = sigmoidf(ldn(gate + e));
                    st(static_cast<TIO *>(p.dgate), e, dov * scale * x * sg * (1.0f - sg));
                    go = dov * sg;
                } else {
                    go = dov;
                }
            }
            b3[xd(i, v)] = go;
        });
    __syncthreads();
    // F = scale Qbar^T go (to scratch), E = scale A_qk^T go (into nu's tile)
    gemm<D, D, 4, SPLIT>(warp, 0, NW, lane, [](int, int, int &lo, int &hi) { lo = 0; hi = C; },
        [&](int c, int i) { return qa[xd(i, c)] * eR[(i >> 4) * D + c]; },
        [&](int, int i, int v) { return b3[xd(i, v)]; },
        [&](int c, int v, float x) { scr[Scratch::F + c * D + v] = scale * x; });
    float *E = ka;
    gemm<C, D, 4, SPLIT>(warp, 0, NW, lane, [](int i0, int, int &lo, int &hi) { lo = i0; hi = C; },
        [&](int j, int i) { return Aq[xc(i, j)]; },
        [&](int, int i, int v) { return b3[xd(i, v)]; },
        [&](int j, int v, float x) { E[xd(j, v)] = scale * x; });
    __syncthreads();
    // Et = Diag(beta) T^T E (to scratch)
    gemm<C, D, 4, SPLIT>(warp, 0, NW, lane, [](int i0, int, int &lo, int &hi) { lo = i0; hi = C; },
        [&](int i, int l) { return Tm[xc(l, i)]; },
        [&](int, int l, int v) { return E[xd(l, v)]; },
        [&](int i, int v, float x) { scr[Scratch::ET + i * D + v] = sb[i] * x; });
}

// The chain: a CTA per (sequence, head, half of the value columns).  dS's
// columns do not mix (dZ = Et + Wt dS_C and dS0 = F + e^{lgam} dS_C - Kbar^T dZ
// act on every column alike), so two CTAs of 256 threads take 64 columns each,
// two per SM.  Shared memory: dS [D][64], dZ [C][64], Wt and Kbar [C][D], e^{lgam}.
constexpr int CHAIN_NT = 256, CHAIN_NW = CHAIN_NT / 32, DVH = D / 2;
struct ChainSmem {
    static constexpr int DS = 0, DZ = DS + D * DVH, WT = DZ + C * DVH, KB = WT + CD, GM = KB + CD;
    static constexpr int FLOATS = GM + D;
    static constexpr size_t BYTES = (size_t)FLOATS * sizeof(float);
    // two CTAs per SM: 228 KB per SM, 1 KB of it reserved per CTA
    static_assert(2 * (BYTES + 1024) <= 233472, "two CTAs fit on an SM");
};
// swizzled offsets of a row-major tile with 64 columns (as xc)
__device__ __forceinline__ int xh(int r, int c) { return xc(r, c); }

template <bool SPLIT>
__global__ void __launch_bounds__(CHAIN_NT, 2) chain_kernel(ChunkBwdParams p) {
    using S = ChainSmem;
    constexpr int NTC = CHAIN_NT;
    extern __shared__ float4 bwdc_smem4[];
    float *sm = reinterpret_cast<float *>(bwdc_smem4);
    float *dS = sm + S::DS, *dZ = sm + S::DZ, *Wt = sm + S::WT, *Kb = sm + S::KB, *gam = sm + S::GM;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t H = p.num_heads, unit = blockIdx.x >> 1, n = unit / H, h = unit % H;
    const int v0 = (blockIdx.x & 1) * DVH;
    const int64_t L = (int64_t)p.cu_seqlens[n + 1] - p.cu_seqlens[n];
    const int64_t nch = (L + C - 1) / C;
    // debug build: the device cu_seqlens agree with the host's chunk table (uniform over the CTA)
    if (kDebugChecks && (p.cu_seqlens[n] < 0 || L < 0 || p.cu_seqlens[n] + L > p.total_tokens ||
                         p.chunk_base[n] + nch != p.chunk_base[n + 1])) {
        if (tid == 0) raise_error(ERR_BOUNDS);
        return;
    }
    const float *dST = p.dS_T ? p.dS_T + (n * H + h) * DD : nullptr;
    for (int i = tid; i < D * DVH / 4; i += NTC) {        // float4 pieces of this half
        const int c = i / (DVH / 4), v = (i % (DVH / 4)) * 4;
        *reinterpret_cast<float4 *>(dS + xh(c, v)) = dST ? ldn4(dST + c * D + v0 + v) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int64_t ci = nch - 1; ci >= 0; --ci) {
        float *scr = p.scratch + ((p.chunk_base[n] + ci) * H + h) * Scratch::FLOATS;
        float *dsc = scr + Scratch::DSC;
        __syncthreads();
        {
            float4 xw[CD / 4 / NTC], xk[CD / 4 / NTC];
#pragma unroll
            for (int u = 0; u < CD / 4 / NTC; ++u) {
                xw[u] = ldn4(scr + Scratch::WT + 4 * (tid + u * NTC));
                xk[u] = ldn4(scr + Scratch::KBAR + 4 * (tid + u * NTC));
            }
            for (int i = tid; i < D * DVH / 4; i += NTC) {
                const int c = i / (DVH / 4), v = (i % (DVH / 4)) * 4;
                *reinterpret_cast<float4 *>(dsc + c * D + v0 + v) = *reinterpret_cast<const float4 *>(dS + xh(c, v));
            }
#pragma unroll
            for (int u = 0; u < CD / 4 / NTC; ++u) {
                const int i = 4 * (tid + u * NTC);
                *reinterpret_cast<float4 *>(Wt + xd(i / D, i % D)) = xw[u];
                *reinterpret_cast<float4 *>(Kb + xd(i / D, i % D)) = xk[u];
            }
            if (tid < D) gam[tid] = ldn(scr + Scratch::GAM + tid);
        }
        __syncthreads();
        // dZ = Et + Wt dS (this half's columns)
        gemm<C, DVH, 4, SPLIT>(warp, 0, CHAIN_NW, lane, [](int, int, int &lo, int &hi) { lo = 0; hi = D; },
            [&](int j, int c) { return Wt[xd(j, c)]; },
            [&](int, int c, int v) { return dS[xh(c, v)]; },
            [&](int j, int v, float x) { dZ[xh(j, v)] = ldn(scr + Scratch::ET + j * D + v0 + v) + x; });
        __syncthreads();
        // dS <- F + e^{lgam} dS - Kbar^T dZ (each element read and written by its own thread)
        gemm<D, DVH, 4, SPLIT>(warp, 0, CHAIN_NW, lane, [](int, int, int &lo, int &hi) { lo = 0; hi = C; },
            [&](int c, int j) { return Kb[xd(j, c)]; },
            [&](int, int j, int v) { return dZ[xh(j, v)]; },
            [&](int c, int v, float x) {
                const int e = xh(c, v);
                dS[e] = ldn(scr + Scratch::F + c * D + v0 + v) + gam[c] * dS[e] - x;
            });
    }
    __syncthreads();
    if (p.dS0) {
        float *out = p.dS0 + (n * H + h) * DD;
        for (int i = tid; i < D * DVH / 4; i += NTC) {
            const int c = i / (DVH / 4), v = (i % (DVH / 4)) * 4;
            *reinterpret_cast<float4 *>(out + c * D + v0 + v) = *reinterpret_cast<const float4 *>(dS + xh(c, v));
        }
    }
}

// shared memory of chain_grad: 5 [C][D] tiles, 3 [C][C] tiles, tables
struct GradSmem {
    static constexpr int B0 = 0, B1 = B0 + CD, B2 = B1 + CD, B3 = B2 + CD, B4 = B3 + CD;
    static constexpr int TT = B4 + CD, S1 = TT + CC, S2 = S1 + CC;
    static constexpr int M = S2 + CC, ER = M + NB * NB * D, EG = ER + NB * D, GM = EG + NB * D;
    static constexpr int BT = GM + D, DL = BT + C, MK = DL + D, FLOATS = MK + C * D / 32;
    static constexpr size_t BYTES = (size_t)FLOATS * sizeof(float);
    static_assert(BYTES <= 232448, "fits in 227 KB");
};

template <typename TIO, bool SPLIT>
__global__ void __launch_bounds__(NT, 1) chain_grad_kernel(ChunkBwdParams p) {
    static_assert(std::is_same<TIO, __nv_bfloat16>::value, "the chunked backward reads bf16 in 16-byte pieces");
    using S = GradSmem;
    extern __shared__ float4 bwdc_smem4[];
    float *sm = reinterpret_cast<float *>(bwdc_smem4);
    float *qa = sm + S::B0, *kb = sm + S::B1, *aa = sm + S::B2, *b3 = sm + S::B3, *b4 = sm + S::B4;
    float *Tm = sm + S::TT, *s1 = sm + S::S1, *s2 = sm + S::S2;
    float *m = sm + S::M, *eR = sm + S::ER, *eG = sm + S::EG, *gam = sm + S::GM, *sb = sm + S::BT;
    float *sdl = sm + S::DL;
    uint32_t *gmask = reinterpret_cast<uint32_t *>(sm + S::MK);   // [g >= floor] bits, [C][D / 32]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const ChunkRef r = chunk_ref(p);
    if (kDebugChecks && !r.ok) {
        if (threadIdx.x == 0) raise_error(ERR_BOUNDS);
        return;
    }
    const int64_t H = p.num_heads;
    float *scr = p.scratch + r.u * Scratch::FLOATS;
    const float *S0p = start_state(p, r);
    const float *dSC = scr + Scratch::DSC;
    const TIO *qin = static_cast<const TIO *>(p.q);
    const TIO *kin = static_cast<const TIO *>(p.k);
    const TIO *gate = static_cast<const TIO *>(p.gate);
    const float scale = p.scale;
    auto row = [&](int i) { return ((r.tok0 + i) * H + r.h) * D; };

    // every load first: dout and the gate, T and A_qk, then q, k, g (staged); the
    // decay tables (a into aa); qa, kb, and go = dout sigmoid(z) into b3
    const Tile8 tdo = load_tile8(static_cast<const __nv_bfloat16 *>(p.dout), r, H, tid);
    Tile8 tz;
    if (gate) tz = load_tile8(static_cast<const __nv_bfloat16 *>(p.gate), r, H, tid);
    {
        float4 tt[2], ta[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            tt[u] = ldn4(scr + Scratch::T + 4 * (tid + u * NT));
            ta[u] = ldn4(scr + Scratch::AQK + 4 * (tid + u * NT));
        }
        stage_qkg(p, r, tid, qa, kb, b4, sb, gmask);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int i = 4 * (tid + u * NT), a = i / C, b = i % C;
            *reinterpret_cast<float4 *>(Tm + xc(a, b)) = tt[u];
            *reinterpret_cast<float4 *>(s2 + xc(a, b)) = ta[u];      // A_qk, for dnu
        }
    }
    __syncthreads();
    decay_tables(tid, b4, aa, m, eR, eG, gam);
    __syncthreads();
    for (int i = tid; i < CD; i += NT) {
        const int x = xd(i / D, i % D);
        const float a = aa[x];
        qa[x] *= a;
        kb[x] /= a;
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int piece = tid + u * NT, t = piece >> 4, c8 = (piece & 15) * 8;
        float f[8];
        unpack8(tdo.v[u], f);
        if (gate) {
            float z[8];
            unpack8(tz.v[u], z);
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] *= sigmoidf(z[e]);
        }
        put8(b3, t, c8, f);
    }
    __syncthreads();
    // dnu = scale A_qk^T go + Khat dS_C (into b4; A_qk staged in s2)
    gemm<C, D, 4, SPLIT>(warp, 0, NW, lane, [](int i0, int, int &lo, int &hi) { lo = i0; hi = C + D; },
        [&](int j, int k) { return k < C ? scale * s2[xc(k, j)] : kb[xd(j, k - C)] * eG[(j >> 4) * D + k - C]; },
        [&](int, int k, int v) { return k < C ? b3[xd(k, v)] : ldn(dSC + (k - C) * D + v); },
        [&](int j, int v, float x) { b4[xd(j, v)] = x; });
    __syncthreads();
    // dY = T^T dnu: dv = Diag(beta) dY, dY to scratch;  dT = dnu (Diag(beta) Z)^T (into s1)
    const float *Zg = scr + Scratch::Z;
    gemm<C, D, 4, SPLIT>(warp, 0, NW, lane, [](int i0, int, int &lo, int &hi) { lo = i0; hi = C; },
        [&](int i, int l) { return Tm[xc(l, i)]; },
        [&](int, int l, int v) { return b4[xd(l, v)]; },
        [&](int i, int v, float x) {
            scr[Scratch::DY + i * D + v] = x;
            if (i < r.Lc) st(static_cast<TIO *>(p.dv), row(i) + v, sb[i] * x);
        });
    gemm<C, C, 4, SPLIT>(warp, 0, NW, lane, [](int i0, int j0, int &lo, int &hi) { lo = 0; hi = j0 > i0 + 15 ? 0 : D; },
        [&](int i, int v) { return b4[xd(i, v)]; },
        [&](int, int v, int j) { return sb[j] * ldn(Zg + j * D + v); },
        [&](int i, int j, float x) { s1[xc(i, j)] = x; });
    __syncthreads();
    // nu (scratch) into b4 for dA_qk (dnu is done with), beside X
    const float *nug = scr + Scratch::NU;
    {
        float4 xn[CD / 4 / NT];
#pragma unroll
        for (int u = 0; u < CD / 4 / NT; ++u) xn[u] = ldn4(nug + 4 * (tid + u * NT));
#pragma unroll
        for (int u = 0; u < CD / 4 / NT; ++u) {
            const int i = 4 * (tid + u * NT);
            *reinterpret_cast<float4 *>(b4 + xd(i / D, i % D)) = xn[u];
        }
    }
    // X = dT T^T (into s2), then dA_kk = -T^T X, j < i (into s1)
    gemm<C, C, 4, SPLIT>(warp, 0, NW, lane, [](int, int, int &lo, int &hi) { lo = 0; hi = C; },
        [&](int i, int b) { return s1[xc(i, b)]; },
        [&](int, int b, int j) { return Tm[xc(j, b)]; },
        [&](int i, int j, float x) { s2[xc(i, j)] = x; });
    __syncthreads();
    gemm<C, C, 4, SPLIT>(warp, 0, NW, lane, [](int i0, int j0, int &lo, int &hi) { lo = i0; hi = j0 > i0 + 15 ? i0 : C; },
        [&](int i, int a) { return Tm[xc(a, i)]; },
        [&](int, int a, int j) { return s2[xc(a, j)]; },
        [&](int i, int j, float x) { s1[xc(i, j)] = j < i ? -x : 0.0f; });
    __syncthreads();
    // dA_qk = scale go nu^T, j <= i (into s2; nu staged in b4)
    gemm<C, C, 4, SPLIT>(warp, 0, NW, lane, [](int i0, int j0, int &lo, int &hi) { lo = 0; hi = j0 > i0 + 15 ? 0 : D; },
        [&](int i, int v) { return b3[xd(i, v)]; },
        [&](int, int v, int j) { return b4[xd(j, v)]; },
        [&](int i, int j, float x) { s2[xc(i, j)] = j <= i ? scale * x : 0.0f; });
    __syncthreads();
    // dbeta = rowsum(dY o Z) + rowsum(dA_kk o At): a warp per row
    {
        const float *dYg = scr + Scratch::DY, *Atg = scr + Scratch::AT;
        for (int i = warp; i < r.Lc; i += NW) {
            float s = 0.0f;
#pragma unroll
            for (int e = 0; e < D / 32; ++e) s = fmaf(dYg[i * D + lane + 32 * e], ldn(Zg + i * D + lane + 32 * e), s);
#pragma unroll
            for (int e = 0; e < C / 32; ++e) s = fmaf(s1[xc(i, lane + 32 * e)], ldn(Atg + i * C + lane + 32 * e), s);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (lane == 0) st(static_cast<TIO *>(p.dbeta), (r.tok0 + i) * H + r.h, s);
        }
    }
    // dq = a (e^r scale go S0^T + dA_qk m kb); q dq into b4 (dlG)
    auto kr_pair = [&](int i0, int, int &lo, int &hi) { lo = S0p ? 0 : D; hi = D + i0 + 16; };
    auto fb_pair = [&](int i0, int k, int c) {
        return k < D ? ldn(S0p + c * D + k) * eR[(i0 >> 4) * D + c]
                     : m[((i0 >> 4) * NB + ((k - D) >> 4)) * D + c] * kb[xd(k - D, c)];
    };
    gemm<C, D, 4, true>(warp, 0, NW, lane, kr_pair,
        [&](int i, int k) { return k < D ? scale * b3[xd(i, k)] : s2[xc(i, k - D)]; }, fb_pair,
        [&](int i, int c, float x) {
            const float dq = aa[xd(i, c)] * x;
            float ql = 0.0f;
            if (i < r.Lc) {
                st(static_cast<TIO *>(p.dq), row(i) + c, dq);
                ql = ldn(qin + row(i) + c);
            }
            b4[xd(i, c)] = ql * dq;
        });
    __syncthreads();
    // dk1 = a (-e^r Diag(beta) dY S0^T + Diag(beta) dA_kk m kb) (into b3); dlG += k dk1
    const float *dYg = scr + Scratch::DY;
    gemm<C, D, 4, true>(warp, 0, NW, lane, kr_pair,
        [&](int i, int k) { return k < D ? -sb[i] * dYg[i * D + k] : sb[i] * s1[xc(i, k - D)]; }, fb_pair,
        [&](int i, int c, float x) {
            const int e = xd(i, c);
            const float d1 = aa[e] * x;
            b3[e] = d1;
            if (i < r.Lc) b4[e] += ldn(kin + row(i) + c) * d1;
        });
    __syncthreads();
    // dk2 through Kbrev: bf (dA_qk^T m qa + (Diag(beta) dA_kk)^T m ka); b3 <- dk1 + that
    gemm<C, D, 4, true>(warp, 0, NW, lane, [](int, int, int &lo, int &hi) { lo = 0; hi = 2 * C; },
        [&](int j, int k) { return k < C ? s2[xc(k, j)] : sb[k - C] * s1[xc(k - C, j)]; },
        [&](int j0, int k, int c) {
            if (k < C) return m[((k >> 4) * NB + (j0 >> 4)) * D + c] * qa[xd(k, c)];
            const int i = k - C, e = xd(i, c);
            return m[((i >> 4) * NB + (j0 >> 4)) * D + c] * ((kb[e] * aa[e]) * aa[e]);   // k a
        },
        [&](int j, int c, float x) {
            const int e = xd(j, c);
            const float d2 = x / aa[e];
            b3[e] += d2;
            if (j < r.Lc) b4[e] -= ldn(kin + row(j) + c) * d2;
        });
    __syncthreads();
    // nu and dS_C into shared memory (qa, kb and the small tiles are done with): nu over
    // s1 | s2, dS_C over qa | kb
    float *snu = s1, *sds = qa;
    {
        float4 xn[CD / 4 / NT], xs[DD / 4 / NT];
#pragma unroll
        for (int u = 0; u < CD / 4 / NT; ++u) xn[u] = ldn4(nug + 4 * (tid + u * NT));
#pragma unroll
        for (int u = 0; u < DD / 4 / NT; ++u) xs[u] = ldn4(dSC + 4 * (tid + u * NT));
#pragma unroll
        for (int u = 0; u < CD / 4 / NT; ++u) {
            const int i = 4 * (tid + u * NT);
            *reinterpret_cast<float4 *>(snu + xd(i / D, i % D)) = xn[u];
        }
#pragma unroll
        for (int u = 0; u < DD / 4 / NT; ++u) {
            const int i = 4 * (tid + u * NT);
            *reinterpret_cast<float4 *>(sds + xd(i / D, i % D)) = xs[u];
        }
    }
    __syncthreads();
    // dkh = bf e^{lgam - r} nu dS_C^T (through Khat): dk = b3 + dkh; k dkh into b3 for dlgam
    gemm<C, D, 4, true>(warp, 0, NW, lane, [](int, int, int &lo, int &hi) { lo = 0; hi = D; },
        [&](int j, int v) { return snu[xd(j, v)]; },
        [&](int j0, int v, int c) { return sds[xd(c, v)] * eG[(j0 >> 4) * D + c]; },
        [&](int j, int c, float x) {
            const int e = xd(j, c);
            const float dh = x / aa[e];
            float kdh = 0.0f;
            if (j < r.Lc) {
                st(static_cast<TIO *>(p.dk), row(j) + c, b3[e] + dh);
                kdh = ldn(kin + row(j) + c) * dh;
                b4[e] -= kdh;
            }
            b3[e] = kdh;
        });
    // e^{lgam} rowsum(dS_C o S0): warp w the channels w + 16 n, a float4 of each row per lane
    {
        float rs[D / NW];
        if (S0p) {
            float4 xa[D / NW], xb[D / NW];
#pragma unroll
            for (int n = 0; n < D / NW; ++n) {
                xa[n] = ldn4(dSC + (warp + NW * n) * D + 4 * lane);
                xb[n] = ldn4(S0p + (warp + NW * n) * D + 4 * lane);
            }
#pragma unroll
            for (int n = 0; n < D / NW; ++n) {
                float s = xa[n].x * xb[n].x + xa[n].y * xb[n].y + xa[n].z * xb[n].z + xa[n].w * xb[n].w;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                rs[n] = s;
            }
        }
        if (lane == 0) {
#pragma unroll
            for (int n = 0; n < D / NW; ++n) sdl[warp + NW * n] = S0p ? gam[warp + NW * n] * rs[n] : 0.0f;
        }
    }
    __syncthreads();
    // dg_s = [g_s >= floor] (sum_{t >= s} dlG_t + dlgam), one channel per thread
    if (tid < D) {
        const int c = tid;
        float run = sdl[c];
        for (int t = 0; t < C; ++t) run += b3[xd(t, c)];      // + sum_t k_t dkh_t
        for (int t = C - 1; t >= 0; --t) {
            run += b4[xd(t, c)];
            if (t < r.Lc) {
                const int64_t e = row(t) + c;
                const bool pass = (gmask[t * (D / 32) + (c >> 5)] >> (c & 31)) & 1u;
                st(static_cast<TIO *>(p.dg), e, pass ? run : 0.0f);
            }
        }
    }
}

}  // namespace bwdc
}  // namespace kda
