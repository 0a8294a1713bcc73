// kda_chunk_tc.cuh -- chunked KDA prefill on the sm_100a tensor cores
// (tcgen05 + TMEM, operands fed by TMA), chunk C = 64 in 16-token blocks,
// dk = dv = 128, bf16 I/O, fp32 state.
//
// Math per chunk (G = inclusive cumulative max(g, floor) inside the chunk,
// r_b = G at the last token before 16-token block b, r_0 = 0, r_4 = G_63):
//   Gt_i   = e^{G_i - r_{b(i)}}                 (<= 1)
//   Kbar_j = k_j e^{r_{b(j)} - G_j}             (<= e^{-16 floor}: bf16/fp32 range
//                                                because of the floor, fupanwang.com
//                                                Kimi K3 report digest, KDA section,
//                                                Fig. 3)
//   K^(b)_j = Kbar_j e^{r_b - r_{b(j)}}  for b(j) <= b   ( = k_j e^{r_b - G_j} )
//   A_qk[i,j] = (q_i Gt_i) . K^(b(i))_j   (j <= i),   A_kk[i,j] = beta_i (k_i Gt_i) . K^(b(i))_j  (j < i)
//   T' = (I + A_kk)^-1 Diag(beta);  W = T' (k Gt e^{r_b}),  U = T' V
//   Vn = U - W S;   O = scale ((q Gt e^{r_b}) S + A_qk Vn) [* sigmoid(z)]
//   S  = Diag(e^{r_4}) S + K^(4)^T Vn
// which equals the token recurrence in real arithmetic (the intra-chunk part
// in parallel, then the state carried to the next chunk: fupanwang.com digest,
// section 基础设施, FlashKDA).
//
// Precision: the products the outputs are sensitive to run in tf32 (A_qk /
// A_kk operands, A_qk Vn, K^(4)^T Vn); W S, (Q e^G) S, W and U run in bf16.
//
// Orientation: the state products are computed transposed so that the value
// channel v is the TMEM lane (M = 128): S^T and Vn^T live in TMEM as the A
// operand, everything token-indexed is a shared-memory B operand.
//
// One CTA (512 threads) carries one (sequence, head) unit; its phases per
// chunk run in order:
//   prep (2 passes of 64 key channels; TMA tiles of q, k, g)  ->  A MMAs (tf32)
//   -> A readout + block-triangular inverse (CUDA cores)  ->  W, U MMAs (bf16)
//   -> W readout  ->  W S, (Q e^G) S MMAs  ->  Vn  ->  A_qk Vn, K^T Vn MMAs (tf32)
//   -> state update + output epilogue.
// The next chunk's q, k, g, v tiles are loaded by TMA while the current
// chunk's later phases run.
#pragma once

#include <cuda.h>

#include "kda_common.cuh"
#include "kda_tc.cuh"

namespace kda {
namespace tck {

using namespace kda::tc;

constexpr int C = 64;
constexpr int D = 128;
constexpr int NB = 4;
constexpr int NT = 512;

// ---- shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_QKG0 = 0;          // pass 0: q | k | g, channels 0-63 (3 x 8 KB)
constexpr uint32_t OFF_QKG1 = 24576;      // pass 1: channels 64-127
constexpr uint32_t QKG_Q = 0, QKG_K = 8192, QKG_G = 16384;
constexpr uint32_t OFF_V = 49152;         // v: MN-major A operand, 2 MN blocks x 8 KB
constexpr uint32_t OFF_INTRA = 65536;     // 72 KB, reused after the A MMAs
//   during prep / A MMAs (per pass of 64 channels = 2 tf32 K-blocks):
constexpr uint32_t OFF_XT = OFF_INTRA;             // X~ [128 rows x 64 ch] tf32 K-major: 2 x 16 KB
constexpr uint32_t OFF_KB = OFF_INTRA + 32768;     // K^(b), b = 0..3, packed rows 16(b+1): 40 KB
//   after the A MMAs:
constexpr uint32_t OFF_SCR = OFF_INTRA;            // A_kk -> T, fp32 [64][68]
constexpr uint32_t SCR_LD = 68;                    // 16-byte aligned rows
constexpr uint32_t OFF_TP = OFF_INTRA + 17408;     // T' bf16 K-major [64 i x 64 j]: 8 KB
constexpr uint32_t OFF_W = OFF_INTRA + 41984;      // W bf16 MN-major [128 c x 64 j]: 16 KB
constexpr uint32_t OFF_QG = OFF_INTRA + 73728;     // Q e^G bf16 MN-major [128 c x 64 i]: 16 KB
constexpr uint32_t OFF_KG = OFF_QG + 16384;        // K e^G bf16 K-major [128 c x 64 j]: 16 KB
// B operand of the second state MMA: rows 0-63 = A_qk [i x j], rows 64-191 =
// K^(4)^T [c x j]; tf32 K-major with two 128-byte K-blocks of 192 rows each
constexpr uint32_t OFF_AK = OFF_KG + 16384;
constexpr uint32_t AK_KBLK = 192u * 128u;          // 24 KB per K-block
constexpr uint32_t OFF_AQK = OFF_AK;               // + kb * AK_KBLK + row * 128
constexpr uint32_t OFF_KHT = OFF_AK + 64u * 128u;  // + kb * AK_KBLK + row * 128
constexpr uint32_t OFF_SMALL = OFF_AK + 2u * AK_KBLK;  // beta[64], gamma[128], barriers, tmem base
constexpr uint32_t OFF_TOT = OFF_SMALL + 1024;     // per-row-group decay totals [8][64] fp32
constexpr uint32_t SMEM_BYTES = OFF_TOT + 2048;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024; // slack for aligning the base
static_assert(OFF_W + 16384 <= OFF_INTRA + 73728, "post-MMA tiles fit the intra region");
static_assert(OFF_QG - OFF_W < (1u << 18) && (OFF_QG - OFF_W) % 16 == 0, "W | Q e^G as one MN-major operand");
static_assert(OFF_KB + 40960 <= OFF_INTRA + 73728, "intra tiles fit");
static_assert(SMEM_ALLOC <= 232448, "fits in 227 KB");

// K^(b) packed layout: tile b has 16(b+1) valid rows; its two 128-byte
// K-blocks are stored back to back.  The MMA (M = 64) reads 64 rows from each
// K-block start; rows past the valid ones read neighbouring bytes of this
// area, which only feed accumulator rows that are never used.
__host__ __device__ constexpr uint32_t kb_rows(int b) { return 16u * (b + 1); }
// start of tile b: sum over b' < b of 2 K-blocks x 16(b'+1) rows x 128 B
__host__ __device__ constexpr uint32_t kb_base(int b) { return 2048u * (uint32_t)b * (uint32_t)(b + 1); }
static_assert(kb_base(1) == 4096u && kb_base(2) == 12288u && kb_base(3) == 24576u, "packing");
static_assert(kb_base(3) + 128u * 64u + 64u * 128u <= 40960u, "K^(b) reads stay in the area");

// ---- TMEM columns
constexpr uint32_t T_DB = 0;      // A MMAs: 4 x 32 columns (M = 64 layout)
constexpr uint32_t T_O2 = 0;      // (A_qk Vn)^T   [v x i]   } one MMA (N = 192), after the
constexpr uint32_t T_DS = 64;     // dS^T          [v x c]   } A readout and the Vn step
constexpr uint32_t T_U = 128;     // U^T     [v x i]
constexpr uint32_t T_W = 192;     // W^T     [c x i]
constexpr uint32_t T_P = 256;     // P^T = (W S)^T, then Vn^T (tf32 A operand)  } one MMA
constexpr uint32_t T_O1 = 320;    // ((Q e^G) S)^T                              } (N = 128)
constexpr uint32_t T_S = 384;     // S^T bf16 A operand (2 per column)
constexpr uint32_t TMEM_COLS = 512;

// One explicit work unit (used by the long-sequence segment split): a token
// range of one head, where its state starts and ends, and what to produce.
enum : int32_t {
    UNIT_STORE_O = 1,      // write the outputs of the range
    UNIT_ZERO_V = 2,       // treat v as zero (U = 0): the run then maps S0 -> M S0
    UNIT_S0_IDENTITY = 4,  // start from S0 = I (with UNIT_ZERO_V: the final state is M)
};
struct TcUnit {
    int64_t t_begin, t_end;
    const float *S0;       // [dk x dv] start state or nullptr (zeros / identity)
    float *S_out;          // [dk x dv] final state or nullptr
    int32_t head, flags;
};

struct TcParams {
    const void *beta, *gate;
    const float *S0;
    const int32_t *cu_seqlens;
    const int32_t *seq_order;
    void *o;
    float *S_T;
    int32_t num_heads;
    float scale, g_floor;
    const TcUnit *units;   // when set, block b runs units[b] instead of a (sequence, head)
};

// byte offset of (row, byte kb within a 128-byte K-block row) in a swizzled block
__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t kbyte) {
    return row * 128u + ((((kbyte >> 4) & 7u) ^ (row & 7u)) << 4) + (kbyte & 15u);
}

// fp32 -> tf32, round to nearest with ties away from zero, on the integer
// pipe: adding half a tf32 ulp to the magnitude bits and truncating the low
// 13 bits gives that rounding for every finite value (a carry into the
// exponent is the correct round-up).
__device__ __forceinline__ float to_tf32(float x) {
    return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}

__device__ __forceinline__ float bf16_at(const unsigned char *tile, uint32_t row, uint32_t col) {
    // element (row, col) of a [64 x 64] bf16 TMA tile (128-byte swizzle)
    const __nv_bfloat16 *p = reinterpret_cast<const __nv_bfloat16 *>(tile + sw128(row, col * 2));
    return __bfloat162float(*p);
}

// D[16x8] += A[16x8] B[8x8] on the warp-level tensor-core path (tf32 inputs,
// fp32 accumulation); fragments: g = lane / 4, t = lane % 4,
//   a = {A[g][t], A[g+8][t], A[g][t+4], A[g+8][t+4]},  b = {B[t][g], B[t+4][g]},
//   d = {D[g][2t], D[g][2t+1], D[g+8][2t], D[g+8][2t+1]}.
__device__ __forceinline__ void mma_16x8x8_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
                 "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// e^x through the hardware exp2 (inputs here are differences of log-decays,
// results are used at tf32 / bf16 operand precision or as decay factors).
__device__ __forceinline__ float fexp(float x) { return __expf(x); }

// two fp32 -> one 32-bit word of bf16 (round to nearest even), lo in the low half
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

__global__ void __launch_bounds__(NT, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_v,
                TcParams p)
{
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float *s_beta = reinterpret_cast<float *>(sm + OFF_SMALL);          // [64]
    float *s_gam = s_beta + 64;                                          // [128]
    uint64_t *bar_qkg = reinterpret_cast<uint64_t *>(sm + OFF_SMALL + 768);   // [2]
    uint64_t *bar_v = bar_qkg + 2;
    uint64_t *bar_mma = bar_qkg + 3;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + OFF_SMALL + 832);
    float *s_tot = reinterpret_cast<float *>(sm + OFF_TOT);              // [8][64]
    float *scr = reinterpret_cast<float *>(sm + OFF_SCR);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.num_heads;
    int hh;
    int64_t t_begin, t_end;
    const float *S0p;
    float *S_outp;
    int32_t flags;
    if (p.units) {
        const TcUnit u = p.units[blockIdx.x];
        hh = u.head; t_begin = u.t_begin; t_end = u.t_end;
        S0p = u.S0; S_outp = u.S_out; flags = u.flags;
    } else {
        const int n_slot = blockIdx.x / H;
        hh = blockIdx.x % H;
        const int n = p.seq_order ? p.seq_order[n_slot] : n_slot;
        t_begin = p.cu_seqlens[n]; t_end = p.cu_seqlens[n + 1];
        const int64_t unit = (int64_t)n * H + hh;
        S0p = p.S0 ? p.S0 + unit * D * D : nullptr;
        S_outp = p.S_T ? p.S_T + unit * D * D : nullptr;
        flags = UNIT_STORE_O;
    }
    const bool store_o = (flags & UNIT_STORE_O) != 0;
    const bool zero_v = (flags & UNIT_ZERO_V) != 0;
    const int nchunks = (int)((t_end - t_begin + C - 1) / C);
    const __nv_bfloat16 *beta = static_cast<const __nv_bfloat16 *>(p.beta);
    const __nv_bfloat16 *gate = static_cast<const __nv_bfloat16 *>(p.gate);
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.o);

    // Lane-parallel coordinates: TMEM lane (value channel v, or key channel c
    // for W^T) = 32 (warp % 4) + lane; the 4 warps sharing a lane quarter split
    // the columns in quarters (cq).
    const int lq = warp & 3;
    const int cq = warp >> 2;
    const int vlane = lq * 32 + lane;
    const uint32_t lane_base = (uint32_t)(lq * 32) << 16;
    // Prep coordinates: 8-row group and 32-channel half of the pass.
    const int rg = warp & 7;
    const int cl = (warp >> 3) * 32 + lane;        // channel within the pass, 0..63

    if (warp == 0) {
        tmem_alloc(s_tmem, TMEM_COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&bar_qkg[0], 1);
        mbar_init(&bar_qkg[1], 1);
        mbar_init(bar_v, 1);
        mbar_init(bar_mma, 1);
        mbar_fence_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *s_tmem;
    const uint32_t smb = smem_u32(sm);

    // issue the TMA loads of chunk `ci` (mask bit 0: pass 0, bit 1: pass 1, bit 2: v)
    auto issue_loads = [&](int ci, int mask) {
        const int y = (int)(t_begin + (int64_t)ci * C);
        const int xk = hh * D;
        for (int pp = 0; pp < 2; ++pp) {
            if (!(mask & (1 << pp))) continue;
            uint64_t *bar = &bar_qkg[pp];
            const uint32_t base = smb + (pp ? OFF_QKG1 : OFF_QKG0);
            mbar_expect_tx(bar, 3 * 8192);
            tma_load_2d(base + QKG_Q, &tm_q, xk + 64 * pp, y, bar);
            tma_load_2d(base + QKG_K, &tm_k, xk + 64 * pp, y, bar);
            tma_load_2d(base + QKG_G, &tm_g, xk + 64 * pp, y, bar);
        }
        if (mask & 4) {
            mbar_expect_tx(bar_v, 2 * 8192);
            tma_load_2d(smb + OFF_V, &tm_v, xk, y, bar_v);
            tma_load_2d(smb + OFF_V + 8192, &tm_v, xk + 64, y, bar_v);
        }
    };

    // ---- state: thread (v, cq) keeps rows c in [32 cq, 32 cq + 32) in registers
    float S[32];
#pragma unroll
    for (int r = 0; r < 32; ++r)
        S[r] = S0p ? S0p[(cq * 32 + r) * D + vlane]
                   : ((flags & UNIT_S0_IDENTITY) && cq * 32 + r == vlane ? 1.0f : 0.0f);
    auto store_state_bf16 = [&]() {        // S^T as the bf16 A operand (2 rows c per column)
        uint32_t r16[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) r16[e] = pack_bf16(S[2 * e], S[2 * e + 1]);
        tmem_st16(tbase + lane_base + T_S + cq * 16, r16);
        tmem_wait_st();
    };
    store_state_bf16();

    // Issued-but-not-yet-waited asynchronous work, tracked identically by all
    // threads (the issue points are uniform), so a timeout can drain it.
    uint32_t qkg_issued[2] = {0, 0}, qkg_done[2] = {0, 0}, v_issued = 0, v_done = 0;
    auto note_loads = [&](int mask) {
        if (mask & 1) ++qkg_issued[0];
        if (mask & 2) ++qkg_issued[1];
        if (mask & 4) ++v_issued;
    };
    if (nchunks > 0) {
        if (tid == 0) issue_loads(0, 7);
        note_loads(7);
    }

    uint32_t mma_phase = 0, mma_issued = 0;
    bool failed = false;
    // beta of the next chunk, loaded one chunk ahead (64 strided values)
    auto load_beta = [&](int ci) -> float {
        const int64_t tb = t_begin + (int64_t)ci * C + tid;
        return (tid < C && ci < nchunks && tb < t_end) ? __bfloat162float(beta[tb * H + hh]) : 0.0f;
    };
    float beta_next = load_beta(0);
    // One thread polls the barrier while the others block in bar.sync (which
    // costs no issue slots); afterwards every thread observes the completed
    // phase once, which acquires the TMA / MMA results for it.
    auto wait_all = [&](uint64_t *bar, uint32_t parity) -> bool {
        const bool ok = tid == 0 ? mbar_wait(bar, parity) : true;
        const bool all = __syncthreads_and(ok) != 0;
        if (all && tid != 0) (void)mbar_try_wait(bar, parity);
        return all;
    };
    auto wait_mma = [&]() -> bool {
        bool ok = wait_all(bar_mma, mma_phase & 1);
        ++mma_phase;
        tc_fence_after();
        return ok;
    };
    auto sync_for_mma = [&]() {            // generic smem / TMEM writes -> MMA issue
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    };

    // MMA descriptors that do not depend on the chunk (start addresses advance per K-step)
    const uint32_t id_a = instr_desc(FMT_TF32, K_MAJOR, K_MAJOR, 64, 32);
    const uint32_t id_w = instr_desc(FMT_BF16, K_MAJOR, K_MAJOR, 128, 64);
    const uint32_t id_u = instr_desc(FMT_BF16, MN_MAJOR, K_MAJOR, 128, 64);
    const uint32_t id_1 = instr_desc(FMT_BF16, K_MAJOR, MN_MAJOR, 128, 128);
    const uint32_t id_2 = instr_desc(FMT_TF32, K_MAJOR, K_MAJOR, 128, 192);
    const uint64_t d_k16 = smem_desc_sw128(smb, 16, 1024);          // K-major template
    const uint64_t d_mnv = smem_desc_sw128(smb, 8192, 1024);        // v: MN blocks 8 KB apart
    const uint64_t d_wq = smem_desc_sw128(smb, OFF_QG - OFF_W, 1024);  // [W | Q e^G] MN-major
    auto at = [](uint64_t tmpl, uint32_t byte_off) -> uint64_t {     // same descriptor, moved start
        return tmpl + (uint64_t)(byte_off >> 4);
    };

    const float g_floor = p.g_floor;
    const float L2E = 1.4426950408889634f;
    (void)L2E;

    for (int ci = 0; ci < nchunks && !failed; ++ci) {
        const int64_t t0 = t_begin + (int64_t)ci * C;
        const int L = (int)min((int64_t)C, t_end - t0);
        const uint32_t ld_par = (uint32_t)(ci & 1);

        // ================================================= prep + A MMAs, 2 passes of 64 key channels
        bool loads_ok = true;
        for (int pass = 0; pass < 2 && !failed; ++pass) {
            // every thread observes the TMA barrier itself (no block barrier here, so
            // this pass's first part overlaps the previous pass's MMA issue); a
            // timeout is folded into the next block-wide barrier
            loads_ok = mbar_wait(&bar_qkg[pass], ld_par) && loads_ok;
            ++qkg_done[pass];
            const unsigned char *raw = sm + (pass ? OFF_QKG1 : OFF_QKG0);
            const int c = pass * 64 + cl;
            if (pass == 0) {
                if (tid < C) s_beta[tid] = beta_next;
                beta_next = load_beta(ci + 1);
            }
            // local inclusive cumulative decay over this thread's 8 rows
            float G[8];
            {
                float acc = 0.0f;
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const int i = rg * 8 + r;
                    const float gi = i < L ? fmaxf(bf16_at(raw + QKG_G, i, cl), g_floor) : 0.0f;
                    acc += gi;
                    G[r] = acc;
                }
                s_tot[rg * 64 + cl] = acc;
            }
            // q, k of the 8 rows (issued before the barrier to overlap its latency)
            float qv[8], kv[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                qv[r] = bf16_at(raw + QKG_Q, rg * 8 + r, cl);
                kv[r] = bf16_at(raw + QKG_K, rg * 8 + r, cl);
            }
            if (pass == 1) {                       // pass-0 A MMAs done (also syncs s_tot)
                const bool ok = tid == 0 ? mbar_wait(bar_mma, mma_phase & 1) : true;
                const bool all = __syncthreads_and(ok && loads_ok) != 0;
                if (all && tid != 0) (void)mbar_try_wait(bar_mma, mma_phase & 1);
                ++mma_phase;
                tc_fence_after();
                if (!all) { failed = true; break; }
            } else if (!__syncthreads_and(loads_ok)) {
                failed = true;
                break;
            }
            // prefix over row groups: P[k] = sum of the first k group totals
            float P[9];
            P[0] = 0.0f;
#pragma unroll
            for (int k = 0; k < 8; ++k) P[k + 1] = P[k] + s_tot[k * 64 + cl];
            const int b = rg >> 1;                 // 16-token block of these rows
            float rg_pre = 0.0f;                   // P[rg]
#pragma unroll
            for (int k = 0; k < 8; ++k) rg_pre = (k == rg) ? P[k] : rg_pre;
            float rb = 0.0f;                       // r_b = P[2b]
#pragma unroll
            for (int k = 0; k < 4; ++k) rb = (k == b) ? P[2 * k] : rb;
            const float r4 = P[8];
            float dfac[NB];                        // e^{r_b' - r_b}, b' >= b
#pragma unroll
            for (int k = 0; k < NB; ++k) dfac[k] = k >= b ? fexp(P[2 * k] - rb) : 0.0f;
            const float eb = fexp(rb);             // e^{r_b}: rebases Gt to the chunk start
            const float e4 = fexp(r4 - rb);        // e^{r_4 - r_b}
            if (rg == 0) s_gam[c] = fexp(r4);
            const uint32_t kbyte = (uint32_t)(cl & 31) * 4u;
            const uint32_t kblk = (uint32_t)(cl >> 5);
            unsigned char *xt = sm + OFF_XT + kblk * 16384u;
            float qg[8], kg[8], kh[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int i = rg * 8 + r;
                const float Gi = rg_pre + G[r];
                const float gt = fexp(Gi - rb);            // Gt_i
                const float kbar = kv[r] * fexp(rb - Gi);   // Kbar_i
                const float qt = qv[r] * gt, kt = kv[r] * gt;
                const uint32_t row = 32u * b + (uint32_t)(i & 15);
                *reinterpret_cast<float *>(xt + sw128(row, kbyte)) = to_tf32(qt);
                *reinterpret_cast<float *>(xt + sw128(row + 16, kbyte)) = to_tf32(kt);
                qg[r] = qt * eb;
                kg[r] = kt * eb;
                kh[r] = kbar * e4;
#pragma unroll
                for (int bp = 0; bp < NB; ++bp) {
                    if (bp < b) continue;
                    unsigned char *tile = sm + OFF_KB + kb_base(bp) + kblk * kb_rows(bp) * 128u;
                    *reinterpret_cast<float *>(tile + sw128(i, kbyte)) = to_tf32(kbar * dfac[bp]);
                }
            }
            // Q e^G (MN-major [c x i]) and K e^G (K-major [c x j]): 8 tokens = one 16-byte chunk
            *reinterpret_cast<uint4 *>(sm + OFF_QG + sw128(c, rg * 16)) =
                make_uint4(pack_bf16(qg[0], qg[1]), pack_bf16(qg[2], qg[3]), pack_bf16(qg[4], qg[5]),
                           pack_bf16(qg[6], qg[7]));
            *reinterpret_cast<uint4 *>(sm + OFF_KG + sw128(c, rg * 16)) =
                make_uint4(pack_bf16(kg[0], kg[1]), pack_bf16(kg[2], kg[3]), pack_bf16(kg[4], kg[5]),
                           pack_bf16(kg[6], kg[7]));
            // K^(4)^T (K-major [c x j], tf32): 8 tokens = 32 bytes
            {
                const uint32_t jb = (uint32_t)rg * 32u;
                unsigned char *dst = sm + OFF_KHT + (jb >> 7) * AK_KBLK;
                *reinterpret_cast<float4 *>(dst + sw128(c, jb & 127u)) =
                    make_float4(to_tf32(kh[0]), to_tf32(kh[1]), to_tf32(kh[2]), to_tf32(kh[3]));
                *reinterpret_cast<float4 *>(dst + sw128(c, (jb & 127u) + 16u)) =
                    make_float4(to_tf32(kh[4]), to_tf32(kh[5]), to_tf32(kh[6]), to_tf32(kh[7]));
            }
            sync_for_mma();
            if (ci + 1 < nchunks) note_loads(1 << pass);
            ++mma_issued;
            if (tid == 0) {
                // q, k, g of this pass are consumed: prefetch the next chunk's
                if (ci + 1 < nchunks) issue_loads(ci + 1, 1 << pass);
#pragma unroll
                for (int bb = 0; bb < NB; ++bb) {
#pragma unroll
                    for (int s = 0; s < 8; ++s) {      // 8 tf32 K-steps of 8 channels
                        const uint32_t kb = (uint32_t)(s >> 2), koff = (uint32_t)(s & 3) * 32u;
                        const uint64_t ad = at(d_k16, OFF_KB + kb_base(bb) + kb * kb_rows(bb) * 128u + koff);
                        const uint64_t bd = at(d_k16, OFF_XT + kb * 16384u + 32u * bb * 128u + koff);
                        mma_tf32_ss(tbase + T_DB + 32 * bb, ad, bd, id_a, (pass > 0 || s > 0) ? 1u : 0u);
                    }
                }
                mma_commit(bar_mma);
            }
        }
        if (failed) break;
        if (!wait_mma()) { failed = true; break; }

        // ================================================= A readout: warp (lq, cq): rows j, row block b = cq
        {
            uint32_t ra[16], rk[16];
            tmem_ld16(tbase + lane_base + T_DB + 32 * cq, ra);
            tmem_ld16(tbase + lane_base + T_DB + 32 * cq + 16, rk);
            tmem_wait_ld();
            if (lane < 16) {
                const int j = lq * 16 + lane;
                const uint32_t kbj = (uint32_t)j * 4u;
                unsigned char *aqk = sm + OFF_AQK + (kbj >> 7) * AK_KBLK;
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int i = 16 * cq + e;
                    const float aq = j <= i ? __uint_as_float(ra[e]) : 0.0f;
                    const float ak = j < i ? s_beta[i] * __uint_as_float(rk[e]) : 0.0f;
                    *reinterpret_cast<float *>(aqk + sw128(i, kbj & 127u)) = to_tf32(aq);
                    scr[i * SCR_LD + j] = ak;
                }
            }
        }
        tc_fence_before();
        __syncthreads();

        // ================================================= T = (I + A_kk)^-1 in place, blocked
        {
            // (1) 16x16 diagonal blocks by forward substitution: thread (block, column)
            float t[16];
            const bool act = tid < 64;
            const int bb = tid >> 4, jj = tid & 15;
            if (act) {
                const float *A = scr + (16 * bb) * SCR_LD + 16 * bb;
#pragma unroll
                for (int i = 0; i < 16; ++i) t[i] = (i == jj) ? 1.0f : 0.0f;
#pragma unroll
                for (int i = 1; i < 16; ++i) {
                    float acc = 0.0f;
#pragma unroll
                    for (int m = 0; m < 15; ++m)
                        if (m < i) acc = fmaf(A[i * SCR_LD + m], t[m], acc);
                    if (i > jj) t[i] = -acc;
                }
            }
            __syncthreads();
            if (act) {
                float *Tb = scr + (16 * bb) * SCR_LD + 16 * bb;
#pragma unroll
                for (int i = 0; i < 16; ++i) Tb[i * SCR_LD + jj] = t[i];
            }
            __syncthreads();
            // Off-diagonal blocks by block products on the warp-level tensor cores
            // (tf32; T' only needs bf16 precision).  tile(...) returns one 16x8
            // tile of D[dr0.., dc0..] E[er0.., ec0..] over a K-wide inner range.
            const int gq = lane >> 2, tq = lane & 3;
            auto tile = [&](int dr0, int dc0, int er0, int ec0, int K, float (&acc)[4]) {
                acc[0] = acc[1] = acc[2] = acc[3] = 0.0f;
                for (int k0 = 0; k0 < K; k0 += 8) {
                    uint32_t a[4], b[2];
                    a[0] = __float_as_uint(scr[(dr0 + gq) * SCR_LD + dc0 + k0 + tq]);
                    a[1] = __float_as_uint(scr[(dr0 + gq + 8) * SCR_LD + dc0 + k0 + tq]);
                    a[2] = __float_as_uint(scr[(dr0 + gq) * SCR_LD + dc0 + k0 + tq + 4]);
                    a[3] = __float_as_uint(scr[(dr0 + gq + 8) * SCR_LD + dc0 + k0 + tq + 4]);
                    b[0] = __float_as_uint(scr[(er0 + k0 + tq) * SCR_LD + ec0 + gq]);
                    b[1] = __float_as_uint(scr[(er0 + k0 + tq + 4) * SCR_LD + ec0 + gq]);
                    mma_16x8x8_tf32(acc, a, b);
                }
            };
            auto put = [&](int r0, int c0, const float (&acc)[4], float sign) {
                scr[(r0 + gq) * SCR_LD + c0 + 2 * tq] = sign * acc[0];
                scr[(r0 + gq) * SCR_LD + c0 + 2 * tq + 1] = sign * acc[1];
                scr[(r0 + gq + 8) * SCR_LD + c0 + 2 * tq] = sign * acc[2];
                scr[(r0 + gq + 8) * SCR_LD + c0 + 2 * tq + 1] = sign * acc[3];
            };
            // (2) 16 -> 32 for the pairs (0,1), (2,3): T10 = -T11 (A10 T00); warps 0-3
            {
                const int o0 = 32 * (warp >> 1), n0 = o0 + 8 * (warp & 1);
                float acc[4];
                if (warp < 4) tile(o0 + 16, o0, o0, n0, 16, acc);
                __syncthreads();
                if (warp < 4) put(o0 + 16, n0, acc, 1.0f);
                __syncthreads();
                if (warp < 4) tile(o0 + 16, o0 + 16, o0 + 16, n0, 16, acc);
                __syncthreads();
                if (warp < 4) put(o0 + 16, n0, acc, -1.0f);
                __syncthreads();
            }
            // (3) 32 -> 64: T[32:, :32] = -T[32:, 32:] (A[32:, :32] T[:32, :32]); warps 0-7
            {
                const int r0 = 32 + 16 * (warp >> 2), n0 = 8 * (warp & 3);
                float acc[4];
                if (warp < 8) tile(r0, 0, 0, n0, 32, acc);
                __syncthreads();
                if (warp < 8) put(r0, n0, acc, 1.0f);
                __syncthreads();
                if (warp < 8) tile(r0, 32, 32, n0, 32, acc);
                __syncthreads();
                if (warp < 8) put(r0, n0, acc, -1.0f);
                __syncthreads();
            }
            // (4) T' = T Diag(beta) as bf16, K-major [i x j], zero above the diagonal; 8 per thread
            {
                const int i = tid >> 3, j0 = (tid & 7) * 8;
                uint32_t pk[4];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    const int j = j0 + e;
                    const float a = j <= i ? scr[i * SCR_LD + j] * s_beta[j] : 0.0f;
                    const float a2 = j + 1 <= i ? scr[i * SCR_LD + j + 1] * s_beta[j + 1] : 0.0f;
                    pk[e / 2] = pack_bf16(a, a2);
                }
                *reinterpret_cast<uint4 *>(sm + OFF_TP + sw128(i, j0 * 2)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
        }
        sync_for_mma();

        // ================================================= W^T = (K e^G)^T T'^T, U^T = V^T T'^T (bf16)
        if (!wait_all(bar_v, ld_par)) { failed = true; break; }
        ++v_done;
        ++mma_issued;
        if (tid == 0) {
#pragma unroll
            for (int s = 0; s < 4; ++s) {          // K = 64 tokens in steps of 16
                const uint64_t bd = at(d_k16, OFF_TP + 32u * s);
                mma_bf16_ss(tbase + T_W, at(d_k16, OFF_KG + 32u * s), bd, id_w, s > 0);
                mma_bf16_ss(tbase + T_U, at(d_mnv, OFF_V + 2048u * s), bd, id_u, s > 0);
            }
            mma_commit(bar_mma);
        }
        if (!wait_mma()) { failed = true; break; }
        if (ci + 1 < nchunks) {                      // v consumed: prefetch the next chunk's
            if (tid == 0) issue_loads(ci + 1, 4);
            note_loads(4);
        }

        // ================================================= W readout: lane c, tokens j in [16 cq, 16 cq + 16)
        {
            uint32_t rw[16];
            tmem_ld16(tbase + lane_base + T_W + cq * 16, rw);
            tmem_wait_ld();
            uint32_t pk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) pk[e] = pack_bf16(__uint_as_float(rw[2 * e]), __uint_as_float(rw[2 * e + 1]));
            *reinterpret_cast<uint4 *>(sm + OFF_W + sw128(vlane, cq * 32)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            *reinterpret_cast<uint4 *>(sm + OFF_W + sw128(vlane, cq * 32 + 16)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
        sync_for_mma();

        // ================================================= P^T = S^T W^T, O1^T = S^T (Q e^G)^T (bf16, A from TMEM)
        ++mma_issued;
        if (tid == 0) {
#pragma unroll
            for (int s = 0; s < 8; ++s)            // K = 128 key channels in steps of 16
                mma_bf16_ts(tbase + T_P, tbase + T_S + 8u * s, at(d_wq, OFF_W + 2048u * s), id_1, s > 0);
            mma_commit(bar_mma);
        }
        if (!wait_mma()) { failed = true; break; }

        // ================================================= Vn^T = U^T - P^T (tf32, in place of P^T)
        {
            uint32_t rp[16], ru[16];
            tmem_ld16(tbase + lane_base + T_P + cq * 16, rp);
            tmem_ld16(tbase + lane_base + T_U + cq * 16, ru);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e)
                rp[e] = __float_as_uint(to_tf32((zero_v ? 0.0f : __uint_as_float(ru[e])) - __uint_as_float(rp[e])));
            tmem_st16(tbase + lane_base + T_P + cq * 16, rp);
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ================================================= O2^T = Vn^T A_qk^T, dS^T = Vn^T K^(4) (tf32)
        ++mma_issued;
        if (tid == 0) {
#pragma unroll
            for (int s = 0; s < 8; ++s) {          // K = 64 tokens in steps of 8
                const uint32_t kb = (uint32_t)(s >> 2), koff = (uint32_t)(s & 3) * 32u;
                mma_tf32_ts(tbase + T_O2, tbase + T_P + 8u * s, at(d_k16, OFF_AK + kb * AK_KBLK + koff), id_2, s > 0);
            }
            mma_commit(bar_mma);
        }
        if (!wait_mma()) { failed = true; break; }

        // ================================================= state update and outputs
        {
#pragma unroll
            for (int hq = 0; hq < 2; ++hq) {       // dS^T rows c in [32 cq + 16 hq, +16)
                uint32_t rd[16];
                tmem_ld16(tbase + lane_base + T_DS + cq * 32 + hq * 16, rd);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    S[hq * 16 + e] = fmaf(s_gam[cq * 32 + hq * 16 + e], S[hq * 16 + e], __uint_as_float(rd[e]));
            }
            store_state_bf16();
            uint32_t r1[16], r2[16];
            tmem_ld16(tbase + lane_base + T_O1 + cq * 16, r1);
            tmem_ld16(tbase + lane_base + T_O2 + cq * 16, r2);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int i = cq * 16 + e;
                if (store_o && i < L) {
                    const int64_t off = ((t0 + i) * H + hh) * D + vlane;
                    float x = p.scale * (__uint_as_float(r1[e]) + __uint_as_float(r2[e]));
                    if (gate) x *= sigmoidf(__bfloat162float(gate[off]));
                    o[off] = __float2bfloat16_rn(x);
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (!failed && S_outp) {
#pragma unroll
        for (int r = 0; r < 32; ++r) S_outp[(cq * 32 + r) * D + vlane] = S[r];
    }
    if (failed && tid == 0) {
        // drain what is still in flight (bounded) before TMEM and shared memory go away
        for (int pp = 0; pp < 2; ++pp)
            for (uint32_t k2 = qkg_done[pp]; k2 < qkg_issued[pp]; ++k2) mbar_wait(&bar_qkg[pp], k2 & 1u, 1u << 20);
        for (uint32_t k2 = v_done; k2 < v_issued; ++k2) mbar_wait(bar_v, k2 & 1u, 1u << 20);
        for (uint32_t k2 = mma_phase; k2 < mma_issued; ++k2) mbar_wait(bar_mma, k2 & 1u, 1u << 20);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, TMEM_COLS);
}

}  // namespace tck
}  // namespace kda
