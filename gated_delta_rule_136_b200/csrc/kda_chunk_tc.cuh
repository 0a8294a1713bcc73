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
//   T' = (I + A_kk)^-1 Diag(beta)
//   Vn = T' V - T' ((k Gt e^{r_b}) S)   (= U - W S of the WY form, U = T' V, W = T' K e^G)
//   O  = scale ((q Gt e^{r_b}) S + A_qk Vn) [* sigmoid(z)]
//   S  = Diag(e^{r_4}) S + K^(4)^T Vn
// which equals the token recurrence in real arithmetic (the intra-chunk part
// in parallel, then the state carried to the next chunk: fupanwang.com digest,
// section 基础设施, FlashKDA).
//
// Precision: the products the outputs are sensitive to run in tf32 or fp16 (the
// A_qk / A_kk operands: tf32 rounded to nearest on the diagonal 16 x 16 blocks,
// fp16 -- the same 11-bit significand -- on the off-diagonal ones, whose
// operands are all at most 1; T' (K e^G) S, A_qk Vn, K^(4)^T Vn in tf32);
// T' V, (K e^G) S and (Q e^G) S run in bf16, with S carried as a
// leading bf16 part plus a bf16 low part (each state product issued once per
// part into the same accumulator).  On the full-size workloads the bf16
// off-diagonal A operands and the bf16 state were the largest terms of the
// output error.
//
// Orientation: the state products are computed transposed so that the value
// channel v is the TMEM lane (M = 128): S^T and Vn^T live in TMEM as the A
// operand, everything token-indexed is a shared-memory B operand.
//
// One CTA (512 threads) carries one (sequence, head) unit; its phases per
// chunk run in order:
//   prep (2 passes of 64 key channels; TMA tiles of q, k, g)  ->  A MMAs (tf32 diagonal
//   blocks, fp16 off-diagonal)
//   -> A readout -> block-triangular inverse (warps 0-7)
//   -> Vn = T' V - T' Y MMAs (Y = (K e^G) S from an MMA issued behind the A MMAs)
//   -> A_qk Vn, K^T Vn MMAs (fp16, power-of-two scales)
//   -> state update + output epilogue.
// The next chunk's q, k, g, v tiles are loaded by TMA while the current
// chunk's later phases run.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>

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
//   during prep / A MMAs (per pass of 64 channels):
constexpr uint32_t OFF_XT = OFF_INTRA;             // X~ [128 rows x 64 ch] tf32 K-major: 2 x 16 KB
constexpr uint32_t OFF_KD = OFF_INTRA + 32768;     // Kbar [64 rows j x 64 ch] tf32 K-major: 2 x 8 KB
constexpr uint32_t OFF_XB = OFF_INTRA + 49152;     // X~ rows 32-127 (blocks 1-3) fp16 K-major: 12 KB
constexpr uint32_t OFF_KO = OFF_INTRA + 61440;     // K^(b) rows j < 16 b, b = 1..3, fp16 K-major: 12 KB
//   after the A MMAs:
constexpr uint32_t OFF_SCR = OFF_INTRA;            // A_kk -> T, fp32 [64][68]
constexpr uint32_t SCR_LD = 68;                    // 16-byte aligned rows
constexpr uint32_t OFF_TP = OFF_INTRA + 17408;     // T' tf32 K-major [64 i x 64 j]: 2 x 8 KB
constexpr uint32_t OFF_XS = OFF_INTRA + 33792;     // inverse scratch: 4 warps x [32 x 8] fp32: 4 KB
constexpr uint32_t XS_LD = 8;
constexpr uint32_t OFF_TPB = OFF_INTRA + 37888;    // T' bf16 K-major [64 i x 64 j]: 8 KB
constexpr uint32_t OFF_QG = OFF_INTRA + 73728;     // Q e^G bf16 MN-major [128 c x 64 i]: 16 KB
constexpr uint32_t OFF_KG = OFF_QG + 16384;        // K e^G bf16 K-major [128 c x 64 j]: 16 KB
// B operand of the second state MMA: rows 0-63 = 2^8 A_qk [i x j], rows 64-191
// = 2^8 K^(4)^T [c x j]; fp16 K-major, one 128-byte K-block of 64 tokens (its A
// operand is 2^-8 Vn^T in fp16: the scales cancel exactly, and fp16 keeps
// tf32's 11-bit significand for these values, |A_qk| and |K^| being at most 1)
constexpr uint32_t OFF_AK = OFF_KG + 16384;
constexpr uint32_t OFF_AQK = OFF_AK;               // + row * 128
constexpr uint32_t OFF_KHT = OFF_AK + 64u * 128u;  // + row * 128
// The output tile waits here for its TMA store, bf16 [64 tokens x 64 v] per
// half (v in [0, 64), then [64, 128)).
constexpr uint32_t OFF_OST = OFF_AK + 192u * 128u;
constexpr uint32_t OFF_SMALL = OFF_OST + 2u * 8192u;   // beta[64], gamma[2][128], barriers, tmem base
constexpr uint32_t SMEM_BYTES = OFF_SMALL + 2048;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024; // slack for aligning the base
static_assert(OFF_TP % 1024 == 0 && OFF_TP + 16384 <= OFF_XS && OFF_XS + 4096 <= OFF_TPB &&
              OFF_TPB % 1024 == 0 && OFF_TPB + 8192 <= OFF_INTRA + 73728, "post-MMA tiles fit the intra region");
static_assert((OFF_KG - OFF_QG) % 16 == 0, "Q e^G | K e^G as one MN-major operand");
static_assert(OFF_KO + 12288 == OFF_INTRA + 73728, "intra tiles fit");
static_assert(SMEM_ALLOC <= 232448, "fits in 227 KB");

// Off-diagonal operands, fp16: tile b (b = 1..3) holds K^(b) rows j < 16 b
// (tokens of the blocks before b), one 128-byte K-block of 64 channels; tiles
// are packed back to back.  The row operand is an fp16 copy of X~ rows of
// blocks 1-3.  Every value is at most |q| or |k| (<= 1: the decays only shrink
// it), so fp16 holds it without overflow, with tf32's 11-bit significand; a
// value below fp16's range is below 6e-8 and so is its every product.  The
// MMA (M = 64) reads 64 rows from a tile's start; rows past the valid ones
// read neighbouring bytes (the next tile, or for b = 3 the first 2 KB after
// the intra region), which only feed accumulator rows that are never used.
__host__ __device__ constexpr uint32_t ko_base(int b) { return 1024u * (uint32_t)b * (uint32_t)(b - 1); }
static_assert(ko_base(1) == 0u && ko_base(2) == 2048u && ko_base(3) == 6144u, "packing");
static_assert(OFF_KO + ko_base(3) + 64u * 128u <= OFF_QG + 16384u, "K^(b) reads stay in shared memory");

// ---- TMEM columns
constexpr uint32_t T_DD = 0;      // diagonal A MMA [64 j x 128 X~ rows] (M = 64 layout)
constexpr uint32_t T_DO = 128;    // off-diagonal A MMAs: 3 x 32 columns (blocks 1-3)
constexpr uint32_t T_O2 = 0;      // (A_qk Vn)^T   [v x i]   } one MMA (N = 192), after the
constexpr uint32_t T_DS = 64;     // dS^T          [v x c]   } A readout and Vn
constexpr uint32_t T_VN = 192;    // Vn^T = V^T T'^T - Y^T T'^T (fp32; its fp16 copy goes to T_LO)
constexpr uint32_t T_O1 = 256;    // ((Q e^G) S)^T  [v x i]  } one MMA (N = 128)
constexpr uint32_t T_Z = 320;     // -((K e^G) S)^T  [v x j] (read as a tf32 A operand)
constexpr uint32_t T_S = 384;     // S^T bf16 A operand (2 per column): the leading bf16 part
constexpr uint32_t T_LO = 448;    // S^T - bf16(S^T) in bf16, the low part of the same operand; then,
                                  // its MMAs done, 2^-8 Vn^T in fp16 (32 columns: two tokens each)
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
    int32_t seq;           // sequence index (snapshot slots)
    int64_t seq_start;     // the sequence's first token (snapshot positions)
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
    SnapOut snap;          // state snapshots (units with UNIT_STORE_O only)
    int64_t total_tokens;  // extents, for the debug build's unit checks
    int32_t num_seqs;
};

// byte offset of (row, byte kb within a 128-byte K-block row) in a swizzled block
__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t kbyte) {
    return row * 128u + ((((kbyte >> 4) & 7u) ^ (row & 7u)) << 4) + (kbyte & 15u);
}

// fp32 -> tf32, round to nearest with ties away from zero, on the integer
// pipe: adding half a tf32 ulp to the magnitude bits and truncating the low
// 13 bits gives that rounding for every finite value (a carry into the
// exponent is the correct round-up).
// two fp32 -> one 32-bit word of fp16 (round to nearest even), lo in the low half
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
          "r"(r[7]) : "memory");
}

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

// D[16x8] += A[16x16] B[16x8], bf16 inputs, fp32 accumulation; fragments:
//   a = {A[g][2t..2t+1], A[g+8][2t..], A[g][2t+8..], A[g+8][2t+8..]},
//   b = {B[2t..2t+1][g], B[2t+8..2t+9][g]},  d as for the tf32 form above.
__device__ __forceinline__ void mma_16x8x16_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
                 "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// four 8x8 b16 matrices, transposed on the way in: lane l gives the address
// of row l % 8 of matrix l / 8 (16 contiguous bytes); lane (g, t) receives
// elements (2t, g) and (2t + 1, g) of each matrix
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}

// two 8x8 b16 matrices from the fragment layout (lane (g, t) holds elements
// (g, 2t) and (g, 2t + 1)), stored transposed: lane l (< 16) gives the address
// of stored row l % 8 of matrix l / 8
__device__ __forceinline__ void stsm_x2_trans(uint32_t addr, uint32_t r0, uint32_t r1) {
    asm volatile("stmatrix.sync.aligned.m8n8.x2.trans.shared.b16 [%0], {%1, %2};"
                 :: "r"(addr), "r"(r0), "r"(r1) : "memory");
}

__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

// bf16 pair in one 32-bit word -> two floats (low half first)
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// 2^x on the special-function unit (approximate; denormal results flush to zero)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// waits (bounded) for the barrier phases [done, issued) of `bar` to complete
__device__ __noinline__ void drain_phases(uint64_t *bar, uint32_t done, uint32_t issued) {
    for (uint32_t k = done; k < issued; ++k) mbar_wait(bar, k & 1u, 1u << 20);
}

// sigmoid on the special-function unit (relative error a few fp32 ulp, far
// below the bf16 rounding of the gated output)
__device__ __forceinline__ float sigmoid_fast(float z) { return __fdividef(1.0f, 1.0f + __expf(-z)); }

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar)) : "memory");
}

// TMA tile store from shared memory (bulk-group completion)
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, uint32_t src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];"
                 ::"l"(map), "r"(x), "r"(y), "r"(src) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// the shared-memory sources of this thread's committed stores may be reused
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// this thread's committed stores are complete
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

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

// SNAP: the variant that stores state snapshots (TcParams::snap); the other
// compiles without that code.  NOOUT: for launches whose units store no outputs
// (the long-sequence split's first pass, context-parallel summaries): the q
// side (Q~, Q e^G, A_qk, O1, O2) is not formed; the state products run as their
// K e^G and K^ parts alone (N = 64 and N = 128).
template <bool SNAP, bool NOOUT = false>
__global__ void __launch_bounds__(NT, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ CUtensorMap tm_o, TcParams p)
{
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float *s_beta = reinterpret_cast<float *>(sm + OFF_SMALL);          // [64]
    float *s_gam = s_beta + 64;                                          // [2][128], by chunk parity
    uint64_t *bar_qkg = reinterpret_cast<uint64_t *>(sm + OFF_SMALL + 1280);  // [2]
    uint64_t *bar_v = bar_qkg + 2;
    uint64_t *bar_mma = bar_qkg + 3;
    uint64_t *bar_y = bar_qkg + 4;       // the (Q e^G | K e^G) S MMA
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + OFF_SMALL + 1344);
    float *scr = reinterpret_cast<float *>(sm + OFF_SCR);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.num_heads;
    int hh;
    int64_t t_begin, t_end;
    const float *S0p;
    float *S_outp;
    int32_t flags;
    int snap_n;                          // sequence index and first token, for snapshots
    int64_t seq_start;
    if (p.units) {
        const TcUnit u = p.units[blockIdx.x];
        hh = u.head; t_begin = u.t_begin; t_end = u.t_end;
        S0p = u.S0; S_outp = u.S_out; flags = u.flags;
        snap_n = u.seq; seq_start = u.seq_start;
    } else {
        const int n_slot = blockIdx.x / H;
        hh = blockIdx.x % H;
        const int n = p.seq_order ? p.seq_order[n_slot] : n_slot;
        if (kDebugChecks && (n < 0 || n >= p.num_seqs)) {
            if (tid == 0) raise_error(ERR_BOUNDS);
            return;
        }
        t_begin = p.cu_seqlens[n]; t_end = p.cu_seqlens[n + 1];
        const int64_t unit = (int64_t)n * H + hh;
        S0p = p.S0 ? p.S0 + unit * D * D : nullptr;
        S_outp = p.S_T ? p.S_T + unit * D * D : nullptr;
        flags = UNIT_STORE_O;
        snap_n = n; seq_start = t_begin;
    }
    if (kDebugChecks) {   // the unit must lie inside the launch's extents
        const bool bad = t_begin < 0 || t_end < t_begin || t_end > p.total_tokens || hh < 0 || hh >= H ||
                         snap_n < 0 || snap_n >= p.num_seqs || (NOOUT && (flags & UNIT_STORE_O));
        if (bad) {
            if (tid == 0) raise_error(ERR_BOUNDS);
            return;                      // (uniform over the CTA, before any shared or TMEM state)
        }
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
    // Prep coordinates (mma fragment layout): channel tile nt, block pair mp,
    // lane (gq, tq); channels cA, cA + 1 of the pass.
    const int nt = warp & 7, mp = warp >> 3;
    const int gq = lane >> 2, tq = lane & 3;
    const int cA = nt * 8 + 2 * tq;
    // swizzled byte offset of (a row r with r % 8 == gq, channel cA) in the tf32
    // K-major operand tiles, and the K-block of cA
    const uint32_t kblk = (uint32_t)(cA >> 5);
    const uint32_t kbyte = (uint32_t)(cA & 31) * 4u;
    const uint32_t sw_lane = ((((kbyte >> 4) & 7u) ^ (uint32_t)gq) << 4) + (kbyte & 15u);
    const uint32_t xt_lane = OFF_XT + kblk * 16384u + sw_lane;
    const uint32_t kd_lane = OFF_KD + kblk * 8192u + sw_lane;
    // the same for the fp16 tiles (one 128-byte K-block of 64 channels)
    const uint32_t xb_lane = OFF_XB + (((((uint32_t)cA * 2u) >> 4) ^ (uint32_t)gq) << 4) + (((uint32_t)cA * 2u) & 15u);
    // constant A fragments of the prefix-sum products (bf16 1.0 = 0x3F80):
    //   a_blk: 16x16 lower triangle with diagonal;  a_ref[kb]: rows m < 4 select block kb <= m
    uint32_t a_blk[4];
    a_blk[0] = (2 * tq <= gq ? 0x3F80u : 0u) | (2 * tq + 1 <= gq ? 0x3F800000u : 0u);
    a_blk[1] = 0x3F803F80u;
    a_blk[2] = 0u;
    a_blk[3] = a_blk[0];
    uint32_t a_ref[NB][4];
#pragma unroll
    for (int kb = 0; kb < NB; ++kb) {
        const uint32_t v = (gq < NB && kb <= gq) ? 0x3F803F80u : 0u;
        a_ref[kb][0] = v; a_ref[kb][1] = 0u; a_ref[kb][2] = v; a_ref[kb][3] = 0u;
    }
    // floor: the largest bf16 fb <= floor; max(g, floor) = max(g, fb) + (g <= fb) (floor - fb)
    const __nv_bfloat16 fb = __float2bfloat16_rd(p.g_floor);
    const __nv_bfloat162 floor_b2 = __halves2bfloat162(fb, fb);
    const float floor_gap = p.g_floor - __bfloat162float(fb);
    const bool floor_inexact = floor_gap != 0.0f;

    if (warp == 0) {
        tmem_alloc(s_tmem, TMEM_COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&bar_qkg[0], 1);
        mbar_init(&bar_qkg[1], 1);
        mbar_init(bar_v, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_y, 1);
        mbar_fence_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *s_tmem;
    const uint32_t smb = smem_u32(sm);
    const bool leader = elect_one();       // this warp's MMA-issuing lane (used in warp 0)

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
    auto store_state_bf16 = [&]() {        // S^T as the bf16 A operand (2 rows c per column):
        uint32_t r16[16];                   // the leading part, then the low part
#pragma unroll
        for (int e = 0; e < 16; ++e) r16[e] = pack_bf16(S[2 * e], S[2 * e + 1]);
        tmem_st16(tbase + lane_base + T_S + cq * 16, r16);
        tmem_wait_st();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const float2 hi = unpack_bf16x2(r16[e]);
            r16[e] = pack_bf16(S[2 * e] - hi.x, S[2 * e + 1] - hi.y);
        }
        tmem_st16(tbase + lane_base + T_LO + cq * 16, r16);
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

    uint32_t mma_phase = 0, mma_issued = 0, y_phase = 0, y_issued = 0;
    bool failed = false;
    // first token of the output tile waiting in the staging area (-1: none);
    // tid 0 issues its TMA store after the next block barrier
    int64_t o_row = -1;
    auto store_o_tile = [&]() {            // tid 0; the staging tile is complete and fenced
        const int x = hh * D;
        tma_store_2d(&tm_o, smb + OFF_OST, x, (int)o_row);
        tma_store_2d(&tm_o, smb + OFF_OST + 8192u, x + 64, (int)o_row);
        bulk_commit();
    };
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

    // MMA descriptors that do not depend on the chunk (start addresses advance per K-step)
    const uint32_t id_d = instr_desc(FMT_TF32, K_MAJOR, K_MAJOR, 64, 128);
    const uint32_t id_o = instr_desc(FMT_F16, K_MAJOR, K_MAJOR, 64, 32);
    const uint32_t id_1 = instr_desc(FMT_BF16, K_MAJOR, MN_MAJOR, 128, NOOUT ? 64 : 128);
    const uint32_t id_vn = instr_desc(FMT_TF32, K_MAJOR, K_MAJOR, 128, 64);
    const uint32_t id_u = instr_desc(FMT_BF16, MN_MAJOR, K_MAJOR, 128, 64);
    const uint32_t id_2 = instr_desc(FMT_F16, K_MAJOR, K_MAJOR, 128, NOOUT ? 128 : 192);
    const uint64_t d_k16 = smem_desc_sw128(smb, 16, 1024);          // K-major template
    const uint64_t d_qk = smem_desc_sw128(smb, OFF_KG - OFF_QG, 1024);  // [Q e^G | -K e^G] MN-major
    const uint64_t d_mnv = smem_desc_sw128(smb, 8192, 1024);             // v: MN blocks 8 KB apart
    auto at = [](uint64_t tmpl, uint32_t byte_off) -> uint64_t {     // same descriptor, moved start
        return tmpl + (uint64_t)(byte_off >> 4);
    };
    // Warp 0: the A MMAs of a prep pass, in two parts.
    //   part 0: the diagonal product D[j, n] = Kbar_j . X~_n over the pass's 64
    //           channels (tf32, M = 64, N = 128: every block against every
    //           block, of which the diagonal 16 x 32 tiles are used), and the
    //           off-diagonal product of block 1;
    //   part 1: the off-diagonal products of blocks 2 and 3 (fp16, M = 64, N = 32:
    //           K^(b) rows j < 16 b against X~ rows of block b); then commit.
    auto issue_a = [&](int pass_, int part) {
        if (part == 0) {
#pragma unroll 1
            for (int s = 0; s < 8; ++s) {          // tf32 K-steps of 8 channels
                const uint32_t kb = (uint32_t)(s >> 2), koff = (uint32_t)(s & 3) * 32u;
                if (leader) mma_tf32_ss(tbase + T_DD, at(d_k16, OFF_KD + kb * 8192u + koff),
                                        at(d_k16, OFF_XT + kb * 16384u + koff), id_d, (pass_ > 0 || s > 0) ? 1u : 0u);
            }
        }
#pragma unroll
        for (int bo = 1; bo < NB; ++bo) {
            if ((bo == 1) != (part == 0)) continue;
#pragma unroll
            for (int s = 0; s < 4; ++s)            // fp16 K-steps of 16 channels
                if (leader) mma_bf16_ss(tbase + T_DO + 32u * (bo - 1), at(d_k16, OFF_KO + ko_base(bo) + 32u * s),
                                        at(d_k16, OFF_XB + 32u * (bo - 1) * 128u + 32u * s), id_o,
                                        (pass_ > 0 || s > 0) ? 1u : 0u);
        }
        if (part == 1 && leader) mma_commit(bar_mma);
    };

    const float L2E = 1.4426950408889634f;

    // The loop runs prep stages (chunk ci, pass) in order.  A chunk's state
    // chain ends with the N = 192 MMA; the next chunk's first prep pass runs
    // while that MMA executes, and only then is the previous chunk finished
    // (state update, outputs) -- its tail -- before the next MMAs are issued.
    int64_t t0 = 0, t0p = 0;                 // first token of the prepped / finishing chunk
    int L = 0, Lp = 0;                       // their lengths
    bool loads_ok = true;
    float2 khv[2][2] = {};                   // this thread's K^ values of the current prep pass
    auto store_khat = [&](int pass_, int bb, int hr) {
        const int b = 2 * mp + bb;
        const uint32_t i = (uint32_t)(16 * b + 8 * hr + gq);
        const uint32_t cg = (uint32_t)(pass_ * 64 + cA);
        *reinterpret_cast<__half *>(sm + OFF_KHT + sw128(cg, i * 2u)) = __float2half_rn(khv[bb][hr].x);
        *reinterpret_cast<__half *>(sm + OFF_KHT + sw128(cg + 1u, i * 2u)) = __float2half_rn(khv[bb][hr].y);
    };
#pragma unroll 1
    for (int st = 0; st <= 2 * nchunks && !failed; ++st) {
        const int pass = st & 1;
        const int ci = st >> 1;              // chunk of this prep pass (nchunks: none, tail only)
        const int tci = ci - 1;              // chunk finished by this stage's tail (pass 0)
        if (pass == 0) {
            t0p = t0; Lp = L;
            loads_ok = true;
            if (ci < nchunks) {
                t0 = t_begin + (int64_t)ci * C;
                L = (int)min((int64_t)C, t_end - t0);
            }
        }
        const uint32_t ld_par = (uint32_t)(ci & 1);
        const bool ragged = L < C;

        // ================================================= prep + A MMAs, 2 passes of 64 key channels
        // Warp (nt, mp) of a pass owns channels 8 nt .. 8 nt + 7 of the pass and the
        // 16-token blocks 2 mp, 2 mp + 1; lane (gq, tq) holds channels cA = 8 nt + 2 tq,
        // cA + 1 of tokens 16 b + gq and 16 b + gq + 8 (mma fragment layout).
        if (ci < nchunks) {
                loads_ok = mbar_wait(&bar_qkg[pass], ld_par) && loads_ok;
                ++qkg_done[pass];
                const uint32_t raw = smb + (pass ? OFF_QKG1 : OFF_QKG0);
                if (pass == 0) {
                    if (tid < C) s_beta[tid] = beta_next;
                    beta_next = load_beta(ci + 1);
                }
                // (1) decay prefix sums on the warp-level tensor cores: with
                //     gc = max(g, floor) (zero past the chunk's end),
                //       x_i   = sum of gc over block b(i) up to i      = G_i - r_b(i)
                //       r_b+1 = sum of gc over blocks 0..b
                //     as products of 0/1 matrices with gc (bf16 operands, fp32 sums:
                //     exact up to the fp32 rounding of the sums)
                uint32_t gf[2][4];                     // [tokens 32h..][block 2h + (j>>1), half j&1]
                ldsm_x4_trans(gf[0], raw + QKG_G + sw128((uint32_t)lane, (uint32_t)nt * 16u));
                ldsm_x4_trans(gf[1], raw + QKG_G + sw128((uint32_t)(32 + lane), (uint32_t)nt * 16u));
                if (pass == 1 && warp == 0) {          // the rest of the pass-0 A MMAs
                    __syncwarp();
                    issue_a(0, 1);
                    __syncwarp();
                }
                uint32_t gi[2][4];                     // indicator g <= fb (floor not a bf16 value)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const __nv_bfloat162 gv = *reinterpret_cast<const __nv_bfloat162 *>(&gf[h][j]);
                        __nv_bfloat162 gc = __hmax2(gv, floor_b2);
                        __nv_bfloat162 ind = __hle2(gv, floor_b2);
                        if (ragged) {                  // tokens past the chunk's end contribute nothing
                            const int tok = 32 * h + 8 * j + 2 * tq;
                            const uint32_t keep = (tok < L ? 0x0000FFFFu : 0u) | (tok + 1 < L ? 0xFFFF0000u : 0u);
                            gf[h][j] = *reinterpret_cast<uint32_t *>(&gc) & keep;
                            gi[h][j] = *reinterpret_cast<uint32_t *>(&ind) & keep;
                        } else {
                            gf[h][j] = *reinterpret_cast<uint32_t *>(&gc);
                            gi[h][j] = *reinterpret_cast<uint32_t *>(&ind);
                        }
                    }
                }
                float xs[2][4], rr[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int bb = 0; bb < 2; ++bb) {
                    const uint32_t b0 = mp ? gf[1][2 * bb] : gf[0][2 * bb];
                    const uint32_t b1 = mp ? gf[1][2 * bb + 1] : gf[0][2 * bb + 1];
                    xs[bb][0] = xs[bb][1] = xs[bb][2] = xs[bb][3] = 0.0f;
                    mma_16x8x16_bf16(xs[bb], a_blk, b0, b1);
                }
#pragma unroll
                for (int kb = 0; kb < NB; ++kb) mma_16x8x16_bf16(rr, a_ref[kb], gf[kb >> 1][2 * (kb & 1)], gf[kb >> 1][2 * (kb & 1) + 1]);
                if (floor_inexact) {                   // + (floor - fb) x (the same sums of the indicator)
                    float xi[2][4], ri[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                    for (int bb = 0; bb < 2; ++bb) {
                        const uint32_t b0 = mp ? gi[1][2 * bb] : gi[0][2 * bb];
                        const uint32_t b1 = mp ? gi[1][2 * bb + 1] : gi[0][2 * bb + 1];
                        xi[bb][0] = xi[bb][1] = xi[bb][2] = xi[bb][3] = 0.0f;
                        mma_16x8x16_bf16(xi[bb], a_blk, b0, b1);
                    }
#pragma unroll
                    for (int kb = 0; kb < NB; ++kb) mma_16x8x16_bf16(ri, a_ref[kb], gi[kb >> 1][2 * (kb & 1)], gi[kb >> 1][2 * (kb & 1) + 1]);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        xs[0][e] = fmaf(floor_gap, xi[0][e], xs[0][e]);
                        xs[1][e] = fmaf(floor_gap, xi[1][e], xs[1][e]);
                        rr[e] = fmaf(floor_gap, ri[e], rr[e]);
                    }
                }
                // (2) block decay factors eT_b = e^{r_b+1 - r_b} for this lane's two channels
                //     (rows 0..3 of the r tile sit in lanes 4 m + tq)
                //     lane (gq, tq) evaluates one factor -- block gq % 4 of channel
                //     cA + gq / 4 -- and gathers the other seven with shuffles
                float2 eT[NB];
                {
                    const int m = gq & 3;
                    // r_{m+1} and r_m of channels cA (rr[0]) and cA + 1 (rr[1])
                    const float hiA = __shfl_sync(0xffffffffu, rr[0], 4 * m + tq);
                    const float hiB = __shfl_sync(0xffffffffu, rr[1], 4 * m + tq);
                    const float loA = __shfl_sync(0xffffffffu, rr[0], (4 * m + 28 + tq) & 31);
                    const float loB = __shfl_sync(0xffffffffu, rr[1], (4 * m + 28 + tq) & 31);
                    const float hi = (gq >> 2) ? hiB : hiA;
                    const float lo = m == 0 ? 0.0f : ((gq >> 2) ? loB : loA);
                    const float e = fexp(hi - lo);
#pragma unroll
                    for (int mm = 0; mm < NB; ++mm)
                        eT[mm] = make_float2(__shfl_sync(0xffffffffu, e, 4 * mm + tq),
                                             __shfl_sync(0xffffffffu, e, 4 * (mm + 4) + tq));
                }
                if (mp == 0 && gq == 0) {              // gamma = e^{r_4} for the state update
                    const float2 g4 = __fmul2_rn(__fmul2_rn(eT[0], eT[1]), __fmul2_rn(eT[2], eT[3]));
                    *reinterpret_cast<float2 *>(s_gam + (ci & 1) * D + pass * 64 + cA) = g4;
                }
                // (3) per-element factors; the stores that no MMA in flight reads go first
                float2 qt[2][2], kt[2][2], kbar[2][2];
                const float2 l2e = make_float2(L2E, L2E), nl2e = make_float2(-L2E, -L2E);
#pragma unroll
                for (int bb = 0; bb < 2; ++bb) {
                    const int b = 2 * mp + bb;
                    float2 Eb = make_float2(1.0f, 1.0f), eK = make_float2(1.0f, 1.0f);
#pragma unroll
                    for (int m = 0; m < NB; ++m) {
                        if (m < b) Eb = __fmul2_rn(Eb, eT[m]);
                        else eK = __fmul2_rn(eK, eT[m]);
                    }
                    uint32_t pq[2], pk[2];
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr) {
                        const int i = 16 * b + gq + 8 * hr;
                        const float2 x2 = make_float2(xs[bb][2 * hr], xs[bb][2 * hr + 1]);
                        const float2 t2 = __fmul2_rn(x2, l2e), u2 = __fmul2_rn(x2, nl2e);
                        const float2 gt = make_float2(ex2_approx(t2.x), ex2_approx(t2.y));       // Gt_i
                        const float2 ig = make_float2(ex2_approx(u2.x), ex2_approx(u2.y));       // 1 / Gt_i
                        const uint32_t qoff = raw + QKG_Q + sw128((uint32_t)i, (uint32_t)cA * 2u);
                        if constexpr (!NOOUT) {
                            const float2 q2 = unpack_bf16x2(ld_shared_u32(qoff));
                            const float2 k2 = unpack_bf16x2(ld_shared_u32(qoff + (QKG_K - QKG_Q)));
                            qt[bb][hr] = __fmul2_rn(q2, gt);
                            kt[bb][hr] = __fmul2_rn(k2, gt);
                            kbar[bb][hr] = __fmul2_rn(k2, ig);                                        // Kbar_i
                            const float2 qg = __fmul2_rn(qt[bb][hr], Eb), kg = __fmul2_rn(kt[bb][hr], Eb);
                            pq[hr] = pack_bf16(qg.x, qg.y);
                            pk[hr] = pack_bf16(-kg.x, -kg.y);   // -K e^G: the MMA then yields -Y
                        } else {                                // the k side alone
                            const float2 k2 = unpack_bf16x2(ld_shared_u32(qoff + (QKG_K - QKG_Q)));
                            kt[bb][hr] = __fmul2_rn(k2, gt);
                            kbar[bb][hr] = __fmul2_rn(k2, ig);
                            const float2 kg = __fmul2_rn(kt[bb][hr], Eb);
                            pk[hr] = pack_bf16(-kg.x, -kg.y);
                        }
                        // K^(4)^T [c x j] tf32: two channels of token i; on the first pass the
                        // previous chunk's last MMA may still read these rows: stored later
                        const float2 kh = __fmul2_rn(kbar[bb][hr], eK);
                        khv[bb][hr] = make_float2(kh.x * 256.0f, kh.y * 256.0f);   // 2^8 K^, as fp16
                        if (pass == 1) store_khat(1, bb, hr);
                    }
                    // Q e^G and -K e^G (bf16 [c x i], tokens contiguous): transposing matrix stores
                    {
                        const uint32_t row = (uint32_t)(pass * 64 + nt * 8 + (lane & 7));
                        const uint32_t tb2 = (uint32_t)(16 * b + 8 * ((lane >> 3) & 1)) * 2u;
                        if constexpr (!NOOUT) stsm_x2_trans(smb + OFF_QG + sw128(row, tb2), pq[0], pq[1]);
                        stsm_x2_trans(smb + OFF_KG + sw128(row, tb2), pk[0], pk[1]);
                    }
                }
                if (pass == 1) {                       // pass-0 A MMAs must be done with X~ and K^(b)
                    loads_ok = mbar_wait(bar_mma, mma_phase & 1) && loads_ok;
                    ++mma_phase;
                    tc_fence_after();
                }
                // (4) the A-MMA operands: X~ rows (q~ at 32 b + r, k~ at 32 b + 16 + r) and
                //     Kbar for the diagonal product (tf32, rounded), X~ rows of blocks 1-3
                //     again in fp16 and the K^(b') copies, b' > b, in fp16 for the
                //     off-diagonal products
#pragma unroll
                for (int bb = 0; bb < 2; ++bb) {
                    const int b = 2 * mp + bb;
                    float2 dfac[NB];                   // e^{r_b' - r_b} for b' > b
                    {
                        float2 run = make_float2(1.0f, 1.0f);
#pragma unroll
                        for (int m = 0; m < NB; ++m) {
                            if (m > b) run = __fmul2_rn(run, eT[m - 1]);
                            dfac[m] = run;
                        }
                    }
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr) {
                        const uint32_t i = (uint32_t)(16 * b + 8 * hr) + (uint32_t)gq;
                        const uint32_t xrow = (uint32_t)(32 * b + 8 * hr) + (uint32_t)gq;
                        auto rnd2 = [](float2 x) { return make_float2(to_tf32(x.x), to_tf32(x.y)); };
                        if constexpr (!NOOUT) *reinterpret_cast<float2 *>(sm + xt_lane + xrow * 128u) = rnd2(qt[bb][hr]);
                        *reinterpret_cast<float2 *>(sm + xt_lane + (xrow + 16u) * 128u) = rnd2(kt[bb][hr]);
                        *reinterpret_cast<float2 *>(sm + kd_lane + i * 128u) = rnd2(kbar[bb][hr]);
                        if (b > 0) {
                            if constexpr (!NOOUT)
                                *reinterpret_cast<uint32_t *>(sm + xb_lane + (xrow - 32u) * 128u) = pack_f16(qt[bb][hr].x, qt[bb][hr].y);
                            *reinterpret_cast<uint32_t *>(sm + xb_lane + (xrow - 16u) * 128u) = pack_f16(kt[bb][hr].x, kt[bb][hr].y);
                        }
#pragma unroll
                        for (int m = 1; m < NB; ++m) {
                            if (m <= b) continue;
                            const float2 v = __fmul2_rn(kbar[bb][hr], dfac[m]);
                            *reinterpret_cast<uint32_t *>(sm + xb_lane - OFF_XB + OFF_KO + ko_base(m) + i * 128u) = pack_f16(v.x, v.y);
                        }
                    }
                }
        }
        if (pass == 0) {
            if (ci > 0) {
                if (!wait_mma()) { failed = true; break; }

                // ================================================= state update and outputs
                // (no block barrier after this phase: the next chunk's prep touches none
                // of what it reads -- gamma is double-buffered -- and the next MMA that
                // overwrites these TMEM columns is issued after a block barrier)
                {
                    const float *gam = s_gam + (tci & 1) * D;
#pragma unroll
                    for (int hq = 0; hq < 2; ++hq) {       // dS^T rows c in [32 cq + 16 hq, +16)
                        uint32_t rd[16];
                        tmem_ld16(tbase + lane_base + T_DS + cq * 32 + hq * 16, rd);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            S[hq * 16 + e] = fmaf(gam[cq * 32 + hq * 16 + e], S[hq * 16 + e], __uint_as_float(rd[e]));
                    }
                    store_state_bf16();
                    if (SNAP && store_o) {       // snapshot of the state after this chunk, if due
                        const int64_t slot = snap_slot(p.snap, snap_n, t0p + Lp - seq_start);
                        if (slot >= 0) {
                            float *dst = p.snap.states + ((slot * H + hh) * D + cq * 32) * D + vlane;
#pragma unroll
                            for (int r = 0; r < 32; ++r) dst[r * D] = S[r];
                        }
                    }
                    uint32_t r1[16], r2[16];
                    if constexpr (!NOOUT) {
                        tmem_ld16(tbase + lane_base + T_O1 + cq * 16, r1);
                        tmem_ld16(tbase + lane_base + T_O2 + cq * 16, r2);
                        tmem_wait_ld();
                    }
                    if (!NOOUT && store_o) {
                        float x[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) x[e] = p.scale * (__uint_as_float(r1[e]) + __uint_as_float(r2[e]));
                        const int nv = min(16, Lp - cq * 16);   // tokens of this thread inside the chunk
                        const int64_t off0 = ((t0p + cq * 16) * H + hh) * D + vlane;
                        if (gate) {
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                if (e < nv) x[e] *= sigmoid_fast(__bfloat162float(gate[off0 + (int64_t)e * H * D]));
                        }
                        if (Lp == C) {
                            // full chunk: into the staging tile, stored by TMA after the next block barrier
                            unsigned char *ost = sm + OFF_OST + (uint32_t)(vlane >> 6) * 8192u;
                            const uint32_t vb = (uint32_t)(vlane & 63) * 2u;
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                *reinterpret_cast<__nv_bfloat16 *>(ost + sw128((uint32_t)(cq * 16 + e), vb)) = __float2bfloat16_rn(x[e]);
                            o_row = t0p;
                        } else {
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                if (e < nv) o[off0 + (int64_t)e * H * D] = __float2bfloat16_rn(x[e]);
                        }
                    }
                }
            }
            if (ci == nchunks) break;
#pragma unroll
            for (int bb = 0; bb < 2; ++bb)
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) store_khat(0, bb, hr);
        }
        // block barrier: the MMA issue needs every thread's operands (and the waits' outcome)
        fence_async_smem();
        tc_fence_before();
        if (!__syncthreads_and(loads_ok)) { failed = true; break; }
        tc_fence_after();
        if (ci + 1 < nchunks) note_loads(1 << pass);
        ++mma_issued;
        if (warp == 0) {
            // q, k, g of this pass are consumed: prefetch the next chunk's; the
            // previous chunk's output tile is complete: store it
            if (lane == 0) {
                if (ci + 1 < nchunks) issue_loads(ci + 1, 1 << pass);
                if (pass == 0 && o_row >= 0) store_o_tile();
            }
            __syncwarp();
            // pass 0: part 0 now, part 1 early in warp 0's pass-1 prep (a long run of
            // issues stalls the issuing warp); pass 1: everything now
            issue_a(pass, 0);
            if (pass == 1) issue_a(1, 1);
        }
        if (pass == 0) o_row = -1;
        if (pass == 0) continue;

        if (tid == 0) bulk_wait_read();        // the staged output tile has been read
        if (!wait_mma()) { failed = true; break; }

        // ================================================= A readout: warp (lq, cq): rows j of block lq, rows i of block cq
        {
            // rows j of block lq against X~ rows of block cq: the diagonal product for
            // lq == cq, block cq's off-diagonal product for lq < cq (lq > cq: j > i, masked)
            const uint32_t acol = lq < cq ? T_DO + 32u * (uint32_t)(cq - 1) : T_DD + 32u * (uint32_t)cq;
            uint32_t ra[16], rk[16];
            tmem_ld16(tbase + lane_base + acol, ra);
            tmem_ld16(tbase + lane_base + acol + 16, rk);
            tmem_wait_ld();
            if (lane < 16) {
                const int j = lq * 16 + lane;
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int i = 16 * cq + e;
                    const float aq = j <= i ? __uint_as_float(ra[e]) : 0.0f;
                    const float ak = j < i ? s_beta[i] * __uint_as_float(rk[e]) : 0.0f;
                    if constexpr (!NOOUT)
                        *reinterpret_cast<__half *>(sm + OFF_AQK + sw128(i, (uint32_t)j * 2u)) = __float2half_rn(aq * 256.0f);
                    scr[i * SCR_LD + j] = ak;
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        bool z_ok = true;
        ++y_issued;
        // [O1 | -Y]^T = S^T [Q e^G | -K e^G]^T (bf16, A = S^T from TMEM as its leading and
        // low parts), issued by warp 8 while warps 0-7 run the inverse: the tensor pipe
        // is idle then, and no prep warp waits on the issue
        if (warp == 8) {
#pragma unroll 1
            for (int ks = 0; ks < 8; ++ks) {       // K = 128 key channels in steps of 16
                // (NOOUT: the -K e^G half alone, into -Y's columns)
                const uint32_t dcol = NOOUT ? T_Z : T_O1, bsrc = (NOOUT ? OFF_KG : OFF_QG) + 2048u * (uint32_t)ks;
                if (leader) mma_bf16_ts(tbase + dcol, tbase + T_S + 8u * (uint32_t)ks, at(d_qk, bsrc), id_1, ks > 0);
                if (leader) mma_bf16_ts(tbase + dcol, tbase + T_LO + 8u * (uint32_t)ks, at(d_qk, bsrc), id_1, 1u);
            }
            if (leader) mma_commit(bar_y);
            __syncwarp();
        }
        // ================================================= T = (I + A_kk)^-1, then T' = T Diag(beta) (warps 0-7)
        // Blocked inverse of the unit lower-triangular 64x64 matrix: 16x16
        // diagonal blocks by forward substitution (warps 0-1), then the block merges
        //   [[T11, 0], [T21, T22]]:  T21 = -T22 (A21 T11)
        // for 16 -> 32 (warps 0-3, two per pair) and 32 -> 64 (warps 0-7, two per
        // column group); the warps that share a merge meet at named barriers.
        {
            const int gq = lane >> 2, tq = lane & 3;
            // acc[16 x 8] += X[16 x K] Y[K x 8] on the warp-level tensor cores
            // (tf32; T' only needs bf16 precision); ldx / ldy in floats
            auto mma_tile = [&](float (&acc)[4], const float *X, int ldx, const float *Y, int ldy, int K) {
                for (int k0 = 0; k0 < K; k0 += 8) {
                    uint32_t a[4], bb[2];
                    a[0] = __float_as_uint(X[gq * ldx + k0 + tq]);
                    a[1] = __float_as_uint(X[(gq + 8) * ldx + k0 + tq]);
                    a[2] = __float_as_uint(X[gq * ldx + k0 + tq + 4]);
                    a[3] = __float_as_uint(X[(gq + 8) * ldx + k0 + tq + 4]);
                    bb[0] = __float_as_uint(Y[(k0 + tq) * ldy + gq]);
                    bb[1] = __float_as_uint(Y[(k0 + tq + 4) * ldy + gq]);
                    mma_16x8x8_tf32(acc, a, bb);
                }
            };
            // store a 16x8 accumulator tile (times `sign`) at D (leading dimension ld)
            auto put_tile = [&](float *D, int ld, const float (&acc)[4], float sign) {
                *reinterpret_cast<float2 *>(D + gq * ld + 2 * tq) = make_float2(sign * acc[0], sign * acc[1]);
                *reinterpret_cast<float2 *>(D + (gq + 8) * ld + 2 * tq) = make_float2(sign * acc[2], sign * acc[3]);
            };
            if (warp < 4) {
                // pair p = warp % 2 (blocks 2p, 2p + 1, rows and columns o .. o + 31) is
                // merged by warps p (diagonal blocks; n-tile 0) and p + 2 (n-tile 1),
                // which meet at named barrier 2 + p
                const int p = warp & 1, half = warp >> 1, o = 32 * p;
                auto pair_sync = [&]() { asm volatile("bar.sync %0, 64;" ::"r"(2 + p) : "memory"); };
                if (half == 0) {   // diagonal blocks: lane = (block, column jj)
                    const int d0 = o + 16 * (lane >> 4), jj = lane & 15;
                    const float *A = scr + d0 * SCR_LD + d0;
                    float t[16];
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
                    __syncwarp();
                    float *Tb = scr + d0 * SCR_LD + d0;
#pragma unroll
                    for (int i = 0; i < 16; ++i) Tb[i * SCR_LD + jj] = t[i];
                    __syncwarp();
                }
                pair_sync();                                   // T11, T22 of the pair
                // 16 -> 32, n-tile `half`: X = A[o+16.., o..] T11[:, tile], then
                // T21[:, tile] = -T22 X[:, tile]; X replaces A21 only after both warps read it
                float x[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                mma_tile(x, scr + (o + 16) * SCR_LD + o, SCR_LD, scr + o * SCR_LD + o + 8 * half, SCR_LD, 16);
                float *blk21 = scr + (o + 16) * SCR_LD + o + 8 * half;
                pair_sync();                                   // A21 is read
                put_tile(blk21, SCR_LD, x, 1.0f);
                __syncwarp();
                x[0] = x[1] = x[2] = x[3] = 0.0f;
                mma_tile(x, scr + (o + 16) * SCR_LD + o + 16, SCR_LD, blk21, SCR_LD, 16);
                __syncwarp();
                put_tile(blk21, SCR_LD, x, -1.0f);
                pair_sync();                                   // T21 of the pair is complete
                // T' rows o..o+31 (lane = row), tf32 K-major [i x j] in two 32-column
                // K-blocks: columns o..o+31 from T (this warp: column groups 2 half,
                // 2 half + 1), the other 32 zero for rows 0-31; rows 32-63, columns
                // 0-31 are written by the 32 -> 64 step
                const int i = o + lane;
                // also as bf16 (K-major [i x j], one 128-byte row) for the T' V product
                unsigned char *tpr = sm + OFF_TP + (uint32_t)p * 8192u;   // K-block of columns o..o+31
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int c8 = 2 * half + cc;
                    const int j0 = o + 8 * c8;
                    const float4 ta = *reinterpret_cast<const float4 *>(scr + i * SCR_LD + j0);
                    const float4 tb = *reinterpret_cast<const float4 *>(scr + i * SCR_LD + j0 + 4);
                    const float4 ba = *reinterpret_cast<const float4 *>(s_beta + j0);
                    const float4 bb4 = *reinterpret_cast<const float4 *>(s_beta + j0 + 4);
                    const float4 va = make_float4(ta.x * ba.x, ta.y * ba.y, ta.z * ba.z, ta.w * ba.w);
                    const float4 vb = make_float4(tb.x * bb4.x, tb.y * bb4.y, tb.z * bb4.z, tb.w * bb4.w);
                    *reinterpret_cast<float4 *>(tpr + sw128((uint32_t)i, (uint32_t)c8 * 32u)) = va;
                    *reinterpret_cast<float4 *>(tpr + sw128((uint32_t)i, (uint32_t)c8 * 32u + 16u)) = vb;
                    *reinterpret_cast<uint4 *>(sm + OFF_TPB + sw128((uint32_t)i, (uint32_t)j0 * 2u)) =
                        make_uint4(pack_bf16(va.x, va.y), pack_bf16(va.z, va.w), pack_bf16(vb.x, vb.y), pack_bf16(vb.z, vb.w));
                }
                if (warp == 0) {                               // rows 0-31, columns 32-63: zero
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4)
                        *reinterpret_cast<float4 *>(sm + OFF_TP + 8192u + sw128((uint32_t)i, (uint32_t)c4 * 16u)) =
                            make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                } else if (warp == 2) {
#pragma unroll
                    for (int c8 = 4; c8 < 8; ++c8)
                        *reinterpret_cast<uint4 *>(sm + OFF_TPB + sw128((uint32_t)i, (uint32_t)c8 * 16u)) = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            if (warp < 8) {
                asm volatile("bar.sync 1, 256;" ::: "memory");   // warps 0-7 only
                // 32 -> 64 for columns 8 cg .. 8 cg + 7 (cg = warp % 4), rows 32 + 16 rt ..
                // + 15 (rt = warp / 4):
                //   X = A[32:64, 0:32] T[0:32, cols],  T[32:64, cols] = -T[32:64, 32:64] X;
                // the two row tiles of a column group meet at named barrier 4 + cg
                const int cg = warp & 3, rt = warp >> 2;
                float *xs = reinterpret_cast<float *>(sm + OFF_XS) + cg * 32 * XS_LD;
                const int n0 = 8 * cg;
                float x[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                mma_tile(x, scr + (32 + 16 * rt) * SCR_LD, SCR_LD, scr + n0, SCR_LD, 32);
                put_tile(xs + 16 * rt * XS_LD, XS_LD, x, 1.0f);
                asm volatile("bar.sync %0, 64;" ::"r"(4 + cg) : "memory");   // both row tiles of X
                x[0] = x[1] = x[2] = x[3] = 0.0f;
                mma_tile(x, scr + (32 + 16 * rt) * SCR_LD + 32, SCR_LD, xs, XS_LD, 32);
                const int j = n0 + 2 * tq;                // columns 0-31: K-block 0
                const float b0 = -s_beta[j], b1 = -s_beta[j + 1];
                const int i0 = 32 + 16 * rt + gq;
                *reinterpret_cast<float2 *>(sm + OFF_TP + sw128((uint32_t)i0, (uint32_t)j * 4u)) =
                    make_float2(x[0] * b0, x[1] * b1);
                *reinterpret_cast<float2 *>(sm + OFF_TP + sw128((uint32_t)i0 + 8u, (uint32_t)j * 4u)) =
                    make_float2(x[2] * b0, x[3] * b1);
                *reinterpret_cast<uint32_t *>(sm + OFF_TPB + sw128((uint32_t)i0, (uint32_t)j * 2u)) =
                    pack_bf16(x[0] * b0, x[1] * b1);
                *reinterpret_cast<uint32_t *>(sm + OFF_TPB + sw128((uint32_t)i0 + 8u, (uint32_t)j * 2u)) =
                    pack_bf16(x[2] * b0, x[3] * b1);
            }
        }
        if (tid == 0) z_ok = mbar_wait(bar_v, ld_par) && mbar_wait(bar_y, y_phase & 1);
        ++v_done;
        ++y_phase;
        fence_async_smem();
        tc_fence_before();
        if (!__syncthreads_and(z_ok)) { failed = true; break; }
        tc_fence_after();

        // ================================================= Vn^T = V^T T'^T + (-Y)^T T'^T, then 2^-8 Vn^T in fp16
        // (bf16 with v as the MN-major A operand from its TMA tile, then tf32 with
        // -Y^T from TMEM, into one accumulator)
        ++mma_issued;
        if (warp == 0) {
            if (!zero_v) {                         // (a unit that treats v as zero skips T' V)
#pragma unroll
                for (int s = 0; s < 4; ++s)        // K = 64 tokens in steps of 16
                    if (leader) mma_bf16_ss(tbase + T_VN, at(d_mnv, OFF_V + 2048u * s), at(d_k16, OFF_TPB + 32u * s), id_u, s > 0);
            }
#pragma unroll
            for (int s = 0; s < 8; ++s) {          // K = 64 tokens in steps of 8
                const uint32_t kb = (uint32_t)(s >> 2), koff = (uint32_t)(s & 3) * 32u;
                if (leader) mma_tf32_ts(tbase + T_VN, tbase + T_Z + 8u * s, at(d_k16, OFF_TP + kb * 8192u + koff), id_vn,
                                        (!zero_v || s > 0) ? 1u : 0u);
            }
            if (leader) mma_commit(bar_mma);
        }
        if (!wait_mma()) { failed = true; break; }
        if (ci + 1 < nchunks) {                      // v consumed: prefetch the next chunk's
            if (tid == 0) issue_loads(ci + 1, 4);
            note_loads(4);
        }
        {   // 2^-8 Vn^T in fp16, two tokens per column, over the state's low part (whose
            // MMAs completed before the V_new MMAs)
            uint32_t rv[16], ph[8];
            tmem_ld16(tbase + lane_base + T_VN + cq * 16, rv);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 8; ++e)
                ph[e] = pack_f16(__uint_as_float(rv[2 * e]) * 0.00390625f, __uint_as_float(rv[2 * e + 1]) * 0.00390625f);
            tmem_st8(tbase + lane_base + T_LO + cq * 8, ph);
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ================================================= O2^T = Vn^T A_qk^T, dS^T = Vn^T K^(4) (fp16, scales 2^-8 x 2^8)
        ++mma_issued;
        if (warp == 0) {
#pragma unroll
            for (int s = 0; s < 4; ++s)            // K = 64 tokens in steps of 16
                if (leader)   // (NOOUT: the K^ rows alone, into dS's columns)
                    mma_bf16_ts(tbase + (NOOUT ? T_DS : T_O2), tbase + T_LO + 8u * s,
                                at(d_k16, (NOOUT ? OFF_KHT : OFF_AK) + 32u * s), id_2, s > 0);
            if (leader) mma_commit(bar_mma);
        }
    }

    if (!failed && S_outp) {
#pragma unroll
        for (int r = 0; r < 32; ++r) S_outp[(cq * 32 + r) * D + vlane] = S[r];
    }
    if (!failed && o_row >= 0) {           // the last chunk's output tile
        fence_async_smem();
        __syncthreads();
        if (tid == 0) store_o_tile();
    }
    if (tid == 0) bulk_wait_all();         // every TMA store has completed
    if (failed && tid == 0) {
        // drain what is still in flight (bounded) before TMEM and shared memory go away
        drain_phases(&bar_qkg[0], qkg_done[0], qkg_issued[0]);
        drain_phases(&bar_qkg[1], qkg_done[1], qkg_issued[1]);
        drain_phases(bar_v, v_done, v_issued);
        drain_phases(bar_mma, mma_phase, mma_issued);
        drain_phases(bar_y, y_phase, y_issued);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, TMEM_COLS);
}

}  // namespace tck
}  // namespace kda
