// kda_tc.cuh -- Blackwell (sm_100a) tensor-core building blocks written as
// inline PTX: tensor memory (TMEM) allocation, tcgen05.mma with shared-memory
// or TMEM operands, commit to an mbarrier, TMEM <-> register moves, the
// shared-memory matrix and instruction descriptors, and the 128-byte
// swizzled shared-memory layouts the descriptors describe.
//
// Every wait here is bounded: on timeout it records KDA_ERR_TIMEOUT in the
// device error word and returns false, so a caller can unwind (free TMEM,
// exit) instead of hanging the GPU.
#pragma once

#include <stdint.h>

#include "kda_common.cuh"

namespace kda {
namespace tc {

// ---------------------------------------------------------------- addresses
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// The polling loop of mbar_wait, kept out of line: waits are many and their
// slow path is rare, so inlining it would only grow the kernels' code.
__device__ __noinline__ bool mbar_wait_poll(uint64_t *bar, uint32_t parity, uint32_t max_iters) {
    for (uint32_t i = 0; i < max_iters; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    raise_error(ERR_TIMEOUT);
    return false;
}

// Waits for the phase with the given parity to complete; gives up after
// `max_iters` polls (each try_wait itself blocks for a bounded time slice).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          uint32_t max_iters = (1u << 22)) {
    if (mbar_try_wait(bar, parity)) return true;
    return mbar_wait_poll(bar, parity, max_iters);
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// ---------------------------------------------------------------- fences
__device__ __forceinline__ void fence_async_smem() {   // generic smem writes -> async proxy (MMA/TMA)
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---------------------------------------------------------------- TMEM allocation (one warp)
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// TMEM address: lane in bits [31:16], column in bits [15:0].
__device__ __forceinline__ uint32_t tmem_addr(uint32_t base, uint32_t lane, uint32_t col) {
    return base + (lane << 16) + col;
}

// ---------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor for a 128-byte-swizzled operand tile.
//   start: smem byte address of the (K-slice of the) tile, 16-byte aligned;
//          the tile's swizzle atoms must sit on 1024-byte boundaries.
//   lbo:   K-major: unused (pass 16); MN-major: bytes between 128-byte-wide
//          MN blocks.
//   sbo:   bytes between groups of 8 rows (K-major) / 8 K-rows (MN-major).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t start, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((start >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;          // descriptor version for tcgen05
    d |= (uint64_t)2u << 61;          // layout: 128-byte swizzle
    return d;
}

enum Fmt : uint32_t { FMT_F16 = 0, FMT_BF16 = 1, FMT_TF32 = 2 };
enum Major : uint32_t { K_MAJOR = 0, MN_MAJOR = 1 };

// Instruction descriptor for kind::f16 / kind::tf32 with fp32 accumulation.
__host__ __device__ constexpr uint32_t instr_desc(uint32_t fmt_ab, uint32_t a_major,
                                                  uint32_t b_major, uint32_t M, uint32_t N) {
    return (1u << 4)                  // D format: f32
           | (fmt_ab << 7) | (fmt_ab << 10)
           | (a_major << 15) | (b_major << 16)
           | ((N >> 3) << 17)
           | ((M >> 4) << 24);
}

// ---------------------------------------------------------------- MMA issue (one thread)
// D[tmem] (+)= A * B^T with A, B from shared memory.
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void mma_tf32_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
// D[tmem] (+)= A * B^T with A in tensor memory.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void mma_tf32_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
// One lane of a converged warp, the same on every call with all lanes
// active.  MMA issue runs warp-wide (descriptor arithmetic stays uniform)
// with only the elected lane executing the tcgen05 instructions; this keeps
// the issue sequence short in both instructions and code size.
__device__ __forceinline__ bool elect_one() {
    uint32_t e;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(e));
    return e != 0;
}

// Arrive on `bar` once every MMA this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

// ---------------------------------------------------------------- TMEM <-> registers
// 32 lanes x 32 bits, 16 consecutive columns: thread t of the warp gets lane
// (warp quarter base + t), columns col..col+15.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
          "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
          "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- swizzled layouts
// Byte offset of element (row, k) in a K-major, 128-byte-swizzled tile with
// `rows` rows: K is cut into 128-byte K-blocks stored one after another
// (each rows x 128 B); inside a K-block, row r sits at r * 128 B and its
// 16-byte chunks are XOR-permuted by (r % 8).
__host__ __device__ constexpr uint32_t kmajor_off(uint32_t row, uint32_t kbyte, uint32_t rows) {
    return (kbyte >> 7) * rows * 128u + row * 128u +
           ((((kbyte >> 4) & 7u) ^ (row & 7u)) << 4) + (kbyte & 15u);
}
// Byte offset of element (mn, k) in an MN-major, 128-byte-swizzled tile with
// `krows` K-rows: MN is cut into 128-byte MN-blocks stored one after another
// (each krows x 128 B); inside a block, K-row k sits at k * 128 B with its
// 16-byte chunks XOR-permuted by (k % 8).
__host__ __device__ constexpr uint32_t mnmajor_off(uint32_t mnbyte, uint32_t k, uint32_t krows) {
    return (mnbyte >> 7) * krows * 128u + k * 128u +
           ((((mnbyte >> 4) & 7u) ^ (k & 7u)) << 4) + (mnbyte & 15u);
}

}  // namespace tc
}  // namespace kda
