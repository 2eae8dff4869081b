// Blackwell (sm_100a) 5th-generation tensor-core primitives: tcgen05.mma with operands in shared
// memory and the accumulator in tensor memory (TMEM), used by the tensor-core grouped expert
// kernel (expert_tc.cu) and checked on their own by focr_tc_selftest (tcgen05_selftest.cu).
//
// The encodings follow the PTX forms that the CUTLASS/CuTe sm100 headers issue.  Operands are
// K-major without swizzle: core matrices of 8 rows x 16 bytes stored contiguously, LBO = 128 B
// between the two core matrices of a 16-wide k-step, SBO = 1024 B between 8-row groups, and the
// descriptors advance by 256 B per k-step inside a 64-wide K-block.
#pragma once

#include <stdint.h>

namespace focr {
namespace umma {

// Instruction descriptor of tcgen05.mma kind::f16 with bf16 A and B, fp32 D, both operands K-major:
// D format at bits 4-5 (1 = f32), A and B formats at 7-9 and 10-12 (1 = bf16), N >> 3 at bits 17-22,
// M >> 4 at bits 24-28.
// The same with f16 A and B (format 0).
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
    return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor, K-major without swizzle: the operand is a grid of core matrices
// of 8 rows x 16 bytes (128 contiguous bytes); `lbo` = byte distance between the two core matrices
// along K of one 16-element k-step, `sbo` = byte distance between consecutive 8-row groups.
// Start address, lbo and sbo are stored >> 4 (bits 0-13, 16-29, 32-45); version 1 at bit 46.
__device__ __forceinline__ uint64_t sdesc_kmajor(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// TMEM allocation by one whole warp: `ncols` (a power of two >= 32) columns; the TMEM address
// (lane 0, first column) is written to shared memory at `dst_smem`.
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

// Release by the same warp that allocated (after every read of the accumulator).
__device__ __forceinline__ void tmem_free(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Generic-proxy writes to shared memory made visible to the tensor core's reads.
__device__ __forceinline__ void fence_smem_to_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// D (TMEM) = A B^T (+ D when `accumulate`), issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         bool accumulate) {
    const uint32_t acc = accumulate ? 1u : 0u, zero = 0u;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc), "r"(zero)
        : "memory");
}

// D (TMEM) = A B^T (+ D when `accumulate`) with A read from tensor memory: lane m holds row m of A,
// 32-bit column c of it the bf16 pair (k = 2c, 2c + 1); one MMA consumes K = 16, i.e. 8 columns
// from `a_tmem`.  B from shared memory through its descriptor.  Issued by one thread.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            bool accumulate) {
    const uint32_t acc = accumulate ? 1u : 0u, zero = 0u;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(acc), "r"(zero)
        : "memory");
}

// 32 consecutive 32-bit columns of one TMEM lane per thread, from registers: warp w (of a
// warpgroup) writes lanes 32 w .. 32 w + 31 at `taddr` = base + ((32 w) << 16) + first column.
// Complete with wait_st() before other threads may rely on the data.
__device__ __forceinline__ void st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
        "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// This thread's earlier tcgen05.st have completed.
__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// The mbarrier in shared memory at `bar_smem` receives one arrival once every MMA this thread
// issued before has completed.
__device__ __forceinline__ void commit(uint32_t bar_smem) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_smem)
                 : "memory");
}

// 16 consecutive fp32 columns of one TMEM lane per thread: warp w (of a warpgroup) reads lanes
// 32 w .. 32 w + 31 at `taddr` = base + ((32 w) << 16) + first column.
__device__ __forceinline__ void ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

}  // namespace umma
}  // namespace focr
