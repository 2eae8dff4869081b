// focr_tc_selftest: one tensor-core tile through the same tcgen05 primitives the grouped expert
// kernel uses (umma.cuh), so the instruction and shared-memory descriptors, the TMEM allocation,
// tcgen05.st / tcgen05.ld and the MMA with A from shared memory or from tensor memory can be
// checked against a host GEMM on their own.
//
// D[128][N] = A[128][K] B[N][K]^T in fp32, A and B bf16 (row-major in global memory).  One CTA of
// four warps: the operands are copied into the K-major, unswizzled core-matrix layout in shared
// memory; for a_from_tmem the rows of A are also written into TMEM (thread = row, 32-bit column c
// = elements 2c, 2c + 1); then one thread issues K / 16 MMAs, commits them to an mbarrier, and the
// four warps read the accumulator back with tcgen05.ld.  Every wait is bounded.
#include <cstdio>

#include "common.cuh"
#include "umma.cuh"

namespace focr {
focr_status report_error(focr_status s, const char* msg);
namespace {

constexpr int ST_KMAX = 256, ST_NMAX = 256;

__global__ void __launch_bounds__(128, 1)
    tc_selftest_kernel(const uint16_t* A, const uint16_t* B, int N, int K, int a_from_tmem, float* D, int* err) {
    extern __shared__ __align__(1024) char smem[];
    char* sA = smem;                                // [16 row groups][K/8 k-cores][8 rows][16 B]
    char* sB = smem + 128 * ST_KMAX * 2;            // [N/8 row groups][K/8 k-cores][8 rows][16 B]
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t tbase;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int kc = K / 8;
    // operands into the core-matrix layout: 16-byte pieces (row r, k-core c)
    for (int i = tid; i < 128 * kc; i += 128) {
        const int r = i / kc, c = i % kc;
        *reinterpret_cast<uint4*>(sA + ((r / 8) * kc + c) * 128 + (r % 8) * 16) =
            *reinterpret_cast<const uint4*>(A + (size_t)r * K + c * 8);
    }
    for (int i = tid; i < N * kc; i += 128) {
        const int r = i / kc, c = i % kc;
        *reinterpret_cast<uint4*>(sB + ((r / 8) * kc + c) * 128 + (r % 8) * 16) =
            *reinterpret_cast<const uint4*>(B + (size_t)r * K + c * 8);
    }
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    if (warp == 0) umma::tmem_alloc(smem_u32(&tbase), 512);
    umma::fence_smem_to_async();
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t t0 = tbase;                      // accumulator at columns [0, N); A at [256, 256 + K/2)
    if (a_from_tmem) {
        // thread = row 32 (warp % 4) + lane of A; K/2 columns in chunks of 32
        const int row = 32 * (warp & 3) + lane;
        for (int c0 = 0; c0 < K / 2; c0 += 32) {
            uint32_t r[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = *reinterpret_cast<const uint32_t*>(A + (size_t)row * K + 2 * (c0 + j));
            umma::st32(t0 + ((uint32_t)(32 * (warp & 3)) << 16) + 256u + (uint32_t)c0, r);
        }
        umma::wait_st();
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    if (tid == 0) {
        const uint32_t idesc = umma::idesc_bf16_f32(128, N);
        const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
        for (int j = 0; j < K / 16; ++j) {
            // k-step j: core matrices 2j and 2j + 1 along K; LBO = 128 B between them, SBO = one
            // row group (kc * 128 B)
            const uint64_t bd = umma::sdesc_kmajor(b0 + 256u * j, 128u, (uint32_t)kc * 128u);
            if (a_from_tmem)
                umma::mma_bf16_ts(t0, t0 + 256u + 8u * j, bd, idesc, j > 0);
            else
                umma::mma_bf16(t0, umma::sdesc_kmajor(a0 + 256u * j, 128u, (uint32_t)kc * 128u), bd, idesc, j > 0);
        }
        umma::commit(smem_u32(&bar));
    }
    __syncwarp();
    bool ok = mbar_wait_bounded(&bar, 0, 2000000000ull);
    if (!ok && tid == 0) *err = 1;
    umma::fence_after_sync();
    if (ok) {
        const int row = 32 * (warp & 3) + lane;
        for (int c = 0; c < N; c += 16) {
            float v[16];
            umma::ld16(t0 + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)c, v);
#pragma unroll
            for (int j = 0; j < 16; ++j) D[(size_t)row * N + c + j] = v[j];
        }
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    if (warp == 0) umma::tmem_free(t0, 512);
}

}  // namespace
}  // namespace focr

using namespace focr;

extern "C" focr_status focr_tc_selftest(const uint16_t* a, const uint16_t* b, int32_t n, int32_t k,
                                        int32_t a_from_tmem, float* d, int32_t* err, void* stream) {
    if (!a || !b || !d || !err) return report_error(FOCR_ERR_INVALID_ARG, "NULL argument");
    if (n < 16 || n > ST_NMAX || n % 16 || k < 16 || k > ST_KMAX || k % 64)
        return report_error(FOCR_ERR_INVALID_ARG, "n must be a multiple of 16 in [16, 256], k a multiple of 64 in [64, 256]");
    if (((uintptr_t)a | (uintptr_t)b) % 16) return report_error(FOCR_ERR_INVALID_ARG, "a and b must be 16-byte aligned");
    const int smem = 128 * ST_KMAX * 2 + ST_NMAX * ST_KMAX * 2;
    cudaError_t e = cudaFuncSetAttribute(tc_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) {
        tc_selftest_kernel<<<1, 128, smem, (cudaStream_t)stream>>>(a, b, n, k, a_from_tmem ? 1 : 0, d, err);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) return report_error(FOCR_ERR_CUDA, cudaGetErrorString(e));
    return FOCR_OK;
}
