// Warp-level tensor-core fragment helpers shared by the decode kernels (mma.sync
// m16n8k16 / m16n8k8, f16 and bf16 operands, fp32 accumulators) and the register-level
// dequantisation of int4 / int8 codes into exact f16 A fragments.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace focr {

struct Frag4 {
    uint32_t r[4];
};

__device__ __forceinline__ void mma16816(float (&d)[4], const Frag4& a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a.r[0]), "r"(a.r[1]), "r"(a.r[2]), "r"(a.r[3]), "r"(b0), "r"(b1));
}

// d = A B (the accumulator input is zero)
__device__ __forceinline__ void mma16816_zc(float (&d)[4], const Frag4& a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a.r[0]), "r"(a.r[1]), "r"(a.r[2]), "r"(a.r[3]), "r"(b0), "r"(b1), "f"(0.f));
}

__device__ __forceinline__ void mma1688(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(b0));
}

__device__ __forceinline__ void mma16816_bf16(float (&d)[4], const uint4& a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma1688_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(b0));
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t hsub2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

constexpr uint32_t H2_1032 = 0x64086408u;   // (1032, 1032)
constexpr uint32_t H2_1152 = 0x64806480u;   // (1152, 1152)
constexpr uint32_t H2_1_16 = 0x2C002C00u;   // (1/16, 1/16)
constexpr uint32_t H2_M72 = 0xD480D480u;    // (-72, -72)

// 8 int4 codes (offset-binary, slots 0,4 | 1,5 | 2,6 | 3,7) -> A fragment, exact q in f16.
// (w & mask) | 0x6400 reads as 1024 + n (low nibble) or 1024 + 16 n (second nibble).
__device__ __forceinline__ Frag4 dq_int4(uint32_t w) {
    Frag4 f;
    const uint32_t w8 = w >> 8;
    f.r[0] = hsub2((w & 0x000F000Fu) | 0x64006400u, H2_1032);
    f.r[1] = hfma2((w & 0x00F000F0u) | 0x64006400u, H2_1_16, H2_M72);
    f.r[2] = hsub2((w8 & 0x000F000Fu) | 0x64006400u, H2_1032);
    f.r[3] = hfma2((w8 & 0x00F000F0u) | 0x64006400u, H2_1_16, H2_M72);
    return f;
}

// 8 int8 codes (offset-binary bytes e0..e7) -> A fragment; 0x64bb reads as 1024 + bb
__device__ __forceinline__ Frag4 dq_int8(uint32_t w0, uint32_t w1) {
    Frag4 f;
    f.r[0] = hsub2(__byte_perm(w0, 0x64646464u, 0x4140), H2_1152);
    f.r[1] = hsub2(__byte_perm(w0, 0x64646464u, 0x4342), H2_1152);
    f.r[2] = hsub2(__byte_perm(w1, 0x64646464u, 0x4140), H2_1152);
    f.r[3] = hsub2(__byte_perm(w1, 0x64646464u, 0x4342), H2_1152);
    return f;
}

__device__ __forceinline__ uint32_t f32x2_to_bf16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// bf16 hi + lo split of two fp32 values: returns {hi pair, lo pair}
__device__ __forceinline__ uint2 split_bf16x2(float a, float b) {
    const uint32_t hi = f32x2_to_bf16x2(a, b);
    const float ra = a - __uint_as_float(hi << 16), rb = b - __uint_as_float(hi & 0xFFFF0000u);
    return make_uint2(hi, f32x2_to_bf16x2(ra, rb));
}

}  // namespace focr
