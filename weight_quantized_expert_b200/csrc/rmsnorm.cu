// Final RMSNorm of the decoder: y = x / sqrt(mean(x^2) + eps) * gamma (gamma = 1 when NULL).
//
// Source: frankenocr.pages.dev, "One forward pass", step 7 (the final RMSNorm feeds the
// lm_head) and franken_ocr README, "Architecture" (final RMSNorm).  One CTA per token;
// the sum of squares accumulates in fp32 (warp shuffles, then across warps).
#include "common.cuh"
#include "lm_head.h"

namespace focr {
namespace {

constexpr int RN_THREADS = 320;   // 1280 / 4 columns per thread

__global__ void __launch_bounds__(RN_THREADS) rmsnorm_kernel(const float* x, const float* gamma, float eps,
                                                             float* out) {
    pdl_wait();
    pdl_launch_dependents();
    __shared__ float part[RN_THREADS / 32];
    const int t = blockIdx.x, tid = threadIdx.x;
    const float4 v = reinterpret_cast<const float4*>(x + (size_t)t * H)[tid];
    float ss = v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((tid & 31) == 0) part[tid >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < RN_THREADS / 32; ++w) tot += part[w];
    const float inv = 1.f / sqrtf(tot / (float)H + eps);
    float4 g = make_float4(1.f, 1.f, 1.f, 1.f);
    if (gamma) g = reinterpret_cast<const float4*>(gamma)[tid];
    reinterpret_cast<float4*>(out + (size_t)t * H)[tid] =
        make_float4(v.x * inv * g.x, v.y * inv * g.y, v.z * inv * g.z, v.w * inv * g.w);
}

}  // namespace

cudaError_t launch_rmsnorm(const float* x, const float* gamma, int T, float eps, float* out, cudaStream_t st) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(T);
    cfg.blockDim = dim3(RN_THREADS);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, rmsnorm_kernel, x, gamma, eps, out);
}

}  // namespace focr
