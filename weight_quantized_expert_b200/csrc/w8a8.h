// Internal launchers of the W8A8 GEMV (see w8a8.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace focr {

// Split plan of one GEMV: `S` warps share a 16-row tile's K, each taking `L` k-steps of 32.
struct W8a8Plan {
    int S = 1, L = 1, grid = 1;
};
W8a8Plan w8a8_plan(int64_t tiles, int KS);

// qx (row-major [T, K] int8) and/or qxf (the GEMV's B-fragment order, NBt = ceil(T / 8) token
// groups per k-step) and sx [T]; either code output may be NULL.
cudaError_t launch_w8a8_quantize(const float* x, int T, int K, int8_t* qx, uint32_t* qxf, float* sx,
                                 cudaStream_t st);
// y[T, N] from packed codes (tiles * KS * 512 bytes), row scales, qxf and sx.  acc (int32
// [T, 16 * tiles]) and cnt (uint32 [tiles]) are zero before the launch and left zero; they are
// touched only when the plan splits K (S > 1).  *err is set to 1 if a bounded wait runs out.
cudaError_t launch_w8a8_gemv(const void* codes, const float* sw, int64_t N, int K, const uint32_t* qxf,
                             const float* sx, int T, float* y, int32_t* acc, uint32_t* cnt, uint32_t* err,
                             cudaStream_t st);

}  // namespace focr
