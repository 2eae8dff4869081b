// Internal launchers for the lm_head GEMV + argmax and the RMSNorm (see lm_head.cu, rmsnorm.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace focr {

size_t lm_head_smem_bytes();
int lm_head_grid();
cudaError_t launch_lm_head(const uint4* codes, const float* scales, const float* x, int T, float* logits,
                           int32_t* argmax, void* ws, cudaStream_t st);
// the same with the ticket word (zero before the launch, left zero), the per-CTA keys
// (sizeof(unsigned long long) x grid x T) and the error word (nullable; set to 1 if still 0 when a
// bounded wait runs out) given separately
cudaError_t launch_lm_head(const uint4* codes, const float* scales, const float* x, int T, float* logits,
                           int32_t* argmax, int* ticket, unsigned long long* keys, int32_t* err, cudaStream_t st);
cudaError_t launch_rmsnorm(const float* x, const float* gamma, int T, float eps, float* out, cudaStream_t st);

}  // namespace focr
