// Internal launcher of the R-SWA decode attention (see rswa.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace focr {

// Key chunks of one launch: S chunks of `chunk` keys over the Rcap + 128 possible keys.
struct RswaPlan {
    int S = 1, chunk = 1;
};
RswaPlan rswa_plan(int B, int Rcap);
size_t rswa_part_bytes(int B, int Rcap);   // the partials' scratch of one launch
cudaError_t launch_rswa(const float* q, const float* k_new, const float* v_new, const float* k_ref,
                        const float* v_ref, const int32_t* ref_len, int Rcap, float* k_ring, float* v_ring,
                        const int32_t* n_gen, int B, float* out, float* part, cudaStream_t st);

}  // namespace focr
