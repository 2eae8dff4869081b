// Host packer interface (see pack.cpp).
#pragma once

#include <functional>

#include "common.cuh"

namespace focr {

uint16_t host_f32_to_bf16(float f);
void host_quantize(const float* w, int64_t rows, int64_t cols, int group, int bits, int8_t* q, float* s);
void host_pack_set(const float* gate, const float* up, const float* down, const ItemGeom& g, uint8_t* items,
                   float* dscale, uint8_t* tc_gu = nullptr, uint8_t* tc_dn = nullptr, int tc_grp = 1);
void host_unpack_matrix(const uint8_t* items, const float* dscale, const ItemGeom& g, int which, int8_t* q,
                        uint16_t* b16, float* s);
void parallel_for(int n, const std::function<void(int)>& fn);

}  // namespace focr

namespace focr {
// lm_head: int8 codes with one scale per row, fragment-order tiles of 16 rows
// (codes: V * 1280 bytes, scales: V floats)
void host_pack_lm_head(const float* w, int64_t V, uint8_t* codes, float* scales);
void host_unpack_lm_head(const uint8_t* codes, int64_t V, int8_t* q);
}  // namespace focr

namespace focr {
// W8A8 linear: int8 codes with one scale per row (s = max|w| / 127), N rows padded to tiles of
// 16 and K columns padded to k-steps of 32 with zero codes.  For row tile r and k-step q, lane
// L = 4 gr + c of a warp holds the 16 bytes of an m16n8k32 s8 A fragment: {row gr, row gr + 8}
// x {columns 32q + 4c .. +3, columns 32q + 16 + 4c .. +3}, as four 32-bit registers in the
// order (gr, lo), (gr + 8, lo), (gr, hi), (gr + 8, hi).  codes: tiles * KS * 512 bytes.
int64_t w8a8_code_offset(int64_t row, int64_t col, int64_t KS);
void host_pack_w8a8(const float* w, int64_t N, int64_t K, uint8_t* codes, float* scales);
void host_unpack_w8a8(const uint8_t* codes, int64_t N, int64_t K, int8_t* q);
}  // namespace focr
