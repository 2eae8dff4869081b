// Host-side quantiser and device-layout packer for libfocr_moe.
//
// Quantisation follows "Four bits, one shared scale" (frankenocr.pages.dev): an int4
// weight is a two's-complement nibble sharing one f32 scale with its group of g
// consecutive input-axis elements of one output row.  Scale rule: s = max|w| / Q in
// one fp32 division (Q = 7 int4, 127 int8); q = round-half-even(w / s) clamped;
// an all-zero group has s = 0 and q = 0.  bf16 weights round to nearest-even.
// The layout written here is described in common.cuh (item blocks for bulk copies
// and 16-byte shared-memory loads).
#include <algorithm>
#include <atomic>
#include <cmath>
#include <functional>
#include <cstring>
#include <thread>
#include <vector>

#include "pack.h"

namespace focr {

uint16_t host_f32_to_bf16(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    const uint32_t lsb = (u >> 16) & 1u;
    return (uint16_t)((u + 0x7FFFu + lsb) >> 16);
}

void host_quantize(const float* w, int64_t rows, int64_t cols, int group, int bits, int8_t* q, float* s) {
    const float Q = bits == 4 ? 7.0f : 127.0f;
    const float lo = bits == 4 ? -8.0f : -127.0f;
    const int64_t ng = (cols + group - 1) / group;
    for (int64_t r = 0; r < rows; ++r) {
        const float* wr = w + r * cols;
        for (int64_t g = 0; g < ng; ++g) {
            const int64_t c0 = g * group;
            const int64_t c1 = std::min<int64_t>(cols, c0 + group);
            float amax = 0.0f;
            for (int64_t c = c0; c < c1; ++c) amax = std::max(amax, std::fabs(wr[c]));
            const float sc = amax / Q;
            s[r * ng + g] = sc;
            for (int64_t c = c0; c < c1; ++c) {
                float v = 0.0f;
                if (sc != 0.0f) {
                    v = std::nearbyint(wr[c] / sc);
                    v = std::min(Q, std::max(lo, v));
                }
                q[r * cols + c] = (int8_t)v;
            }
        }
    }
}

namespace {

struct Quantised {
    std::vector<int8_t> q;    // [rows, cols]
    std::vector<float> s;     // [rows, ng]
    std::vector<uint16_t> b;  // bf16 bits [rows, cols]
    int64_t ng = 0;
};

Quantised quantise(const float* w, int64_t rows, int64_t cols, int wtype, int group) {
    Quantised out;
    if (wtype == FOCR_W_BF16) {
        out.b.resize((size_t)(rows * cols));
        for (int64_t i = 0; i < rows * cols; ++i) out.b[(size_t)i] = host_f32_to_bf16(w[i]);
    } else {
        out.ng = (cols + group - 1) / group;
        out.q.resize((size_t)(rows * cols));
        out.s.resize((size_t)(rows * out.ng));
        host_quantize(w, rows, cols, group, wtype == FOCR_W_INT4 ? 4 : 8, out.q.data(), out.s.data());
    }
    return out;
}

// write the 8 input columns [c, c+8) of one row in the unit encoding of `wtype`
void put_unit(const Quantised& m, int wtype, int64_t cols, int64_t row, int64_t c, uint8_t* dst) {
    if (wtype == FOCR_W_INT4) {
        const int8_t* q = m.q.data() + row * cols + c;
        for (int b = 0; b < 4; ++b)
            dst[b] = (uint8_t)(((q[2 * b] + 8) & 0xF) | (((q[2 * b + 1] + 8) & 0xF) << 4));
    } else if (wtype == FOCR_W_INT8) {
        const int8_t* q = m.q.data() + row * cols + c;
        for (int b = 0; b < 8; ++b) dst[b] = (uint8_t)(q[b] + 128);
    } else {
        std::memcpy(dst, m.b.data() + row * cols + c, 16);
    }
}

void get_unit(int wtype, const uint8_t* src, int8_t* q8, uint16_t* b16) {
    if (wtype == FOCR_W_INT4) {
        for (int b = 0; b < 4; ++b) {
            q8[2 * b] = (int8_t)((src[b] & 0xF) - 8);
            q8[2 * b + 1] = (int8_t)((src[b] >> 4) - 8);
        }
    } else if (wtype == FOCR_W_INT8) {
        for (int b = 0; b < 8; ++b) q8[b] = (int8_t)((int)src[b] - 128);
    } else {
        std::memcpy(b16, src, 16);
    }
}

}  // namespace

// Pack one SwiGLU weight set (gate/up [inter, H], down [H, inter]) into item blocks.
void host_pack_set(const float* gate, const float* up, const float* down, const ItemGeom& g, uint8_t* items,
                   float* dscale) {
    const int wt = g.wtype;
    const Quantised qg = quantise(gate, g.inter, H, wt, g.group);
    const Quantised qu = quantise(up, g.inter, H, wt, g.group);
    const Quantised qd = quantise(down, H, g.inter, wt, g.group);
    const int ub = unit_row_bytes(wt);
    const int ngk = is_quant(wt) ? H / g.group : 0;
    for (int sl = 0; sl < g.slices; ++sl) {
        uint8_t* blk = items + (size_t)sl * g.item_bytes;
        std::memset(blk, 0, g.item_bytes);
        const int i0 = sl * g.S;
        for (int quad = 0; quad < g.S / 2; ++quad) {
            for (int u = 0; u < UNITS; ++u) {
                for (int r = 0; r < 4; ++r) {
                    const Quantised& m = (r < 2) ? qg : qu;
                    const int64_t row = i0 + 2 * quad + (r & 1);
                    put_unit(m, wt, H, row, 8 * u, blk + ((size_t)(quad * UNITS + u) * 4 + r) * ub);
                }
            }
            if (is_quant(wt)) {
                float* sc = (float*)(blk + g.gu_w_bytes) + (size_t)quad * ngk * 4;
                for (int grp = 0; grp < ngk; ++grp)
                    for (int r = 0; r < 4; ++r) {
                        const Quantised& m = (r < 2) ? qg : qu;
                        const int64_t row = i0 + 2 * quad + (r & 1);
                        sc[grp * 4 + r] = m.s[(size_t)(row * m.ng + grp)];
                    }
            }
        }
        uint8_t* dw = blk + g.gu_w_bytes + g.gu_s_bytes;
        for (int h = 0; h < H; ++h) {
            uint8_t* dst = dw + (size_t)h * 16;
            // the row slice down[h, i0 : i0 + S] is S codes = 16 bytes in every format
            for (int c = 0; c < g.S; c += 8) put_unit(qd, wt, g.inter, h, i0 + c, dst + (c / 8) * ub);
        }
    }
    if (is_quant(wt)) {
        const int ngd = g.inter / g.group;
        for (int grp = 0; grp < ngd; ++grp)
            for (int h = 0; h < H; ++h) dscale[(size_t)grp * H + h] = qd.s[(size_t)(h * qd.ng + grp)];
    }
}

// Recover the canonical codes/scales of one matrix (0 gate, 1 up, 2 down) of a set.
void host_unpack_matrix(const uint8_t* items, const float* dscale, const ItemGeom& g, int which, int8_t* q,
                        uint16_t* b16, float* s) {
    const int wt = g.wtype;
    const int ub = unit_row_bytes(wt);
    const int ngk = is_quant(wt) ? H / g.group : 0;
    int8_t q8[8];
    uint16_t bb[8];
    for (int sl = 0; sl < g.slices; ++sl) {
        const uint8_t* blk = items + (size_t)sl * g.item_bytes;
        const int i0 = sl * g.S;
        if (which < 2) {
            for (int quad = 0; quad < g.S / 2; ++quad)
                for (int rr = 0; rr < 2; ++rr) {
                    const int r = which * 2 + rr;
                    const int64_t row = i0 + 2 * quad + rr;
                    for (int u = 0; u < UNITS; ++u) {
                        get_unit(wt, blk + ((size_t)(quad * UNITS + u) * 4 + r) * ub, q8, bb);
                        for (int j = 0; j < 8; ++j) {
                            if (is_quant(wt)) q[row * H + 8 * u + j] = q8[j];
                            else b16[row * H + 8 * u + j] = bb[j];
                        }
                    }
                    if (is_quant(wt)) {
                        const float* sc = (const float*)(blk + g.gu_w_bytes) + (size_t)quad * ngk * 4;
                        for (int grp = 0; grp < ngk; ++grp) s[row * ngk + grp] = sc[grp * 4 + r];
                    }
                }
        } else {
            const uint8_t* dw = blk + g.gu_w_bytes + g.gu_s_bytes;
            for (int h = 0; h < H; ++h)
                for (int c = 0; c < g.S; c += 8) {
                    get_unit(wt, dw + (size_t)h * 16 + (c / 8) * ub, q8, bb);
                    for (int j = 0; j < 8; ++j) {
                        if (is_quant(wt)) q[(int64_t)h * g.inter + i0 + c + j] = q8[j];
                        else b16[(int64_t)h * g.inter + i0 + c + j] = bb[j];
                    }
                }
        }
    }
    if (which == 2 && is_quant(wt)) {
        const int ngd = g.inter / g.group;
        for (int grp = 0; grp < ngd; ++grp)
            for (int h = 0; h < H; ++h) s[(int64_t)h * ngd + grp] = dscale[(size_t)grp * H + h];
    }
}

void parallel_for(int n, const std::function<void(int)>& fn) {
    unsigned hw = std::thread::hardware_concurrency();
    int nt = (int)std::max(1u, std::min<unsigned>(hw, 32u));
    nt = std::min(nt, n);
    std::vector<std::thread> th;
    std::atomic<int> next{0};
    for (int t = 0; t < nt; ++t)
        th.emplace_back([&] {
            for (int i = next++; i < n; i = next++) fn(i);
        });
    for (auto& t : th) t.join();
}

}  // namespace focr
