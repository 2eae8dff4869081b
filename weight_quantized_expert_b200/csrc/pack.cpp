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

// Where every code of one item lives.  `fn(matrix, row, col, byte_offset, nibble_slot)` is
// called once per weight of the item: matrix 0 gate / 1 up / 2 down (row, col in that
// matrix), byte_offset from the item block start, nibble_slot in 0..7 (int4) or -1.
template <class Fn>
void visit_item(const ItemGeom& g, int slice, Fn&& fn) {
    const int wt = g.wtype;
    const int fb = frag_bytes(wt), kpv = ksteps_per_vec(wt);
    const int i0 = slice * g.S;
    for (int t = 0; t < g.S / 8; ++t)
        for (int q = 0; q < KSTEPS; ++q)
            for (int L = 0; L < 32; ++L) {
                const int gr = L >> 2, c = L & 3;
                const size_t vec = ((size_t)(t * (KSTEPS / kpv) + q / kpv) * 32 + L) * 16 + (q % kpv) * fb;
                for (int j = 0; j < 8; ++j) {
                    const int trow = gr + 8 * ((j >> 1) & 1);
                    const int col = 16 * q + 2 * c + (j & 1) + 8 * (j >> 2);
                    const int mat = trow < 8 ? 0 : 1;
                    const int row = i0 + 8 * t + (trow & 7);
                    if (wt == FOCR_W_INT4) fn(mat, row, col, vec, nibble_slot(j));
                    else if (wt == FOCR_W_INT8) fn(mat, row, col, vec + j, -1);
                    else fn(mat, row, col, vec + 2 * j, -1);
                }
            }
    const size_t d0 = g.gu_w_bytes + g.gu_s_bytes;
    for (int m = 0; m < OTILES; ++m)
        for (int L = 0; L < 32; ++L) {
            const int gr = L >> 2, c = L & 3;
            const size_t base = d0 + ((size_t)m * 32 + L) * 8;
            if (wt == FOCR_W_BF16) {
                for (int j = 0; j < 4; ++j)
                    fn(2, 16 * m + gr + 8 * (j >> 1), i0 + 2 * c + (j & 1), base + 2 * j, -1);
            } else {
                const int nq = wt == FOCR_W_INT4 ? 2 : 1;
                for (int q = 0; q < nq; ++q)
                    for (int j = 0; j < 8; ++j) {
                        const int row = 16 * m + gr + 8 * ((j >> 1) & 1);
                        const int col = i0 + 16 * q + 2 * c + (j & 1) + 8 * (j >> 2);
                        if (wt == FOCR_W_INT4) fn(2, row, col, base + 4 * q, nibble_slot(j));
                        else fn(2, row, col, base + j, -1);
                    }
            }
        }
}

// GU scale slot of (tile t, group gi, tile-row gr, matrix 0 gate / 1 up), in floats.
inline size_t gu_scale_index(int ngk, int t, int gi, int gr, int mat) {
    return ((size_t)(t * ngk + gi) * 8 + gr) * 2 + mat;
}

}  // namespace

namespace {

// One block (128 rows x 64 input columns, K-block kb) of the tensor-core layout (common.cuh).
// row_of(r) -> (matrix, row) of block row r.
// f32 -> f16 bits, round to nearest even; finite values beyond the f16 range saturate to
// +-65504 (no weight of a supported model comes near it), NaN stays NaN and +-inf stays inf.
uint16_t host_f32_to_f16(float f) {
    uint32_t x;
    std::memcpy(&x, &f, 4);
    const uint32_t sign = (x >> 16) & 0x8000u, ax = x & 0x7FFFFFFFu;
    if (ax >= 0x7F800000u) return (uint16_t)(sign | (ax > 0x7F800000u ? 0x7E00u : 0x7C00u));
    if (ax >= 0x477FF000u) return (uint16_t)(sign | 0x7BFFu);   // >= 65520 would round to inf
    if (ax < 0x38800000u) {                                     // below 2^-14: a subnormal f16 (or zero)
        float af;
        std::memcpy(&af, &ax, 4);
        return (uint16_t)(sign | (uint32_t)std::nearbyint(af * 16777216.0f));   // units of 2^-24
    }
    uint32_t h = ((((ax >> 23) - 127u + 15u) << 10) | ((ax & 0x7FFFFFu) >> 13));
    const uint32_t rem = ax & 0x1FFFu;
    if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) h += 1u;
    return (uint16_t)(sign | h);
}

// One tensor-core block; 16-bit weights are written as bf16, or as f16 when `f16` (the gate/up
// operands of the tensor-core kernel are f16).
template <class RowOf>
void tc_block(const Quantised* const* m3, const int64_t* cols3, const TcGeom& g, int kb, RowOf&& row_of,
              uint8_t* blk, bool f16) {
    const int wt = g.wtype;
    std::memset(blk, 0, g.blk);
    if (wt == FOCR_W_BF16) {
        for (int r = 0; r < TC_M; ++r) {
            int mat;
            int64_t row;
            row_of(r, mat, row);
            const Quantised& m = *m3[mat];
            for (int k = 0; k < TC_KB; ++k) {
                uint16_t v = m.b[(size_t)(row * cols3[mat] + kb * TC_KB + k)];
                if (f16) {
                    const uint32_t u = (uint32_t)v << 16;
                    float fv;
                    std::memcpy(&fv, &u, 4);
                    v = host_f32_to_f16(fv);
                }
                const size_t off = ((size_t)(r / 8) * 8 + k / 8) * 128 + (size_t)(r % 8) * 16 + (size_t)(k % 8) * 2;
                std::memcpy(blk + off, &v, 2);
            }
        }
        return;
    }
    const int spk = tc_spk(g.group);
    const uint32_t rb = tc_row_bytes(wt);
    float* sc = reinterpret_cast<float*>(blk + (size_t)TC_M * rb);
    for (int r = 0; r < TC_M; ++r) {
        int mat;
        int64_t row;
        row_of(r, mat, row);
        const Quantised& m = *m3[mat];
        const int64_t c0 = (int64_t)kb * TC_KB;
        for (int k = 0; k < TC_KB; ++k) {
            const int q = m.q[(size_t)(row * cols3[mat] + c0 + k)];
            const int kc = k / 8, e = k % 8;
            const int pair = kc & 3, word = kc >> 2;
            if (wt == FOCR_W_INT4) {
                const int nib = (e >> 1) + 4 * (e & 1);
                uint8_t* wp = blk + (size_t)r * rb + pair * 8 + word * 4;
                uint32_t w;
                std::memcpy(&w, wp, 4);
                w |= (uint32_t)((q + 8) & 0xF) << (4 * nib);
                std::memcpy(wp, &w, 4);
            } else {
                blk[(size_t)r * rb + pair * 16 + word * 8 + e] = (uint8_t)(q + 128);
            }
        }
        for (int h = 0; h < spk; ++h) {
            const int64_t col = c0 + (int64_t)h * (TC_KB / spk);
            sc[r * spk + h] = m.s[(size_t)(row * m.ng + col / g.group)];
        }
    }
}

void tc_pack(const Quantised& qg, const Quantised& qu, const Quantised& qd, const TcGeom& g, uint8_t* gu,
             uint8_t* dn) {
    const Quantised* m3[3] = {&qg, &qu, &qd};
    const int64_t cols3[3] = {H, H, g.inter};
    for (int p = 0; p < g.tiles; ++p)
        for (int kb = 0; kb < TC_KBH; ++kb)
            tc_block(m3, cols3, g, kb,
                     [&](int r, int& mat, int64_t& row) {
                         mat = (r >> 3) & 1;                      // rows 16 j + 8 h + r': h = 1 is up
                         row = (int64_t)TC_KB * p + 8 * (r >> 4) + (r & 7);
                     },
                     gu + tc_block_index(g.tiles, TC_KBH, p, kb, g.grp) * g.blk, true);
    for (int mt = 0; mt < TC_MT; ++mt)
        for (int kb = 0; kb < g.tiles; ++kb)
            tc_block(m3, cols3, g, kb,
                     [&](int r, int& mat, int64_t& row) {
                         mat = 2;
                         row = (int64_t)TC_M * mt + r;
                     },
                     dn + tc_block_index(TC_MT, g.tiles, mt, kb, g.grp) * g.blk, false);
}

}  // namespace

// Pack one SwiGLU weight set (gate/up [inter, H], down [H, inter]) into item blocks and, when
// tc_gu/tc_dn are given, into the tensor-core layout with tile groups of tc_grp as well (one
// quantisation for both).
void host_pack_set(const float* gate, const float* up, const float* down, const ItemGeom& g, uint8_t* items,
                   float* dscale, uint8_t* tc_gu, uint8_t* tc_dn, int tc_grp) {
    const int wt = g.wtype;
    const Quantised qg = quantise(gate, g.inter, H, wt, g.group);
    const Quantised qu = quantise(up, g.inter, H, wt, g.group);
    const Quantised qd = quantise(down, H, g.inter, wt, g.group);
    if (tc_gu && tc_dn) tc_pack(qg, qu, qd, make_tc_geom(wt, g.group, g.inter, tc_grp), tc_gu, tc_dn);
    const Quantised* m3[3] = {&qg, &qu, &qd};
    const int64_t cols3[3] = {H, H, g.inter};
    const int ngk = is_quant(wt) ? H / g.group : 0;
    for (int sl = 0; sl < g.slices; ++sl) {
        uint8_t* blk = items + (size_t)sl * g.item_bytes;
        std::memset(blk, 0, g.item_bytes);
        visit_item(g, sl, [&](int mat, int row, int col, size_t off, int slot) {
            const Quantised& m = *m3[mat];
            const size_t e = (size_t)row * cols3[mat] + col;
            if (wt == FOCR_W_INT4) {
                const uint32_t code = (uint32_t)((m.q[e] + 8) & 0xF);
                uint32_t w;
                std::memcpy(&w, blk + off, 4);
                w |= code << (4 * slot);
                std::memcpy(blk + off, &w, 4);
            } else if (wt == FOCR_W_INT8) {
                blk[off] = (uint8_t)(m.q[e] + 128);
            } else {
                std::memcpy(blk + off, &m.b[e], 2);
            }
        });
        if (is_quant(wt)) {
            float* sc = reinterpret_cast<float*>(blk + g.gu_w_bytes);
            const int i0 = sl * g.S;
            for (int t = 0; t < g.S / 8; ++t)
                for (int gi = 0; gi < ngk; ++gi)
                    for (int gr = 0; gr < 8; ++gr) {
                        const int64_t row = i0 + 8 * t + gr;
                        sc[gu_scale_index(ngk, t, gi, gr, 0)] = qg.s[(size_t)(row * qg.ng + gi)];
                        sc[gu_scale_index(ngk, t, gi, gr, 1)] = qu.s[(size_t)(row * qu.ng + gi)];
                    }
        }
    }
    if (is_quant(wt)) {
        const int ngd = (g.inter + g.group - 1) / g.group;
        for (int grp = 0; grp < ngd; ++grp)
            for (int h = 0; h < H; ++h) dscale[(size_t)grp * H + h] = qd.s[(size_t)(h * qd.ng + grp)];
    }
}

// Recover the canonical codes/scales of one matrix (0 gate, 1 up, 2 down) of a set.
void host_unpack_matrix(const uint8_t* items, const float* dscale, const ItemGeom& g, int which, int8_t* q,
                        uint16_t* b16, float* s) {
    const int wt = g.wtype;
    const int ngk = is_quant(wt) ? H / g.group : 0;
    const int64_t cols = which == 2 ? g.inter : H;
    for (int sl = 0; sl < g.slices; ++sl) {
        const uint8_t* blk = items + (size_t)sl * g.item_bytes;
        visit_item(g, sl, [&](int mat, int row, int col, size_t off, int slot) {
            if (mat != which) return;
            const size_t e = (size_t)row * cols + col;
            if (wt == FOCR_W_INT4) {
                uint32_t w;
                std::memcpy(&w, blk + off, 4);
                q[e] = (int8_t)((int)((w >> (4 * slot)) & 0xF) - 8);
            } else if (wt == FOCR_W_INT8) {
                q[e] = (int8_t)((int)blk[off] - 128);
            } else {
                std::memcpy(&b16[e], blk + off, 2);
            }
        });
        if (which < 2 && is_quant(wt)) {
            const float* sc = reinterpret_cast<const float*>(blk + g.gu_w_bytes);
            const int i0 = sl * g.S;
            for (int t = 0; t < g.S / 8; ++t)
                for (int gi = 0; gi < ngk; ++gi)
                    for (int gr = 0; gr < 8; ++gr)
                        s[(int64_t)(i0 + 8 * t + gr) * ngk + gi] = sc[gu_scale_index(ngk, t, gi, gr, which)];
        }
    }
    if (which == 2 && is_quant(wt)) {
        const int ngd = (g.inter + g.group - 1) / g.group;
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

// lm_head codes: tile r (16 rows), k-step q, lane L = 4 gr + c hold the A-fragment
// elements e0..e7 of rows 16r+gr, 16r+gr+8 and columns 16q+2c(+1), 16q+2c+8(+9), two
// k-steps per 16-byte lane vector, offset-binary (q + 128).
static size_t lm_code_offset(int64_t row, int col) {
    const int64_t r = row / 16;
    const int rr = (int)(row % 16);
    const int gr = rr & 7, hi = rr >> 3;
    const int q = col / 16, kc = col % 16;
    const int c = (kc & 7) >> 1, odd = kc & 1, up = kc >> 3;
    const int L = 4 * gr + c;
    const int j = odd + 2 * hi + 4 * up;   // inverse of the e0..e7 element order
    return ((size_t)(r * (KSTEPS / 2) + q / 2) * 32 + L) * 16 + (q % 2) * 8 + j;
}

void host_pack_lm_head(const float* w, int64_t V, uint8_t* codes, float* scales) {
    const int64_t tiles = V / 16;
    parallel_for((int)tiles, [&](int r) {
        std::vector<int8_t> q(16 * H);
        host_quantize(w + (size_t)r * 16 * H, 16, H, H, 8, q.data(), scales + (size_t)r * 16);
        for (int rr = 0; rr < 16; ++rr)
            for (int col = 0; col < H; ++col)
                codes[lm_code_offset((int64_t)r * 16 + rr, col)] = (uint8_t)(q[(size_t)rr * H + col] + 128);
    });
}

void host_unpack_lm_head(const uint8_t* codes, int64_t V, int8_t* q) {
    parallel_for((int)(V / 16), [&](int r) {
        for (int rr = 0; rr < 16; ++rr)
            for (int col = 0; col < H; ++col) {
                const int64_t row = (int64_t)r * 16 + rr;
                q[(size_t)row * H + col] = (int8_t)((int)codes[lm_code_offset(row, col)] - 128);
            }
    });
}

}  // namespace focr

namespace focr {

int64_t w8a8_code_offset(int64_t row, int64_t col, int64_t KS) {
    const int64_t tile = row / 16, rr = row % 16, q = col / 32, kl = col % 32;
    const int64_t gr = rr % 8, hi_row = rr / 8, half = kl / 16, c = (kl % 16) / 4, e = kl % 4;
    const int64_t lane = 4 * gr + c, reg = 2 * half + hi_row;
    return ((tile * KS + q) * 32 + lane) * 16 + reg * 4 + e;
}

void host_pack_w8a8(const float* w, int64_t N, int64_t K, uint8_t* codes, float* scales) {
    const int64_t KS = (K + 31) / 32, tiles = (N + 15) / 16;
    std::memset(codes, 0, (size_t)(tiles * KS * 512));
    std::memset(scales, 0, sizeof(float) * (size_t)(tiles * 16));
    parallel_for((int)tiles, [&](int r) {
        const int64_t r0 = (int64_t)r * 16, rows = std::min<int64_t>(16, N - r0);
        std::vector<int8_t> q((size_t)(rows * K));
        host_quantize(w + r0 * K, rows, K, (int)K, 8, q.data(), scales + r0);
        for (int64_t rr = 0; rr < rows; ++rr)
            for (int64_t col = 0; col < K; ++col)
                codes[w8a8_code_offset(r0 + rr, col, KS)] = (uint8_t)q[(size_t)(rr * K + col)];
    });
}

void host_unpack_w8a8(const uint8_t* codes, int64_t N, int64_t K, int8_t* q) {
    const int64_t KS = (K + 31) / 32;
    parallel_for((int)((N + 15) / 16), [&](int r) {
        const int64_t r1 = std::min<int64_t>(N, (int64_t)r * 16 + 16);
        for (int64_t row = (int64_t)r * 16; row < r1; ++row)
            for (int64_t col = 0; col < K; ++col) q[row * K + col] = (int8_t)codes[w8a8_code_offset(row, col, KS)];
    });
}

}  // namespace focr
