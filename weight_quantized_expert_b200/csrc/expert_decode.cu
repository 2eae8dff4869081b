// Grouped expert kernel for decode-sized batches: the shared expert and every
// selected routed expert, SwiGLU fused, weights dequantised in registers straight
// into 16x8x16 tensor-core fragments (f16 operands, fp32 accumulation).
//
// Sources: frankenocr.pages.dev, "One forward pass", step 6 (64 routed experts + 2 fused
// shared experts, top-6 without renormalisation); franken_ocr README, "Architecture"
// (each expert 1280 -> 896 SiLU-gated); "Four bits, one shared scale" (int4 nibble +
// f32 group scale; int8 and bf16 formats).
//
// Work: an "item" is one slice of S intermediate rows of one expert (common.cuh; ~60-77
// KB).  Items are numbered shared-expert slices first, then the slices of every expert
// that received tokens (ascending id); CTA b of a persistent grid (one per SM) takes
// items b, b+G, ...  A producer warp streams item blocks into a two-slot shared-memory
// ring with bulk async copies (cp.async.bulk + mbarrier) and publishes each item's
// expert id next to it; 16 consumer warps compute:
//   phase 1  [g; u] = [G; U]_slice x  -- warp (tile, k-part): mma.sync m16n8k16; int4/int8
//            codes become exact f16 values in registers and are multiplied by their group
//            scale (f16); bf16 weights feed bf16 MMAs as stored; k-parts summed in shared memory
//   swiglu   a = silu(g) * u * w_route  (fp32, then f16 phase-2 B fragments)
//   phase 2  y = D[:, slice] a          -- warp owns 5 of the 80 output tiles
// Tokens are the 8 columns of the n8 fragments.  With T <= 8 every item uses the same
// columns (the batch), routed weights of tokens that did not pick the expert are 0, and
// the layer output stays in registers across all of a CTA's items: one flush of atomics
// at the end.  With T > 8 items walk their tokens in groups of 8 (gathered) and add every
// group's result into the output with atomics.
// The shared-expert slices need no routing, so they run while the router kernel is still
// working (programmatic dependent launch); routed items start after griddepcontrol.wait,
// and no output is added before it (the router zeroes `out`).  Every mbarrier wait is
// bounded in time; on expiry the kernel records an error word and stops.
//
// Precision: int4/int8 weights enter the MMA as f16(q * s) (one rounding, relative 2^-11;
// scales below f16's normal range lose bits) with x and a rounded to f16; bf16 weights
// enter unchanged and x and a are split into bf16 hi + lo parts (two MMAs, about 16
// significant bits); every product accumulates in fp32.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"

namespace focr {
namespace {

constexpr int NCW = 16;                      // consumer warps
constexpr int NCT = NCW * 32;                // consumer threads
constexpr int NTHREADS = NCT + 32;           // + producer warp
constexpr int NSLOT = 2;
constexpr int NTOK = 8;                      // tokens per fragment (n8)
constexpr uint32_t SLOT_BYTES = 76800;       // largest item (int4 g32) + its down scales
constexpr uint32_t DSC_BYTES = H * 4;        // one group's down scales
constexpr int TILES_PER_WARP = OTILES / NCW; // 5
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // 2 s

template <int RW, int SW>
struct SmemLayout {
    static constexpr bool F16 = is_quant(RW) || is_quant(SW);     // some expert uses f16 MMAs
    static constexpr bool BF16 = !is_quant(RW) || !is_quant(SW);  // some expert uses bf16 MMAs
    static constexpr uint32_t slots = 0;
    static constexpr uint32_t xh = slots + NSLOT * SLOT_BYTES;          // [80][32] uint2: f16 x B frags
    static constexpr uint32_t xb = xh + (F16 ? KSTEPS * 32 * 8 : 0);    // [80][32] uint4: bf16 x hi, lo frags
    static constexpr uint32_t red = xb + (BF16 ? KSTEPS * 32 * 16 : 0); // [16 tasks][32] float4
    static constexpr uint32_t ah = red + 16 * 32 * 16;                  // [2][32] uint2: f16 a B frags
    static constexpr uint32_t abf = ah + 2 * 32 * 8;                    // [32] uint2: bf16 a hi, lo frags
    static constexpr uint32_t wn = abf + 32 * 8;                        // [NTOK] f32 route weights
    static constexpr uint32_t tok = wn + NTOK * 4;                      // [NTOK] i32 token ids
    static constexpr uint32_t ridx = tok + NTOK * 4;                    // [NTOK][6] i32 (T <= 8)
    static constexpr uint32_t rw = ridx + NTOK * K * 4;                 // [NTOK][6] f32 (T <= 8)
    static constexpr uint32_t rec = rw + NTOK * K * 4;                  // [NSLOT] i32 expert of the slot's item
    static constexpr uint32_t bars = rec + 16;                          // full[NSLOT], empty[NSLOT]
    static constexpr uint32_t misc = bars + 2 * NSLOT * 8;
    static constexpr uint32_t total = misc + 16;
    static_assert(total <= 232448, "shared memory budget");
};

struct ExpertParams {
    const float* x;
    int T;
    float* out;
    LayerView L;
    RouteView R;
};

// ------------------------------------------------------------------ fragments
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

// ------------------------------------------------------------------ phase 1: gate/up
// QN k-steps starting at q0 of tile t; PH = q0 % (G / 16) is a compile-time phase so every
// group boundary, and the scale register it uses, is known at compile time.
template <int W, int G, int PH>
__device__ __forceinline__ void gate_up_quant(const char* slot, const uint2* xh, float (&tot)[4], int t, int q0,
                                              int lane) {
    constexpr int NT = slice_rows(W) / 8;
    constexpr int KP = NCW / NT;
    constexpr int QN = KSTEPS / KP;
    constexpr int KPV = ksteps_per_vec(W);
    constexpr int SPG = G / 16;
    constexpr int NGK = H / G;
    constexpr int NGW = (PH + QN - 1) / SPG + 1;      // groups this warp touches
    const int gr = lane >> 2;
    const uint4* gw = reinterpret_cast<const uint4*>(slot) + (t * (KSTEPS / KPV) + q0 / KPV) * 32 + lane;
    const uint2* xb = xh + q0 * 32 + lane;
    const float2* gs = reinterpret_cast<const float2*>(slot + gu_w_bytes_of(W)) + (t * NGK + (q0 - PH) / SPG) * 8 + gr;
    uint32_t sg[NGW], su[NGW];   // (gate, gate) and (up, up) scales as f16x2
#pragma unroll
    for (int g = 0; g < NGW; ++g) {
        const float2 v = gs[g * 8];
        sg[g] = f32x2_to_f16x2(v.x, v.x);
        su[g] = f32x2_to_f16x2(v.y, v.y);
    }
    float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};   // even / odd k-steps
#pragma unroll
    for (int qv = 0; qv < QN / KPV; ++qv) {
        const uint4 v = gw[qv * 32];
        const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < KPV; ++j) {
            const int qq = qv * KPV + j;
            const int g = (PH + qq) / SPG;
            const uint2 b = xb[qq * 32];
            Frag4 a;
            if constexpr (W == FOCR_W_INT4) a = dq_int4(vv[j]);
            else a = dq_int8(vv[2 * j], vv[2 * j + 1]);
            a.r[0] = hmul2(a.r[0], sg[g]);
            a.r[1] = hmul2(a.r[1], su[g]);
            a.r[2] = hmul2(a.r[2], sg[g]);
            a.r[3] = hmul2(a.r[3], su[g]);
            if (qq & 1) mma16816(acc1, a, b.x, b.y);
            else mma16816(acc0, a, b.x, b.y);
        }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) tot[r] = acc0[r] + acc1[r];
}

template <int W, int G>
__device__ __forceinline__ void phase_gate_up(const char* slot, const uint2* xh, const uint4* xbf, float4* red,
                                              int warp, int lane) {
    constexpr int NT = slice_rows(W) / 8;       // tiles per item
    constexpr int KP = NCW / NT;                // k-parts
    constexpr int QN = KSTEPS / KP;             // k-steps per warp
    const int t = warp % NT, part = warp / NT;
    const int q0 = part * QN;
    float tot[4];
    if constexpr (!is_quant(W)) {
        // bf16 weights as stored; x as bf16 hi + lo
        const uint4* gw = reinterpret_cast<const uint4*>(slot) + (t * KSTEPS + q0) * 32 + lane;
        const uint4* xb = xbf + q0 * 32 + lane;
        float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int q = 0; q < QN; ++q) {
            const uint4 a = gw[q * 32];
            const uint4 b = xb[q * 32];
            if (q & 1) {
                mma16816_bf16(acc1, a, b.x, b.y);
                mma16816_bf16(acc1, a, b.z, b.w);
            } else {
                mma16816_bf16(acc0, a, b.x, b.y);
                mma16816_bf16(acc0, a, b.z, b.w);
            }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) tot[r] = acc0[r] + acc1[r];
    } else {
        constexpr int SPG = G / 16;
        switch (q0 % SPG) {
            case 0: gate_up_quant<W, G, 0>(slot, xh, tot, t, q0, lane); break;
            case 2: if constexpr (SPG > 2) gate_up_quant<W, G, 2 % SPG>(slot, xh, tot, t, q0, lane); break;
            case 4: if constexpr (SPG > 4) gate_up_quant<W, G, 4 % SPG>(slot, xh, tot, t, q0, lane); break;
            default: if constexpr (SPG > 6) gate_up_quant<W, G, 6 % SPG>(slot, xh, tot, t, q0, lane); break;
        }
    }
    red[warp * 32 + lane] = make_float4(tot[0], tot[1], tot[2], tot[3]);
}

// ------------------------------------------------------------------ swiglu -> phase-2 B fragments
template <int W>
__device__ __forceinline__ void swiglu_to_frag(const float4* red, __half* ah, __nv_bfloat16* abf, const float* wn,
                                               int ctid) {
    constexpr int NT = slice_rows(W) / 8;
    constexpr int KP = NCW / NT;
    if (ctid >= NT * 32) return;
    const int t = ctid >> 5, lane = ctid & 31;
    const int gr = lane >> 2, c = lane & 3;
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int p = 0; p < KP; ++p) {
        const float4 v = red[(p * NT + t) * 32 + lane];
        s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
    }
    // s.x, s.y: gate of intermediate 8t+gr for tokens 2c, 2c+1; s.z, s.w: up
    const float a[2] = {s.x / (1.f + __expf(-s.x)) * s.z * wn[2 * c], s.y / (1.f + __expf(-s.y)) * s.w * wn[2 * c + 1]};
    const int i = 8 * t + gr;                     // slice-local intermediate index = k of phase 2
    if constexpr (is_quant(W)) {
        const int q2 = i >> 4, kin = i & 15;
        const int reg = kin >> 3, half = kin & 1, cl = (kin & 7) >> 1;
#pragma unroll
        for (int h = 0; h < 2; ++h)
            ah[((q2 * 32 + 4 * (2 * c + h) + cl) * 2 + reg) * 2 + half] = __float2half_rn(a[h]);
    } else {
        // one 16x8x8 step: lane 4n + i/2 holds k = i in half i % 2 of its hi and lo registers
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const __nv_bfloat16 hi = __float2bfloat16_rn(a[h]);
            const __nv_bfloat16 lo = __float2bfloat16_rn(a[h] - __bfloat162float(hi));
            const int ln = 4 * (2 * c + h) + (i >> 1);
            abf[(ln * 2 + 0) * 2 + (i & 1)] = hi;
            abf[(ln * 2 + 1) * 2 + (i & 1)] = lo;
        }
    }
}

// ------------------------------------------------------------------ phase 2: down
template <int W, int G>
__device__ __forceinline__ void phase_down(const char* slot, const uint2* ah, const uint2* abf, int warp, int lane,
                                           float (&y)[TILES_PER_WARP][4], bool accumulate) {
    const uint2* dw = reinterpret_cast<const uint2*>(slot + gu_w_bytes_of(W) + gu_s_bytes_of(W, G)) + warp * 32 + lane;
    const float* dsc = reinterpret_cast<const float*>(slot + blk_bytes_of(W, G)) + 16 * warp + (lane >> 2);
    uint2 b0 = make_uint2(0u, 0u), b1 = make_uint2(0u, 0u);
    if constexpr (is_quant(W)) b0 = ah[lane];
    else b0 = abf[lane];
    if constexpr (W == FOCR_W_INT4) b1 = ah[32 + lane];
#pragma unroll
    for (int j = 0; j < TILES_PER_WARP; ++j) {
        const uint2 v = dw[j * NCW * 32];
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (W == FOCR_W_INT4) {
            mma16816(d, dq_int4(v.x), b0.x, b0.y);
            mma16816(d, dq_int4(v.y), b1.x, b1.y);
        } else if constexpr (W == FOCR_W_INT8) {
            mma16816(d, dq_int8(v.x, v.y), b0.x, b0.y);
        } else {
            mma1688_bf16(d, v.x, v.y, b0.x);   // a hi
            mma1688_bf16(d, v.x, v.y, b0.y);   // a lo
        }
        float s0 = 1.f, s1 = 1.f;
        if constexpr (is_quant(W)) {
            s0 = dsc[j * NCW * 16];
            s1 = dsc[j * NCW * 16 + 8];
        }
        if (accumulate) {
            y[j][0] = fmaf(d[0], s0, y[j][0]);
            y[j][1] = fmaf(d[1], s0, y[j][1]);
            y[j][2] = fmaf(d[2], s1, y[j][2]);
            y[j][3] = fmaf(d[3], s1, y[j][3]);
        } else {
            y[j][0] = d[0] * s0;
            y[j][1] = d[1] * s0;
            y[j][2] = d[2] * s1;
            y[j][3] = d[3] * s1;
        }
    }
}

__device__ __forceinline__ void consumer_sync() { named_bar_sync(1, NCT); }

// x rows of up to 8 tokens -> B fragments.  Entry (q, lane), n = lane / 4, c = lane % 4, holds
// columns 16q+2c, +1 (first register) and 16q+2c+8, +9 (second) of token column n:
// xh as f16, xb as bf16 hi then lo.  tok[n] < 0 gives a zero column.  All loads of a thread
// are issued before any conversion.
template <bool F16, bool BF16>
__device__ __forceinline__ void build_x_frags(const float* x, const int* tok, uint2* xh, uint4* xb, int ctid) {
    constexpr int PER = KSTEPS * 32 / NCT;   // 5 entries per thread
    float2 lo[PER], hi[PER];
#pragma unroll
    for (int r = 0; r < PER; ++r) {
        const int i = ctid + r * NCT;
        const int q = i >> 5, ln = i & 31;
        const int tk = tok[ln >> 2];
        lo[r] = hi[r] = make_float2(0.f, 0.f);
        if (tk >= 0) {
            const float* row = x + (size_t)tk * H + 16 * q + 2 * (ln & 3);
            lo[r] = __ldg(reinterpret_cast<const float2*>(row));
            hi[r] = __ldg(reinterpret_cast<const float2*>(row + 8));
        }
    }
#pragma unroll
    for (int r = 0; r < PER; ++r) {
        const int i = ctid + r * NCT;
        if constexpr (F16) xh[i] = make_uint2(f32x2_to_f16x2(lo[r].x, lo[r].y), f32x2_to_f16x2(hi[r].x, hi[r].y));
        if constexpr (BF16) {
            const uint2 a = split_bf16x2(lo[r].x, lo[r].y), b = split_bf16x2(hi[r].x, hi[r].y);
            xb[i] = make_uint4(a.x, b.x, a.y, b.y);
        }
    }
}

// one item's phases, dispatched on whether it is a routed or a shared-expert item
template <int RW, int SW, int G>
struct ItemOps {
    static __device__ __forceinline__ void gate_up(bool routed, const char* slot, const uint2* xh, const uint4* xb,
                                                   float4* red, int warp, int lane) {
        if (routed) phase_gate_up<RW, G>(slot, xh, xb, red, warp, lane);
        else phase_gate_up<SW, G>(slot, xh, xb, red, warp, lane);
    }
    static __device__ __forceinline__ void swiglu(bool routed, const float4* red, __half* ah, __nv_bfloat16* abf,
                                                  const float* wn, int ctid) {
        if (routed) swiglu_to_frag<RW>(red, ah, abf, wn, ctid);
        else swiglu_to_frag<SW>(red, ah, abf, wn, ctid);
    }
    static __device__ __forceinline__ void down(bool routed, const char* slot, const uint2* ah, const uint2* abf,
                                                int warp, int lane, float (&y)[TILES_PER_WARP][4], bool accumulate) {
        if (routed) phase_down<RW, G>(slot, ah, abf, warp, lane, y, accumulate);
        else phase_down<SW, G>(slot, ah, abf, warp, lane, y, accumulate);
    }
};

template <int RW, int SW, int G>
__global__ void __launch_bounds__(NTHREADS, 1) expert_decode_kernel(ExpertParams p) {
    using SL = SmemLayout<RW, SW>;
    extern __shared__ __align__(128) char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + SL::bars);
    uint64_t* empty = full + NSLOT;
    volatile int* okflag = reinterpret_cast<volatile int*>(smem + SL::misc);
    int* rec = reinterpret_cast<int*>(smem + SL::rec);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_shared = p.L.sg.slices;
    const bool small = p.T <= NTOK;   // one token group for every item, output kept in registers

    if (tid == 0) {
        for (int s = 0; s < NSLOT; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        fence_barrier_init();
        okflag[0] = 1;   // consumer wait result
        okflag[1] = 0;   // abort
    }
    __syncthreads();

    if (warp == NCW) {
        // ------------------------------------------------------------ producer
        if (lane != 0) return;
        const uint64_t pol = policy_evict_first();
        const ItemGeom& rg = p.L.rg;
        const ItemGeom& sg = p.L.sg;
        constexpr uint32_t r_bytes = blk_bytes_of(RW, G), s_bytes = blk_bytes_of(SW, G);
        // Every item this CTA will stream is prefetched into L2 first, so the ring copies
        // below see L2 latency instead of HBM latency (the ring holds only two items).
        auto prefetch_item = [&](int item) {
            if (item < n_shared) {
                bulk_prefetch_l2(p.L.shared_items + (size_t)item * sg.item_bytes, s_bytes);
                if (is_quant(SW)) bulk_prefetch_l2(p.L.shared_dscale + (size_t)(item * sg.S / G) * H, DSC_BYTES);
            } else {
                const int k = item - n_shared;
                const int a = k / rg.slices, s = k % rg.slices;
                const int e = p.R.active[a];
                bulk_prefetch_l2(p.L.routed_items + ((size_t)e * rg.slices + s) * rg.item_bytes, r_bytes);
                if (is_quant(RW))
                    bulk_prefetch_l2(p.L.routed_dscale + (size_t)e * rg.dscale_expert_floats +
                                         (size_t)(s * rg.S / G) * H,
                                     DSC_BYTES);
            }
        };
        for (int item = blockIdx.x; item < n_shared; item += gridDim.x) prefetch_item(item);
        int n_items = 0x7fffffff;
        bool waited = false;
        int issued = 0;
        for (int it = 0;; ++it) {
            const int item = blockIdx.x + it * gridDim.x;
            if (item >= n_shared && !waited) {
                pdl_wait();
                waited = true;
                n_items = n_shared + p.R.active[E] * rg.slices;
                for (int pi = item; pi < n_items; pi += gridDim.x) prefetch_item(pi);
            }
            if (item >= n_items) break;
            const int slot = it % NSLOT;
            if (it >= NSLOT && !mbar_wait_bounded(&empty[slot], ((it / NSLOT) - 1) & 1, WAIT_LIMIT_NS)) {
                atomicExch(&p.R.ctrl[CTRL_ERROR], DEVERR_EMPTY_WAIT);
                okflag[1] = 1;
                break;
            }
            if (okflag[1]) break;
            const uint8_t* blk;
            const float* dsc = nullptr;
            uint32_t bytes;
            int expert;
            if (item < n_shared) {
                blk = p.L.shared_items + (size_t)item * sg.item_bytes;
                if (is_quant(SW)) dsc = p.L.shared_dscale + (size_t)(item * sg.S / G) * H;
                bytes = s_bytes;
                expert = -1;
            } else {
                const int k = item - n_shared;
                const int a = k / rg.slices, s = k % rg.slices;
                expert = p.R.active[a];
                blk = p.L.routed_items + ((size_t)expert * rg.slices + s) * rg.item_bytes;
                if (is_quant(RW))
                    dsc = p.L.routed_dscale + (size_t)expert * rg.dscale_expert_floats + (size_t)(s * rg.S / G) * H;
                bytes = r_bytes;
            }
            rec[slot] = expert;   // published to the consumers by the full barrier
            char* dst = smem + SL::slots + slot * SLOT_BYTES;
            mbar_arrive_expect_tx(&full[slot], bytes + (dsc ? DSC_BYTES : 0u));
            bulk_g2s(dst, blk, bytes, &full[slot], pol);
            if (dsc) bulk_g2s(dst + bytes, dsc, DSC_BYTES, &full[slot], pol);
            issued = it + 1;
        }
        // never leave copies in flight: wait (bounded) for the last issued ones
        for (int it = max(0, issued - NSLOT); it < issued; ++it)
            (void)mbar_wait_bounded(&full[it % NSLOT], (it / NSLOT) & 1, WAIT_LIMIT_NS);
        return;
    }

    // ---------------------------------------------------------------- consumers
    using Ops = ItemOps<RW, SW, G>;
    const int ctid = tid;
    int* tok = reinterpret_cast<int*>(smem + SL::tok);
    float* wn = reinterpret_cast<float*>(smem + SL::wn);
    int* ridx = reinterpret_cast<int*>(smem + SL::ridx);
    float* rw = reinterpret_cast<float*>(smem + SL::rw);
    uint2* xh = reinterpret_cast<uint2*>(smem + SL::xh);
    uint4* xbf = reinterpret_cast<uint4*>(smem + SL::xb);
    float4* red = reinterpret_cast<float4*>(smem + SL::red);
    __half* ahh = reinterpret_cast<__half*>(smem + SL::ah);
    __nv_bfloat16* abfh = reinterpret_cast<__nv_bfloat16*>(smem + SL::abf);
    const uint2* ah = reinterpret_cast<const uint2*>(smem + SL::ah);
    const uint2* abf = reinterpret_cast<const uint2*>(smem + SL::abf);
    float y[TILES_PER_WARP][4];
#pragma unroll
    for (int j = 0; j < TILES_PER_WARP; ++j) y[j][0] = y[j][1] = y[j][2] = y[j][3] = 0.f;

    if (small) {
        if (ctid < NTOK) tok[ctid] = ctid < p.T ? ctid : -1;
        consumer_sync();
        build_x_frags<SL::F16, SL::BF16>(p.x, tok, xh, xbf, ctid);   // visible after the first item's barrier
    }
    int n_items = 0x7fffffff;
    bool waited = false;
    for (int it = 0;; ++it) {
        const int item = blockIdx.x + it * gridDim.x;
        if (item >= n_shared && !waited) {
            pdl_wait();
            waited = true;
            n_items = n_shared + p.R.active[E] * p.L.rg.slices;
            if (small && ctid < p.T * K) {
                ridx[ctid] = p.R.topk_idx[ctid];
                rw[ctid] = p.R.topk_w[ctid];
            }
            consumer_sync();
        }
        if (item >= n_items) break;
        const int slot = it % NSLOT;
        const uint32_t par = (it / NSLOT) & 1;
        if (ctid == 0) {
            const bool ok = mbar_wait_bounded(&full[slot], par, WAIT_LIMIT_NS);
            if (!ok) {
                atomicExch(&p.R.ctrl[CTRL_ERROR], DEVERR_FULL_WAIT);
                okflag[1] = 1;
            }
            okflag[0] = ok ? 1 : 0;
        }
        consumer_sync();
        if (!okflag[0]) break;
        while (!mbar_try_wait(&full[slot], par)) {
        }
        const int expert = rec[slot];
        const bool routed = expert >= 0;
        const char* sbuf = smem + SL::slots + slot * SLOT_BYTES;

        int ntok = NTOK, seg = 0;
        if (!small && routed) {
            ntok = p.R.counts[expert];
            seg = p.R.offsets[expert];
        } else if (!small) {
            ntok = p.T;
        }
        for (int b0 = 0; b0 < ntok; b0 += NTOK) {
            if (ctid < NTOK) {
                // routing weight of every column for this item's expert (0 if not routed)
                float w = 0.f;
                if (small) {
                    if (ctid < p.T) {
                        if (!routed) {
                            w = 1.f;
                        } else {
#pragma unroll
                            for (int j = 0; j < K; ++j)
                                if (ridx[ctid * K + j] == expert) w = rw[ctid * K + j];
                        }
                    }
                } else {
                    int tk = -1;
                    if (b0 + ctid < ntok) {
                        if (!routed) {
                            tk = b0 + ctid;
                            w = 1.f;
                        } else {
                            const int e = p.R.perm[seg + b0 + ctid];
                            tk = e / K;
                            w = p.R.topk_w[e];
                        }
                    }
                    tok[ctid] = tk;
                }
                wn[ctid] = w;
            }
            if (!small) {
                consumer_sync();
                build_x_frags<SL::F16, SL::BF16>(p.x, tok, xh, xbf, ctid);
                consumer_sync();
            }
            Ops::gate_up(routed, sbuf, xh, xbf, red, warp, lane);
            consumer_sync();
            Ops::swiglu(routed, red, ahh, abfh, wn, ctid);
            consumer_sync();
            if (small) {
                Ops::down(routed, sbuf, ah, abf, warp, lane, y, true);
            } else {
                Ops::down(routed, sbuf, ah, abf, warp, lane, y, false);
                if (!waited) {
                    pdl_wait();   // the router zeroes `out` first
                    waited = true;
                    n_items = n_shared + p.R.active[E] * p.L.rg.slices;
                }
                const int gr = lane >> 2, c = lane & 3;
                const int t0 = tok[2 * c], t1 = tok[2 * c + 1];
#pragma unroll
                for (int j = 0; j < TILES_PER_WARP; ++j) {
                    const int row = 16 * (warp + NCW * j) + gr;
                    if (t0 >= 0) {
                        atomicAdd(p.out + (size_t)t0 * H + row, y[j][0]);
                        atomicAdd(p.out + (size_t)t0 * H + row + 8, y[j][2]);
                    }
                    if (t1 >= 0) {
                        atomicAdd(p.out + (size_t)t1 * H + row, y[j][1]);
                        atomicAdd(p.out + (size_t)t1 * H + row + 8, y[j][3]);
                    }
                }
            }
            consumer_sync();
        }
        if (ctid == 0) mbar_arrive(&empty[slot]);
    }
    if (small && okflag[1] == 0) {
        if (!waited) pdl_wait();   // the router zeroes `out` first
        const int gr = lane >> 2, c = lane & 3;
#pragma unroll
        for (int j = 0; j < TILES_PER_WARP; ++j) {
            const int row = 16 * (warp + NCW * j) + gr;
            if (2 * c < p.T) {
                atomicAdd(p.out + (size_t)(2 * c) * H + row, y[j][0]);
                atomicAdd(p.out + (size_t)(2 * c) * H + row + 8, y[j][2]);
            }
            if (2 * c + 1 < p.T) {
                atomicAdd(p.out + (size_t)(2 * c + 1) * H + row, y[j][1]);
                atomicAdd(p.out + (size_t)(2 * c + 1) * H + row + 8, y[j][3]);
            }
        }
    }
}

int g_num_sms = 0;

template <int RW, int SW, int G>
cudaError_t launch_typed(const ExpertParams& p, cudaStream_t st) {
    static_assert(blk_bytes_of(RW, G) + DSC_BYTES <= SLOT_BYTES && blk_bytes_of(SW, G) + DSC_BYTES <= SLOT_BYTES,
                  "item does not fit a ring slot");
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(expert_decode_kernel<RW, SW, G>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)SmemLayout<RW, SW>::total);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(g_num_sms);
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = SmemLayout<RW, SW>::total;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, expert_decode_kernel<RW, SW, G>, p);
}

}  // namespace

cudaError_t launch_expert_decode(const float* x, int T, const LayerView& L, const RouteView& R, float* out,
                                 cudaStream_t st) {
    if (g_num_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    }
    const ExpertParams p{x, T, out, L, R};
    const int rw = L.rg.wtype, sw = L.sg.wtype;
    const int g = is_quant(rw) ? L.rg.group : (is_quant(sw) ? L.sg.group : 128);
#define FOCR_CASE(A, B, GG) \
    if (rw == A && sw == B && g == GG) return launch_typed<A, B, GG>(p, st);
    FOCR_CASE(FOCR_W_INT4, FOCR_W_BF16, 32)
    FOCR_CASE(FOCR_W_INT4, FOCR_W_BF16, 64)
    FOCR_CASE(FOCR_W_INT4, FOCR_W_BF16, 128)
    FOCR_CASE(FOCR_W_INT4, FOCR_W_INT4, 32)
    FOCR_CASE(FOCR_W_INT4, FOCR_W_INT4, 64)
    FOCR_CASE(FOCR_W_INT4, FOCR_W_INT4, 128)
    FOCR_CASE(FOCR_W_INT4, FOCR_W_INT8, 128)
    FOCR_CASE(FOCR_W_INT8, FOCR_W_INT8, 128)
    FOCR_CASE(FOCR_W_INT8, FOCR_W_BF16, 128)
    FOCR_CASE(FOCR_W_INT8, FOCR_W_INT4, 128)
    FOCR_CASE(FOCR_W_BF16, FOCR_W_BF16, 128)
    FOCR_CASE(FOCR_W_BF16, FOCR_W_INT4, 32)
    FOCR_CASE(FOCR_W_BF16, FOCR_W_INT4, 64)
    FOCR_CASE(FOCR_W_BF16, FOCR_W_INT4, 128)
    FOCR_CASE(FOCR_W_BF16, FOCR_W_INT8, 128)
#undef FOCR_CASE
    return cudaErrorInvalidValue;
}

}  // namespace focr
