// Decode path for T <= 8 tokens: a gate/up kernel and a down kernel, chained behind the
// router by programmatic dependent launch.
//
// Sources: frankenocr.pages.dev, "One forward pass", step 6 (64 routed experts + 2 fused
// shared experts, top-6 without renormalisation); franken_ocr README, "Architecture"
// (each expert 1280 -> 896 SiLU-gated); "Four bits, one shared scale" (int4 nibble + f32
// group scale; int8 and bf16 formats).
//
// The batch's tokens are the 8 columns of m16n8 tensor-core fragments (tokens that did not
// pick an expert get routing weight 0).  Both kernels read the packed item layout of
// common.cuh.
//
// decode_gu: a unit is one tile of 8 intermediates (8 gate rows over 8 up rows) of the
//   shared set or of a selected expert over a range of input columns (all 1280 for int4,
//   halves for int8, quarters for bf16) -- about 10 KB of codes.  Each warp works alone: it
//   bulk-copies a unit into its own shared-memory buffer (cp.async.bulk, own mbarrier,
//   bounded wait), turns int4/int8 codes into exact f16 A fragments (bf16 weights enter
//   bf16 MMAs with x split into hi + lo), scales each group's fp32 sum, and applies
//   a = silu(g) * u * w_route to whole rows; tiles split along K write each part's sums to
//   its own workspace slot, and the warp that completes a tile (arrival counter) adds the
//   parts in a fixed order and applies it.  a goes to the workspace as the down projection's B
//   fragments.  Shared-set units run while the router is still working, routed units after
//   griddepcontrol.wait; the first unit of every slice prefetches the slice's
//   down-projection bytes into L2.
// decode_down: a unit is one 16-row output tile of one set (shared, or a selected expert)
//   over a chunk of 8-16 slices.  The 8 warps of a CTA take 8 tiles of one chunk; each
//   loads its codes and scales (the first step before waiting on decode_gu), one bulk copy
//   stages the chunk's B fragments of a in shared memory for all of them, and y = D a is
//   scaled per row and group and added into fixed-point sums per output element; the unit that
//   completes a 16-row tile (arrival counter) adds the tile's totals to the output the router
//   initialised, once, and clears them.  So repeated calls give bit-identical outputs.
//
// Precision: int4/int8 codes exact in f16 with fp32 group scales and f16 activations; bf16
// weights exact with bf16 hi + lo activations; fp32 accumulation throughout.
#include "common.cuh"
#include "fragments.cuh"
#include "launch_state.h"

namespace focr {
namespace {

constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // 2 s
constexpr uint32_t GU_SMEM_BUDGET = 200 * 1024;     // leaves room for a small router CTA on the same SM
constexpr int GU_MAX_WARPS = 16;
constexpr int DN_WARPS = 8;                         // down kernel: 8 warps, two CTAs per SM
constexpr int DN_BFRAGS = 16 * 2 * 32;              // B fragments of one chunk (<= 16 slices x 2 steps)

struct SmallParams {
    const float* x;
    int T;
    float* out;
    LayerView L;
    RouteView R;
    int shared_only;
    int deterministic;   // fixed-point output sums (bit-identical repeats) instead of fp32 atomics
};

// Workspace indexing (shared set first, then the routed experts' active slots a = 0..U-1):
// gate/up tile sums and counters, f16 a steps of 16 intermediates, bf16 a steps of 8.
__device__ __forceinline__ int gu_tile_base(bool routed, int a) { return routed ? IS_MAX / 8 + a * (I / 8) : 0; }
__device__ __forceinline__ int a16_base(bool routed, int a) { return routed ? IS_MAX / 16 + a * (I / 16) : 0; }
__device__ __forceinline__ int abf_base(bool routed, int a) { return routed ? IS_MAX / 8 + a * (I / 8) : 0; }

// x of the batch in B-fragment order: for k-step q and lane = 4n + c, columns 16q+2c, +1,
// +8, +9 of token n (zero for n >= T) -- as f16 pairs (xh, the quantised sets' operand)
// and/or fp32 (xs, split into bf16 hi + lo at use by the bf16 sets).  All loads of a
// thread are issued before its stores.
template <int NT, bool F16, bool F32>
__device__ __forceinline__ void build_x(const float* x, int T, uint2* xh, float4* xs, int* err) {
    constexpr int PER = (KSTEPS * 32 + NT - 1) / NT;
    float4 v[PER];
#pragma unroll
    for (int k = 0; k < PER; ++k) {
        const int i = threadIdx.x + k * NT;
        const int q = i >> 5, ln = i & 31, n = ln >> 2, c = ln & 3;
        v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < KSTEPS * 32 && n < T) {
            const float* row = x + (size_t)n * H + 16 * q + 2 * c;
            const float2 lo = __ldg(reinterpret_cast<const float2*>(row));
            const float2 hi = __ldg(reinterpret_cast<const float2*>(row + 8));
            v[k] = make_float4(lo.x, lo.y, hi.x, hi.y);
        }
    }
#pragma unroll
    for (int k = 0; k < PER; ++k) {
        const int i = threadIdx.x + k * NT;
        if (i < KSTEPS * 32) {
            if constexpr (F16) {
                xh[i] = make_uint2(f32x2_to_f16x2(v[k].x, v[k].y), f32x2_to_f16x2(v[k].z, v[k].w));
                if (f16_out_of_range(v[k].x) || f16_out_of_range(v[k].y) || f16_out_of_range(v[k].z) ||
                    f16_out_of_range(v[k].w))
                    atomicExch(err, DEVERR_RANGE);   // beyond the f16 operand range (reported, not fatal)
            }
            if constexpr (F32) xs[i] = v[k];
        }
    }
}

__device__ __forceinline__ uint2 ldg_nc2(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

// routing weight of batch columns 2c and 2c+1 for `expert` (0 when the token did not pick it)
__device__ __forceinline__ float2 route_w(const RouteView& R, int T, int expert, int c) {
    float w[2] = {0.f, 0.f};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int t = 2 * c + h;
        if (t < T) {
#pragma unroll
            for (int j = 0; j < K; ++j)
                if (R.topk_idx[t * K + j] == expert) w[h] = R.topk_w[t * K + j];
        }
    }
    return make_float2(w[0], w[1]);
}

// ------------------------------------------------------------------ gate/up units
// A unit is one tile (8 gate rows over the 8 matching up rows) over QN of the 80 k-steps:
// all of them for int4, halves for int8, quarters for bf16 -- 10 KB of codes either way.
template <int W>
constexpr int gu_parts() {   // column parts of a unit
    return W == FOCR_W_INT4 ? 1 : (W == FOCR_W_INT8 ? 2 : 4);
}

template <int W, int G, int PARTS = gu_parts<W>()>
struct GuUnit {
    static constexpr int KP = PARTS;
    static constexpr int QN = KSTEPS / KP;                 // k-steps per unit
    static constexpr int KPV = ksteps_per_vec(W);          // k-steps per 16-byte lane vector
    static constexpr int NV = QN / KPV;                    // lane vectors per unit (20)
    static constexpr uint32_t W_BYTES = (uint32_t)NV * 32 * 16;
    static constexpr int NG = is_quant(W) ? QN * 16 / G : 0;   // scale groups in the unit
    static constexpr uint32_t S_BYTES = (uint32_t)NG * 64;     // [group][8 gr][gate, up] f32
    static constexpr uint32_t BYTES = W_BYTES + S_BYTES;
    static_assert(!is_quant(W) || (QN * 16) % G == 0, "a unit holds whole scale groups");
};

template <int RW, int SW, int G>
struct GuCfg {
    using RU = GuUnit<RW, G>;
    using SU = GuUnit<SW, G>;
    static constexpr bool F16 = is_quant(RW) || is_quant(SW);    // x as f16 B fragments
    static constexpr bool F32 = !is_quant(RW) || !is_quant(SW);  // x in fp32 (bf16 hi/lo split at use)
    static constexpr uint32_t BUF = ((RU::BYTES > SU::BYTES ? RU::BYTES : SU::BYTES) + 127u) & ~127u;
    static constexpr uint32_t xh = 0;                                           // [80][32] uint2
    static constexpr uint32_t xs = xh + (F16 ? (uint32_t)KSTEPS * 32 * 8 : 0u);  // [80][32] float4
    static constexpr uint32_t bufs = xs + (F32 ? (uint32_t)KSTEPS * 32 * 16 : 0u);
    static constexpr int NW_FIT = (int)((GU_SMEM_BUDGET - bufs - 256u) / BUF);
    static constexpr int NW = NW_FIT < GU_MAX_WARPS ? NW_FIT : GU_MAX_WARPS;
    static constexpr uint32_t bars = bufs + (uint32_t)NW * BUF;
    static constexpr uint32_t total = bars + (uint32_t)NW * 8;
    static_assert(xs % 16 == 0 && bufs % 128 == 0 && BUF % 128 == 0 && bars % 8 == 0, "region alignment");
    static_assert(NW >= 4, "shared memory budget");
};

// [g; u] partial sums of one unit: tot[0], tot[1] = gate row gr of tokens 2c, 2c+1;
// tot[2], tot[3] = the up row.  int4/int8 codes become exact f16 A fragments and each
// scale group's fp32 sum is scaled; bf16 weights meet x's bf16 hi and lo parts.
template <int W, int G, int PARTS = gu_parts<W>()>
__device__ __forceinline__ void gu_compute(const char* buf, const uint2* xh, const float4* xs, int q0, int lane,
                                           float (&tot)[4]) {
    using U = GuUnit<W, G, PARTS>;
    if constexpr (!is_quant(W)) {
        // four independent accumulators (hi/lo x even/odd k-step) keep the MMA pipe busy
        float acc[4][4] = {};
#pragma unroll 4
        for (int v = 0; v < U::NV; v += 2) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint4 a = lds128(buf + ((v + h) * 32 + lane) * 16);
                const float4 xv = lds128f(xs + (q0 + v + h) * 32 + lane);
                const uint2 l = split_bf16x2(xv.x, xv.y), hh = split_bf16x2(xv.z, xv.w);
                mma16816_bf16(acc[2 * h], a, l.x, hh.x);       // x hi
                mma16816_bf16(acc[2 * h + 1], a, l.y, hh.y);   // x lo
            }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) tot[r] = (acc[0][r] + acc[1][r]) + (acc[2][r] + acc[3][r]);
    } else {
        // each scale group's sum is built in two accumulators (even / odd k-steps; the first
        // MMA of each starts from zero), then scaled into tot
        constexpr int QPG = G / 16;                  // k-steps per scale group (>= 2)
        constexpr int VB = U::NV % 4 == 0 ? 4 : 2;   // vectors per loop step: whole scale groups
        static_assert(QPG >= 2 && (VB * U::KPV) % QPG == 0 && U::NV % VB == 0, "loop step holds whole groups");
        const float2* sc = reinterpret_cast<const float2*>(buf + U::W_BYTES) + (lane >> 2);
        float acc[2][4];
#pragma unroll 1
        for (int v0 = 0; v0 < U::NV; v0 += VB) {
#pragma unroll
            for (int vv = 0; vv < VB; ++vv) {
                const uint4 w = lds128(buf + ((v0 + vv) * 32 + lane) * 16);
                const uint32_t wr[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int j = 0; j < U::KPV; ++j) {
                    const int qq = vv * U::KPV + j;     // compile-time position in the step
                    const int ql = v0 * U::KPV + qq;    // unit-local k-step
                    Frag4 a;
                    if constexpr (W == FOCR_W_INT4) a = dq_int4(wr[j]);
                    else a = dq_int8(wr[2 * j], wr[2 * j + 1]);
                    const uint2 xb = xh[(q0 + ql) * 32 + lane];
                    if (qq % QPG < 2) mma16816_zc(acc[qq & 1], a, xb.x, xb.y);
                    else mma16816(acc[qq & 1], a, xb.x, xb.y);
                    if ((qq + 1) % QPG == 0) {
                        const float2 s = sc[(ql / QPG) * 8];
                        tot[0] = fmaf(acc[0][0] + acc[1][0], s.x, tot[0]);
                        tot[1] = fmaf(acc[0][1] + acc[1][1], s.x, tot[1]);
                        tot[2] = fmaf(acc[0][2] + acc[1][2], s.y, tot[2]);
                        tot[3] = fmaf(acc[0][3] + acc[1][3], s.y, tot[3]);
                    }
                }
            }
        }
    }
}

// a = silu(g) * u * w_route for intermediate 8 ti + gr of tokens 2c, 2c+1, stored as the
// down projection's B fragments: f16 m16n8k16 steps for int4/int8 sets (step ti / 2,
// register ti % 2), bf16 hi + lo m16n8k8 steps for bf16 sets (step ti).
template <int W>
__device__ __forceinline__ void store_a(const RouteView& R, bool routed, int a_slot, int ti, int lane,
                                        const float (&s)[4], float2 wr) {
    const int gr = lane >> 2, c = lane & 3;
    const float av[2] = {s[0] / (1.f + __expf(-s[0])) * s[2] * wr.x, s[1] / (1.f + __expf(-s[1])) * s[3] * wr.y};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int ln = 4 * (2 * c + h) + (gr >> 1);
        if constexpr (is_quant(W)) {
            __half* a16 = reinterpret_cast<__half*>(R.a16);
            const int step = a16_base(routed, a_slot) + (ti >> 1);
            a16[((step * 32 + ln) * 2 + (ti & 1)) * 2 + (gr & 1)] = __float2half_rn(av[h]);
            if (f16_out_of_range(av[h])) atomicExch(R.ctrl + CTRL_ERROR, DEVERR_RANGE);
        } else {
            __nv_bfloat16* abf = reinterpret_cast<__nv_bfloat16*>(R.abf);
            const int step = abf_base(routed, a_slot) + ti;
            const __nv_bfloat16 hi = __float2bfloat16_rn(av[h]);
            const __nv_bfloat16 lo = __float2bfloat16_rn(av[h] - __bfloat162float(hi));
            abf[((step * 32 + ln) * 2 + 0) * 2 + (gr & 1)] = hi;
            abf[((step * 32 + ln) * 2 + 1) * 2 + (gr & 1)] = lo;
        }
    }
}

// One gate/up unit of a warp, in two halves.  gu_issue bulk-copies its codes (and scale
// groups) into the warp's buffer and, for the first unit of a slice, prefetches the
// slice's down-projection bytes into L2.  gu_finish waits for the copy, computes, and
// either applies SwiGLU (whole rows) or adds into the tile's sums, the last of the KP
// parts applying it.  gu_finish returns false if the copy did not complete in time.
template <int W, int G, int PARTS = gu_parts<W>()>
__device__ __forceinline__ const uint8_t* gu_block(const SmallParams& p, bool routed, int expert, int u) {
    constexpr int S = slice_rows(W);
    const ItemGeom& g = routed ? p.L.rg : p.L.sg;
    const int s = (u / PARTS) / (S / 8);
    return (routed ? p.L.routed_items + (size_t)expert * g.slices * g.item_bytes : p.L.shared_items) +
           (size_t)s * g.item_bytes;
}

template <int W, int G, int PARTS = gu_parts<W>()>
__device__ __forceinline__ void gu_issue(const SmallParams& p, bool routed, int expert, int u, char* buf,
                                         uint64_t* bar, int lane, uint64_t pol) {
    using U = GuUnit<W, G, PARTS>;
    constexpr int S = slice_rows(W);
    const int ti = u / U::KP, part = u % U::KP;
    const int s = ti / (S / 8), t = ti % (S / 8);
    const uint8_t* blk = gu_block<W, G, PARTS>(p, routed, expert, u);
    __syncwarp();   // every lane is done with the previous unit's buffer
    if (lane == 0) {
        mbar_arrive_expect_tx(bar, U::BYTES);
        bulk_g2s(buf, blk + ((size_t)t * (KSTEPS / U::KPV) + (size_t)part * U::NV) * 512, U::W_BYTES, bar, pol);
        if constexpr (U::NG > 0)
            bulk_g2s(buf + U::W_BYTES, blk + gu_w_bytes_of(W) + ((size_t)t * (H / G) + (size_t)part * U::NG) * 64,
                     U::S_BYTES, bar, pol);
    } else if (lane == 1 && t == 0 && part == 0) {
        bulk_prefetch_l2(blk + gu_w_bytes_of(W) + gu_s_bytes_of(W, G), d_w_bytes_of());
        if (is_quant(W) && (s * S) % G == 0) {
            const ItemGeom& g = routed ? p.L.rg : p.L.sg;
            const float* dsc = routed ? p.L.routed_dscale + (size_t)expert * g.dscale_expert_floats : p.L.shared_dscale;
            bulk_prefetch_l2(dsc + (size_t)(s * S / G) * H, H * 4);
        }
    }
}

template <int W, int G>
__device__ __forceinline__ bool gu_finish(const SmallParams& p, bool routed, int a_slot, int expert, int u,
                                          const char* buf, uint64_t* bar, uint32_t& phase, const uint2* xh,
                                          const float4* xs, int lane) {
    using U = GuUnit<W, G>;
    const int ti = u / U::KP, part = u % U::KP;
    const float2 wr = routed ? route_w(p.R, p.T, expert, lane & 3) : make_float2(1.f, 1.f);
    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar, phase, WAIT_LIMIT_NS));
    phase ^= 1u;
    if (!ok) {
        if (lane == 0) atomicExch(&p.R.ctrl[CTRL_ERROR], DEVERR_FULL_WAIT);
        (void)mbar_wait_bounded(bar, phase ^ 1u, WAIT_LIMIT_NS);   // never leave the copy in flight
        return false;
    }
    float tot[4] = {0.f, 0.f, 0.f, 0.f};
    gu_compute<W, G>(buf, xh, xs, part * U::QN, lane, tot);
    if constexpr (U::KP == 1) {
        store_a<W>(p.R, routed, a_slot, ti, lane, tot, wr);
    } else {
        // each part's sums go to their own slot; the warp that completes the tile adds the parts in
        // a fixed order, so the total does not depend on the order they arrive in
        const int tile = gu_tile_base(routed, a_slot) + ti;
        float4* gp = reinterpret_cast<float4*>(p.R.gpart) + ((size_t)tile * 4) * 32 + lane;
        __stcg(gp + part * 32, make_float4(tot[0], tot[1], tot[2], tot[3]));
        __threadfence();
        __syncwarp();
        int old = 0;
        if (lane == 0) old = atomicAdd(&p.R.tcnt[tile], 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old == U::KP - 1) {   // the other parts' sums are in: apply
            __threadfence();
            float sum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int q = 0; q < U::KP; ++q) {
                const float4 v = __ldcg(gp + q * 32);
                sum[0] += v.x;
                sum[1] += v.y;
                sum[2] += v.z;
                sum[3] += v.w;
            }
            if (lane == 0) p.R.tcnt[tile] = 0;
            store_a<W>(p.R, routed, a_slot, ti, lane, sum, wr);
        }
    }
    return true;
}

// Warps are ranked across SMs first (rho = warp * grid + block) so that both the
// shared-set units, which take the low ranks, and the routed units, which take the high
// ranks, spread over every SM.  A warp's first shared unit is in flight while x is staged.
template <int RW, int SW, int G>
__global__ void __launch_bounds__(GuCfg<RW, SW, G>::NW * 32, 2) decode_gu_kernel(SmallParams p) {
    using C = GuCfg<RW, SW, G>;
    extern __shared__ __align__(128) char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint2* xh = reinterpret_cast<const uint2*>(smem + C::xh);
    const float4* xs = reinterpret_cast<const float4*>(smem + C::xs);
    char* buf = smem + C::bufs + warp * C::BUF;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::bars) + warp;
    const int nwt = gridDim.x * C::NW;
    const int rho = warp * gridDim.x + blockIdx.x;
    const uint64_t pol = policy_evict_first();
    const int s_units = (p.L.sg.inter / 8) * C::SU::KP;
    if (lane == 0) {
        mbar_init(bar, 1);
        fence_barrier_init();
    }
    __syncwarp();
    if (rho < s_units) gu_issue<SW, G>(p, false, -1, rho, buf, bar, lane, pol);
    build_x<C::NW * 32, C::F16, C::F32>(p.x, p.T, reinterpret_cast<uint2*>(smem + C::xh),
                                         reinterpret_cast<float4*>(smem + C::xs), p.R.ctrl + CTRL_ERROR);
    __syncthreads();

    uint32_t phase = 0;
    bool ok = true;
    for (int u = rho; ok && u < s_units; u += nwt) {
        if (u != rho) gu_issue<SW, G>(p, false, -1, u, buf, bar, lane, pol);
        ok = gu_finish<SW, G>(p, false, 0, -1, u, buf, bar, phase, xh, xs, lane);
    }
    pdl_wait();                 // the router's selection is complete and visible
    pdl_launch_dependents();    // the down kernel may read it from now on
    if (p.shared_only || !ok) return;
    constexpr int per_expert = (I / 8) * C::RU::KP;
    const int r_units = p.R.active[E] * per_expert;
    for (int r = nwt - 1 - rho; ok && r < r_units; r += nwt) {
        const int a = r / per_expert;
        const int e = p.R.active[a];
        gu_issue<RW, G>(p, true, e, r % per_expert, buf, bar, lane, pol);
        ok = gu_finish<RW, G>(p, true, a, e, r % per_expert, buf, bar, phase, xh, xs, lane);
    }
}

// ------------------------------------------------------------------ down units
// A unit is one output tile (16 rows) of one set over a chunk of CH consecutive slices:
// per slice one 8-byte A load per lane (int4: two k16 steps, int8: one k16 step, bf16:
// one k8 step) and the matching B fragments of a.  Scale groups never straddle a chunk.
template <int W, int G>
struct DownUnit {
    static constexpr int S = slice_rows(W);
    // slices per chunk (int4 g64: 14, so an expert's 28 slices make two equal chunks)
    static constexpr int CH = W == FOCR_W_INT4 ? (G == 32 ? 8 : (G == 64 ? 14 : 16)) : 16;
    static constexpr int SPG = is_quant(W) ? (G / S < CH ? G / S : CH) : CH;   // slices per scale group
    static constexpr int NGC = CH / SPG;                                  // scale groups per chunk
    static constexpr int BPS = W == FOCR_W_INT4 ? 2 : 1;                  // B fragments (uint2) per slice
    static_assert(!is_quant(W) || (CH * S) % G == 0, "chunks hold whole scale groups");
};

// A loads (codes, and scale groups) of one unit: independent of the gate/up kernel, so a
// warp's first unit issues them before waiting on that kernel
template <int W, int G>
struct DownA {
    uint2 v[DownUnit<W, G>::CH];
    float sc[is_quant(W) ? DownUnit<W, G>::NGC : 1][2];
    int ns;
};

template <int W, int G>
__device__ __forceinline__ void down_load(const uint8_t* items, const ItemGeom& g, const float* dsc, int chunk, int m,
                                          int lane, DownA<W, G>& A) {
    using D = DownUnit<W, G>;
    const int s0 = chunk * D::CH;
    A.ns = min(D::CH, g.slices - s0);
    const uint8_t* dw = items + (size_t)s0 * g.item_bytes + gu_w_bytes_of(W) + gu_s_bytes_of(W, G) + (m * 32 + lane) * 8;
#pragma unroll
    for (int j = 0; j < D::CH; ++j) A.v[j] = j < A.ns ? ldg_nc2(dw + (size_t)j * g.item_bytes) : make_uint2(0u, 0u);
    if constexpr (is_quant(W)) {
#pragma unroll
        for (int jg = 0; jg < D::NGC; ++jg) {
            A.sc[jg][0] = A.sc[jg][1] = 0.f;
            if (jg * D::SPG < A.ns) {
                const float* r = dsc + (size_t)((s0 + jg * D::SPG) * D::S / G) * H + 16 * m + (lane >> 2);
                A.sc[jg][0] = __ldg(r);
                A.sc[jg][1] = __ldg(r + 8);
            }
        }
    }
}

// B fragments of a (written by the gate/up kernel), the MMAs (two independent accumulators),
// the group scales, and the atomic adds into the output rows 16m .. 16m+15
template <int W, int G>
__device__ __forceinline__ void down_finish(const DownA<W, G>& A, const uint2* bsm, int m, int T, float* out,
                                            const RouteView& R, bool det, int lane) {
    using D = DownUnit<W, G>;
    constexpr int CH = D::CH;
    const int gr = lane >> 2, c = lane & 3;
    uint2 b[CH][D::BPS];
#pragma unroll
    for (int j = 0; j < CH; ++j)
#pragma unroll
        for (int h = 0; h < D::BPS; ++h)
            b[j][h] = j < A.ns ? bsm[(j * D::BPS + h) * 32 + lane] : make_uint2(0u, 0u);

    float y[4] = {0.f, 0.f, 0.f, 0.f};
    float acc[2][4] = {};
#pragma unroll
    for (int j = 0; j < CH; ++j) {
        if (j < A.ns) {
            if constexpr (W == FOCR_W_INT4) {
                mma16816(acc[0], dq_int4(A.v[j].x), b[j][0].x, b[j][0].y);
                mma16816(acc[1], dq_int4(A.v[j].y), b[j][1].x, b[j][1].y);
            } else if constexpr (W == FOCR_W_INT8) {
                mma16816(acc[j & 1], dq_int8(A.v[j].x, A.v[j].y), b[j][0].x, b[j][0].y);
            } else {
                mma1688_bf16(acc[0], A.v[j].x, A.v[j].y, b[j][0].x);   // a hi
                mma1688_bf16(acc[1], A.v[j].x, A.v[j].y, b[j][0].y);   // a lo
            }
        }
        if constexpr (is_quant(W)) {
            if ((j + 1) % D::SPG == 0) {
                const int jg = j / D::SPG;
                y[0] = fmaf(acc[0][0] + acc[1][0], A.sc[jg][0], y[0]);
                y[1] = fmaf(acc[0][1] + acc[1][1], A.sc[jg][0], y[1]);
                y[2] = fmaf(acc[0][2] + acc[1][2], A.sc[jg][1], y[2]);
                y[3] = fmaf(acc[0][3] + acc[1][3], A.sc[jg][1], y[3]);
#pragma unroll
                for (int k = 0; k < 2; ++k) acc[k][0] = acc[k][1] = acc[k][2] = acc[k][3] = 0.f;
            }
        }
    }
    if constexpr (!is_quant(W)) {
#pragma unroll
        for (int r = 0; r < 4; ++r) y[r] = acc[0][r] + acc[1][r];
    }
    // deterministic: into the fixed-point sums of tile m (any arrival order gives the same totals),
    // counted against the tile after the warp's last unit; otherwise fp32 atomics into the output
    const int row = 16 * m + gr;
    const int tok[4] = {2 * c, 2 * c + 1, 2 * c, 2 * c + 1}, rr[4] = {row, row, row + 8, row + 8};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (tok[i] >= T) continue;
        const size_t idx = (size_t)tok[i] * H + rr[i];
        if (!det) atomicAdd(out + idx, y[i]);
        else if (fx_ok(y[i])) red_add_u64(R.dacc + idx, fx_of(y[i]));
        else R.dflag[idx] = 1;
    }
}

// The warp that completes 16-row tile m adds the tile's fixed-point totals to the output the
// router initialised, once, and clears them.
__device__ __forceinline__ void down_convert(const RouteView& R, float* out, int T, int m, int lane) {
    __threadfence();
    for (int i = lane; i < 16 * T; i += 32) {
        const size_t idx = (size_t)(i >> 4) * H + 16 * m + (i & 15);
        const unsigned long long a = __ldcg(R.dacc + idx);
        const int f = __ldcg(R.dflag + idx);
        out[idx] += f ? __int_as_float(0x7fc00000) : fx_to_float(a);
        R.dacc[idx] = 0ull;
        if (f) R.dflag[idx] = 0;
    }
    if (lane == 0) R.dcnt[m] = 0;
}

// One step of a CTA: its 8 warps take 8 consecutive output tiles of one chunk of one set.
// Each warp loads its A codes and scales; on the first step the CTA then waits on the
// gate/up kernel; one thread bulk-copies the chunk's B fragments of a (contiguous in the
// workspace) into shared memory for all eight warps.  Returns false if that copy did not
// complete in time.
template <int W, int G>
__device__ __forceinline__ bool down_step(const SmallParams& p, const uint8_t* items, const ItemGeom& g,
                                          const float* dsc, const uint2* bset, int chunk, int m, bool first,
                                          uint2* bsm, uint64_t* bar, uint32_t& phase, int lane) {
    using D = DownUnit<W, G>;
    DownA<W, G> A;
    down_load<W, G>(items, g, dsc, chunk, m, lane, A);
    if (first) pdl_wait();
    __syncthreads();   // the previous step's readers are done with bsm
    if (threadIdx.x == 0) {
        const uint32_t bytes = (uint32_t)A.ns * D::BPS * 256u;
        mbar_arrive_expect_tx(bar, bytes);
        bulk_g2s(bsm, bset + (size_t)chunk * D::CH * D::BPS * 32, bytes, bar, policy_evict_first());
    }
    // the wait's outcome is made CTA-uniform, so every warp leaves the step loop together
    const bool ok = __syncthreads_and(mbar_wait_bounded(bar, phase, WAIT_LIMIT_NS)) != 0;
    phase ^= 1u;
    if (!ok) {
        if (threadIdx.x == 0) atomicExch(&p.R.ctrl[CTRL_ERROR], DEVERR_FULL_WAIT);
        (void)mbar_wait_bounded(bar, phase ^ 1u, WAIT_LIMIT_NS);   // never leave the copy in flight
        return false;
    }
    down_finish<W, G>(A, bsm, m, p.T, p.out, p.R, p.deterministic != 0, lane);
    return true;
}

// Units: the shared set's (chunk, tile) pairs, then every selected expert's, 80 output
// tiles per chunk; the 8 warps of a CTA take 8 consecutive units, which share the chunk
// (80, the number of units per chunk and the totals are multiples of 8, so the loop is
// uniform over the CTA).  This grid is scheduled only after every gate/up CTA has passed
// its own wait on the router, so the expert list is final and can be read (from L2)
// before this grid's wait; the codes of a CTA's first step are then in flight while the
// gate/up kernel finishes.
template <int RW, int SW, int G>
__global__ void __launch_bounds__(DN_WARPS * 32, 2) decode_down_kernel(SmallParams p) {
    using DR = DownUnit<RW, G>;
    using DS = DownUnit<SW, G>;
    __shared__ __align__(128) uint2 bsm[DN_BFRAGS];
    __shared__ uint64_t bar;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    pdl_launch_dependents();   // the next forward's router may launch; it waits for this grid
    const int nwt = gridDim.x * DN_WARPS;
    const int nch_s = (p.L.sg.slices + DS::CH - 1) / DS::CH;
    const int nch_r = (p.L.rg.slices + DR::CH - 1) / DR::CH;
    const int n_s = OTILES * nch_s;
    const int per_expert = OTILES * nch_r;
    const int n_act = p.shared_only ? 0 : __ldcg(&p.R.active[E]);
    const int total = n_s + n_act * per_expert;
    const int tile_units = nch_s + n_act * nch_r;   // units adding into each 16-row output tile
    const uint2* bs = is_quant(SW) ? p.R.a16 : p.R.abf;
    const uint2* br = is_quant(RW) ? p.R.a16 : p.R.abf;
    uint32_t phase = 0;
    bool first = true, ok = true;
    for (int base = blockIdx.x * DN_WARPS; ok && base < total; base += nwt) {
        const int u = base + warp;
        if (u < n_s) {
            ok = down_step<SW, G>(p, p.L.shared_items, p.L.sg, p.L.shared_dscale, bs, u / OTILES, u % OTILES, first,
                                  bsm, &bar, phase, lane);
        } else {
            const int r = u - n_s;
            const int a = r / per_expert, rem = r % per_expert;
            const int e = __ldcg(&p.R.active[a]);
            const ItemGeom& g = p.L.rg;
            ok = down_step<RW, G>(p, p.L.routed_items + (size_t)e * g.slices * g.item_bytes, g,
                                  p.L.routed_dscale + (size_t)e * g.dscale_expert_floats,
                                  br + (size_t)(is_quant(RW) ? a16_base(true, a) : abf_base(true, a)) * 32,
                                  rem / OTILES, rem % OTILES, first, bsm, &bar, phase, lane);
        }
        first = false;
    }
    if (ok && p.deterministic) {
        // a warp's units are counted against their tiles once, after all of them: one fence, then
        // one counter increment per unit with the units spread over the lanes
        __syncwarp();
        __threadfence();   // this warp's sums are visible before its units are counted
        const int nunits = total > blockIdx.x * DN_WARPS ? (total - blockIdx.x * DN_WARPS + nwt - 1) / nwt : 0;
        for (int j0 = 0; j0 < nunits; j0 += 32) {
            const int j = j0 + lane;
            int m = -1;
            bool done = false;
            if (j < nunits) {
                m = (blockIdx.x * DN_WARPS + j * nwt + warp) % OTILES;
                done = atomicAdd(&p.R.dcnt[m], 1) == tile_units - 1;
            }
            unsigned mask = __ballot_sync(0xffffffffu, done);
            while (mask) {
                const int src = __ffs(mask) - 1;
                mask &= mask - 1;
                down_convert(p.R, p.out, p.T, __shfl_sync(0xffffffffu, m, src), lane);
            }
        }
    }
    if (first) pdl_wait();   // every CTA waits before exiting (keeps the chain of forwards ordered)
}

template <int RW, int SW, int G>
cudaError_t launch_small_typed(const SmallParams& p, int sms, cudaStream_t st) {
    using C = GuCfg<RW, SW, G>;
    cudaError_t e0 = once_per_device((const void*)decode_gu_kernel<RW, SW, G>, [] {
        cudaError_t e = cudaFuncSetAttribute(decode_gu_kernel<RW, SW, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)C::total);
        if (e != cudaSuccess) return e;
        // the whole unified L1 as shared memory for all kernels of the path, so an SM never
        // has to change its split between consecutive kernels
        e = cudaFuncSetAttribute(decode_gu_kernel<RW, SW, G>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        return cudaFuncSetAttribute(decode_down_kernel<RW, SW, G>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                    cudaSharedmemCarveoutMaxShared);
    });
    if (e0 != cudaSuccess) return e0;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(sms);
    cfg.blockDim = dim3(C::NW * 32);
    cfg.dynamicSmemBytes = C::total;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, decode_gu_kernel<RW, SW, G>, p);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(2 * sms);
    cfg.blockDim = dim3(DN_WARPS * 32);
    cfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&cfg, decode_down_kernel<RW, SW, G>, p);
}

}  // namespace

cudaError_t launch_decode_small(const float* x, int T, const LayerView& L, const RouteView& R, float* out,
                                bool shared_only, bool deterministic, cudaStream_t st) {
    if (T < 1 || T > 8 || L.sg.inter > IS_MAX || L.sg.inter % 8 != 0) return cudaErrorInvalidValue;
    const int sms = device_sms();
    if (sms <= 0) return cudaErrorInvalidDevice;
    const SmallParams p{x, T, out, L, R, shared_only ? 1 : 0, deterministic ? 1 : 0};
    const int rw = L.rg.wtype, sw = L.sg.wtype;
    const int g = is_quant(rw) ? L.rg.group : (is_quant(sw) ? L.sg.group : 128);
#define FOCR_CASE(A, B, GG) \
    if (rw == A && sw == B && g == GG) return launch_small_typed<A, B, GG>(p, sms, st);
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
