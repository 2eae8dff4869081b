// Decode path for T <= 8 tokens: two streaming kernels with no CTA-wide synchronisation.
//
// Sources: frankenocr.pages.dev, "One forward pass", step 6 (64 routed experts + 2 fused
// shared experts, top-6 without renormalisation); franken_ocr README, "Architecture"
// (each expert 1280 -> 896 SiLU-gated); "Four bits, one shared scale" (int4 nibble + f32
// group scale; int8 and bf16 formats).
//
// The batch's tokens are the 8 columns of m16n8 tensor-core fragments (tokens that did not
// pick an expert get routing weight 0).  Both kernels read the packed item layout of
// common.cuh straight from global memory with 16-byte loads; every warp works alone on
// ~10 KB units.
//
// decode_gu (router -> gu, programmatic dependent launch): a unit is one tile of 8
//   intermediates (8 gate rows over 8 up rows) of the shared set or of a selected expert
//   over a range of input columns (all 1280 for int4, halves for int8, quarters for bf16).
//   int4/int8 codes become exact f16 A fragments, each scale group's fp32 accumulator is
//   scaled, bf16 weights enter bf16 MMAs with x split into hi + lo.  A unit that covers the
//   whole row applies a = silu(g) * u * w_route itself; k-split tiles add their partial
//   sums into the workspace with vector atomics, and the warp that completes a tile
//   (arrival counter) applies it and clears the sums and the counter.  a goes to the
//   workspace as the B fragments of the down projection.  Shared-set units run while the
//   router is still working; routed units start after griddepcontrol.wait.  Warps of
//   routed units also prefetch their expert's down-projection bytes into L2.
// decode_down (gu -> down): a unit is one output tile of 16 rows of one selected expert
//   (all 896 intermediates) or of a quarter of the shared set; y = D a is scaled per row
//   and group and added into the output with atomics (the router initialised it).
//
// Precision: as the grouped expert kernel -- int4/int8 codes exact in f16 with fp32 group
// scales and f16 activations; bf16 weights exact with bf16 hi + lo activations; fp32
// accumulation throughout.
#include "common.cuh"
#include "fragments.cuh"

namespace focr {
namespace {

constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // 2 s
constexpr uint32_t GU_SMEM_BUDGET = 180 * 1024;     // leaves room for a router CTA on the same SM
constexpr int GU_MAX_WARPS = 16;
constexpr int DN_WARPS = 8;                         // down kernel: 8 warps, two CTAs per SM

struct SmallParams {
    const float* x;
    int T;
    float* out;
    LayerView L;
    RouteView R;
    int shared_only;
};

// Workspace indexing (shared set first, then the routed experts' active slots a = 0..U-1):
// gate/up tile sums and counters, f16 a steps of 16 intermediates, bf16 a steps of 8.
__device__ __forceinline__ int gu_tile_base(bool routed, int a) { return routed ? IS_MAX / 8 + a * (I / 8) : 0; }
__device__ __forceinline__ int a16_base(bool routed, int a) { return routed ? IS_MAX / 16 + a * (I / 16) : 0; }
__device__ __forceinline__ int abf_base(bool routed, int a) { return routed ? IS_MAX / 8 + a * (I / 8) : 0; }

// x of the batch in B-fragment order, fp32: xs[q][lane] = columns 16q+2c, +1, +8, +9 of
// token n (lane = 4n + c), zero for n >= T.  Both the f16 and the bf16 hi/lo operands
// are formed from it at use.
__device__ __forceinline__ void build_xs(const float* x, int T, float4* xs, int nthreads) {
    for (int i = threadIdx.x; i < KSTEPS * 32; i += nthreads) {
        const int q = i >> 5, ln = i & 31, n = ln >> 2, c = ln & 3;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (n < T) {
            const float* row = x + (size_t)n * H + 16 * q + 2 * c;
            const float2 lo = __ldg(reinterpret_cast<const float2*>(row));
            const float2 hi = __ldg(reinterpret_cast<const float2*>(row + 8));
            v = make_float4(lo.x, lo.y, hi.x, hi.y);
        }
        xs[i] = v;
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
template <int W, int G>
struct GuUnit {
    static constexpr int KP = W == FOCR_W_INT4 ? 1 : (W == FOCR_W_INT8 ? 2 : 4);   // column parts
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
    static constexpr uint32_t BUF = ((RU::BYTES > SU::BYTES ? RU::BYTES : SU::BYTES) + 127u) & ~127u;
    static constexpr uint32_t XS_BYTES = (uint32_t)KSTEPS * 32 * 16;
    static constexpr int NW_FIT = (int)((GU_SMEM_BUDGET - XS_BYTES - 256u) / BUF);
    static constexpr int NW = NW_FIT < GU_MAX_WARPS ? NW_FIT : GU_MAX_WARPS;
    static constexpr uint32_t bufs = XS_BYTES;
    static constexpr uint32_t bars = bufs + (uint32_t)NW * BUF;
    static constexpr uint32_t total = bars + (uint32_t)NW * 8;
    static_assert(NW >= 4, "shared memory budget");
};

// [g; u] partial sums of one unit: tot[0], tot[1] = gate row gr of tokens 2c, 2c+1;
// tot[2], tot[3] = the up row.  int4/int8 codes become exact f16 A fragments and each
// scale group's fp32 sum is scaled; bf16 weights meet x's bf16 hi and lo parts.
template <int W, int G>
__device__ __forceinline__ void gu_compute(const char* buf, const float4* xs, int q0, int lane, float (&tot)[4]) {
    using U = GuUnit<W, G>;
    if constexpr (!is_quant(W)) {
#pragma unroll 5
        for (int v = 0; v < U::NV; ++v) {
            const uint4 a = lds128(buf + (v * 32 + lane) * 16);
            const float4 xv = lds128f(xs + (q0 + v) * 32 + lane);
            const uint2 l = split_bf16x2(xv.x, xv.y), h = split_bf16x2(xv.z, xv.w);
            mma16816_bf16(tot, a, l.x, h.x);   // x hi
            mma16816_bf16(tot, a, l.y, h.y);   // x lo
        }
    } else {
        constexpr int QPG = G / 16;          // k-steps per scale group
        constexpr int VB = 4;                // vectors per loop step: whole scale groups
        static_assert((VB * U::KPV) % QPG == 0 && U::NV % VB == 0, "loop step holds whole groups");
        const float2* sc = reinterpret_cast<const float2*>(buf + U::W_BYTES) + (lane >> 2);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
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
                    const float4 xv = lds128f(xs + (q0 + ql) * 32 + lane);
                    mma16816(acc, a, f32x2_to_f16x2(xv.x, xv.y), f32x2_to_f16x2(xv.z, xv.w));
                    if ((qq + 1) % QPG == 0) {
                        const float2 s = sc[(ql / QPG) * 8];
                        tot[0] = fmaf(acc[0], s.x, tot[0]);
                        tot[1] = fmaf(acc[1], s.x, tot[1]);
                        tot[2] = fmaf(acc[2], s.y, tot[2]);
                        tot[3] = fmaf(acc[3], s.y, tot[3]);
                        acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
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

// One gate/up unit of a warp: bulk-copy its codes (and scale groups) into the warp's
// buffer, prefetch the slice's down-projection bytes into L2 (first unit of a slice),
// compute, and either apply SwiGLU (whole rows) or add into the tile's sums, the last of
// the KP parts applying it.  Returns false if the copy did not complete in time.
template <int W, int G>
__device__ __forceinline__ bool gu_unit(const SmallParams& p, bool routed, int a_slot, int expert, int u, char* buf,
                                        uint64_t* bar, uint32_t& phase, const float4* xs, int lane, uint64_t pol) {
    using U = GuUnit<W, G>;
    constexpr int S = slice_rows(W);
    const ItemGeom& g = routed ? p.L.rg : p.L.sg;
    const int ti = u / U::KP, part = u % U::KP;   // set-local tile, column part
    const int s = ti / (S / 8), t = ti % (S / 8);
    const uint8_t* blk = (routed ? p.L.routed_items + (size_t)expert * g.slices * g.item_bytes : p.L.shared_items) +
                         (size_t)s * g.item_bytes;
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
            const float* dsc = routed ? p.L.routed_dscale + (size_t)expert * g.dscale_expert_floats : p.L.shared_dscale;
            bulk_prefetch_l2(dsc + (size_t)(s * S / G) * H, H * 4);
        }
    }
    const float2 wr = routed ? route_w(p.R, p.T, expert, lane & 3) : make_float2(1.f, 1.f);
    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar, phase, WAIT_LIMIT_NS));
    phase ^= 1u;
    if (!ok) {
        if (lane == 0) atomicExch(&p.R.ctrl[CTRL_ERROR], DEVERR_FULL_WAIT);
        (void)mbar_wait_bounded(bar, phase ^ 1u, WAIT_LIMIT_NS);   // never leave the copy in flight
        return false;
    }
    float tot[4] = {0.f, 0.f, 0.f, 0.f};
    gu_compute<W, G>(buf, xs, part * U::QN, lane, tot);
    if constexpr (U::KP == 1) {
        store_a<W>(p.R, routed, a_slot, ti, lane, tot, wr);
    } else {
        const int tile = gu_tile_base(routed, a_slot) + ti;
        float* ga = p.R.gacc + ((size_t)tile * 32 + lane) * 4;
        red_add_v4(ga, tot[0], tot[1], tot[2], tot[3]);
        __threadfence();
        __syncwarp();
        int old = 0;
        if (lane == 0) old = atomicAdd(&p.R.tcnt[tile], 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old == U::KP - 1) {   // the other parts' sums are in: apply and clear
            __threadfence();
            const float4 v = __ldcg(reinterpret_cast<const float4*>(ga));
            __stcg(reinterpret_cast<float4*>(ga), make_float4(0.f, 0.f, 0.f, 0.f));
            if (lane == 0) p.R.tcnt[tile] = 0;
            const float sum[4] = {v.x, v.y, v.z, v.w};
            store_a<W>(p.R, routed, a_slot, ti, lane, sum, wr);
        }
    }
    return true;
}

// Warps are ranked across SMs first (rho = warp * grid + block) so that both the
// shared-set units, which take the low ranks, and the routed units, which take the high
// ranks, spread over every SM.
template <int RW, int SW, int G>
__global__ void __launch_bounds__(GuCfg<RW, SW, G>::NW * 32, 2) decode_gu_kernel(SmallParams p) {
    using C = GuCfg<RW, SW, G>;
    extern __shared__ __align__(128) char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float4* xs = reinterpret_cast<const float4*>(smem);
    char* buf = smem + C::bufs + warp * C::BUF;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::bars) + warp;
    if (lane == 0) {
        mbar_init(bar, 1);
        fence_barrier_init();
    }
    build_xs(p.x, p.T, reinterpret_cast<float4*>(smem), C::NW * 32);
    __syncthreads();

    const int nwt = gridDim.x * C::NW;
    const int rho = warp * gridDim.x + blockIdx.x;
    const uint64_t pol = policy_evict_first();
    uint32_t phase = 0;
    bool ok = true;
    const int s_units = (p.L.sg.inter / 8) * C::SU::KP;
    for (int u = rho; ok && u < s_units; u += nwt)
        ok = gu_unit<SW, G>(p, false, 0, -1, u, buf, bar, phase, xs, lane, pol);
    pdl_wait();                 // the router's selection is complete and visible
    pdl_launch_dependents();    // the down kernel may read it from now on
    if (p.shared_only || !ok) return;
    constexpr int per_expert = (I / 8) * C::RU::KP;
    const int r_units = p.R.active[E] * per_expert;
    for (int r = nwt - 1 - rho; ok && r < r_units; r += nwt) {
        const int a = r / per_expert;
        ok = gu_unit<RW, G>(p, true, a, p.R.active[a], r % per_expert, buf, bar, phase, xs, lane, pol);
    }
}

// ------------------------------------------------------------------ down units
// A unit is one output tile (16 rows) of one set over a chunk of CH consecutive slices:
// per slice one 8-byte A load per lane (int4: two k16 steps, int8: one k16 step, bf16:
// one k8 step) and the matching B fragments of a.  Scale groups never straddle a chunk.
template <int W, int G>
struct DownUnit {
    static constexpr int S = slice_rows(W);
    static constexpr int CH = (W == FOCR_W_INT4 && G == 32) ? 8 : 16;    // slices per chunk
    static constexpr int SPG = is_quant(W) ? (G / S < CH ? G / S : CH) : CH;   // slices per scale group
    static constexpr int NGC = CH / SPG;                                  // scale groups per chunk
    static constexpr int BPS = W == FOCR_W_INT4 ? 2 : 1;                  // B fragments (uint2) per slice
    static_assert(!is_quant(W) || (CH * S) % G == 0, "chunks hold whole scale groups");
};

template <int W, int G>
__device__ __forceinline__ void down_unit(const uint8_t* items, const ItemGeom& g, const float* dsc, const uint2* bfr,
                                          int chunk, int m, int T, float* out, int lane) {
    using D = DownUnit<W, G>;
    constexpr int CH = D::CH;
    const int gr = lane >> 2, c = lane & 3;
    const int s0 = chunk * CH;
    const int ns = min(CH, g.slices - s0);
    const uint8_t* dw = items + (size_t)s0 * g.item_bytes + gu_w_bytes_of(W) + gu_s_bytes_of(W, G) + (m * 32 + lane) * 8;
    uint2 v[CH];
#pragma unroll
    for (int j = 0; j < CH; ++j) v[j] = j < ns ? ldg_nc2(dw + (size_t)j * g.item_bytes) : make_uint2(0u, 0u);
    float sc[is_quant(W) ? D::NGC : 1][2];
    if constexpr (is_quant(W)) {
#pragma unroll
        for (int jg = 0; jg < D::NGC; ++jg) {
            sc[jg][0] = sc[jg][1] = 0.f;
            if (jg * D::SPG < ns) {
                const float* r = dsc + (size_t)((s0 + jg * D::SPG) * D::S / G) * H + 16 * m + gr;
                sc[jg][0] = __ldg(r);
                sc[jg][1] = __ldg(r + 8);
            }
        }
    }
    uint2 b[CH][D::BPS];
#pragma unroll
    for (int j = 0; j < CH; ++j)
#pragma unroll
        for (int h = 0; h < D::BPS; ++h)
            b[j][h] = j < ns ? bfr[((s0 + j) * D::BPS + h) * 32 + lane] : make_uint2(0u, 0u);

    float y[4] = {0.f, 0.f, 0.f, 0.f};
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < CH; ++j) {
        if (j < ns) {
            if constexpr (W == FOCR_W_INT4) {
                mma16816(acc, dq_int4(v[j].x), b[j][0].x, b[j][0].y);
                mma16816(acc, dq_int4(v[j].y), b[j][1].x, b[j][1].y);
            } else if constexpr (W == FOCR_W_INT8) {
                mma16816(acc, dq_int8(v[j].x, v[j].y), b[j][0].x, b[j][0].y);
            } else {
                mma1688_bf16(acc, v[j].x, v[j].y, b[j][0].x);   // a hi
                mma1688_bf16(acc, v[j].x, v[j].y, b[j][0].y);   // a lo
            }
        }
        if constexpr (is_quant(W)) {
            if ((j + 1) % D::SPG == 0) {
                const int jg = j / D::SPG;
                y[0] = fmaf(acc[0], sc[jg][0], y[0]);
                y[1] = fmaf(acc[1], sc[jg][0], y[1]);
                y[2] = fmaf(acc[2], sc[jg][1], y[2]);
                y[3] = fmaf(acc[3], sc[jg][1], y[3]);
                acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
            }
        }
    }
    if constexpr (!is_quant(W)) {
        y[0] = acc[0]; y[1] = acc[1]; y[2] = acc[2]; y[3] = acc[3];
    }
    const int row = 16 * m + gr;
    if (2 * c < T) {
        atomicAdd(out + (size_t)(2 * c) * H + row, y[0]);
        atomicAdd(out + (size_t)(2 * c) * H + row + 8, y[2]);
    }
    if (2 * c + 1 < T) {
        atomicAdd(out + (size_t)(2 * c + 1) * H + row, y[1]);
        atomicAdd(out + (size_t)(2 * c + 1) * H + row + 8, y[3]);
    }
}

// Units: the shared set's (chunk, tile) pairs, then every selected expert's; consecutive
// warps of a CTA take consecutive output tiles of one chunk, so they read the same a
// fragments.
template <int RW, int SW, int G>
__global__ void __launch_bounds__(DN_WARPS * 32, 2) decode_down_kernel(SmallParams p) {
    using DR = DownUnit<RW, G>;
    using DS = DownUnit<SW, G>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();   // a fragments of the gate/up kernel (and, through it, the router's output)
    const int nwt = gridDim.x * DN_WARPS;
    const int gw = blockIdx.x * DN_WARPS + warp;
    const int nch_s = (p.L.sg.slices + DS::CH - 1) / DS::CH;
    const int nch_r = (p.L.rg.slices + DR::CH - 1) / DR::CH;
    const int n_s = OTILES * nch_s;
    const int per_expert = OTILES * nch_r;
    const int total = n_s + (p.shared_only ? 0 : p.R.active[E] * per_expert);
    const uint2* bs = is_quant(SW) ? p.R.a16 : p.R.abf;
    const uint2* br = is_quant(RW) ? p.R.a16 : p.R.abf;
    for (int u = gw; u < total; u += nwt) {
        if (u < n_s) {
            down_unit<SW, G>(p.L.shared_items, p.L.sg, p.L.shared_dscale, bs, u / OTILES, u % OTILES, p.T, p.out, lane);
        } else {
            const int r = u - n_s;
            const int a = r / per_expert, rem = r % per_expert;
            const int e = p.R.active[a];
            const ItemGeom& g = p.L.rg;
            down_unit<RW, G>(p.L.routed_items + (size_t)e * g.slices * g.item_bytes, g,
                             p.L.routed_dscale + (size_t)e * g.dscale_expert_floats,
                             br + (size_t)(is_quant(RW) ? a16_base(true, a) : abf_base(true, a)) * 32, rem / OTILES,
                             rem % OTILES, p.T, p.out, lane);
        }
    }
}

int g_sms = 0;

template <int RW, int SW, int G>
cudaError_t launch_small_typed(const SmallParams& p, cudaStream_t st) {
    using C = GuCfg<RW, SW, G>;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(decode_gu_kernel<RW, SW, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)C::total);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(g_sms);
    cfg.blockDim = dim3(C::NW * 32);
    cfg.dynamicSmemBytes = C::total;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, decode_gu_kernel<RW, SW, G>, p);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(2 * g_sms);
    cfg.blockDim = dim3(DN_WARPS * 32);
    cfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&cfg, decode_down_kernel<RW, SW, G>, p);
}

}  // namespace

cudaError_t launch_decode_small(const float* x, int T, const LayerView& L, const RouteView& R, float* out,
                                bool shared_only, cudaStream_t st) {
    if (T < 1 || T > 8 || L.sg.inter > IS_MAX || L.sg.inter % 8 != 0) return cudaErrorInvalidValue;
    if (g_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev);
    }
    const SmallParams p{x, T, out, L, R, shared_only ? 1 : 0};
    const int rw = L.rg.wtype, sw = L.sg.wtype;
    const int g = is_quant(rw) ? L.rg.group : (is_quant(sw) ? L.sg.group : 128);
#define FOCR_CASE(A, B, GG) \
    if (rw == A && sw == B && g == GG) return launch_small_typed<A, B, GG>(p, st);
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
