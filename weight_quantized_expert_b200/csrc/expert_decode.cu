// Grouped expert kernel for batches of 9 to MID_T tokens (batched decode; the tensor-core kernel in
// expert_tc.cu serves larger batches, where it is faster): the
// shared expert and every selected routed expert, SwiGLU fused, weights dequantised in
// registers straight into 16x8x16 tensor-core fragments (fp32 accumulation).
//
// Sources: frankenocr.pages.dev, "One forward pass", step 6 (64 routed experts + 2 fused
// shared experts, top-6 without renormalisation); franken_ocr README, "Architecture"
// (each expert 1280 -> 896 SiLU-gated); "Four bits, one shared scale" (int4 nibble +
// f32 group scale; int8 and bf16 formats).
//
// Work: an "item" is one slice of S intermediate rows of one expert (common.cuh; ~60-77
// KB).  Items are numbered shared-expert slices first, then the slices of every expert
// that received tokens (ascending id); CTA b of a persistent grid (one per SM) takes
// items b, b+G, ...  A producer warp streams item blocks into a 2- or 3-slot shared-memory
// ring with bulk async copies (cp.async.bulk + mbarrier) and publishes each item's
// expert id next to it.  20 consumer warps walk the item's tokens (all tokens for the
// shared expert, the expert's segment of the dispatch permutation otherwise) in passes of
// NG x 8 tokens, each group of 8 being the columns of one set of n8 fragments:
//   phase 1  [g; u] = [G; U]_slice x  -- warp w covers input columns [64w, 64w + 64) of every
//            tile with mma.sync m16n8k16; each A fragment (int4/int8 codes as exact f16,
//            bf16 weights as stored) serves every token group of the pass; each scale
//            group's fp32 sum is scaled; the twenty column parts meet in shared memory
//   swiglu   a = silu(g) * u * w_route  (fp32, then the phase-2 B fragments)
//   phase 2  y = D[:, slice] a          -- warp owns 4 of the 80 output tiles
// and adds every token's result into its output row with atomics.  The shared-expert
// slices need no routing, so they run while the router kernel is still working
// (programmatic dependent launch); routed items start after griddepcontrol.wait, and no
// output is added before it (the router initialises `out`).  Every mbarrier wait is
// bounded in time; on expiry the kernel records an error word and stops.
//
// Precision: int4/int8 codes are exact in f16 and scales are applied in fp32; x and a are
// rounded to f16 (relative 2^-11) for them.  bf16 weights enter unchanged and x and a are
// split into bf16 hi + lo parts (two MMAs, about 16 significant bits).  Every product
// accumulates in fp32.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "fragments.cuh"
#include "launch_state.h"

namespace focr {
namespace {

constexpr int NCW = 20;                      // consumer warps
constexpr int NCT = NCW * 32;                // consumer threads
constexpr int NTHREADS = NCT + 32;           // + producer warp
constexpr int NTOK = 8;                      // tokens per fragment (n8)
constexpr int NG = 2;                        // token groups per pass
constexpr int NTP = NG * NTOK;               // tokens per pass
constexpr uint32_t DSC_BYTES = H * 4;        // one group's down scales
constexpr int TILES_PER_WARP = OTILES / NCW; // 4
constexpr int KSW = KSTEPS / NCW;            // 4 k-steps of phase 1 per warp
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // 2 s

// Ring slots are sized for the kernel's own item types; three slots when they fit.
template <int RW, int SW, int G>
struct SmemLayout {
    static constexpr uint32_t item_r = blk_bytes_of(RW, G) + (is_quant(RW) ? DSC_BYTES : 0u);
    static constexpr uint32_t item_s = blk_bytes_of(SW, G) + (is_quant(SW) ? DSC_BYTES : 0u);
    static constexpr uint32_t slot_bytes = ((item_r > item_s ? item_r : item_s) + 127u) & ~127u;
    static constexpr uint32_t rest = NG * (4 * 4 * 32 * 4 + 2 * 32 * 8 + 32 * 8) + 2 * NTP * 4 + 16 + 2 * 3 * 8 + 16;
    static constexpr int nslot = 3 * slot_bytes + rest <= 232448 ? 3 : 2;
    static constexpr uint32_t slots = 0;
    static constexpr uint32_t acc = slots + nslot * slot_bytes;         // [NG][4 tiles][4 comps][32] f32 sums
    static constexpr uint32_t ah = acc + NG * 4 * 4 * 32 * 4;           // [NG][2][32] uint2: f16 a B frags
    static constexpr uint32_t abf = ah + NG * 2 * 32 * 8;               // [NG][32] uint2: bf16 a hi, lo frags
    static constexpr uint32_t wn = abf + NG * 32 * 8;                   // [NTP] f32 route weights
    static constexpr uint32_t tok = wn + NTP * 4;                       // [NTP] i32 token ids
    static constexpr uint32_t rec = tok + NTP * 4;                      // [nslot] i32 expert of the slot's item
    static constexpr uint32_t bars = rec + 16;                          // full[nslot], empty[nslot]
    static constexpr uint32_t misc = bars + 2 * 3 * 8;
    static constexpr uint32_t total = misc + 16;
    static_assert(total <= 232448, "shared memory budget");
};

struct ExpertParams {
    const float* x;
    int T;
    float* out;
    LayerView L;
    RouteView R;
    int shared_only;   // a single dense SwiGLU (the "shared" weight set), no routing
};

// ------------------------------------------------------------------ x fragments (registers)
// Warp w owns k-steps 4w .. 4w+3 of phase 1, so its B fragments of the pass's x stay in
// registers, in the form the item's weights need: v[g][j] = f16 (b0, b1) for int4/int8
// items, bf16 hi (b0, b1), lo (b0, b1) for bf16 items, for token group g.  Lane
// (n = lane / 4, c = lane % 4) holds columns 16q+2c, +1 and 16q+2c+8, +9 of token
// tok[8g + n]; tok < 0 gives zeros.
struct XFrags {
    uint32_t v[NG][KSW][4];
};

template <bool F16, bool BF16>
__device__ __forceinline__ void load_x_frags(const float* x, const int* tok, int warp, int lane, bool as_bf16,
                                             XFrags& xf) {
    float2 lo[NG][KSW], hi[NG][KSW];
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        const int tk = tok[NTOK * g + (lane >> 2)];
#pragma unroll
        for (int j = 0; j < KSW; ++j) {
            lo[g][j] = hi[g][j] = make_float2(0.f, 0.f);
            if (tk >= 0) {
                const float* row = x + (size_t)tk * H + 16 * (KSW * warp + j) + 2 * (lane & 3);
                lo[g][j] = __ldg(reinterpret_cast<const float2*>(row));
                hi[g][j] = __ldg(reinterpret_cast<const float2*>(row + 8));
            }
        }
    }
#pragma unroll
    for (int g = 0; g < NG; ++g)
#pragma unroll
        for (int j = 0; j < KSW; ++j) {
            if (BF16 && (!F16 || as_bf16)) {
                const uint2 a = split_bf16x2(lo[g][j].x, lo[g][j].y), b = split_bf16x2(hi[g][j].x, hi[g][j].y);
                xf.v[g][j][0] = a.x;
                xf.v[g][j][1] = b.x;
                xf.v[g][j][2] = a.y;
                xf.v[g][j][3] = b.y;
            } else {
                xf.v[g][j][0] = f32x2_to_f16x2(lo[g][j].x, lo[g][j].y);
                xf.v[g][j][1] = f32x2_to_f16x2(hi[g][j].x, hi[g][j].y);
                xf.v[g][j][2] = xf.v[g][j][3] = 0u;
            }
        }
}

// ------------------------------------------------------------------ phase 1: gate/up
// Every tile of the item over this warp's four k-steps, for the pass's ng token groups.
// int4/int8 codes become exact f16 values and the fp32 sum of each scale group is multiplied
// by its scale (the four k-steps lie in one group for g >= 64, in two for g = 32).
template <int W, int G>
__device__ __forceinline__ void phase_gate_up(const char* slot, const XFrags& xf, float* acc_s, int warp, int lane,
                                              int ng) {
    constexpr int NT = slice_rows(W) / 8;
    const int gr = lane >> 2;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        float tot[NG][4] = {};
        if constexpr (!is_quant(W)) {
            const uint4* gw = reinterpret_cast<const uint4*>(slot) + (t * KSTEPS + KSW * warp) * 32 + lane;
#pragma unroll
            for (int j = 0; j < KSW; ++j) {
                const uint4 a = gw[j * 32];
#pragma unroll
                for (int g = 0; g < NG; ++g) {
                    if (g < ng) {
                        mma16816_bf16(tot[g], a, xf.v[g][j][0], xf.v[g][j][1]);   // x hi
                        mma16816_bf16(tot[g], a, xf.v[g][j][2], xf.v[g][j][3]);   // x lo
                    }
                }
            }
        } else {
            constexpr int NGK = H / G;
            uint32_t wv[8];
            if constexpr (W == FOCR_W_INT4) {
                const uint4 v = reinterpret_cast<const uint4*>(slot)[(t * (KSTEPS / 4) + warp) * 32 + lane];
                wv[0] = v.x; wv[1] = v.y; wv[2] = v.z; wv[3] = v.w;
            } else {
                const uint4* g8 = reinterpret_cast<const uint4*>(slot) + (t * (KSTEPS / 2) + 2 * warp) * 32 + lane;
                const uint4 v0 = g8[0], v1 = g8[32];
                wv[0] = v0.x; wv[1] = v0.y; wv[2] = v0.z; wv[3] = v0.w;
                wv[4] = v1.x; wv[5] = v1.y; wv[6] = v1.z; wv[7] = v1.w;
            }
            const float2* gs = reinterpret_cast<const float2*>(slot + gu_w_bytes_of(W)) + t * NGK * 8 + gr;
            constexpr int NH = G == 32 ? 2 : 1;   // scale groups among the warp's four k-steps
            float acc[NG][NH][4] = {};
#pragma unroll
            for (int j = 0; j < KSW; ++j) {
                Frag4 a;
                if constexpr (W == FOCR_W_INT4) a = dq_int4(wv[j]);
                else a = dq_int8(wv[2 * j], wv[2 * j + 1]);
#pragma unroll
                for (int g = 0; g < NG; ++g)
                    if (g < ng) mma16816(acc[g][G == 32 ? j >> 1 : 0], a, xf.v[g][j][0], xf.v[g][j][1]);
            }
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                const int gi = G == 32 ? 2 * warp + h : (KSW * warp * 16) / G;
                const float2 sc = gs[gi * 8];
#pragma unroll
                for (int g = 0; g < NG; ++g) {
                    tot[g][0] = fmaf(acc[g][h][0], sc.x, tot[g][0]);
                    tot[g][1] = fmaf(acc[g][h][1], sc.x, tot[g][1]);
                    tot[g][2] = fmaf(acc[g][h][2], sc.y, tot[g][2]);
                    tot[g][3] = fmaf(acc[g][h][3], sc.y, tot[g][3]);
                }
            }
        }
        // the twenty warps' partial sums meet in shared memory ([group][tile][component][lane])
#pragma unroll
        for (int g = 0; g < NG; ++g)
            if (g < ng)
#pragma unroll
                for (int r = 0; r < 4; ++r) atomicAdd(acc_s + ((g * 4 + t) * 4 + r) * 32 + lane, tot[g][r]);
    }
}

// ------------------------------------------------------------------ swiglu -> phase-2 B fragments
// One thread per (group, tile, lane) reads the summed g and u (and clears them for the next
// pass); a = silu(g) * u * w_route goes into the group's phase-2 B fragments.
template <int W>
__device__ __forceinline__ void swiglu_to_frag(float* acc_s, __half* ah, __nv_bfloat16* abf, const float* wn,
                                               int ctid, int ng, int* err) {
    constexpr int NT = slice_rows(W) / 8;
    if (ctid >= ng * NT * 32) return;
    const int g = ctid / (NT * 32), t = (ctid >> 5) % NT, lane = ctid & 31;
    float4 s;
    float* a4 = acc_s + ((g * 4 + t) * 4) * 32 + lane;
    s.x = a4[0]; s.y = a4[32]; s.z = a4[64]; s.w = a4[96];
    a4[0] = a4[32] = a4[64] = a4[96] = 0.f;
    const int gr = lane >> 2, c = lane & 3;
    // s.x, s.y: gate of intermediate 8t+gr for tokens 2c, 2c+1 of the group; s.z, s.w: up
    const float* w = wn + NTOK * g;
    const float a[2] = {s.x / (1.f + __expf(-s.x)) * s.z * w[2 * c], s.y / (1.f + __expf(-s.y)) * s.w * w[2 * c + 1]};
    const int i = 8 * t + gr;                     // slice-local intermediate index = k of phase 2
    if constexpr (is_quant(W)) {
        const int q2 = i >> 4, kin = i & 15;
        const int reg = kin >> 3, half = kin & 1, cl = (kin & 7) >> 1;
        __half* ahg = ah + g * (2 * 32 * 4);
#pragma unroll
        for (int h = 0; h < 2; ++h)
        {
            ahg[((q2 * 32 + 4 * (2 * c + h) + cl) * 2 + reg) * 2 + half] = __float2half_rn(a[h]);
            if (f16_out_of_range(a[h])) atomicExch(err, DEVERR_RANGE);   // reported, not fatal
        }
    } else {
        // one 16x8x8 step: lane 4n + i/2 holds k = i in half i % 2 of its hi and lo registers
        __nv_bfloat16* abg = abf + g * (32 * 4);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const __nv_bfloat16 hi = __float2bfloat16_rn(a[h]);
            const __nv_bfloat16 lo = __float2bfloat16_rn(a[h] - __bfloat162float(hi));
            const int ln = 4 * (2 * c + h) + (i >> 1);
            abg[(ln * 2 + 0) * 2 + (i & 1)] = hi;
            abg[(ln * 2 + 1) * 2 + (i & 1)] = lo;
        }
    }
}

// ------------------------------------------------------------------ phase 2: down
// Each of the warp's four output tiles: one A fragment (one load, one dequantisation) for
// every token group of the pass; the down scales of the slice's group are applied in fp32.
template <int W, int G>
__device__ __forceinline__ void phase_down(const char* slot, const uint2* ah, const uint2* abf, int warp, int lane,
                                           float (&y)[TILES_PER_WARP][NG][4], int ng) {
    const uint2* dw = reinterpret_cast<const uint2*>(slot + gu_w_bytes_of(W) + gu_s_bytes_of(W, G)) + warp * 32 + lane;
    const float* dsc = reinterpret_cast<const float*>(slot + blk_bytes_of(W, G)) + 16 * warp + (lane >> 2);
    uint2 b0[NG], b1[NG];
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        b0[g] = b1[g] = make_uint2(0u, 0u);
        if constexpr (is_quant(W)) b0[g] = ah[g * 64 + lane];
        else b0[g] = abf[g * 32 + lane];
        if constexpr (W == FOCR_W_INT4) b1[g] = ah[g * 64 + 32 + lane];
    }
#pragma unroll
    for (int j = 0; j < TILES_PER_WARP; ++j) {
        const uint2 v = dw[j * NCW * 32];
        float s0 = 1.f, s1 = 1.f;
        if constexpr (is_quant(W)) {
            s0 = dsc[j * NCW * 16];
            s1 = dsc[j * NCW * 16 + 8];
        }
        Frag4 a0, a1;
        if constexpr (W == FOCR_W_INT4) {
            a0 = dq_int4(v.x);
            a1 = dq_int4(v.y);
        } else if constexpr (W == FOCR_W_INT8) {
            a0 = dq_int8(v.x, v.y);
        }
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            if (g < ng) {
                if constexpr (W == FOCR_W_INT4) {
                    mma16816(d, a0, b0[g].x, b0[g].y);
                    mma16816(d, a1, b1[g].x, b1[g].y);
                } else if constexpr (W == FOCR_W_INT8) {
                    mma16816(d, a0, b0[g].x, b0[g].y);
                } else {
                    mma1688_bf16(d, v.x, v.y, b0[g].x);   // a hi
                    mma1688_bf16(d, v.x, v.y, b0[g].y);   // a lo
                }
            }
            y[j][g][0] = d[0] * s0;
            y[j][g][1] = d[1] * s0;
            y[j][g][2] = d[2] * s1;
            y[j][g][3] = d[3] * s1;
        }
    }
}

__device__ __forceinline__ void consumer_sync() { named_bar_sync(1, NCT); }

// one item's phases, dispatched on whether it is a routed or a shared-expert item
template <int RW, int SW, int G>
struct ItemOps {
    static constexpr bool F16 = is_quant(RW) || is_quant(SW);
    static constexpr bool BF16 = !is_quant(RW) || !is_quant(SW);
    using XF = XFrags;
    static __device__ __forceinline__ void gate_up(bool routed, const char* slot, const XF& xf, float* acc, int warp,
                                                   int lane, int ng) {
        if (routed) phase_gate_up<RW, G>(slot, xf, acc, warp, lane, ng);
        else phase_gate_up<SW, G>(slot, xf, acc, warp, lane, ng);
    }
    static __device__ __forceinline__ void swiglu(bool routed, float* acc, __half* ah, __nv_bfloat16* abf,
                                                  const float* wn, int ctid, int ng, int* err) {
        if (routed) swiglu_to_frag<RW>(acc, ah, abf, wn, ctid, ng, err);
        else swiglu_to_frag<SW>(acc, ah, abf, wn, ctid, ng, err);
    }
    static __device__ __forceinline__ void down(bool routed, const char* slot, const uint2* ah, const uint2* abf,
                                                int warp, int lane, float (&y)[TILES_PER_WARP][NG][4], int ng) {
        if (routed) phase_down<RW, G>(slot, ah, abf, warp, lane, y, ng);
        else phase_down<SW, G>(slot, ah, abf, warp, lane, y, ng);
    }
};

template <int RW, int SW, int G>
__global__ void __launch_bounds__(NTHREADS, 1) expert_decode_kernel(ExpertParams p) {
    using SL = SmemLayout<RW, SW, G>;
    constexpr int NSLOT = SL::nslot;
    constexpr uint32_t SLOT_BYTES = SL::slot_bytes;
    using Ops = ItemOps<RW, SW, G>;
    extern __shared__ __align__(128) char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + SL::bars);
    uint64_t* empty = full + NSLOT;
    volatile int* okflag = reinterpret_cast<volatile int*>(smem + SL::misc);
    int* rec = reinterpret_cast<int*>(smem + SL::rec);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_shared = p.L.sg.slices;

    if (tid == 0) {
        for (int s = 0; s < NSLOT; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NCW);   // every consumer warp releases the slot
        }
        fence_barrier_init();
        okflag[0] = 1;   // consumer wait result
        okflag[1] = 0;   // abort
    }
    for (int i = tid; i < NG * 4 * 4 * 32; i += NTHREADS) reinterpret_cast<float*>(smem + SL::acc)[i] = 0.f;
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
        int n_items = p.shared_only ? n_shared : 0x7fffffff;
        bool waited = p.shared_only != 0;
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
    const int ctid = tid;
    int* tok = reinterpret_cast<int*>(smem + SL::tok);
    float* wn = reinterpret_cast<float*>(smem + SL::wn);
    float* acc = reinterpret_cast<float*>(smem + SL::acc);
    __half* ahh = reinterpret_cast<__half*>(smem + SL::ah);
    __nv_bfloat16* abfh = reinterpret_cast<__nv_bfloat16*>(smem + SL::abf);
    const uint2* ah = reinterpret_cast<const uint2*>(smem + SL::ah);
    const uint2* abf = reinterpret_cast<const uint2*>(smem + SL::abf);
    typename Ops::XF xf;
    float y[TILES_PER_WARP][NG][4];

    int n_items = p.shared_only ? n_shared : 0x7fffffff;
    bool waited = false;
    for (int it = 0;; ++it) {
        const int item = blockIdx.x + it * gridDim.x;
        if (item >= n_shared && !waited && !p.shared_only) {
            pdl_wait();
            waited = true;
            n_items = n_shared + p.R.active[E] * p.L.rg.slices;
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
        const int ntok = routed ? p.R.counts[expert] : p.T;
        const int seg = routed ? p.R.offsets[expert] : 0;
        for (int b0 = 0; b0 < ntok; b0 += NTP) {
            const int ng = min(NG, (ntok - b0 + NTOK - 1) / NTOK);   // token groups with tokens (CTA-uniform)
            consumer_sync();   // the previous pass is done with tok / wn
            if (ctid < NTP) {
                int tk = -1;
                float w = 0.f;
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
                wn[ctid] = w;
            }
            consumer_sync();
            load_x_frags<Ops::F16, Ops::BF16>(p.x, tok, warp, lane, !is_quant(routed ? RW : SW), xf);
            Ops::gate_up(routed, sbuf, xf, acc, warp, lane, ng);
            consumer_sync();
            Ops::swiglu(routed, acc, ahh, abfh, wn, ctid, ng, p.R.ctrl + CTRL_ERROR);
            consumer_sync();
            Ops::down(routed, sbuf, ah, abf, warp, lane, y, ng);
            if (!waited) {
                pdl_wait();   // the router initialises `out` first
                waited = true;
                if (!p.shared_only) n_items = n_shared + p.R.active[E] * p.L.rg.slices;
            }
            const int gr = lane >> 2, c = lane & 3;
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                if (g >= ng) break;
                const int t0 = tok[NTOK * g + 2 * c], t1 = tok[NTOK * g + 2 * c + 1];
#pragma unroll
                for (int j = 0; j < TILES_PER_WARP; ++j) {
                    const int row = 16 * (warp + NCW * j) + gr;
                    if (t0 >= 0) {
                        atomicAdd(p.out + (size_t)t0 * H + row, y[j][g][0]);
                        atomicAdd(p.out + (size_t)t0 * H + row + 8, y[j][g][2]);
                    }
                    if (t1 >= 0) {
                        atomicAdd(p.out + (size_t)t1 * H + row, y[j][g][1]);
                        atomicAdd(p.out + (size_t)t1 * H + row + 8, y[j][g][3]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);   // this warp is done with the slot
    }
    if (!waited) pdl_wait();   // every CTA waits before exiting (keeps the chain of forwards ordered)
}

template <int RW, int SW, int G>
cudaError_t launch_typed(const ExpertParams& p, int sms, cudaStream_t st) {
    const cudaError_t e = once_per_device((const void*)expert_decode_kernel<RW, SW, G>, [] {
        return cudaFuncSetAttribute(expert_decode_kernel<RW, SW, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)SmemLayout<RW, SW, G>::total);
    });
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(sms);
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = SmemLayout<RW, SW, G>::total;
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
                                 bool shared_only, cudaStream_t st) {
    if (T <= SMALL_T) return cudaErrorInvalidValue;   // batches of up to 8 tokens take the decode kernels
    const int sms = device_sms();
    if (sms <= 0) return cudaErrorInvalidDevice;
    const ExpertParams p{x, T, out, L, R, shared_only ? 1 : 0};
    const int rw = L.rg.wtype, sw = L.sg.wtype;
    const int g = is_quant(rw) ? L.rg.group : (is_quant(sw) ? L.sg.group : 128);
#define FOCR_CASE(A, B, GG) \
    if (rw == A && sw == B && g == GG) return launch_typed<A, B, GG>(p, sms, st);
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
