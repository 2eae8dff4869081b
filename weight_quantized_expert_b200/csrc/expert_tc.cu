// Tensor-core grouped expert kernel for batches of more than 8 tokens (batched decode,
// prefill): the shared expert and every selected routed expert as tcgen05 GEMMs with the
// accumulators in tensor memory, SwiGLU fused into the gate/up epilogue, and a combine that
// sums each token's parts in a fixed order (no atomics on the output, so repeated calls are
// bit-identical).
//
// Sources: frankenocr.pages.dev, "One forward pass", step 6 (64 routed experts + 2 fused
// shared experts, softmax top-6 without renormalisation, weighted sum of the experts); franken_ocr
// README, "Architecture" (each expert 1280 -> 896 SiLU-gated; the shared experts always on);
// "Four bits, one shared scale" (int4 nibble + f32 group scale; int8 and bf16 formats).
//
// The contraction is swapped so that the weights fill the MMA's M = 128 rows and a chunk of at
// most 128 of an expert's tokens fills N (a multiple of 16):
//   gate/up unit  (set, tile of 64 intermediates, token chunk): D[128 x N] = [G; U]_tile X^T over
//                 K = 1280 (block rows interleave gate and up by 8, see the tensor-core layout
//                 in common.cuh); the epilogue pairs each gate lane with its up lane (shuffle
//                 by 8) and writes a = silu(g) * u * w_route as bf16 into the "a image"
//   down unit     (set, m-tile of 128 output rows, [K part,] token chunk): D = Down_mtile a^T
//                 over the set's intermediates (the shared set's in up to 8 K parts); the
//                 epilogue writes fp32 rows y per (token, slot) or per (token, part)
//   combine       out[t] = resid + sum_parts y_shared + sum_{j<6} y_slot[t*6+j]
// Units are handed out by a global atomic counter (largest classes first: shared gate/up,
// routed gate/up, shared down, routed down), so a unit only ever waits on units with smaller
// numbers, which running CTAs hold: a down unit's B load waits (bounded) for its expert's
// gate/up units to have written their a rows.
//
// Warp roles (one CTA per SM, 448 threads):
//   warp 0      loader: takes units, publishes their descriptors, streams quantised weight
//               blocks (codes + scales, 4.5-8.5 KB per 128 x 64 block) into a ring with bulk
//               async copies (cp.async.bulk + mbarrier), and prefetches bf16 blocks into L2
//   warp 1      MMA: one thread issues tcgen05.mma (kind::f16, bf16 operands, fp32 accumulate
//               in TMEM; 4 k-steps of 16 per block) and commits stages and accumulators
//   warps 2-9   stagers: dequantise a block (q * s rounded to bf16; int4 by the exponent-bias
//               method, int8 through fp32) into the K-major core-matrix layout, gather the
//               chunk's token rows of x (bf16) as the B operand, or bulk-copy bf16 blocks and
//               a-image rows
//   warps 10-13 epilogue: tcgen05.ld of a 128-column accumulator (four in TMEM, so the MMA
//               runs ahead), SwiGLU or output rows, then the unit's completion counter
// Every wait is bounded in time (%globaltimer); on expiry the kernel records an error word,
// stops taking work, waits (bounded) for its own copies in flight, frees TMEM and returns.
#include <cuda_bf16.h>

#include "common.cuh"
#include "fragments.cuh"
#include "umma.cuh"

namespace focr {
namespace {

constexpr int NSTG = 8;                          // stager warps
constexpr int NEPI = 4;                          // epilogue warps
constexpr int WARP_LOAD = 0, WARP_MMA = 1, WARP_STG = 2, WARP_EPI = WARP_STG + NSTG;
constexpr int WARP_COPY = WARP_EPI + NEPI;       // streams quantised blocks into the raw ring
constexpr int WARP_BLD = WARP_COPY + 1;          // fills operand stages by copy: bf16 A, token rows, a rows
constexpr int NWARPS = WARP_BLD + 1;
constexpr int NTHREADS = NWARPS * 32;
constexpr int NCH = 128;                         // tokens of one unit at most (the MMA's N)
constexpr int NAB = 5;                           // operand stages
constexpr int NPAIR = NSTG / 2;                  // stager warp pairs, one operand stage each in turn
constexpr uint32_t A_BYTES = TC_M * TC_KB * 2;   // 16 KB bf16 A block
constexpr uint32_t B_BYTES = NCH * TC_KB * 2;    // 16 KB bf16 B block
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t RAW_BUDGET = 46 * 1024;       // quantised blocks in flight (plus L2 prefetch)
constexpr int UR = 6;                            // unit descriptors in flight
constexpr int NACC = 4;                          // TMEM accumulators of 128 columns
constexpr uint32_t TMEM_COLS = 512;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // 2 s
constexpr int DEVERR_TC_WAIT = 3;

enum UnitKind { UK_GU_S = 0, UK_GU_R = 1, UK_DN_S = 2, UK_DN_R = 3, UK_XG = 4, UK_END = 5 };

struct Unit {
    int kind, expert, tile, part;
    int kb0, nkb;        // K-blocks [kb0, kb0 + nkb) of the set's matrix
    int ntok, N;         // tokens of the chunk, N = ntok rounded up to 16
    int c0;              // first token of the chunk: shared, a token id; routed, an index in the expert's segment
    int arow;            // first row of the chunk in the a image
    int wdep, wtarget;   // counter (index into the tensor-core control words) to wait for before the B loads, -1: none
    int ddep;            // counter this unit's completion adds to
    int seg;             // routed: first dispatch entry of the chunk (index into the permutation)
    int ent[NCH];        // routed: dispatch entries t * 6 + j of the chunk's tokens
    float w[NCH];        // routed gate/up: their routing weights
};

struct Sched {
    int T, U, nchs, cs_s, P, KPP;
    int n_xg, n_gu_s, n_gu_r, n_dn_s, n_dn_r, total;
    int e[E], n[E], off[E], poff[E], nch[E], cs[E];
    int gu_pre[E + 1], dn_pre[E + 1];
};

struct TcParams {
    const float* x;      // [T][1280] fp32
    int T;
    float* out;
    int resid;
    int shared_only;
    TcView V;
    RouteView R;
    TcWork W;
};

__host__ __device__ constexpr uint32_t cmax(uint32_t a, uint32_t b) { return a > b ? a : b; }

template <int RW, int SW, int G>
struct TcSmem {
    static constexpr uint32_t raw_r = is_quant(RW) ? tc_block_bytes(RW, G) : 0u;
    static constexpr uint32_t raw_s = is_quant(SW) ? tc_block_bytes(SW, G) : 0u;
    static constexpr uint32_t raw_slot = (cmax(cmax(raw_r, raw_s), 128u) + 127u) & ~127u;
    static constexpr int NR = (is_quant(RW) || is_quant(SW))
                                  ? ((int)(RAW_BUDGET / raw_slot) > 32 ? 32 : (int)(RAW_BUDGET / raw_slot))
                                  : 2;
    static constexpr uint32_t ab = 0;                                        // [NAB][A | B]
    static constexpr uint32_t raw = ab + NAB * STAGE_BYTES;                  // [NR][raw_slot]
    static constexpr uint32_t units = raw + NR * raw_slot;                   // [UR] Unit
    static constexpr uint32_t sched = (units + UR * (uint32_t)sizeof(Unit) + 15u) & ~15u;
    static constexpr uint32_t bars = (sched + (uint32_t)sizeof(Sched) + 7u) & ~7u;
    static constexpr int NBARS = 2 * NAB + 2 * NR + 2 * UR + 2 * NACC + 1;
    static constexpr uint32_t misc = bars + 8u * NBARS;                      // tmem base, abort flag
    static constexpr uint32_t total = misc + 16u;
    static_assert(total <= 232448, "shared memory budget");
};

// ------------------------------------------------------------------ small PTX helpers

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void fence_proxy_async_all() { asm volatile("fence.proxy.async;" ::: "memory"); }

__device__ __forceinline__ void sts128(void* p, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(p)), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint2 lds64(const void* p) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(smem_u32(p)));
    return v;
}

// Wait (bounded) until the counter reaches `target`.
__device__ __forceinline__ bool wait_counter(const int* p, int target) {
    if (ld_acquire(p) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire(p) < target) {
        if (globaltimer_ns() - t0 > WAIT_LIMIT_NS) return false;
        __nanosleep(100);
    }
    return true;
}

// ------------------------------------------------------------------ dequantisation to bf16
__device__ __forceinline__ uint32_t bf2_sub(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t bf2_mul(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

constexpr uint32_t BF2_MAGIC = 0x43004300u;   // (128, 128): a nibble n under it reads as 128 + n
constexpr uint32_t BF2_136 = 0x43084308u;     // (136, 136)

// One k-core of int4 codes (element 2m in nibble m, 2m+1 in nibble m+4, q + 8) -> 8 bf16 q * s.
// q = (128 + n) - 136 is exact in bf16; the product is rounded once (s2 = bf16 pair of the scale).
__device__ __forceinline__ uint4 dq_int4_bf16(uint32_t w, uint32_t s2) {
    uint4 r;
    r.x = bf2_mul(bf2_sub((w & 0x000F000Fu) | BF2_MAGIC, BF2_136), s2);
    r.y = bf2_mul(bf2_sub(((w >> 4) & 0x000F000Fu) | BF2_MAGIC, BF2_136), s2);
    r.z = bf2_mul(bf2_sub(((w >> 8) & 0x000F000Fu) | BF2_MAGIC, BF2_136), s2);
    r.w = bf2_mul(bf2_sub(((w >> 12) & 0x000F000Fu) | BF2_MAGIC, BF2_136), s2);
    return r;
}

// One k-core of int8 codes (q + 128 in bytes 0..7) -> 8 bf16 q * s (fp32 product, one rounding).
__device__ __forceinline__ uint4 dq_int8_bf16(uint32_t w0, uint32_t w1, float s) {
    float f[8];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        f[b] = (byte_to_float(w0, b) - 8388736.0f) * s;
        f[4 + b] = (byte_to_float(w1, b) - 8388736.0f) * s;
    }
    return make_uint4(f32x2_to_bf16x2(f[0], f[1]), f32x2_to_bf16x2(f[2], f[3]), f32x2_to_bf16x2(f[4], f[5]),
                      f32x2_to_bf16x2(f[6], f[7]));
}

// Warp hw (0, 1) of a stager pair turns block rows 64 hw .. 64 hw + 63 of a quantised block into
// the bf16 A operand: lane (pr = lane / 8, rr = lane % 8) writes k-cores pr and pr + 4 of rows
// 8 g + rr of each of the warp's eight row groups g; every warp store covers 512 contiguous bytes.
template <int W, int G>
__device__ __forceinline__ void dequant_half(const uint8_t* raw, char* A, int hw, int lane) {
    constexpr int SPK = tc_spk(G);
    constexpr uint32_t RB = tc_row_bytes(W);
    const float* sc = reinterpret_cast<const float*>(raw + TC_M * RB);
    const int pr = lane >> 3, rr = lane & 7;
#pragma unroll 4
    for (int gg = 0; gg < 8; ++gg) {
        const int g = 8 * hw + gg;          // row group
        const int row = 8 * g + rr;
        const float s0 = sc[row * SPK], s1 = sc[row * SPK + SPK - 1];
        char* d0 = A + g * 1024 + pr * 128 + rr * 16;
        if constexpr (W == FOCR_W_INT4) {
            const uint2 c = lds64(raw + row * 32 + pr * 8);
            const uint32_t b0 = f32x2_to_bf16x2(s0, s0);
            sts128(d0, dq_int4_bf16(c.x, b0));
            sts128(d0 + 512, dq_int4_bf16(c.y, SPK == 1 ? b0 : f32x2_to_bf16x2(s1, s1)));
        } else {
            const uint4 c = lds128(raw + row * 64 + pr * 16);
            sts128(d0, dq_int8_bf16(c.x, c.y, s0));
            sts128(d0 + 512, dq_int8_bf16(c.z, c.w, s1));
        }
    }
}

// weight block kb (absolute) of a unit's A operand
__device__ __forceinline__ const uint8_t* a_block(const TcView& V, const Unit& U, int kb) {
    const bool routed = U.kind == UK_GU_R || U.kind == UK_DN_R;
    const TcSetView& S = routed ? V.r : V.s;
    if (U.kind <= UK_GU_R)
        return S.gu + (routed ? (size_t)U.expert * S.g.gu_bytes : 0) + ((size_t)U.tile * TC_KBH + kb) * S.g.blk;
    return S.dn + (routed ? (size_t)U.expert * S.g.dn_bytes : 0) + ((size_t)U.tile * S.g.tiles + kb) * S.g.blk;
}

// ------------------------------------------------------------------ the kernel
template <int RW, int SW, int G>
__global__ void __launch_bounds__(NTHREADS, 1) expert_tc_kernel(TcParams p) {
    using SL = TcSmem<RW, SW, G>;
    constexpr int NR = SL::NR;
    extern __shared__ __align__(1024) char smem[];
    Unit* units = reinterpret_cast<Unit*>(smem + SL::units);
    Sched& S = *reinterpret_cast<Sched*>(smem + SL::sched);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SL::bars);
    uint64_t* ab_full = bars;
    uint64_t* ab_empty = ab_full + NAB;
    uint64_t* raw_full = ab_empty + NAB;
    uint64_t* raw_empty = raw_full + NR;
    uint64_t* u_full = raw_empty + NR;
    uint64_t* u_empty = u_full + UR;
    uint64_t* acc_full = u_empty + UR;
    uint64_t* acc_empty = acc_full + NACC;
    uint64_t* drain = acc_empty + NACC;   // the MMA thread's last commit before TMEM is freed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SL::misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SL::misc + 4);
    int* ctrl = p.R.ctrl + CTRL_TC;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < NAB; ++i) {
            mbar_init(&ab_full[i], 2 + 1);   // the dequantising pair's two warps + the loader
            mbar_init(&ab_empty[i], 1);
        }
        for (int i = 0; i < NR; ++i) {
            mbar_init(&raw_full[i], 1);
            mbar_init(&raw_empty[i], 2);
        }
        for (int i = 0; i < UR; ++i) {
            mbar_init(&u_full[i], 1);
            mbar_init(&u_empty[i], NSTG + 1 + NEPI + 2);
        }
        for (int i = 0; i < NACC; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], NEPI);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == WARP_MMA) umma::tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();   // routing, x rows and the output of the previous kernel are complete

    auto fail = [&](int code) {
        atomicExch(&p.R.ctrl[CTRL_ERROR], code);
        *abort_flag = 1;
    };

    if (warp == WARP_LOAD) {
        // ------------------------------------------------------------ schedule (whole warp)
        const TcGeom& rg = p.V.r.g;
        const TcGeom& sg = p.V.s.g;
        const int T = p.T;
        const int U = p.shared_only ? 0 : p.R.active[E];
        int pad[2], gu[2], dn[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int a = lane + 32 * h;
            pad[h] = gu[h] = dn[h] = 0;
            if (a < U) {
                const int e = p.R.active[a];
                const int n = p.R.counts[e];
                const int nch0 = (n + NCH - 1) / NCH;
                const int cs = ((n + nch0 - 1) / nch0 + 15) & ~15;   // chunk size, a multiple of 16
                const int nch = (n + cs - 1) / cs;
                S.e[a] = e;
                S.n[a] = n;
                S.off[a] = p.R.offsets[e];
                S.nch[a] = nch;
                S.cs[a] = cs;
                pad[h] = (n + 15) & ~15;
                gu[h] = rg.tiles * nch;
                dn[h] = TC_MT * nch;
            }
        }
        // exclusive prefix sums over the active experts a = lane + 32 h (padded a-image rows,
        // gate/up units, down units)
        int sp[2] = {pad[0], pad[1]}, sgu[2] = {gu[0], gu[1]}, sdn[2] = {dn[0], dn[1]};
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int vp = __shfl_up_sync(0xffffffffu, sp[h], o);
                const int vg = __shfl_up_sync(0xffffffffu, sgu[h], o);
                const int vd = __shfl_up_sync(0xffffffffu, sdn[h], o);
                if (lane >= o) {
                    sp[h] += vp;
                    sgu[h] += vg;
                    sdn[h] += vd;
                }
            }
        sp[1] += __shfl_sync(0xffffffffu, sp[0], 31);
        sgu[1] += __shfl_sync(0xffffffffu, sgu[0], 31);
        sdn[1] += __shfl_sync(0xffffffffu, sdn[0], 31);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int a = lane + 32 * h;
            if (a < U) {
                S.poff[a] = sp[h] - pad[h];
                S.gu_pre[a] = sgu[h] - gu[h];
                S.dn_pre[a] = sdn[h] - dn[h];
            }
        }
        if (lane == 31) {
            S.gu_pre[U] = sgu[1];
            S.dn_pre[U] = sdn[1];
            S.T = T;
            S.U = U;
            const int nch0 = (T + NCH - 1) / NCH;
            S.cs_s = ((T + nch0 - 1) / nch0 + 15) & ~15;
            S.nchs = (T + S.cs_s - 1) / S.cs_s;
            S.P = tc_parts(sg.inter);
            S.KPP = tc_kpp(sg.inter);
            S.n_xg = U;
            S.n_gu_s = sg.tiles * S.nchs;
            S.n_gu_r = sgu[1];
            S.n_dn_s = TC_MT * S.P * S.nchs;
            S.n_dn_r = sdn[1];
            S.total = S.n_xg + S.n_gu_s + S.n_gu_r + S.n_dn_s + S.n_dn_r;
        }
        __syncwarp();

        // ------------------------------------------------------------ loader loop
        for (int k = 0;; ++k) {
            int u = 0;
            if (lane == 0) u = *abort_flag ? S.total : atomicAdd(&ctrl[TC_WORK], 1);
            u = __shfl_sync(0xffffffffu, u, 0);
            const int slot = k % UR;
            bool ok = true;
            if (lane == 0) ok = mbar_wait_bounded(&u_empty[slot], ((k / UR) & 1) ^ 1, WAIT_LIMIT_NS);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) {
                if (lane == 0) fail(DEVERR_TC_WAIT);
                break;
            }
            Unit& Un = units[slot];
            int kind = UK_END;
            if (u < S.total) {
                int v = u;
                if (v < S.n_xg) {
                    // gather unit of active expert v: its token rows of x into dispatch order
                    kind = UK_XG;
                    if (lane == 0) {
                        Un.expert = S.e[v];
                        Un.tile = Un.part = 0;
                        Un.kb0 = Un.nkb = 0;
                        Un.c0 = 0;
                        Un.ntok = S.n[v];
                        Un.arow = S.poff[v];
                        Un.seg = S.off[v];
                        Un.wdep = -1;
                        Un.wtarget = 0;
                        Un.ddep = TC_DEP_X + S.e[v];
                    }
                } else if ((v -= S.n_xg) < S.n_gu_s) {
                    kind = UK_GU_S;
                    const int tile = v / S.nchs, ch = v % S.nchs;
                    if (lane == 0) {
                        Un.expert = -1;
                        Un.tile = tile;
                        Un.part = tile / S.KPP;
                        Un.kb0 = 0;
                        Un.nkb = TC_KBH;
                        Un.c0 = ch * S.cs_s;
                        Un.ntok = min(S.cs_s, T - Un.c0);
                        Un.arow = Un.c0;
                        Un.wdep = -1;
                        Un.wtarget = 0;
                        Un.ddep = TC_DEP_S + Un.part;
                    }
                } else if ((v -= S.n_gu_s) < S.n_gu_r) {
                    kind = UK_GU_R;
                } else if ((v -= S.n_gu_r) < S.n_dn_s) {
                    kind = UK_DN_S;
                    const int mt = v / (S.P * S.nchs), rem = v % (S.P * S.nchs);
                    const int part = rem / S.nchs, ch = rem % S.nchs;
                    if (lane == 0) {
                        Un.expert = -1;
                        Un.tile = mt;
                        Un.part = part;
                        Un.kb0 = part * S.KPP;
                        Un.nkb = min(S.KPP, sg.tiles - Un.kb0);
                        Un.c0 = ch * S.cs_s;
                        Un.ntok = min(S.cs_s, T - Un.c0);
                        Un.arow = Un.c0;
                        Un.wdep = TC_DEP_S + part;
                        Un.wtarget = Un.nkb * S.nchs * NEPI;
                        Un.ddep = TC_DN_DONE;
                    }
                } else {
                    v -= S.n_dn_s;
                    kind = UK_DN_R;
                }
                if (kind == UK_GU_R || kind == UK_DN_R) {
                    const int* pre = kind == UK_GU_R ? S.gu_pre : S.dn_pre;
                    int lo = 0, hi = S.U - 1;   // last a with pre[a] <= v
                    while (lo < hi) {
                        const int mid = (lo + hi + 1) >> 1;
                        if (pre[mid] <= v) lo = mid;
                        else hi = mid - 1;
                    }
                    const int a = lo, w = v - pre[a];
                    const int nch = S.nch[a];
                    const int tile = w / nch, ch = w % nch;
                    const int c0 = ch * S.cs[a];
                    const int ntok = min(S.cs[a], S.n[a] - c0);
                    const int seg = S.off[a] + c0;
                    if (lane == 0) {
                        Un.expert = S.e[a];
                        Un.tile = tile;
                        Un.part = 0;
                        Un.kb0 = 0;
                        Un.nkb = kind == UK_GU_R ? TC_KBH : rg.tiles;
                        Un.c0 = c0;
                        Un.ntok = ntok;
                        Un.arow = S.poff[a] + c0;
                        Un.seg = seg;
                        // gate/up waits for the expert's gathered rows, down for all its gate/up units
                        Un.wdep = kind == UK_DN_R ? TC_DEP_R + S.e[a] : TC_DEP_X + S.e[a];
                        Un.wtarget = kind == UK_DN_R ? rg.tiles * nch * NEPI : NEPI;
                        Un.ddep = kind == UK_DN_R ? TC_DN_DONE : TC_DEP_R + S.e[a];
                    }
                    for (int n = lane; n < ntok; n += 32) {
                        const int ent = p.R.perm[seg + n];
                        Un.ent[n] = ent;
                        Un.w[n] = p.R.topk_w[ent];
                    }
                }
                if (lane == 0) Un.N = (Un.ntok + 15) & ~15;
            }
            if (lane == 0) Un.kind = kind;
            __syncwarp();
            if (lane == 0) mbar_arrive(&u_full[slot]);
            if (kind == UK_END) break;
            if (lane == 0 && kind != UK_XG) {
                // the copier will stream this unit's blocks a few units from now: bring them into L2
                const bool routed = kind == UK_GU_R || kind == UK_DN_R;
                const int wt = routed ? RW : SW;
                const uint32_t blk = is_quant(wt) ? (routed ? p.V.r.g.blk : p.V.s.g.blk) : A_BYTES;
                const uint8_t* b0 = a_block(p.V, Un, Un.kb0);
                const uint32_t bytes = (uint32_t)Un.nkb * blk;   // the unit's blocks are contiguous
                for (uint32_t o = 0; o < bytes; o += 64u * 1024u)
                    bulk_prefetch_l2(b0 + o, min(64u * 1024u, bytes - o));
            }
            if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;
        }
    } else if (warp == WARP_COPY) {
        // ------------------------------------------------------------ raw-ring copier (one thread)
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            int raw_i = 0;
            for (int k = 0;; ++k) {
                const int slot = k % UR;
                if (!mbar_wait_bounded(&u_full[slot], (k / UR) & 1, WAIT_LIMIT_NS)) {
                    fail(DEVERR_TC_WAIT);
                    break;
                }
                const Unit& Un = units[slot];
                const int kind = Un.kind;
                if (kind == UK_END) {
                    mbar_arrive(&u_empty[slot]);
                    break;
                }
                const bool routed = kind == UK_GU_R || kind == UK_DN_R;
                const int wt = routed ? RW : SW;
                bool ok = true;
                if (is_quant(wt)) {
                    const uint32_t blk = routed ? p.V.r.g.blk : p.V.s.g.blk;
                    const int nkb = Un.nkb, kb0 = Un.kb0;
                    for (int kb = 0; kb < nkb; ++kb, ++raw_i) {
                        const int r = raw_i % NR;
                        if (!mbar_wait_bounded(&raw_empty[r], ((raw_i / NR) & 1) ^ 1, WAIT_LIMIT_NS)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&raw_full[r], blk);
                        bulk_g2s(smem + SL::raw + r * SL::raw_slot, a_block(p.V, Un, kb0 + kb), blk, &raw_full[r],
                                 pol);
                    }
                }
                mbar_arrive(&u_empty[slot]);
                if (!ok) {
                    fail(DEVERR_TC_WAIT);
                    break;
                }
                if (*abort_flag) break;
            }
            // never leave copies in flight: the last NR issued blocks must have landed
            for (int i = max(0, raw_i - NR); i < raw_i; ++i)
                (void)mbar_wait_bounded(&raw_full[i % NR], (i / NR) & 1, WAIT_LIMIT_NS);
        }
        __syncwarp();
    } else if (warp == WARP_BLD) {
        // ------------------------------------------------------------ operand-stage loader (one thread)
        // Every stage in order: the B operand (N rows of an operand image: x in token order for the
        // shared set, x in dispatch order for routed experts, a for down projections) and, for
        // bf16 weights, the A block, by bulk copies completing on the stage barrier.
        if (lane == 0) {
            int ab_i = 0;
            for (int k = 0;; ++k) {
                const int slot = k % UR;
                if (!mbar_wait_bounded(&u_full[slot], (k / UR) & 1, WAIT_LIMIT_NS)) {
                    fail(DEVERR_TC_WAIT);
                    break;
                }
                const Unit& Un = units[slot];
                const int kind = Un.kind;
                if (kind == UK_END) {
                    mbar_arrive(&u_empty[slot]);
                    break;
                }
                const bool routed = kind == UK_GU_R || kind == UK_DN_R;
                const bool is_gu = kind <= UK_GU_R;
                const bool quant = is_quant(routed ? RW : SW);
                const int N = Un.N, kb0 = Un.kb0, nkb = Un.nkb;
                const uint16_t* img = is_gu ? (routed ? p.W.x_img_r : p.W.x_img) : (routed ? p.W.a_img : p.W.a_sh);
                const int rows = routed ? p.W.arows : p.W.tpad;
                const uint32_t bbytes = (uint32_t)N * 128u;
                bool ok = true;
                if (nkb > 0 && Un.wdep >= 0) {
                    // the rows come from other units' epilogues: wait until they are all written
                    ok = wait_counter(&ctrl[Un.wdep], Un.wtarget);
                    fence_proxy_async_all();
                }
                for (int kb = 0; kb < nkb && ok; ++kb, ++ab_i) {
                    const int s = ab_i % NAB;
                    char* Ast = smem + SL::ab + s * STAGE_BYTES;
                    if (!mbar_wait_bounded(&ab_empty[s], ((ab_i / NAB) & 1) ^ 1, WAIT_LIMIT_NS)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&ab_full[s], bbytes + (quant ? 0u : A_BYTES));
                    if (!quant) bulk_g2s(Ast, a_block(p.V, Un, kb0 + kb), A_BYTES, &ab_full[s], policy_evict_first());
                    bulk_g2s(Ast + A_BYTES, img + ((size_t)(kb0 + kb) * rows + Un.arow) * TC_KB, bbytes, &ab_full[s],
                             policy_evict_last());
                }
                if (!ok) {
                    fail(DEVERR_TC_WAIT);
                    break;
                }
                mbar_arrive(&u_empty[slot]);
                if (*abort_flag) break;
            }
        }
        __syncwarp();
    } else if (warp == WARP_MMA) {
        // ------------------------------------------------------------ MMA issuer (one thread)
        if (lane == 0) {
            int ab_i = 0, acc_i = 0;
            for (int k = 0;; ++k) {
                const int slot = k % UR;
                if (!mbar_wait_bounded(&u_full[slot], (k / UR) & 1, WAIT_LIMIT_NS)) {
                    fail(DEVERR_TC_WAIT);
                    break;
                }
                const Unit& Un = units[slot];
                if (Un.kind == UK_END) {
                    mbar_arrive(&u_empty[slot]);
                    break;
                }
                if (Un.kind == UK_XG) {   // no MMA work
                    mbar_arrive(&u_empty[slot]);
                    continue;
                }
                const int b = acc_i % NACC;
                if (!mbar_wait_bounded(&acc_empty[b], ((acc_i / NACC) & 1) ^ 1, WAIT_LIMIT_NS)) {
                    fail(DEVERR_TC_WAIT);
                    break;
                }
                umma::fence_after_sync();
                const uint32_t idesc = umma::idesc_bf16_f32(TC_M, Un.N);
                const uint32_t d = tmem_base + (uint32_t)(b * 128);
                bool ok = true;
                for (int kb = 0; kb < Un.nkb; ++kb, ++ab_i) {
                    const int s = ab_i % NAB;
                    if (!mbar_wait_bounded(&ab_full[s], (ab_i / NAB) & 1, WAIT_LIMIT_NS)) {
                        ok = false;
                        break;
                    }
                    umma::fence_after_sync();
                    const uint32_t a0 = smem_u32(smem + SL::ab + s * STAGE_BYTES);
                    const uint32_t b0 = a0 + A_BYTES;
#pragma unroll
                    for (int j = 0; j < TC_KB / 16; ++j)
                        umma::mma_bf16(d, umma::sdesc_kmajor(a0 + 256u * j, 128u, 1024u),
                                       umma::sdesc_kmajor(b0 + 256u * j, 128u, 1024u), idesc, kb > 0 || j > 0);
                    umma::commit(smem_u32(&ab_empty[s]));
                }
                if (!ok) {
                    fail(DEVERR_TC_WAIT);
                    break;
                }
                umma::commit(smem_u32(&acc_full[b]));
                ++acc_i;
                mbar_arrive(&u_empty[slot]);
                if (*abort_flag) break;
            }
            // every MMA this thread issued has completed before TMEM can be freed
            umma::commit(smem_u32(drain));
            (void)mbar_wait_bounded(drain, 0, WAIT_LIMIT_NS);
        }
        __syncwarp();
    } else if (warp < WARP_EPI) {
        // ------------------------------------------------------------ dequantising stagers
        // Warp pair pp = (sw / 2) takes every NPAIR-th operand stage in turn; warp hw = sw % 2 of
        // the pair dequantises block rows 64 hw .. 64 hw + 63 of a quantised A block (for a bf16
        // block the pair only takes its turn: the loader warp copies it).  The pair's stores are
        // ordered before the tensor core's reads by a proxy fence, then each warp arrives.
        const int sw = warp - WARP_STG;
        const int pp = sw >> 1, hw = sw & 1;
        int ab_i = 0, raw_i = 0;
        for (int k = 0;; ++k) {
            const int slot = k % UR;
            bool ok = true;
            if (lane == 0) ok = mbar_wait_bounded(&u_full[slot], (k / UR) & 1, WAIT_LIMIT_NS);
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
                if (lane == 0) fail(DEVERR_TC_WAIT);
                break;
            }
            const Unit& Un = units[slot];
            const int kind = Un.kind;
            if (kind == UK_END) {
                if (lane == 0) mbar_arrive(&u_empty[slot]);
                break;
            }
            const bool routed = kind == UK_GU_R || kind == UK_DN_R;
            const bool quant = is_quant(routed ? RW : SW);
            const int nkb = Un.nkb;
            for (int kb = 0; kb < nkb && ok; ++kb, ++ab_i) {
                const int r = raw_i;
                if (quant) ++raw_i;
                if (ab_i % NPAIR != pp) continue;
                const int s = ab_i % NAB;
                char* Ast = smem + SL::ab + s * STAGE_BYTES;
                if (lane == 0) ok = mbar_wait_bounded(&ab_empty[s], ((ab_i / NAB) & 1) ^ 1, WAIT_LIMIT_NS);
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) break;
                if (quant) {
                    const int rs = r % NR;
                    if (lane == 0) ok = mbar_wait_bounded(&raw_full[rs], (r / NR) & 1, WAIT_LIMIT_NS);
                    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                    if (!ok) break;
                    const uint8_t* raw = reinterpret_cast<const uint8_t*>(smem + SL::raw + rs * SL::raw_slot);
                    if (routed) {
                        if constexpr (is_quant(RW)) dequant_half<RW, G>(raw, Ast, hw, lane);
                    } else {
                        if constexpr (is_quant(SW)) dequant_half<SW, G>(raw, Ast, hw, lane);
                    }
                    umma::fence_smem_to_async();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&raw_empty[rs]);
                }
                if (lane == 0) mbar_arrive(&ab_full[s]);
            }
            if (!ok) {
                if (lane == 0) fail(DEVERR_TC_WAIT);
                break;
            }
            if (lane == 0) mbar_arrive(&u_empty[slot]);
            if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;   // TMEM lane quarter this warp may access
        int acc_i = 0;
        for (int k = 0;; ++k) {
            const int slot = k % UR;
            bool ok = true;
            if (lane == 0) ok = mbar_wait_bounded(&u_full[slot], (k / UR) & 1, WAIT_LIMIT_NS);
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
                if (lane == 0) fail(DEVERR_TC_WAIT);
                break;
            }
            const Unit& Un = units[slot];
            const int kind = Un.kind;
            if (kind == UK_END) {
                if (lane == 0) mbar_arrive(&u_empty[slot]);
                break;
            }
            if (kind == UK_XG) {
                // the expert's token rows of x, in dispatch order, into its padded segment of the
                // dispatch-order image: 16-byte pieces, consecutive threads writing consecutive pieces
                const int et = (warp - WARP_EPI) * 32 + lane, n = Un.ntok, r8 = (n + 7) & ~7;
                const int per_kb = r8 * 8;   // pieces of one K-block
                const uint4* src = reinterpret_cast<const uint4*>(p.W.x_img);
                uint4* dst = reinterpret_cast<uint4*>(p.W.x_img_r);
                for (int c = et; c < TC_KBH * per_kb; c += NEPI * 32) {
                    const int kb = c / per_kb, rem = c % per_kb;
                    const int row = (rem >> 6) * 8 + (rem & 7), kc = (rem >> 3) & 7;
                    if (row < n) {
                        const int t = p.R.perm[Un.seg + row] / K;
                        dst[img_index(p.W.arows, Un.arow + row, kb * TC_KB + kc * 8) / 8] =
                            __ldg(src + img_index(p.W.tpad, t, kb * TC_KB + kc * 8) / 8);
                    }
                }
                fence_proxy_async_all();
                __threadfence();
                __syncwarp();
                if (lane == 0) {
                    atomicAdd(&ctrl[Un.ddep], 1);
                    mbar_arrive(&u_empty[slot]);
                }
                continue;
            }
            const int b = acc_i % NACC;
            if (lane == 0) ok = mbar_wait_bounded(&acc_full[b], (acc_i / NACC) & 1, WAIT_LIMIT_NS);
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
                if (lane == 0) fail(DEVERR_TC_WAIT);
                break;
            }
            umma::fence_after_sync();
            const bool routed = kind == UK_GU_R || kind == UK_DN_R;
            const int ntok = Un.ntok, N = Un.N;
            const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * 128);
            if (kind <= UK_GU_R) {
                const bool gate = (lane & 8) == 0;
                const int i = TC_KB * Un.tile + 16 * q + 8 * (lane >> 4) + (lane & 7);   // intermediate
                uint16_t* img = routed ? p.W.a_img : p.W.a_sh;
                const int rows = routed ? p.W.arows : p.W.tpad;
                uint16_t* col = img + (size_t)(i / TC_KB) * rows * TC_KB + ((i % TC_KB) / 8) * 64 + (i % 8);
                for (int c = 0; c < N; c += 16) {
                    float v[16];
                    umma::ld16(taddr + (uint32_t)c, v);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float other = __shfl_xor_sync(0xffffffffu, gate ? v[8 + j] : v[j], 8);
                        const float g = gate ? v[j] : other;
                        const float u = gate ? other : v[8 + j];
                        const int n = c + (gate ? j : 8 + j);
                        if (n < ntok) {
                            const float w = routed ? Un.w[n] : 1.0f;
                            const float a = __fdividef(g, 1.0f + __expf(-g)) * u * w;
                            const int row = Un.arow + n;
                            col[(size_t)(row >> 3) * 512 + (row & 7) * 8] =
                                __bfloat16_as_ushort(__float2bfloat16_rn(a));
                        }
                    }
                }
            } else {
                const int m = TC_M * Un.tile + 32 * q + lane;   // output row
                for (int c = 0; c < N; c += 16) {
                    float v[16];
                    umma::ld16(taddr + (uint32_t)c, v);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int n = c + j;
                        if (n < ntok) {
                            float* dst = routed ? p.W.y_slot + (size_t)Un.ent[n] * H + m
                                                : p.W.y_sh + ((size_t)Un.part * p.T + Un.c0 + n) * H + m;
                            *dst = v[j];
                        }
                    }
                }
            }
            umma::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[b]);
            ++acc_i;
            // publish: this warp's rows, then its completion count (a unit is complete when all
            // NEPI epilogue warps have counted it)
            fence_proxy_async_all();
            __threadfence();
            __syncwarp();
            if (lane == 0) atomicAdd(&ctrl[Un.ddep], 1);
            if (lane == 0) mbar_arrive(&u_empty[slot]);
            if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;
        }
    }

    // ---------------------------------------------------------------- combine (all threads)
    umma::fence_before_sync();
    __syncthreads();
    pdl_launch_dependents();
    __shared__ int go;
    if (tid == 0) {
        go = 0;
        if (!*abort_flag) {
            if (wait_counter(&ctrl[TC_DN_DONE], (S.n_dn_s + S.n_dn_r) * NEPI)) go = 1;
            else fail(DEVERR_TC_WAIT);
        }
    }
    __syncthreads();
    if (go) {
        const int T = p.T, P = S.P;
        const int n4 = T * (H / 4);
        const float4* x4 = reinterpret_cast<const float4*>(p.x);
        const float4* ys4 = reinterpret_cast<const float4*>(p.W.y_sh);
        const float4* yr4 = reinterpret_cast<const float4*>(p.W.y_slot);
        float4* o4 = reinterpret_cast<float4*>(p.out);
        for (int i = blockIdx.x * NTHREADS + tid; i < n4; i += gridDim.x * NTHREADS) {
            const int t = i / (H / 4), c = i % (H / 4);
            float4 a = p.resid ? __ldg(x4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            for (int pp = 0; pp < P; ++pp) {
                const float4 v = __ldcg(ys4 + ((size_t)pp * T + t) * (H / 4) + c);
                a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
            }
            if (!p.shared_only) {
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    const float4 v = __ldcg(yr4 + ((size_t)t * K + j) * (H / 4) + c);
                    a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
                }
            }
            o4[i] = a;
        }
    }
    __syncthreads();
    if (warp == WARP_MMA) {
        umma::fence_after_sync();
        umma::tmem_free(tmem_base, TMEM_COLS);
    }
    if (tid == 0) {
        // the last CTA returns the counters to zero for the next forward
        __threadfence();
        if (atomicAdd(&ctrl[TC_EXIT], 1) == (int)gridDim.x - 1) {
            __threadfence();
            for (int i = 0; i < TC_WORDS; ++i) ctrl[i] = 0;
            __threadfence();
        }
    }
}

// x (fp32) -> the bf16 operand image in token order (the dense layer has no router to write it)
__global__ void x_image_kernel(const float* x, int T, int rows, uint16_t* img) {
    pdl_wait();
    pdl_launch_dependents();
    const int n = T * (H / 8);   // 16-byte pieces: 8 columns of one token
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const int t = i / (H / 8), k = (i % (H / 8)) * 8;
        const float4 a = __ldg(reinterpret_cast<const float4*>(x + (size_t)t * H + k));
        const float4 b = __ldg(reinterpret_cast<const float4*>(x + (size_t)t * H + k + 4));
        reinterpret_cast<uint4*>(img)[img_index(rows, t, k) / 8] =
            make_uint4(f32x2_to_bf16x2(a.x, a.y), f32x2_to_bf16x2(a.z, a.w), f32x2_to_bf16x2(b.x, b.y),
                       f32x2_to_bf16x2(b.z, b.w));
    }
}

int g_tc_sms = 0;

template <int RW, int SW, int G>
cudaError_t launch_tc_typed(const TcParams& p, cudaStream_t st) {
    using SL = TcSmem<RW, SW, G>;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(expert_tc_kernel<RW, SW, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)SL::total);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(g_tc_sms);
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = SL::total;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, expert_tc_kernel<RW, SW, G>, p);
}

}  // namespace

cudaError_t launch_expert_tc(const float* x, int T, const TcView& V, const RouteView& R, const TcWork& W, float* out,
                             bool resid, bool shared_only, cudaStream_t st) {
    if (T <= SMALL_T) return cudaErrorInvalidValue;
    if (g_tc_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_tc_sms, cudaDevAttrMultiProcessorCount, dev);
    }
    if (shared_only) {
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(g_tc_sms);
        cfg.blockDim = dim3(256);
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const cudaError_t e = cudaLaunchKernelEx(&cfg, x_image_kernel, x, T, W.tpad, W.x_img);
        if (e != cudaSuccess) return e;
    }
    const TcParams p{x, T, out, resid ? 1 : 0, shared_only ? 1 : 0, V, R, W};
    const int rw = V.r.g.wtype, sw = V.s.g.wtype;
    const int g = is_quant(rw) ? V.r.g.group : (is_quant(sw) ? V.s.g.group : 128);
#define FOCR_CASE(A, B, GG) \
    if (rw == A && sw == B && g == GG) return launch_tc_typed<A, B, GG>(p, st);
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
