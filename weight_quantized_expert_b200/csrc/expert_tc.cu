// Tensor-core grouped expert kernel for batches of more than MID_T tokens (prefill; the dense
// layer for more than 8): the shared expert and every selected routed expert as tcgen05 GEMMs with the
// dequantised weights and the accumulators in tensor memory, SwiGLU fused into the gate/up
// epilogue, and a combine that sums each token's parts in a fixed order (no atomics on the
// output, so repeated calls are bit-identical).
//
// Sources: frankenocr.pages.dev, "One forward pass", step 6 (64 routed experts + 2 fused
// shared experts, softmax top-6 without renormalisation, weighted sum of the experts); franken_ocr
// README, "Architecture" (each expert 1280 -> 896 SiLU-gated; the shared experts always on);
// "Four bits, one shared scale" (int4 nibble + f32 group scale; int8 and bf16 formats).
//
// The contraction is swapped so that the weights fill the MMA's M = 128 rows and a chunk of at
// most 128 of an expert's tokens fills N (a multiple of 16).  A work unit covers MT <= 4 weight
// tiles of one set that share the unit's token chunk (MT = 128 / N rounded down to 1, 2 or 4),
// so each K-block of token rows is loaded once for MT tiles:
//   gate/up unit  (set, MT tiles of 64 intermediates, token chunk): D_t[128 x N] = [G; U]_t X^T over
//                 K = 1280 (block rows interleave gate and up by 8, see the tensor-core layout in
//                 common.cuh); the epilogue pairs each gate lane with its up lane (shuffle by 8)
//                 and writes a = silu(g) * u * w_route as bf16 into the "a image"
//                 (x arrives as an f16 image: the router writes it in token order, the prologue
//                 copies each expert's rows into dispatch order)
//   down unit     (set, MT m-tiles of 128 output rows, [K part,] token chunk): D_t = Down_t a^T over
//                 the set's intermediates (the shared set's in up to 8 K parts); the epilogue
//                 writes fp32 rows y per (token, slot) or per (token, part)
//   dispatch      (prologue of every CTA, epilogue warps): a share of the token -> expert entries
//                 placed in their experts' segments (perm) and their x rows copied into an operand image
//   combine       out[t] = resid + sum_parts y_shared + sum_{j<6} y_slot[t*6+j]
// Units are handed out by a global atomic counter (shared gate/up, routed gate/up, shared down,
// routed down), so a unit only ever waits on units with smaller numbers, which running CTAs hold,
// or on the prologue, which every CTA runs first: a unit's token-row loads wait (bounded) until
// the units (or dispatch entries) that write those rows are done.
//
// Operand types: gate/up MMAs take f16 (x rounded to f16, weights q * s formed in f16), down MMAs
// bf16 (the SwiGLU output a and q * s rounded to bf16, for a's range); accumulation is fp32.
//
// Warp roles (one CTA per SM, 640 threads):
//   warp 0       scheduler: takes units, publishes their descriptors
//   warp 1       MMA: one thread issues tcgen05.mma (kind::f16, A from TMEM, B from shared
//                memory, fp32 accumulate in TMEM; 4 k-steps of 16 per 64-wide K-block), waiting
//                once per A stage of two blocks: a single issuing thread is bound by the
//                latency of each wait, not by the tensor pipe, at these small N
//   warp 2       weight copier: bulk copies (cp.async.bulk + mbarrier) of super-slots of about
//                16-18 KB (a few K-blocks of the unit's tiles) into a ~110 KB ring, so enough
//                HBM reads are in flight to stream at full bandwidth
//   warp 3       token-row loader: one bulk copy per K-block of N rows of an operand image
//   warps 4-15   dequantisers, three groups of four (one warp per TMEM lane quarter): thread = one
//                of the block's 128 rows; int4 (exponent-bias method) or int8 codes times the group
//                scale (q * s in f16 for gate/up, bf16 for down), written to a TMEM A stage with
//                tcgen05.st; 16-bit blocks are stored in their units' type and moved as they are
//   warps 16-19  epilogue: tcgen05.ld of the accumulators, SwiGLU or output rows, completion
//                counts; first the prologue share of the dispatch
// Every wait is bounded in time (%globaltimer); on expiry the kernel records an error word,
// stops taking work, waits (bounded) for its own copies in flight, frees TMEM and returns.
#include <cuda_bf16.h>

#include "common.cuh"
#include "fragments.cuh"
#include "umma.cuh"
#include "launch_state.h"

namespace focr {
namespace {

constexpr int NDQG = 3;                          // dequantiser groups
constexpr int NEPI = 4;                          // epilogue warps
constexpr int WARP_SCHED = 0, WARP_MMA = 1, WARP_COPY = 2, WARP_BLD = 3, WARP_DQ = 4;
constexpr int WARP_EPI = WARP_DQ + 4 * NDQG;
constexpr int NWARPS = WARP_EPI + NEPI;
constexpr int NTHREADS = NWARPS * 32;
constexpr int NCH = 128;                         // tokens of one unit at most (the MMA's N)
constexpr int NA = 4;                            // TMEM A stages (64 columns: two blocks of 128 rows x 64 bf16)
constexpr int NACC = 2;                          // TMEM accumulators (128 columns)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_A0 = NACC * 128;           // first column of the A stages
constexpr int NB = 6;                            // token-row stages in shared memory
constexpr uint32_t B_SLOT = NCH * TC_KB * 2;     // 16 KB
constexpr uint32_t RAW_BUDGET = 110 * 1024;      // weight super-slots in flight
constexpr int UR = 4;                            // unit descriptors in flight
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // 2 s
constexpr int DEVERR_TC_WAIT = 3;

static_assert(WARP_DQ % 4 == 0 && WARP_EPI % 4 == 0, "a group of four warps covers the four TMEM lane quarters");
static_assert(TM_A0 + NA * 64 <= TMEM_COLS, "TMEM budget");

enum UnitKind { UK_GU_S = 0, UK_GU_R = 1, UK_DN_S = 2, UK_DN_R = 3, UK_END = 5 };

// A stages: a unit's weight blocks (K-block kb, tile t) pass through TMEM two at a time, tiles
// (2 i, 2 i + 1) of one K-block per stage (a single tile where mt is odd), so that the MMA issuer
// waits once per pair of blocks.
__device__ __forceinline__ int stages_per_kb(int mt) { return (mt + 1) >> 1; }

// tiles a unit may cover for a chunk of N token rows: the MT accumulators fit 128 TMEM columns
__device__ __forceinline__ int mt_for(int N, int cap) {
    const int m = N <= 32 ? 4 : (N <= 64 ? 2 : 1);
    return m < cap ? m : cap;
}

struct Unit {
    int kind, expert;
    int tile, mt;        // first weight tile and tiles covered (gate/up: 64 intermediates; down: 128 rows)
    int part;            // shared down: K part
    int kb0, nkb;        // K-blocks [kb0, kb0 + nkb) of the set's matrix
    int ntok, N;         // tokens of the chunk, N = ntok rounded up to 16
    int c0;              // first token of the chunk: shared, a token id; routed, an index in the expert's segment
    int arow;            // first row of the chunk in the operand images
    int seg;             // routed: first dispatch entry of the chunk (index into the permutation)
    int wdep, wtarget;   // counter (index into the tensor-core control words) to wait for before the B loads, -1: none
    int ddep;            // counter this unit's completion adds to
    int ent[NCH];        // routed: dispatch entries t * 6 + j of the chunk's tokens
    float w[NCH];        // routed gate/up: their routing weights
};

struct Sched {
    int T, U, nchs, cs_s, P, KPP;
    unsigned m0, m1;     // experts 0-31 / 32-63 with tokens
    int n_gu_s, n_gu_r, n_dn_s, n_dn_r, total;
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
    static constexpr uint32_t raw_r = (uint32_t)tc_tile_group(RW) * tc_block_bytes(RW, G);
    static constexpr uint32_t raw_s = (uint32_t)tc_tile_group(SW) * tc_block_bytes(SW, G);
    static constexpr uint32_t raw_slot = (cmax(raw_r, raw_s) + 127u) & ~127u;
    static constexpr int cap_r = (int)(raw_slot / tc_block_bytes(RW, G));   // blocks one super-slot holds
    static constexpr int cap_s = (int)(raw_slot / tc_block_bytes(SW, G));
    static constexpr int cap = cap_r > cap_s ? cap_r : cap_s;
    static constexpr int NR = (int)(RAW_BUDGET / raw_slot);
    static constexpr uint32_t braw = 0;                                           // [NR][raw_slot]
    static constexpr uint32_t bstage = (braw + NR * raw_slot + 1023u) & ~1023u;   // [NB][B_SLOT]
    static constexpr uint32_t units = bstage + NB * B_SLOT;                       // [UR] Unit
    static constexpr uint32_t sched = (units + UR * (uint32_t)sizeof(Unit) + 15u) & ~15u;
    static constexpr uint32_t bars = (sched + (uint32_t)sizeof(Sched) + 7u) & ~7u;
    static constexpr int NBARS = 2 * NR + 2 * NB + 2 * NA + 2 * UR + 2 * NACC + 2;
    static constexpr uint32_t misc = bars + 8u * NBARS;                           // tmem base, abort flag
    static constexpr uint32_t total = misc + 16u;
    static_assert(NR >= 4, "weight ring depth");
    static_assert(total <= 232448, "shared memory budget");
};

// ------------------------------------------------------------------ small PTX helpers

__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void fence_proxy_async_all() { asm volatile("fence.proxy.async;" ::: "memory"); }

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

__device__ __forceinline__ uint32_t h2_sub(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t h2_mul(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
constexpr uint32_t H2_MAGIC = 0x64006400u;    // f16 (1024, 1024): a nibble n under it reads as 1024 + n
constexpr uint32_t H2_1032 = 0x64086408u;     // f16 (1032, 1032)
constexpr uint32_t BF2_MAGIC = 0x43004300u;   // (128, 128): a nibble n under it reads as 128 + n
constexpr uint32_t BF2_136 = 0x43084308u;     // (136, 136)

// One k-core of int4 codes (element 2m in nibble m, 2m+1 in nibble m+4, q + 8) -> 8 bf16 q * s.
// q = (128 + n) - 136 is exact in bf16; the product is rounded once (s2 = bf16 pair of the scale).
template <bool F16>
__device__ __forceinline__ void dq_int4_bf16(uint32_t w, uint32_t s2, uint32_t* r) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t nib = (w >> (4 * i)) & 0x000F000Fu;
        r[i] = F16 ? h2_mul(h2_sub(nib | H2_MAGIC, H2_1032), s2) : bf2_mul(bf2_sub(nib | BF2_MAGIC, BF2_136), s2);
    }
}

// One k-core of int8 codes (q + 128 in bytes 0..7) -> 8 bf16 q * s (fp32 product, one rounding).
template <bool F16>
__device__ __forceinline__ void dq_int8_bf16(uint32_t w0, uint32_t w1, float s, uint32_t* r) {
    float f[8];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        f[b] = (byte_to_float(w0, b) - 8388736.0f) * s;
        f[4 + b] = (byte_to_float(w1, b) - 8388736.0f) * s;
    }
#pragma unroll
    for (int m = 0; m < 4; ++m)
        r[m] = F16 ? f32x2_to_f16x2(f[2 * m], f[2 * m + 1]) : f32x2_to_bf16x2(f[2 * m], f[2 * m + 1]);
}

// One row of a 16-bit weight block (stored as the operand image: k-core c of row r at
// [(r / 8) * 8 + c][r % 8] in 16-byte pieces) into 32 registers: 32-bit column c of the TMEM A
// stage holds elements 2c, 2c + 1 of the 64-wide K-block.  Thread = block row `row`.
__device__ __forceinline__ void block_row_copy(const uint8_t* blk, int row, uint32_t (&r)[32]) {
    const uint8_t* base = blk + (row >> 3) * 1024 + (row & 7) * 16;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 v = lds128(base + c * 128);
        r[4 * c] = v.x;
        r[4 * c + 1] = v.y;
        r[4 * c + 2] = v.z;
        r[4 * c + 3] = v.w;
    }
}

// One row of a quantised weight block held in registers between its shared-memory load and its
// conversion, so that both blocks of an A stage are loaded before either is converted.
template <int W, int G>
struct RowRaw {
    static constexpr int NC = W == FOCR_W_INT8 ? 4 : 2;
    uint4 c[NC];
    float s0, s1;
    __device__ __forceinline__ void load(const uint8_t* blk, int row) {
        constexpr int SPK = tc_spk(G);
        constexpr uint32_t RB = tc_row_bytes(W);
        const float* sc = reinterpret_cast<const float*>(blk + TC_M * RB) + row * SPK;
#pragma unroll
        for (int i = 0; i < NC; ++i) c[i] = lds128(blk + row * RB + 16 * i);
        s0 = sc[0];
        s1 = sc[SPK - 1];
    }
    // q * s in f16 (gate/up operands) or bf16 (down operands)
    template <bool F16>
    __device__ __forceinline__ void cvt(uint32_t (&r)[32]) const {
        if constexpr (W == FOCR_W_INT4) {
            // pairs (c, c + 4), 8 bytes each: words k-core c, k-core c + 4
            const uint32_t b0 = F16 ? f32x2_to_f16x2(s0, s0) : f32x2_to_bf16x2(s0, s0);
            const uint32_t b1 = tc_spk(G) == 1 ? b0 : (F16 ? f32x2_to_f16x2(s1, s1) : f32x2_to_bf16x2(s1, s1));
            dq_int4_bf16<F16>(c[0].x, b0, r + 0);
            dq_int4_bf16<F16>(c[0].y, b1, r + 16);
            dq_int4_bf16<F16>(c[0].z, b0, r + 4);
            dq_int4_bf16<F16>(c[0].w, b1, r + 20);
            dq_int4_bf16<F16>(c[1].x, b0, r + 8);
            dq_int4_bf16<F16>(c[1].y, b1, r + 24);
            dq_int4_bf16<F16>(c[1].z, b0, r + 12);
            dq_int4_bf16<F16>(c[1].w, b1, r + 28);
        } else {
            // pairs (c, c + 4), 16 bytes each
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                dq_int8_bf16<F16>(c[i].x, c[i].y, s0, r + 4 * i);
                dq_int8_bf16<F16>(c[i].z, c[i].w, s1, r + 4 * (i + 4));
            }
        }
    }
};

// This thread's row of the `nb` (1 or 2) adjacent weight blocks at `bp` (`blk` bytes apart) into
// the two 32-column halves of a TMEM A stage at `ta` (this warp's lane quarter), as f16 for gate/up
// units (`f16`) and bf16 for down units; 16-bit blocks are stored in the format their units use.
// Completes with tcgen05.wait::st by the caller.
template <int W, int G>
__device__ __forceinline__ void dq_stage(const uint8_t* bp, uint32_t blk, int nb, int row, uint32_t ta, bool f16) {
    uint32_t r[32];
    if constexpr (W == FOCR_W_BF16) {
        block_row_copy(bp, row, r);
        umma::st32(ta, r);
        if (nb > 1) {
            block_row_copy(bp + blk, row, r);
            umma::st32(ta + 32u, r);
        }
    } else {
        RowRaw<W, G> x0, x1;
        x0.load(bp, row);
        if (nb > 1) x1.load(bp + blk, row);
        if (f16) x0.template cvt<true>(r);
        else x0.template cvt<false>(r);
        umma::st32(ta, r);
        if (nb > 1) {
            if (f16) x1.template cvt<true>(r);
            else x1.template cvt<false>(r);
            umma::st32(ta + 32u, r);
        }
    }
}

// weight block kb (absolute) of tile `tile` of a unit's set
__device__ __forceinline__ const uint8_t* w_block(const TcView& V, const Unit& U, int tile, int kb) {
    const bool routed = U.kind == UK_GU_R || U.kind == UK_DN_R;
    const TcSetView& S = routed ? V.r : V.s;
    if (U.kind <= UK_GU_R)
        return S.gu + (routed ? (size_t)U.expert * S.g.gu_bytes : 0) +
               tc_block_index(S.g.tiles, TC_KBH, tile, kb, S.g.grp) * S.g.blk;
    return S.dn + (routed ? (size_t)U.expert * S.g.dn_bytes : 0) +
           tc_block_index(TC_MT, S.g.tiles, tile, kb, S.g.grp) * S.g.blk;
}

// Active index of expert e (its rank among the experts with tokens).
__device__ __forceinline__ int active_index(const Sched& S, int e) {
    return e < 32 ? __popc(S.m0 & ((1u << e) - 1u)) : __popc(S.m0) + __popc(S.m1 & ((1u << (e - 32)) - 1u));
}

// The epilogue warps' share of the dispatch (see the prologue in the kernel): warp ew of this CTA
// takes entries i = blockIdx + gridDim * (ew + NEPI * j), GE of them per pass, each pass one
// sweep over the entries before its last one.
__device__ __forceinline__ void epilogue_gather(const TcParams& p, const Sched& S, int* ctrl, int ew, int lane) {
    constexpr int GE = 4;    // entries per pass
    constexpr int LB = 8;    // 16-byte index loads per lane in flight
    const int ntot = p.T * K;
    const int4* idx4 = reinterpret_cast<const int4*>(p.R.topk_idx);
    const uint4* src = reinterpret_cast<const uint4*>(p.W.x_img);
    uint4* dst = reinterpret_cast<uint4*>(p.W.x_img_r);
    for (int j0 = ew;; j0 += NEPI * GE) {
        int ii[GE], ee[GE], rk[GE];
        int lim = 0;
#pragma unroll
        for (int g = 0; g < GE; ++g) {
            const long long i = (long long)blockIdx.x + (long long)gridDim.x * (j0 + NEPI * g);
            ii[g] = i < ntot ? (int)i : -1;
            ee[g] = ii[g] >= 0 ? __ldcg(&p.R.topk_idx[ii[g]]) : -1;
            rk[g] = 0;
            if (ii[g] >= 0) lim = ii[g];
        }
        if (ii[0] < 0) break;
        // rank of each entry among the earlier entries of its expert
        for (int c0 = 0; c0 * 4 < lim; c0 += 32 * LB) {
            int4 v[LB];
#pragma unroll
            for (int m = 0; m < LB; ++m) {
                const int c = c0 + m * 32 + lane;
                v[m] = c * 4 < lim ? __ldcg(idx4 + c) : make_int4(-1, -1, -1, -1);
            }
#pragma unroll
            for (int m = 0; m < LB; ++m) {
                const int i = (c0 + m * 32 + lane) * 4;
#pragma unroll
                for (int g = 0; g < GE; ++g) {
                    rk[g] += (int)(v[m].x == ee[g] && i < ii[g]) + (int)(v[m].y == ee[g] && i + 1 < ii[g]) +
                             (int)(v[m].z == ee[g] && i + 2 < ii[g]) + (int)(v[m].w == ee[g] && i + 3 < ii[g]);
                }
            }
        }
#pragma unroll
        for (int g = 0; g < GE; ++g)
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) rk[g] += __shfl_xor_sync(0xffffffffu, rk[g], o);
        // perm entries and the rows: 20 K-blocks x 8 pieces of 16 bytes per row, 5 per lane, two
        // rows in flight at a time
#pragma unroll
        for (int g0 = 0; g0 < GE; g0 += 2) {
            uint4 buf[2][5];
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                if (ii[g0 + g] < 0) continue;
                const int t = ii[g0 + g] / K;
#pragma unroll
                for (int m = 0; m < 5; ++m) {
                    const int pc = m * 32 + lane, kb = pc >> 3, kc = pc & 7;
                    buf[g][m] = __ldg(src + img_index(p.W.tpad, t, kb * TC_KB + kc * 8) / 8);
                }
            }
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                if (ii[g0 + g] < 0) continue;
                const int a = active_index(S, ee[g0 + g]);
                const int row = S.poff[a] + rk[g0 + g];
                if (lane == 0) p.R.perm[S.off[a] + rk[g0 + g]] = ii[g0 + g];
#pragma unroll
                for (int m = 0; m < 5; ++m) {
                    const int pc = m * 32 + lane, kb = pc >> 3, kc = pc & 7;
                    dst[img_index(p.W.arows, row, kb * TC_KB + kc * 8) / 8] = buf[g][m];
                }
            }
        }
        // publish: the rows (read by the tensor-memory copies) and perm, then the counters
        fence_proxy_async_all();
        __threadfence();
        __syncwarp();
        if (lane == 0) {
#pragma unroll
            for (int g = 0; g < GE; ++g)
                if (ii[g] >= 0) atomicAdd(&ctrl[TC_DEP_X + ee[g]], 1);
        }
    }
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
    uint64_t* raw_full = bars;
    uint64_t* raw_empty = raw_full + NR;
    uint64_t* b_full = raw_empty + NR;
    uint64_t* b_empty = b_full + NB;
    uint64_t* a_full = b_empty + NB;
    uint64_t* a_empty = a_full + NA;
    uint64_t* u_full = a_empty + NA;
    uint64_t* u_empty = u_full + UR;
    uint64_t* acc_full = u_empty + UR;
    uint64_t* acc_empty = acc_full + NACC;
    uint64_t* drain = acc_empty + NACC;   // the MMA thread's last commit before TMEM is freed
    uint64_t* s_ready = drain + 1;        // the schedule summary S is written
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SL::misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SL::misc + 4);
    int* ctrl = p.R.ctrl + CTRL_TC;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < NR; ++i) {
            mbar_init(&raw_full[i], 1);
            mbar_init(&raw_empty[i], 4 * SL::cap);   // 4 warps per block; the copier fills in for absent blocks
        }
        for (int i = 0; i < NB; ++i) {
            mbar_init(&b_full[i], 1);
            mbar_init(&b_empty[i], 1);
        }
        for (int i = 0; i < NA; ++i) {
            mbar_init(&a_full[i], 4);
            mbar_init(&a_empty[i], 1);
        }
        for (int i = 0; i < UR; ++i) {
            mbar_init(&u_full[i], 1);
            mbar_init(&u_empty[i], 4 * NDQG + NEPI + 3);   // dequantisers, epilogue, MMA, copier, loader
        }
        for (int i = 0; i < NACC; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], NEPI);
        }
        mbar_init(drain, 1);
        mbar_init(s_ready, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == WARP_MMA) umma::tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();   // routing, x image and the output of the previous kernel are complete

    auto fail = [&](int code) {
        atomicExch(&p.R.ctrl[CTRL_ERROR], code);
        *abort_flag = 1;
    };

    if (warp == WARP_SCHED) {
        // ------------------------------------------------------------ schedule (whole warp)
        const TcGeom& rg = p.V.r.g;
        const TcGeom& sg = p.V.s.g;
        const int T = p.T;
        // lane l owns experts l and l + 32; the active experts (with tokens) are numbered in
        // ascending expert order.  The router left per-expert assignment counts; each expert's
        // segment of the dispatch order starts at the exclusive prefix sum of the counts.
        int cnt[2], offs[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) cnt[h] = p.shared_only ? 0 : __ldcg(&ctrl[TC_CNT + lane + 32 * h]);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            int incl = cnt[h];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            offs[h] = incl - cnt[h];
        }
        offs[1] += __shfl_sync(0xffffffffu, offs[0] + cnt[0], 31);
        const unsigned m0 = __ballot_sync(0xffffffffu, cnt[0] > 0), m1 = __ballot_sync(0xffffffffu, cnt[1] > 0);
        const int U = __popc(m0) + __popc(m1);
        if (blockIdx.x == 0 && !p.shared_only) {
            // the routing summary for callers: counts, segment offsets, experts with tokens
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int e = lane + 32 * h;
                p.R.counts[e] = cnt[h];
                p.R.offsets[e] = offs[h];
                if (cnt[h] > 0)
                    p.R.active[h == 0 ? __popc(m0 & ((1u << lane) - 1u))
                                      : __popc(m0) + __popc(m1 & ((1u << lane) - 1u))] = e;
            }
            if (lane == 31) {
                p.R.offsets[E] = offs[1] + cnt[1];
                p.R.active[E] = U;
            }
        }
        int pad[2], gu[2], dn[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int e = lane + 32 * h;
            const int a = h == 0 ? __popc(m0 & ((1u << lane) - 1u)) : __popc(m0) + __popc(m1 & ((1u << lane) - 1u));
            pad[h] = gu[h] = dn[h] = 0;
            if (cnt[h] > 0) {
                const int n = cnt[h];
                const int nch0 = (n + NCH - 1) / NCH;
                const int cs = ((n + nch0 - 1) / nch0 + 15) & ~15;   // chunk size, a multiple of 16
                const int nch = (n + cs - 1) / cs;
                S.e[a] = e;
                S.n[a] = n;
                S.off[a] = offs[h];
                S.nch[a] = nch;
                S.cs[a] = cs;
                pad[h] = (n + 15) & ~15;
                for (int c = 0; c < nch; ++c) {
                    const int mt = mt_for((min(cs, n - c * cs) + 15) & ~15, tc_tile_group(RW));
                    gu[h] += (rg.tiles + mt - 1) / mt;
                    dn[h] += (TC_MT + mt - 1) / mt;
                }
            }
        }
        // exclusive prefix sums in expert order (inactive experts add nothing), stored at the active
        // index: padded image rows, gate/up units, down units
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
            const int a = h == 0 ? __popc(m0 & ((1u << lane) - 1u)) : __popc(m0) + __popc(m1 & ((1u << lane) - 1u));
            if (cnt[h] > 0) {
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
            S.m0 = m0;
            S.m1 = m1;
            S.n_gu_s = sg.tiles * S.nchs;
            S.n_gu_r = sgu[1];
            S.n_dn_s = TC_MT * S.P * S.nchs;
            S.n_dn_r = sdn[1];
            S.total = S.n_gu_s + S.n_gu_r + S.n_dn_s + S.n_dn_r;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(s_ready);

        // ------------------------------------------------------------ scheduler loop
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
                if (v < S.n_gu_s) {
                    kind = UK_GU_S;
                    const int tile = v / S.nchs, ch = v % S.nchs;
                    if (lane == 0) {
                        Un.expert = -1;
                        Un.tile = tile;
                        Un.mt = 1;
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
                    const int mtile = v / (S.P * S.nchs), rem = v % (S.P * S.nchs);
                    const int part = rem / S.nchs, ch = rem % S.nchs;
                    if (lane == 0) {
                        Un.expert = -1;
                        Un.tile = mtile;
                        Un.mt = 1;
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
                    const bool g_u = kind == UK_GU_R;
                    const int* pre = g_u ? S.gu_pre : S.dn_pre;
                    int lo = 0, hi = S.U - 1;   // last a with pre[a] <= v
                    while (lo < hi) {
                        const int mid = (lo + hi + 1) >> 1;
                        if (pre[mid] <= v) lo = mid;
                        else hi = mid - 1;
                    }
                    const int a = lo;
                    int w = v - pre[a];
                    const int ntiles = g_u ? rg.tiles : TC_MT;
                    int ch = 0, mt = 1;
                    for (;; ++ch) {   // the chunk of the expert this unit falls in
                        mt = mt_for((min(S.cs[a], S.n[a] - ch * S.cs[a]) + 15) & ~15, tc_tile_group(RW));
                        const int per = (ntiles + mt - 1) / mt;
                        if (w < per || ch + 1 >= S.nch[a]) break;
                        w -= per;
                    }
                    const int c0 = ch * S.cs[a];
                    const int ntok = min(S.cs[a], S.n[a] - c0);
                    const int seg = S.off[a] + c0;
                    if (lane == 0) {
                        Un.expert = S.e[a];
                        Un.tile = w * mt;
                        Un.mt = min(mt, ntiles - w * mt);
                        Un.part = 0;
                        Un.kb0 = 0;
                        Un.nkb = g_u ? TC_KBH : rg.tiles;
                        Un.c0 = c0;
                        Un.ntok = ntok;
                        Un.arow = S.poff[a] + c0;
                        Un.seg = seg;
                        // gate/up waits for the expert's gathered rows, down for all its gate/up units
                        Un.wdep = g_u ? TC_DEP_X + S.e[a] : TC_DEP_R + S.e[a];
                        Un.wtarget = g_u ? S.n[a] : (S.gu_pre[a + 1] - S.gu_pre[a]) * NEPI;
                        Un.ddep = g_u ? TC_DEP_R + S.e[a] : TC_DN_DONE;
                    }
                    // the expert's permutation segment is written as its rows are gathered
                    bool dep = true;
                    if (lane == 0) dep = wait_counter(&ctrl[TC_DEP_X + S.e[a]], S.n[a]);
                    if (!__shfl_sync(0xffffffffu, dep ? 1 : 0, 0)) {
                        if (lane == 0) fail(DEVERR_TC_WAIT);
                        kind = UK_END;
                    } else {
                        for (int n = lane; n < ntok; n += 32) {
                            const int ent = __ldcg(&p.R.perm[seg + n]);
                            Un.ent[n] = ent;
                            Un.w[n] = __ldcg(&p.R.topk_w[ent]);
                        }
                    }
                }
                if (lane == 0) Un.N = (Un.ntok + 15) & ~15;
            }
            if (lane == 0) Un.kind = kind;
            __syncwarp();
            if (lane == 0) mbar_arrive(&u_full[slot]);
            if (kind == UK_END) break;
            if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;
        }
    } else if (warp == WARP_COPY) {
        // ------------------------------------------------------------ weight copier (one thread)
        // Per unit: super-slots of a few K-blocks x the unit's tiles, one bulk copy per K-block
        // (or one per super-slot where the K-blocks of a single tile are adjacent).
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
                const TcGeom& gg = routed ? p.V.r.g : p.V.s.g;
                const int mt = Un.mt, kq = max(1, (routed ? SL::cap_r : SL::cap_s) / mt);
                const bool whole = gg.grp == 1 && mt == 1;   // K-blocks of one tile are adjacent
                bool ok = true;
                for (int kb = 0; kb < Un.nkb; kb += kq, ++raw_i) {
                    // super-slot: K-blocks [kb, kb + nk) x the unit's mt tiles, block (j, t) at j mt + t
                    const int nk = min(kq, Un.nkb - kb);
                    const int r = raw_i % NR;
                    if (!mbar_wait_bounded(&raw_empty[r], ((raw_i / NR) & 1) ^ 1, WAIT_LIMIT_NS)) {
                        ok = false;
                        break;
                    }
                    for (int i = nk * mt; i < SL::cap; ++i)   // blocks this super-slot does not hold
                        for (int j = 0; j < 4; ++j) mbar_arrive(&raw_empty[r]);
                    mbar_arrive_expect_tx(&raw_full[r], (uint32_t)(nk * mt) * gg.blk);
                    char* dst = smem + SL::braw + r * SL::raw_slot;
                    if (whole) {
                        bulk_g2s(dst, w_block(p.V, Un, Un.tile, Un.kb0 + kb), (uint32_t)nk * gg.blk, &raw_full[r], pol);
                    } else {
                        for (int j = 0; j < nk; ++j)   // the unit's tiles of one K-block are adjacent
                            bulk_g2s(dst + (size_t)j * mt * gg.blk, w_block(p.V, Un, Un.tile, Un.kb0 + kb + j),
                                     (uint32_t)mt * gg.blk, &raw_full[r], pol);
                    }
                }
                mbar_arrive(&u_empty[slot]);
                if (!ok) {
                    fail(DEVERR_TC_WAIT);
                    break;
                }
                if (*abort_flag) break;
            }
            // never leave copies in flight: the last NR issued super-slots must have landed
            for (int i = max(0, raw_i - NR); i < raw_i; ++i)
                (void)mbar_wait_bounded(&raw_full[i % NR], (i / NR) & 1, WAIT_LIMIT_NS);
        }
        __syncwarp();
    } else if (warp == WARP_BLD) {
        // ------------------------------------------------------------ token-row loader (one thread)
        // Per K-block: N rows of an operand image (x in token order for the shared set, x in
        // dispatch order for routed experts, a for down projections).
        if (lane == 0) {
            int b_i = 0;
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
                const uint16_t* img = is_gu ? (routed ? p.W.x_img_r : p.W.x_img) : (routed ? p.W.a_img : p.W.a_sh);
                const int rows = routed ? p.W.arows : p.W.tpad;
                const uint32_t bytes = (uint32_t)Un.N * 128u;
                bool ok = true;
                if (Un.nkb > 0 && Un.wdep >= 0) {
                    // the rows come from other units' epilogues: wait until they are all written
                    ok = wait_counter(&ctrl[Un.wdep], Un.wtarget);
                    fence_proxy_async_all();
                }
                for (int kb = 0; kb < Un.nkb && ok; ++kb, ++b_i) {
                    const int s = b_i % NB;
                    if (!mbar_wait_bounded(&b_empty[s], ((b_i / NB) & 1) ^ 1, WAIT_LIMIT_NS)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&b_full[s], bytes);
                    bulk_g2s(smem + SL::bstage + s * B_SLOT, img + ((size_t)(Un.kb0 + kb) * rows + Un.arow) * TC_KB,
                             bytes, &b_full[s], policy_evict_last());
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
            int a_i = 0, b_i = 0, acc_i = 0;
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
                const int b = acc_i % NACC;
                if (!mbar_wait_bounded(&acc_empty[b], ((acc_i / NACC) & 1) ^ 1, WAIT_LIMIT_NS)) {
                    fail(DEVERR_TC_WAIT);
                    break;
                }
                umma::fence_after_sync();
                const int N = Un.N, mt = Un.mt;
                // gate/up: f16 weights and x; down: bf16 weights and a (range of the SwiGLU output)
                const uint32_t idesc =
                    Un.kind <= UK_GU_R ? umma::idesc_f16_f32(TC_M, N) : umma::idesc_bf16_f32(TC_M, N);
                const uint32_t d0 = tmem_base + (uint32_t)(b * 128);
                const int pp = stages_per_kb(mt), nst = Un.nkb * pp;
                bool ok = true;
                uint32_t b0 = 0;
                for (int st = 0; st < nst; ++st, ++a_i) {
                    const int kb = st / pp, t0 = 2 * (st % pp);
                    const int bs = b_i % NB;
                    if (t0 == 0) {   // first stage of a K-block: its token rows
                        if (!mbar_wait_bounded(&b_full[bs], (b_i / NB) & 1, WAIT_LIMIT_NS)) {
                            ok = false;
                            break;
                        }
                        b0 = smem_u32(smem + SL::bstage + bs * B_SLOT);
                    }
                    const int as = a_i % NA;
                    if (!mbar_wait_bounded(&a_full[as], (a_i / NA) & 1, WAIT_LIMIT_NS)) {
                        ok = false;
                        break;
                    }
                    umma::fence_after_sync();
                    const uint32_t a0 = tmem_base + TM_A0 + (uint32_t)(as * 64);
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        if (t0 + i >= mt) break;
#pragma unroll
                        for (int j = 0; j < TC_KB / 16; ++j)
                            umma::mma_bf16_ts(d0 + (uint32_t)((t0 + i) * N), a0 + 32u * i + 8u * j,
                                              umma::sdesc_kmajor(b0 + 256u * j, 128u, 1024u), idesc, kb > 0 || j > 0);
                    }
                    umma::commit(smem_u32(&a_empty[as]));
                    if (t0 + 2 >= mt) {   // last stage of the K-block: release its token rows
                        umma::commit(smem_u32(&b_empty[bs]));
                        ++b_i;
                    }
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
        // ------------------------------------------------------------ dequantisers
        // Group dg takes every NDQG-th A stage (the unit's stages in K-block-major order, two
        // tiles of one K-block each); warp q of the group converts block rows 32 q .. 32 q + 31
        // (thread = row) of the stage's blocks and writes them to its TMEM columns.
        const int dg = (warp - WARP_DQ) >> 2, q = warp & 3;
        const int row = 32 * q + lane;
        int a_i = 0, raw_i = 0;   // blocks and super-slots of all units so far
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
            const int nkb = Un.nkb, mt = Un.mt;
            const uint32_t blk = routed ? p.V.r.g.blk : p.V.s.g.blk;
            const int kq = max(1, (routed ? SL::cap_r : SL::cap_s) / mt);   // K-blocks per super-slot
            const int pp = stages_per_kb(mt), nst = nkb * pp;
            for (int st = 0; st < nst && ok; ++st, ++a_i) {
                if (a_i % NDQG != dg) continue;
                const int kb = st / pp, t0 = 2 * (st % pp), nb = min(2, mt - t0);
                const int as = a_i % NA;
                const int ri = raw_i + kb / kq;   // the super-slot holding K-block kb of every tile
                const int rs = ri % NR;
                if (lane == 0) {
                    ok = mbar_wait_bounded(&a_empty[as], ((a_i / NA) & 1) ^ 1, WAIT_LIMIT_NS) &&
                         mbar_wait_bounded(&raw_full[rs], (ri / NR) & 1, WAIT_LIMIT_NS);
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) break;
                const uint8_t* bp = reinterpret_cast<const uint8_t*>(smem + SL::braw + rs * SL::raw_slot) +
                                    (size_t)((kb % kq) * mt + t0) * blk;
                const uint32_t ta = tmem_base + ((uint32_t)(32 * q) << 16) + TM_A0 + (uint32_t)(as * 64);
                if (routed) dq_stage<RW, G>(bp, blk, nb, row, ta, kind <= UK_GU_R);
                else dq_stage<SW, G>(bp, blk, nb, row, ta, kind <= UK_GU_R);
                umma::wait_st();
                umma::fence_before_sync();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&a_full[as]);
                    for (int i = 0; i < nb; ++i) mbar_arrive(&raw_empty[rs]);
                }
            }
            raw_i += (nkb + kq - 1) / kq;
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
        bool go_on = true;
        if (!p.shared_only) {
            // Prologue: every CTA places a share of the dispatch entries.  Entry i = t * 6 + j of
            // expert e goes to rank r = #{entries i' < i of expert e} of e's segment: perm[off_e + r]
            // = i, and token t's row of the x image is copied to row poff_e + r of the dispatch-
            // order image.  Each placed entry adds one to e's gathered-rows counter.
            bool ok = true;
            if (lane == 0) ok = mbar_wait_bounded(s_ready, 0, WAIT_LIMIT_NS);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) {
                if (lane == 0) fail(DEVERR_TC_WAIT);
                go_on = false;
            } else {
                epilogue_gather(p, S, ctrl, warp - WARP_EPI, lane);
            }
        }
        for (int k = 0; go_on; ++k) {
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
            const int b = acc_i % NACC;
            if (lane == 0) ok = mbar_wait_bounded(&acc_full[b], (acc_i / NACC) & 1, WAIT_LIMIT_NS);
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
                if (lane == 0) fail(DEVERR_TC_WAIT);
                break;
            }
            umma::fence_after_sync();
            const bool routed = kind == UK_GU_R || kind == UK_DN_R;
            const int ntok = Un.ntok, N = Un.N;
            for (int t = 0; t < Un.mt; ++t) {
                const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * 128 + t * N);
                if (kind <= UK_GU_R) {
                    const bool gate = (lane & 8) == 0;
                    const int i = TC_KB * (Un.tile + t) + 16 * q + 8 * (lane >> 4) + (lane & 7);   // intermediate
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
                                const int rr = Un.arow + n;
                                col[(size_t)(rr >> 3) * 512 + (rr & 7) * 8] = __bfloat16_as_ushort(__float2bfloat16_rn(a));
                            }
                        }
                    }
                } else {
                    const int m = TC_M * (Un.tile + t) + 32 * q + lane;   // output row
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
            if (lane == 0) {
                atomicAdd(&ctrl[Un.ddep], 1);
                mbar_arrive(&u_empty[slot]);
            }
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

// x (fp32) -> the f16 operand image in token order (the dense layer has no router to write it);
// a finite |x| beyond the f16 range sets the error word (DEVERR_RANGE)
__global__ void x_image_kernel(const float* x, int T, int rows, uint16_t* img, int* err) {
    pdl_wait();
    pdl_launch_dependents();
    const int n = T * (H / 8);   // 16-byte pieces: 8 columns of one token
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const int t = i / (H / 8), k = (i % (H / 8)) * 8;
        const float4 a = __ldg(reinterpret_cast<const float4*>(x + (size_t)t * H + k));
        const float4 b = __ldg(reinterpret_cast<const float4*>(x + (size_t)t * H + k + 4));
        if (f16_out_of_range(a.x) || f16_out_of_range(a.y) || f16_out_of_range(a.z) || f16_out_of_range(a.w) ||
            f16_out_of_range(b.x) || f16_out_of_range(b.y) || f16_out_of_range(b.z) || f16_out_of_range(b.w))
            atomicExch(err, DEVERR_RANGE);
        reinterpret_cast<uint4*>(img)[img_index(rows, t, k) / 8] =
            make_uint4(f32x2_to_f16x2(a.x, a.y), f32x2_to_f16x2(a.z, a.w), f32x2_to_f16x2(b.x, b.y),
                       f32x2_to_f16x2(b.z, b.w));
    }
}

template <int RW, int SW, int G>
cudaError_t launch_tc_typed(const TcParams& p, int sms, cudaStream_t st) {
    using SL = TcSmem<RW, SW, G>;
    const cudaError_t e = once_per_device((const void*)expert_tc_kernel<RW, SW, G>, [] {
        return cudaFuncSetAttribute(expert_tc_kernel<RW, SW, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)SL::total);
    });
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(sms);
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
    const int sms = device_sms();
    if (sms <= 0) return cudaErrorInvalidDevice;
    if (shared_only) {
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(sms);
        cfg.blockDim = dim3(256);
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const cudaError_t e = cudaLaunchKernelEx(&cfg, x_image_kernel, x, T, W.tpad, W.x_img, R.ctrl + CTRL_ERROR);
        if (e != cudaSuccess) return e;
    }
    const TcParams p{x, T, out, resid ? 1 : 0, shared_only ? 1 : 0, V, R, W};
    const int rw = V.r.g.wtype, sw = V.s.g.wtype;
    const int g = is_quant(rw) ? V.r.g.group : (is_quant(sw) ? V.s.g.group : 128);
#define FOCR_CASE(A, B, GG) \
    if (rw == A && sw == B && g == GG) return launch_tc_typed<A, B, GG>(p, sms, st);
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
