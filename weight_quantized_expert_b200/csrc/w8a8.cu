// W8A8 GEMV: per-token int8 activations against per-row int8 weights, with an exact integer dot.
//
// Source: franken_ocr README, "CPU Backend and Optimizations" (the int8 decode linears run a
// quantise-plus-GEMV pass per token on integer dot products with exact, non-saturating i32
// accumulation) and "Command Reference", `focr robot` (K = 6848 is the accumulation's worst case).
// Readings where the pages are silent: the activation scale mirrors the weights' one.
//
//   s_x[t] = fp32(max_k |x[t, k]|) / 127 (one fp32 division);
//   q_x[t, k] = round-half-even(x[t, k] / s_x[t]) clamped to [-127, 127] (s_x = 0 gives q_x = 0);
//   acc[t, n] = sum_k q_w[n, k] q_x[t, k], exact: |acc| <= K * 127^2 < 2^31 for K <= 133,143;
//   y[t, n]   = fp32((fp64(s_w[n]) * fp64(s_x[t])) * fp64(acc)).
//
// Kernels:
//   w8a8_quantize_kernel  one CTA per token: an order-free block max, then the codes, written
//                         row-major (the public quantiser) and/or in the m16n8k32 B-fragment order
//                         the GEMV reads: for k-step q and token group nb, 32 lanes x 8 bytes, lane
//                         4 gr + c holding token 8 nb + gr at columns 32q + 4c .. +3 and
//                         32q + 16 + 4c .. +3.
//   w8a8_gemv_kernel      an HBM-bound stream of the codes.  A unit is one 16-row tile over a chunk
//                         of k-steps; its codes are contiguous (tile-major packing), so one lane of
//                         a producer warp moves each unit with a single bulk copy (cp.async.bulk,
//                         up to 20 KB) into a ring of shared-memory stages (up to 8, 160 KB in
//                         flight per SM).  Up to eight consumer warps take the units in turn, each
//                         owning the same stages throughout (no phase aliasing): a 16-byte
//                         A fragment per lane per k-step from shared memory, the B fragments (the
//                         activation codes) staged once per CTA in shared memory (read through L1
//                         when they do not fit beside 3 stages), integer tensor-core MMAs
//                         (mma.sync m16n8k32 s8 with s32 accumulate: exact integer arithmetic).  When a tile's K is split over several units,
//                         their partial sums meet by integer atomics (exact, so the order does not
//                         matter) and the tile's last unit (a per-tile counter) applies the scales
//                         and returns the sums and the counter to zero.  The producer starts before
//                         the quantiser has finished (programmatic dependent launch): the codes do
//                         not depend on it; the consumers wait for it.  Every mbarrier wait is
//                         bounded; one that runs out sets the workspace's error word.
#include <algorithm>

#include "common.cuh"
#include "launch_state.h"
#include "w8a8.h"

namespace focr {
namespace {

constexpr int QT = 256;                        // quantiser threads per token
constexpr int NC = 8;                          // GEMV consumer warps per CTA
constexpr int GT = (NC + 1) * 32;              // + one producer warp
constexpr int LMAX = 40;                       // most k-steps of one unit (20 KB of codes)
constexpr int NST_MAX = 10;                    // most ring stages
constexpr int NST_MIN = 3;                     // fewest ring stages with the qx fragments in shared memory
constexpr size_t STAGE_BYTES = (size_t)LMAX * 512;
constexpr size_t SMEM_MAX = 232448;            // 227 KB: the opt-in dynamic shared memory of one CTA
constexpr size_t SX_BYTES = 256;               // FOCR_W8A8_T_MAX fp32 activation scales
constexpr size_t BAR_BYTES = 2 * NST_MAX * sizeof(uint64_t);
constexpr uint64_t WAIT_NS = 200000000ull;     // a bounded wait gives up after 0.2 s
static_assert(NST_MAX * STAGE_BYTES + SX_BYTES + BAR_BYTES <= SMEM_MAX, "ring exceeds shared memory");

// D += A (16 x 32 s8, row) * B (32 x 8 s8, col), s32 accumulate
__device__ __forceinline__ void mma_s8(int (&d)[4], const uint4& a, uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float w8a8_scale(float sw, float sx, int acc) {
    return __double2float_rn(__dmul_rn(__dmul_rn((double)sw, (double)sx), (double)acc));
}

struct QParams {
    const float* x;
    int T, K, KS, NBt;
    int8_t* qx;       // nullable, [T, K]
    uint32_t* qxf;    // nullable, [KS][NBt][32][2] words
    float* sx;        // [T]
};

__global__ void __launch_bounds__(QT) w8a8_quantize_kernel(QParams p) {
    __shared__ float red[QT / 32];
    const int t = blockIdx.x, tid = threadIdx.x;
    const float* xt = p.x + (size_t)t * p.K;
    pdl_launch_dependents();   // the GEMV may start streaming its codes now; it waits for this grid's end
    pdl_wait();                // x may come from the previous kernel
    float m = 0.f;
    for (int k = tid; k < p.K; k += QT) m = fmaxf(m, fabsf(xt[k]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) red[tid >> 5] = m;
    __syncthreads();
    m = red[0];
#pragma unroll
    for (int w = 1; w < QT / 32; ++w) m = fmaxf(m, red[w]);
    const float s = __fdiv_rn(m, 127.0f);
    if (tid == 0) p.sx[t] = s;
    const int nb = t >> 3, gr = t & 7;
    for (int w = tid; w < p.KS * 8; w += QT) {
        uint32_t packed = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int k = 4 * w + e;
            int v = 0;
            if (k < p.K && s != 0.f) v = max(-127, min(127, __float2int_rn(__fdiv_rn(xt[k], s))));
            packed |= (uint32_t)(v & 0xff) << (8 * e);
            if (p.qx && k < p.K) p.qx[(size_t)t * p.K + k] = (int8_t)v;
        }
        if (p.qxf) {
            const int q = w >> 3, c = w & 3, half = (w >> 2) & 1;
            p.qxf[((size_t)(q * p.NBt + nb) * 32 + 4 * gr + c) * 2 + half] = packed;
        }
    }
}

struct GParams {
    const uint8_t* codes;   // [tiles][KS][32 lanes][16 bytes]
    const float* sw;        // [16 * tiles]
    const uint2* qxf;       // [KS][NBt][32]
    const float* sx;        // [T]
    float* y;               // [T, N]
    int32_t* acc;           // [T, 16 * tiles], split plans only
    uint32_t* cnt;          // [tiles], split plans only
    uint32_t* err;          // set to 1 when a bounded wait runs out
    int64_t N;
    int KS, tiles, S, L, T, NBt;
    int nst;                // ring stages of this launch, a multiple of ncons
    int ncons;              // consumer warps that take units (unit i: warp i % ncons, stage i % nst)
    uint32_t xf_bytes;      // qx fragments staged in shared memory (0: read through L1)
};

// shared memory: [qx fragments, xf_bytes][sx, SX_BYTES][ring, nst stages][full / empty barriers]
__host__ __device__ __forceinline__ size_t ring_offset(uint32_t xf_bytes) { return xf_bytes + SX_BYTES; }
__host__ __device__ __forceinline__ size_t bar_offset(uint32_t xf_bytes, int nst) {
    return ring_offset(xf_bytes) + (size_t)nst * STAGE_BYTES;
}

template <int NB, bool XS>
__device__ __forceinline__ void mma_kstep(int (&acc)[NB][4], const uint4& a, const uint2* bq, int nbt, int lane) {
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
        if (nb < nbt) {
            const uint2 b = XS ? bq[nb * 32 + lane] : __ldg(bq + nb * 32 + lane);
            mma_s8(acc[nb], a, b.x, b.y);
        }
}

__device__ __forceinline__ void unit_range(const GParams& p, int64_t u, int& tile, int& q0, int& q1) {
    tile = (int)(u / p.S);
    q0 = (int)(u % p.S) * p.L;
    q1 = min(p.KS, q0 + p.L);
}

// the producer lane: one bulk copy per unit into the ring, nst units ahead of the consumers
__device__ void w8a8_produce(const GParams& p, char* ring, uint64_t* full, uint64_t* empty, int64_t units) {
    const uint64_t policy = policy_evict_first();   // every code byte is read once
    const int nst = p.nst;
    int i = 0;
    bool ok = true;
    for (;; ++i) {
        const int64_t u = blockIdx.x + (int64_t)i * gridDim.x;
        if (u >= units) break;
        const int s = i % nst;
        if (i >= nst && !mbar_wait_bounded(&empty[s], ((i / nst) - 1) & 1, WAIT_NS)) {
            ok = false;
            break;
        }
        int tile, q0, q1;
        unit_range(p, u, tile, q0, q1);
        const uint32_t bytes = (uint32_t)(q1 - q0) * 512u;
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_g2s(ring + (size_t)s * STAGE_BYTES, p.codes + ((size_t)tile * p.KS + q0) * 512, bytes, &full[s], policy);
    }
    // the CTA does not end with copies into its shared memory in flight
    for (int k = max(0, i - nst); k < i; ++k)
        if (!mbar_wait_bounded(&full[k % nst], (k / nst) & 1, WAIT_NS)) ok = false;
    if (!ok) atomicExch(p.err, 1u);
}

template <int NB, bool XS>
__device__ void w8a8_consume(const GParams& p, const uint2* xf, const float* sxs, const char* ring, uint64_t* full,
                             uint64_t* empty, int64_t units, int warp, int lane) {
    const int gr = lane >> 2, c = lane & 3;
    const int nst = p.nst;
    const int64_t NP = 16 * (int64_t)p.tiles;
    const uint2* bsrc = XS ? xf : p.qxf;
    // a stage's successive units all belong to one warp (nst is a multiple of ncons), so no warp
    // waits on a phase of its full barrier more than one phase ahead of the copies
    for (int i = warp;; i += p.ncons) {
        const int64_t u = blockIdx.x + (int64_t)i * gridDim.x;
        if (u >= units) break;
        int tile, q0, q1;
        unit_range(p, u, tile, q0, q1);
        const int64_t r0 = 16 * (int64_t)tile + gr, r1 = r0 + 8;
        float s0 = 0.f, s1 = 0.f;
        if (p.S == 1) {   // row scales in flight while the codes arrive
            s0 = __ldg(p.sw + r0);
            s1 = __ldg(p.sw + r1);
        }
        const int s = i % nst;
        if (!mbar_wait_bounded(&full[s], (i / nst) & 1, WAIT_NS)) {
            if (lane == 0) atomicExch(p.err, 1u);
            break;
        }
        const uint4* a_src = reinterpret_cast<const uint4*>(ring + (size_t)s * STAGE_BYTES) + lane;
        int acc[NB][4];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0;
#pragma unroll 4
        for (int q = q0; q < q1; ++q)
            mma_kstep<NB, XS>(acc, a_src[(q - q0) * 32], bsrc + (size_t)q * p.NBt * 32, p.NBt, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);   // the stage's codes are consumed: refill it

        if (p.S == 1) {
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int t = 8 * nb + 2 * c + h;
                    if (t >= p.T) continue;
                    const float sx = sxs[t];
                    if (r0 < p.N) p.y[(size_t)t * p.N + r0] = w8a8_scale(s0, sx, acc[nb][h]);
                    if (r1 < p.N) p.y[(size_t)t * p.N + r1] = w8a8_scale(s1, sx, acc[nb][2 + h]);
                }
            continue;
        }
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int t = 8 * nb + 2 * c + h;
                if (t >= p.T) continue;
                if (r0 < p.N) atomicAdd(p.acc + (size_t)t * NP + r0, acc[nb][h]);
                if (r1 < p.N) atomicAdd(p.acc + (size_t)t * NP + r1, acc[nb][2 + h]);
            }
        __threadfence();
        __syncwarp();
        uint32_t last = 0;
        if (lane == 0) last = atomicAdd(p.cnt + tile, 1u) == (uint32_t)(p.S - 1);
        last = __shfl_sync(0xffffffffu, last, 0);
        if (!last) continue;
        __threadfence();
        for (int k = lane; k < 16 * p.T; k += 32) {
            const int t = k >> 4;
            const int64_t row = 16 * (int64_t)tile + (k & 15);
            if (row >= p.N) continue;
            int32_t* a = p.acc + (size_t)t * NP + row;
            p.y[(size_t)t * p.N + row] = w8a8_scale(__ldg(p.sw + row), sxs[t], __ldcg(a));
            __stcg(a, 0);
        }
        if (lane == 0) p.cnt[tile] = 0;
    }
}

template <int NB, bool XS>
__global__ void __launch_bounds__(GT, 1) w8a8_gemv_kernel(GParams p) {
    extern __shared__ __align__(128) char smem[];
    uint2* xf = reinterpret_cast<uint2*>(smem);
    float* sxs = reinterpret_cast<float*>(smem + p.xf_bytes);
    char* ring = smem + ring_offset(p.xf_bytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + bar_offset(p.xf_bytes, p.nst));
    uint64_t* empty = full + NST_MAX;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t units = (int64_t)p.tiles * p.S;
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.nst; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        fence_barrier_init();
    }
    __syncthreads();
    if (warp == NC) {   // the codes are weights: streaming starts before the quantiser has finished
        if (lane == 0) w8a8_produce(p, ring, full, empty, units);
        return;
    }
    pdl_wait();   // qx fragments and scales come from the quantiser
    if (XS) {
        const uint4* src = reinterpret_cast<const uint4*>(p.qxf);
        uint4* dst = reinterpret_cast<uint4*>(xf);
        for (int k = threadIdx.x; k < (int)(p.xf_bytes / 16); k += NC * 32) dst[k] = __ldcg(src + k);
    }
    for (int t = threadIdx.x; t < p.T; t += NC * 32) sxs[t] = __ldcg(p.sx + t);
    named_bar_sync(1, NC * 32);
    if (warp < p.ncons) w8a8_consume<NB, XS>(p, xf, sxs, ring, full, empty, units, warp, lane);
}

template <int NB, bool XS>
cudaError_t launch_gemv_nb(const GParams& p, int grid, cudaStream_t st) {
    const cudaError_t e = once_per_device((const void*)w8a8_gemv_kernel<NB, XS>, [] {
        return cudaFuncSetAttribute(w8a8_gemv_kernel<NB, XS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)SMEM_MAX);
    });
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(GT);
    cfg.dynamicSmemBytes = bar_offset(p.xf_bytes, p.nst) + BAR_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, w8a8_gemv_kernel<NB, XS>, p);
}

template <int NB>
cudaError_t launch_gemv_xs(const GParams& p, int grid, cudaStream_t st) {
    return p.xf_bytes ? launch_gemv_nb<NB, true>(p, grid, st) : launch_gemv_nb<NB, false>(p, grid, st);
}

}  // namespace

W8a8Plan w8a8_plan(int64_t tiles, int KS) {
    // cost of a plan: the k-steps on the busiest CTA's critical path, each unit charged a few
    // k-steps for its copy latency and epilogue; fewer splits win ties (no atomics when S = 1)
    constexpr int UNIT_OVERHEAD = 4;
    const int sms = device_sms() > 0 ? device_sms() : 148;
    const int s_min = (KS + LMAX - 1) / LMAX, s_max = std::max(s_min, KS / 8);
    W8a8Plan best;
    int64_t best_cost = -1;
    for (int S = s_min; S <= s_max && S <= s_min + 64; ++S) {
        const int L = (KS + S - 1) / S, S2 = (KS + L - 1) / L;   // L <= LMAX; no empty chunk
        const int64_t units = tiles * S2;
        const int grid = (int)std::min<int64_t>(sms, units);
        const int64_t cost = ((units + grid - 1) / grid) * (L + UNIT_OVERHEAD);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best.S = S2;
            best.L = L;
            best.grid = grid;
        }
    }
    return best;
}

cudaError_t launch_w8a8_quantize(const float* x, int T, int K, int8_t* qx, uint32_t* qxf, float* sx,
                                 cudaStream_t st) {
    QParams p;
    p.x = x;
    p.T = T;
    p.K = K;
    p.KS = (K + 31) / 32;
    p.NBt = (T + 7) / 8;
    p.qx = qx;
    p.qxf = qxf;
    p.sx = sx;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(T);
    cfg.blockDim = dim3(QT);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, w8a8_quantize_kernel, p);
}

cudaError_t launch_w8a8_gemv(const void* codes, const float* sw, int64_t N, int K, const uint32_t* qxf,
                             const float* sx, int T, float* y, int32_t* acc, uint32_t* cnt, uint32_t* err,
                             cudaStream_t st) {
    GParams p;
    p.codes = reinterpret_cast<const uint8_t*>(codes);
    p.sw = sw;
    p.qxf = reinterpret_cast<const uint2*>(qxf);
    p.sx = sx;
    p.y = y;
    p.acc = acc;
    p.cnt = cnt;
    p.err = err;
    p.N = N;
    p.KS = (K + 31) / 32;
    p.tiles = (int)((N + 15) / 16);
    p.T = T;
    p.NBt = (T + 7) / 8;
    const W8a8Plan pl = w8a8_plan(p.tiles, p.KS);
    p.S = pl.S;
    p.L = pl.L;
    // the qx fragments go to shared memory when NST_MIN stages still fit beside them
    const size_t xf = (size_t)p.KS * p.NBt * 256;
    const size_t room = SMEM_MAX - SX_BYTES - BAR_BYTES;
    if (xf + NST_MIN * STAGE_BYTES <= room) {
        p.xf_bytes = (uint32_t)xf;
        p.nst = (int)std::min<size_t>(NST_MAX, (room - xf) / STAGE_BYTES);
    } else {
        p.xf_bytes = 0;
        p.nst = NST_MAX;
    }
    p.ncons = std::min(NC, p.nst);
    p.nst -= p.nst % p.ncons;
    if (p.NBt <= 1) return launch_gemv_xs<1>(p, pl.grid, st);
    if (p.NBt <= 2) return launch_gemv_xs<2>(p, pl.grid, st);
    if (p.NBt <= 4) return launch_gemv_xs<4>(p, pl.grid, st);
    return launch_gemv_xs<8>(p, pl.grid, st);
}

}  // namespace focr
