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
//   w8a8_gemv_kernel      an HBM-bound stream of the codes.  One warp per (16-row tile, k-chunk)
//                         unit loads one 16-byte A fragment per lane per k-step (non-allocating, a
//                         batch of 4 in flight while the previous one is consumed) and issues
//                         integer tensor-core MMAs (mma.sync m16n8k32 s8 with s32 accumulate: exact
//                         integer arithmetic), the B fragments coming from L1.  When a tile's K is
//                         split over several warps, their partial sums meet by integer atomics
//                         (exact, so the order does not matter) and the tile's last warp (a
//                         per-tile counter) applies the scales and returns the sums and the counter
//                         to zero.  The first batch of codes is loaded before the wait on the
//                         quantiser (programmatic dependent launch): the weights do not depend on it.
#include <algorithm>

#include "common.cuh"
#include "launch_state.h"
#include "w8a8.h"

namespace focr {
namespace {

constexpr int QT = 256;        // quantiser threads per token
constexpr int GW = 16;         // GEMV warps per CTA
constexpr int GT = GW * 32;
constexpr int BATCH = 4;       // k-steps per load batch
constexpr int MIN_CHUNK = 8;   // fewest k-steps a split unit takes

__device__ __forceinline__ uint4 ldg_stream16(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// D += A (16 x 32 s8, row) * B (32 x 8 s8, col), s32 accumulate
__device__ __forceinline__ void mma_s8(int (&d)[4], const uint4& a, uint32_t b0, uint32_t b1) {
    asm volatile(
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
    pdl_wait();   // x may come from the previous kernel
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
    pdl_launch_dependents();
}

struct GParams {
    const uint4* codes;   // [tiles][KS][32] lane vectors
    const float* sw;      // [16 * tiles]
    const uint2* qxf;     // [KS][NBt][32]
    const float* sx;      // [T]
    float* y;             // [T, N]
    int32_t* acc;         // [T, 16 * tiles], split plans only
    uint32_t* cnt;        // [tiles], split plans only
    int64_t N;
    int KS, tiles, S, L, T, NBt;
};

template <int NB>
__device__ __forceinline__ void mma_kstep(int (&acc)[NB][4], const uint4& a, const uint2* bq, int nbt, int lane) {
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
        if (nb < nbt) {
            const uint2 b = __ldg(bq + nb * 32 + lane);
            mma_s8(acc[nb], a, b.x, b.y);
        }
}

template <int NB>
__global__ void __launch_bounds__(GT, 1) w8a8_gemv_kernel(GParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gr = lane >> 2, c = lane & 3;
    const int64_t units = (int64_t)p.tiles * p.S, nwarps = (int64_t)gridDim.x * GW;
    bool waited = false;
    for (int64_t u = (int64_t)blockIdx.x * GW + warp; u < units; u += nwarps) {
        const int tile = (int)(u / p.S), j = (int)(u % p.S);
        const int q0 = j * p.L, q1 = min(p.KS, q0 + p.L);
        const uint4* src = p.codes + (size_t)tile * p.KS * 32 + lane;
        uint4 cur[BATCH], nxt[BATCH];
#pragma unroll
        for (int i = 0; i < BATCH; ++i)
            if (q0 + i < q1) cur[i] = ldg_stream16(src + (size_t)(q0 + i) * 32);
        if (!waited) {
            pdl_wait();   // the codes above are weights; the activations come from the quantiser
            waited = true;
        }
        int acc[NB][4];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0;
#pragma unroll 1
        for (int qb = q0; qb < q1; qb += BATCH) {
            if (qb + BATCH < q1) {
#pragma unroll
                for (int i = 0; i < BATCH; ++i)
                    if (qb + BATCH + i < q1) nxt[i] = ldg_stream16(src + (size_t)(qb + BATCH + i) * 32);
            }
#pragma unroll
            for (int i = 0; i < BATCH; ++i)
                if (qb + i < q1) mma_kstep<NB>(acc, cur[i], p.qxf + (size_t)(qb + i) * p.NBt * 32, p.NBt, lane);
#pragma unroll
            for (int i = 0; i < BATCH; ++i) cur[i] = nxt[i];
        }
        const int64_t r0 = 16 * (int64_t)tile + gr, r1 = r0 + 8;
        const int64_t NP = 16 * (int64_t)p.tiles;
        if (p.S == 1) {
            const float s0 = __ldg(p.sw + r0), s1 = __ldg(p.sw + r1);
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int t = 8 * nb + 2 * c + h;
                    if (t >= p.T) continue;
                    const float sx = __ldg(p.sx + t);
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
        for (int i = lane; i < 16 * p.T; i += 32) {
            const int t = i >> 4;
            const int64_t row = 16 * (int64_t)tile + (i & 15);
            if (row >= p.N) continue;
            int32_t* a = p.acc + (size_t)t * NP + row;
            p.y[(size_t)t * p.N + row] = w8a8_scale(__ldg(p.sw + row), __ldg(p.sx + t), __ldcg(a));
            __stcg(a, 0);
        }
        if (lane == 0) p.cnt[tile] = 0;
    }
    if (!waited) pdl_wait();
}

template <int NB>
cudaError_t launch_gemv_nb(const GParams& p, int grid, cudaStream_t st) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(GT);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, w8a8_gemv_kernel<NB>, p);
}

}  // namespace

W8a8Plan w8a8_plan(int64_t tiles, int KS) {
    W8a8Plan pl;
    const int sms = device_sms();
    const int64_t nwarps = (int64_t)(sms > 0 ? sms : 148) * GW;
    int S = 1;
    if (tiles < nwarps) S = (int)std::min<int64_t>((nwarps + tiles - 1) / tiles, std::max(1, KS / MIN_CHUNK));
    pl.L = (KS + S - 1) / S;
    pl.S = (KS + pl.L - 1) / pl.L;   // no empty chunk
    const int64_t units = tiles * pl.S;
    pl.grid = (int)std::min<int64_t>(sms > 0 ? sms : 148, (units + GW - 1) / GW);
    return pl;
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
                             const float* sx, int T, float* y, int32_t* acc, uint32_t* cnt, cudaStream_t st) {
    GParams p;
    p.codes = reinterpret_cast<const uint4*>(codes);
    p.sw = sw;
    p.qxf = reinterpret_cast<const uint2*>(qxf);
    p.sx = sx;
    p.y = y;
    p.acc = acc;
    p.cnt = cnt;
    p.N = N;
    p.KS = (K + 31) / 32;
    p.tiles = (int)((N + 15) / 16);
    p.T = T;
    p.NBt = (T + 7) / 8;
    const W8a8Plan pl = w8a8_plan(p.tiles, p.KS);
    p.S = pl.S;
    p.L = pl.L;
    if (p.NBt <= 1) return launch_gemv_nb<1>(p, pl.grid, st);
    if (p.NBt <= 2) return launch_gemv_nb<2>(p, pl.grid, st);
    if (p.NBt <= 4) return launch_gemv_nb<4>(p, pl.grid, st);
    return launch_gemv_nb<8>(p, pl.grid, st);
}

}  // namespace focr
