// lm_head GEMV 1280 -> 129280 with int8 weights (one f32 scale per row) and the greedy
// argmax, fused.
//
// Source: frankenocr.pages.dev, "One forward pass", step 7 (final RMSNorm feeds an lm_head
// GEMV from 1,280 to 129,280 logits; greedy decoding) and "Four bits, one shared scale"
// (int8 on lm_head).  logit_n = s_n * sum_k q_nk x_k; argmax ties go to the lower index.
//
// Layout (packed on the host): rows in tiles of 16; for tile r, k-step q (16 columns) and
// lane L = 4 gr + c the eight codes of an m16n8k16 A fragment (rows gr, gr+8; columns
// 16q+2c, +1, +8, +9), offset-binary, two k-steps per 16-byte lane vector:
// codes[tile][q / 2][lane][16 bytes]; scales[row] f32.
//
// Kernel: one CTA of 12 warps per SM; warps stream whole tiles with 16-byte non-allocating
// loads (a batch of 4 lane vectors in flight, the next batch issued before the current one
// is consumed).  int8 codes are exact in f16; x is split into f16 hi + lo fragments (two
// MMAs, about 22 significant bits), so logits carry fp32 accuracy.  Tokens are processed in
// chunks of up to 32 (4 n8 fragment columns).  Each lane keeps the best (logit, row) of
// its columns; warps and CTAs reduce packed (ordered logit, ~row) keys, and the last CTA
// to finish (atomic ticket, reset after use) writes argmax[t].
//
// Up to 8 tokens (decode) take lm_head_ring_kernel instead: the same fragments and MMAs, with each
// tile's 20 KB of codes moved by one bulk copy into a shared-memory ring (see below), which keeps
// 160 KB per SM in flight, and each tile's k-steps split over two warps (two partial sums, added
// once).
#include "common.cuh"
#include "launch_state.h"
#include "fragments.cuh"
#include "lm_head.h"

namespace focr {
namespace {

constexpr int LW = 12;                 // warps per CTA
constexpr int LT = LW * 32;
constexpr int VT = FOCR_VOCAB / 16;    // 8080 row tiles
constexpr int VEC_PER_TILE = KSTEPS / 2;   // 40 lane vectors of 16 bytes
constexpr int TCH = 32;                // tokens per chunk

struct LmParams {
    const uint4* codes;
    const float* scales;
    const float* x;
    int T;
    float* logits;       // nullable [T, V]
    int32_t* argmax;     // [T]
    unsigned long long* keys;   // [gridDim][T]
    int* ticket;
    int32_t* err;        // nullable: set to 1 (if still 0) when a bounded wait of the ring kernel runs out
};

__device__ __forceinline__ uint4 ldg_stream(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ unsigned long long pack_key(float v, int row) {
    uint32_t b = __float_as_uint(v);
    b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);   // order-preserving bits
    return ((unsigned long long)b << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)row);
}

constexpr int BATCH = 4;   // 16-byte lane vectors per load batch (two batches in flight)

template <int NB>
__device__ __forceinline__ void lm_chunk(const LmParams& p, int t0, const uint4* xb, unsigned long long* wkeys,
                                         int gwarp, int nwarps, int warp, int lane) {
    const int gr = lane >> 2, c = lane & 3;
    unsigned long long best[NB][2];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) best[nb][0] = best[nb][1] = 0ull;
    for (int tile = gwarp; tile < VT; tile += nwarps) {
        const uint4* src = p.codes + (size_t)tile * VEC_PER_TILE * 32 + lane;
        float acc[NB][4];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0.f;
        uint4 cur[BATCH], nxt[BATCH];
#pragma unroll
        for (int i = 0; i < BATCH; ++i) cur[i] = ldg_stream(src + i * 32);
#pragma unroll 1
        for (int v0 = 0; v0 < VEC_PER_TILE; v0 += BATCH) {
            if (v0 + BATCH < VEC_PER_TILE) {
#pragma unroll
                for (int i = 0; i < BATCH; ++i) nxt[i] = ldg_stream(src + (v0 + BATCH + i) * 32);
            }
#pragma unroll
            for (int i = 0; i < BATCH; ++i) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int q = 2 * (v0 + i) + h;
                    const Frag4 a = h ? dq_int8(cur[i].z, cur[i].w) : dq_int8(cur[i].x, cur[i].y);
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb) {
                        const uint4 b = xb[(q * NB + nb) * 32 + lane];
                        mma16816(acc[nb], a, b.x, b.y);   // x hi
                        mma16816(acc[nb], a, b.z, b.w);   // x lo
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < BATCH; ++i) cur[i] = nxt[i];
        }
        const int r0 = 16 * tile + gr, r1 = r0 + 8;
        const float s0 = __ldg(p.scales + r0), s1 = __ldg(p.scales + r1);
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int t = t0 + 8 * nb + 2 * c + h;
                const float l0 = acc[nb][h] * s0, l1 = acc[nb][2 + h] * s1;
                if (t < p.T) {
                    if (p.logits) {
                        p.logits[(size_t)t * FOCR_VOCAB + r0] = l0;
                        p.logits[(size_t)t * FOCR_VOCAB + r1] = l1;
                    }
                    const unsigned long long k0 = pack_key(l0, r0), k1 = pack_key(l1, r1);
                    unsigned long long& b = best[nb][h];
                    b = k0 > b ? k0 : b;
                    b = k1 > b ? k1 : b;
                }
            }
        }
    }
    // lanes with the same c hold the same two columns of every fragment column block
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            unsigned long long b = best[nb][h];
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                const unsigned long long ob = __shfl_xor_sync(0xffffffffu, b, o);
                b = ob > b ? ob : b;
            }
            if (lane < 4) wkeys[warp * TCH + 8 * nb + 2 * lane + h] = b;
        }
}

__global__ void __launch_bounds__(LT, 1) lm_head_kernel(LmParams p) {
    extern __shared__ __align__(128) char smem[];
    uint4* xb = reinterpret_cast<uint4*>(smem);                                   // [80][NB][32] f16 hi/lo frags
    unsigned long long* wkeys = reinterpret_cast<unsigned long long*>(smem + KSTEPS * 4 * 32 * 16);  // [LW][TCH]
    __shared__ int last;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gwarp = blockIdx.x * LW + warp, nwarps = gridDim.x * LW;
    pdl_wait();   // x comes from the previous kernel (the RMSNorm)

    for (int t0 = 0; t0 < p.T; t0 += TCH) {
        const int nt = min(TCH, p.T - t0);
        const int NB = (nt + 7) / 8;
        __syncthreads();   // previous chunk done with xb / wkeys
        // x fragments of this chunk: entry (q, nb, lane) = columns 16q+2c(+1), 16q+2c+8(+9) of token 8nb + lane/4
        for (int i = tid; i < KSTEPS * NB * 32; i += LT) {
            const int ln = i & 31, qn = i >> 5;
            const int q = qn / NB, nb = qn % NB;
            const int t = t0 + 8 * nb + (ln >> 2);
            float2 lo = make_float2(0.f, 0.f), hi = make_float2(0.f, 0.f);
            if (t < p.T) {
                const float* row = p.x + (size_t)t * H + 16 * q + 2 * (ln & 3);
                lo = *reinterpret_cast<const float2*>(row);
                hi = *reinterpret_cast<const float2*>(row + 8);
            }
            const uint32_t h0 = f32x2_to_f16x2(lo.x, lo.y), h1 = f32x2_to_f16x2(hi.x, hi.y);
            const __half2 hh0 = *reinterpret_cast<const __half2*>(&h0), hh1 = *reinterpret_cast<const __half2*>(&h1);
            const float2 r0 = __half22float2(hh0), r1 = __half22float2(hh1);
            const uint32_t l0 = f32x2_to_f16x2(lo.x - r0.x, lo.y - r0.y), l1 = f32x2_to_f16x2(hi.x - r1.x, hi.y - r1.y);
            xb[i] = make_uint4(h0, h1, l0, l1);
        }
        for (int i = tid; i < LW * TCH; i += LT) wkeys[i] = 0ull;
        __syncthreads();
        switch (NB) {
            case 1: lm_chunk<1>(p, t0, xb, wkeys, gwarp, nwarps, warp, lane); break;
            case 2: lm_chunk<2>(p, t0, xb, wkeys, gwarp, nwarps, warp, lane); break;
            case 3: lm_chunk<3>(p, t0, xb, wkeys, gwarp, nwarps, warp, lane); break;
            default: lm_chunk<4>(p, t0, xb, wkeys, gwarp, nwarps, warp, lane); break;
        }
        __syncthreads();
        if (tid < nt) {
            unsigned long long b = 0ull;
            for (int w = 0; w < LW; ++w) b = wkeys[w * TCH + tid] > b ? wkeys[w * TCH + tid] : b;
            p.keys[(size_t)blockIdx.x * p.T + t0 + tid] = b;
        }
    }
    // the last CTA to finish reduces the per-CTA keys
    __threadfence();
    __syncthreads();
    if (tid == 0) last = (atomicAdd(p.ticket, 1) == (int)gridDim.x - 1);
    __syncthreads();
    if (!last) return;
    __threadfence();
    for (int t = tid; t < p.T; t += LT) {
        unsigned long long b = 0ull;
        for (int g = 0; g < (int)gridDim.x; ++g) {
            const unsigned long long k = __ldcg(p.keys + (size_t)g * p.T + t);
            b = k > b ? k : b;
        }
        p.argmax[t] = (int32_t)(0xFFFFFFFFu - (uint32_t)(b & 0xFFFFFFFFull));
    }
    if (tid == 0) *p.ticket = 0;
}

// ---------------------------------------------------------------- T <= 8: bulk-copy ring
// One producer lane moves each 16-row tile (20 KB of codes, contiguous) with one bulk copy into a
// ring of shared-memory stages.  Stage s belongs to the warp pair (s, s + RNST): both take the
// CTA's tiles s, s + RNST, ... (so neither waits on a full barrier more than one phase ahead of its
// copies), each runs half of the tile's k-steps, the second warp hands its partial sums over in
// shared memory, and the first adds them (first half + second half) and finishes the tile.  The x
// fragments of the (single) token chunk are built once per CTA in shared memory.
constexpr int RNST = 8;                                  // ring stages
constexpr int RNC = 2 * RNST;                            // consumer warps: a pair per stage
constexpr int RT = (RNC + 1) * 32;                       // + one producer warp
constexpr int RHALF = VEC_PER_TILE / 2;                  // lane vectors per warp of a pair
constexpr size_t TILE_BYTES = (size_t)VEC_PER_TILE * 32 * 16;
constexpr size_t R_XB = (size_t)KSTEPS * 32 * 16;        // x fragments of 8 tokens
constexpr size_t R_KEYS = (size_t)RNST * 8 * 8;          // [pair][token] argmax keys
constexpr size_t R_RED = R_XB + R_KEYS;                  // [pair][2][32 lanes][4] partial sums + [pair][2][2] ok flags
constexpr size_t R_RED_BYTES = (size_t)RNST * 2 * 32 * 16 + (size_t)RNST * 2 * 2 * 4;
constexpr size_t R_RING = (R_RED + R_RED_BYTES + 127) & ~(size_t)127;
constexpr size_t R_BARS = R_RING + RNST * TILE_BYTES;
constexpr size_t R_SMEM = R_BARS + 2 * RNST * sizeof(uint64_t);
constexpr uint64_t R_WAIT_NS = 200000000ull;
static_assert(VEC_PER_TILE % 2 == 0, "a tile splits into two halves");
static_assert(RNST + 2 <= 16, "named barriers: 0, 1 and one per pair");
static_assert(R_SMEM <= 232448, "ring exceeds shared memory");

__device__ void lm_ring_produce(const LmParams& p, char* ring, uint64_t* full, uint64_t* empty) {
    const uint64_t policy = policy_evict_first();
    int i = 0;
    bool ok = true;
    for (;; ++i) {
        const int tile = blockIdx.x + i * gridDim.x;
        if (tile >= VT) break;
        const int s = i % RNST;
        if (i >= RNST && !mbar_wait_bounded(&empty[s], ((i / RNST) - 1) & 1, R_WAIT_NS)) {
            ok = false;
            break;
        }
        mbar_arrive_expect_tx(&full[s], (uint32_t)TILE_BYTES);
        bulk_g2s(ring + (size_t)s * TILE_BYTES, p.codes + (size_t)tile * VEC_PER_TILE * 32, (uint32_t)TILE_BYTES,
                 &full[s], policy);
    }
    for (int k = max(0, i - RNST); k < i; ++k)   // no copy into this CTA's shared memory outlives it
        if (!mbar_wait_bounded(&full[k % RNST], (k / RNST) & 1, R_WAIT_NS)) ok = false;
    if (!ok && p.err) atomicCAS(p.err, 0, 1);
}

__global__ void __launch_bounds__(RT, 1) lm_head_ring_kernel(LmParams p) {
    extern __shared__ __align__(128) char smem[];
    uint4* xb = reinterpret_cast<uint4*>(smem);                               // [80][32] f16 hi/lo frags
    unsigned long long* wkeys = reinterpret_cast<unsigned long long*>(smem + R_XB);   // [RNST][8]
    char* ring = smem + R_RING;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + R_BARS);
    uint64_t* empty = full + RNST;
    __shared__ int last;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < RNST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        fence_barrier_init();
    }
    __syncthreads();
    if (warp == RNC) {   // the codes are weights: they stream before the RMSNorm that makes x has finished
        if (lane == 0) lm_ring_produce(p, ring, full, empty);
        return;
    }
    pdl_wait();   // x comes from the previous kernel (the RMSNorm)
    for (int i = tid; i < KSTEPS * 32; i += RNC * 32) {
        const int ln = i & 31, q = i >> 5;
        const int t = ln >> 2;
        float2 lo = make_float2(0.f, 0.f), hi = make_float2(0.f, 0.f);
        if (t < p.T) {
            const float* row = p.x + (size_t)t * H + 16 * q + 2 * (ln & 3);
            lo = *reinterpret_cast<const float2*>(row);
            hi = *reinterpret_cast<const float2*>(row + 8);
        }
        const uint32_t h0 = f32x2_to_f16x2(lo.x, lo.y), h1 = f32x2_to_f16x2(hi.x, hi.y);
        const __half2 hh0 = *reinterpret_cast<const __half2*>(&h0), hh1 = *reinterpret_cast<const __half2*>(&h1);
        const float2 r0 = __half22float2(hh0), r1 = __half22float2(hh1);
        const uint32_t l0 = f32x2_to_f16x2(lo.x - r0.x, lo.y - r0.y), l1 = f32x2_to_f16x2(hi.x - r1.x, hi.y - r1.y);
        xb[i] = make_uint4(h0, h1, l0, l1);
    }
    named_bar_sync(1, RNC * 32);

    const int gr = lane >> 2, c = lane & 3;
    const int pw = warp % RNST, second = warp / RNST;   // pair (= stage) and which half of each tile
    float4* red = reinterpret_cast<float4*>(smem + R_RED);                                // [pair][2][32]
    int32_t* red_ok = reinterpret_cast<int32_t*>(smem + R_RED + (size_t)RNST * 2 * 32 * 16);   // [pair][2][2]
    unsigned long long best[2] = {0ull, 0ull};
    for (int i = pw, n = 0;; i += RNST, ++n) {
        const int tile = blockIdx.x + i * gridDim.x;
        if (tile >= VT) break;
        const int r0 = 16 * tile + gr, r1 = r0 + 8;
        float s0 = 0.f, s1 = 0.f;
        if (!second) {   // in flight during the wait
            s0 = __ldg(p.scales + r0);
            s1 = __ldg(p.scales + r1);
        }
        const int s = pw, buf = n & 1;
        const bool ok = mbar_wait_bounded(&full[s], n & 1, R_WAIT_NS);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (ok) {
            const uint4* a_src = reinterpret_cast<const uint4*>(ring + (size_t)s * TILE_BYTES) + lane;
            const int v0 = second * RHALF;
#pragma unroll 4
            for (int v = v0; v < v0 + RHALF; ++v) {
                const uint4 a = a_src[v * 32];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const Frag4 f = h ? dq_int8(a.z, a.w) : dq_int8(a.x, a.y);
                    const uint4 b = xb[(2 * v + h) * 32 + lane];
                    mma16816(acc, f, b.x, b.y);   // x hi
                    mma16816(acc, f, b.z, b.w);   // x lo
                }
            }
        }
        // the pair meets once per tile (double-buffered hand-over): partial sums and both wait results
        if (second) red[(pw * 2 + buf) * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        if (lane == 0) red_ok[(pw * 2 + buf) * 2 + second] = ok ? 1 : 0;
        named_bar_sync(2 + pw, 64);
        const bool both = red_ok[(pw * 2 + buf) * 2] && red_ok[(pw * 2 + buf) * 2 + 1];
        if (!both) {
            if (lane == 0 && !ok && p.err) atomicCAS(p.err, 0, 1);
            break;
        }
        if (second) continue;
        if (lane == 0) mbar_arrive(&empty[s]);   // both halves of the stage are consumed: refill it
        const float4 o = red[(pw * 2 + buf) * 32 + lane];
        acc[0] += o.x;
        acc[1] += o.y;
        acc[2] += o.z;
        acc[3] += o.w;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int t = 2 * c + h;
            const float l0 = acc[h] * s0, l1 = acc[2 + h] * s1;
            if (t < p.T) {
                if (p.logits) {
                    p.logits[(size_t)t * FOCR_VOCAB + r0] = l0;
                    p.logits[(size_t)t * FOCR_VOCAB + r1] = l1;
                }
                const unsigned long long k0 = pack_key(l0, r0), k1 = pack_key(l1, r1);
                best[h] = k0 > best[h] ? k0 : best[h];
                best[h] = k1 > best[h] ? k1 : best[h];
            }
        }
    }
    if (!second) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            unsigned long long b = best[h];
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                const unsigned long long ob = __shfl_xor_sync(0xffffffffu, b, o);
                b = ob > b ? ob : b;
            }
            if (lane < 4) wkeys[pw * 8 + 2 * lane + h] = b;
        }
    }
    named_bar_sync(1, RNC * 32);
    if (tid < p.T) {
        unsigned long long b = 0ull;
        for (int w = 0; w < RNST; ++w) b = wkeys[w * 8 + tid] > b ? wkeys[w * 8 + tid] : b;
        p.keys[(size_t)blockIdx.x * p.T + tid] = b;
    }
    // the last CTA to finish reduces the per-CTA keys
    __threadfence();
    named_bar_sync(1, RNC * 32);
    if (tid == 0) last = (atomicAdd(p.ticket, 1) == (int)gridDim.x - 1);
    named_bar_sync(1, RNC * 32);
    if (!last) return;
    __threadfence();
    for (int t = tid; t < p.T; t += RNC * 32) {
        unsigned long long b = 0ull;
        for (int g = 0; g < (int)gridDim.x; ++g) {
            const unsigned long long k = __ldcg(p.keys + (size_t)g * p.T + t);
            b = k > b ? k : b;
        }
        p.argmax[t] = (int32_t)(0xFFFFFFFFu - (uint32_t)(b & 0xFFFFFFFFull));
    }
    if (tid == 0) *p.ticket = 0;
}

}  // namespace

size_t lm_head_smem_bytes() { return (size_t)KSTEPS * 4 * 32 * 16 + (size_t)LW * TCH * 8; }

cudaError_t launch_lm_head(const uint4* codes, const float* scales, const float* x, int T, float* logits,
                           int32_t* argmax, void* ws, cudaStream_t st) {
    return launch_lm_head(codes, scales, x, T, logits, argmax, reinterpret_cast<int*>(ws),
                          reinterpret_cast<unsigned long long*>(reinterpret_cast<char*>(ws) + 256),
                          reinterpret_cast<int32_t*>(ws) + 1, st);
}

cudaError_t launch_lm_head(const uint4* codes, const float* scales, const float* x, int T, float* logits,
                           int32_t* argmax, int* ticket, unsigned long long* keys, int32_t* err, cudaStream_t st) {
    const bool ring = T <= 8;
    const void* fn = ring ? (const void*)lm_head_ring_kernel : (const void*)lm_head_kernel;
    const cudaError_t e = once_per_device(fn, [ring] {
        return ring ? cudaFuncSetAttribute(lm_head_ring_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)R_SMEM)
                    : cudaFuncSetAttribute(lm_head_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)lm_head_smem_bytes());
    });
    if (e != cudaSuccess) return e;
    const int sms = device_sms();
    if (sms <= 0) return cudaErrorInvalidDevice;
    LmParams p;
    p.codes = codes;
    p.scales = scales;
    p.x = x;
    p.T = T;
    p.logits = logits;
    p.argmax = argmax;
    p.ticket = ticket;
    p.keys = keys;
    p.err = err;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(sms);
    cfg.blockDim = dim3(ring ? RT : LT);
    cfg.dynamicSmemBytes = ring ? R_SMEM : lm_head_smem_bytes();
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return ring ? cudaLaunchKernelEx(&cfg, lm_head_ring_kernel, p) : cudaLaunchKernelEx(&cfg, lm_head_kernel, p);
}

int lm_head_grid() { return device_sms(); }

}  // namespace focr
