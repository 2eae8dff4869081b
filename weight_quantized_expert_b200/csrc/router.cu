// Router: logits = x W_r^T, softmax, greedy top-6 without renormalisation, and the
// token -> expert dispatch (histogram, exclusive scan, stable permutation).
//
// Source: frankenocr.pages.dev, "One forward pass", step 6 -- a softmax router over
// 64 routed experts picks the top 6 greedily and does not renormalise; the router
// stays bf16 ("Four bits, one shared scale": bf16 on the router).
//
// Precision: every product of a bf16 weight and an fp32 activation is exact in fp64,
// so logits are accumulated in fp64 and rounded once to fp32; experts are ranked by
// (fp32 logit descending, index ascending).  Softmax is evaluated in fp32.
//
// Grid: (ceil(T / 8) token blocks) x (5 column blocks of 256).  Each CTA writes fp64
// partial logits; the last CTA of a token block (atomic ticket) sums the five
// partials in a fixed order, runs softmax + top-6 for its 8 tokens (one warp per
// token), and the last token block to finish performs the dispatch.  Tickets are
// reset by the CTAs that consume them, so the workspace control words end at zero.
#include "common.cuh"

namespace focr {
namespace {

constexpr int RT_THREADS = 256;
constexpr int KCOLS = H / ROUTER_KSPLIT;  // 256

struct RouterParams {
    const float* x;
    int T;
    const uint16_t* wr;
    RouteView R;
    float* out;
};

__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, o);
        const int oi = __shfl_xor_sync(0xffffffffu, i, o);
        if (ov > v || (ov == v && oi < i)) {
            v = ov;
            i = oi;
        }
    }
}

__global__ void __launch_bounds__(RT_THREADS) router_kernel(RouterParams p) {
    pdl_wait();                 // inputs may come from the previous kernel on the stream
    pdl_launch_dependents();    // let the expert kernel start its routing-free work

    __shared__ float xs[ROUTER_TB][KCOLS];
    __shared__ float lg[ROUTER_TB][E];
    __shared__ int flag;
    __shared__ int cnt[E];
    __shared__ int cursor[E];
    __shared__ int wc[RT_THREADS / 32][E];

    const int tid = threadIdx.x;
    const int tb = blockIdx.x, kb = blockIdx.y;
    const int t0 = tb * ROUTER_TB;
    const int nt = min(ROUTER_TB, p.T - t0);
    const int k0 = kb * KCOLS;

    // zero the layer output (the expert kernel adds into it after this grid completes)
    {
        const int nblk = gridDim.x * gridDim.y;
        const int b = blockIdx.y * gridDim.x + blockIdx.x;
        float4* o4 = reinterpret_cast<float4*>(p.out);
        const int n4 = p.T * H / 4;
        for (int i = b * RT_THREADS + tid; i < n4; i += nblk * RT_THREADS) o4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }

    for (int i = tid; i < ROUTER_TB * KCOLS / 4; i += RT_THREADS) {
        const int t = i / (KCOLS / 4), c = (i % (KCOLS / 4)) * 4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (t < nt) v = *reinterpret_cast<const float4*>(p.x + (size_t)(t0 + t) * H + k0 + c);
        *reinterpret_cast<float4*>(&xs[t][c]) = v;
    }
    __syncthreads();

    // thread -> (expert e, quarter of the 256 columns)
    const int e = tid >> 2, part = tid & 3;
    double acc[ROUTER_TB];
#pragma unroll
    for (int t = 0; t < ROUTER_TB; ++t) acc[t] = 0.0;
    const uint16_t* wrow = p.wr + (size_t)e * H + k0 + part * 64;
#pragma unroll 2
    for (int c = 0; c < 64; c += 8) {
        const uint4 wv = *reinterpret_cast<const uint4*>(wrow + c);
        float w[8];
        bf16x2_to_f32(wv.x, w[0], w[1]);
        bf16x2_to_f32(wv.y, w[2], w[3]);
        bf16x2_to_f32(wv.z, w[4], w[5]);
        bf16x2_to_f32(wv.w, w[6], w[7]);
#pragma unroll
        for (int t = 0; t < ROUTER_TB; ++t)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[t] = fma((double)xs[t][part * 64 + c + j], (double)w[j], acc[t]);
    }
#pragma unroll
    for (int t = 0; t < ROUTER_TB; ++t) {
        acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 1);
        acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 2);
    }
    if (part == 0)
        for (int t = 0; t < nt; ++t) p.R.partial[((size_t)kb * p.T + t0 + t) * E + e] = acc[t];

    // ---- last column block of this token block: logits, softmax, top-6
    __threadfence();
    __syncthreads();
    if (tid == 0) flag = (atomicAdd(&p.R.ctrl[tb], 1) == ROUTER_KSPLIT - 1);
    __syncthreads();
    if (!flag) return;
    __threadfence();
    for (int i = tid; i < ROUTER_TB * E; i += RT_THREADS) {
        const int t = i / E, ee = i % E;
        if (t < nt) {
            double s = 0.0;
            for (int b = 0; b < ROUTER_KSPLIT; ++b)
                s += __ldcg(&p.R.partial[((size_t)b * p.T + t0 + t) * E + ee]);
            const float l = (float)s;
            lg[t][ee] = l;
            p.R.logits[(size_t)(t0 + t) * E + ee] = l;
        }
    }
    if (tid == 0) p.R.ctrl[tb] = 0;
    __syncthreads();

    const int warp = tid >> 5, lane = tid & 31;
    if (warp < nt) {
        const int t = warp;
        float v0 = lg[t][lane], v1 = lg[t][lane + 32];
        // softmax denominator (fp32), max over 64
        float m = fmaxf(v0, v1);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float den = expf(v0 - m) + expf(v1 - m);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
        bool taken0 = false, taken1 = false;
        for (int j = 0; j < K; ++j) {
            // best remaining candidate of this lane (lower index first on ties)
            float cv = -INFINITY;
            int ci = 0x7fffffff;
            if (!taken0) { cv = v0; ci = lane; }
            if (!taken1 && (v1 > cv || (v1 == cv && lane + 32 < ci))) { cv = v1; ci = lane + 32; }
            warp_argmax(cv, ci);
            if (ci == lane) taken0 = true;
            if (ci == lane + 32) taken1 = true;
            if (lane == 0) {
                p.R.topk_idx[(size_t)(t0 + t) * K + j] = ci;
                p.R.topk_w[(size_t)(t0 + t) * K + j] = expf(cv - m) / den;
            }
        }
    }

    // ---- last token block overall: dispatch
    __threadfence();
    __syncthreads();
    if (tid == 0) flag = (atomicAdd(&p.R.ctrl[CTRL_GLOBAL_TICKET], 1) == (int)gridDim.x - 1);
    __syncthreads();
    if (!flag) return;
    __threadfence();

    const int n = p.T * K;
    if (tid < E) cnt[tid] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += RT_THREADS) atomicAdd(&cnt[__ldcg(&p.R.topk_idx[i])], 1);
    __syncthreads();
    if (tid == 0) {
        int run = 0, u = 0;
        for (int ee = 0; ee < E; ++ee) {
            p.R.counts[ee] = cnt[ee];
            p.R.offsets[ee] = run;
            cursor[ee] = run;
            if (cnt[ee] > 0) p.R.active[u++] = ee;
            run += cnt[ee];
        }
        p.R.offsets[E] = run;
        p.R.active[E] = u;
        p.R.ctrl[CTRL_GLOBAL_TICKET] = 0;
    }
    __syncthreads();
    // stable scatter in chunks of 256 entries: rank = cursor + earlier warps + earlier lanes
    for (int base = 0; base < n; base += RT_THREADS) {
        for (int i = tid; i < (RT_THREADS / 32) * E; i += RT_THREADS) (&wc[0][0])[i] = 0;
        __syncthreads();
        const int i = base + tid;
        const int ee = i < n ? __ldcg(&p.R.topk_idx[i]) : -1;
        const unsigned same = __match_any_sync(0xffffffffu, ee);
        const unsigned lower = same & ((1u << lane) - 1u);
        if (ee >= 0 && lower == 0) wc[warp][ee] = __popc(same);
        __syncthreads();
        if (ee >= 0) {
            int pos = cursor[ee] + __popc(lower);
            for (int w = 0; w < warp; ++w) pos += wc[w][ee];
            p.R.perm[pos] = i;
        }
        __syncthreads();
        if (tid < E) {
            int add = 0;
            for (int w = 0; w < RT_THREADS / 32; ++w) add += wc[w][tid];
            cursor[tid] += add;
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_router(const float* x, int T, int /*T_ws*/, const LayerView& L, const RouteView& R, float* out,
                          cudaStream_t st) {
    RouterParams p{x, T, L.router, R, out};
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((T + ROUTER_TB - 1) / ROUTER_TB, ROUTER_KSPLIT);
    cfg.blockDim = dim3(RT_THREADS);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, router_kernel, p);
}

}  // namespace focr
