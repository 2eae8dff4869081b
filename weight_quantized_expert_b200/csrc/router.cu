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
// Grid: one thread-block cluster of 8 CTAs per block of TB <= 8 tokens.  CTA r of a
// cluster computes fp64 partial logits over input columns [160 r, 160 r + 160); the seven
// remote CTAs send theirs into CTA 0's shared memory as asynchronous stores (st.async)
// that complete on a CTA-0 mbarrier, armed before the one cluster barrier (which precedes
// the wait on the previous kernel), and then initialise the layer output.  CTA 0 sums the
// eight partials in a fixed order, ranks each token's 64 experts by a strict total-order
// key (one thread per candidate) while other warps compute the softmax statistics, and,
// when the batch has a single token block, one warp does the dispatch from shared memory.
// With several token blocks each cluster publishes its top-6 and the last one to finish
// (atomic ticket, reset after use) does the dispatch.
#include <cooperative_groups.h>

#include "common.cuh"
#include "launch_state.h"

namespace cg = cooperative_groups;

namespace focr {
namespace {

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

constexpr int RT_THREADS = 256;
constexpr int RC = ROUTER_KSPLIT;         // CTAs per cluster
constexpr int KCOLS = H / RC;             // 160 columns per CTA
constexpr int PART_COLS = KCOLS / 4;      // 40 columns per thread
constexpr int NVEC = PART_COLS / 8;       // 5 vectors of 8 bf16
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // 2 s

struct RouterParams {
    const float* x;
    int T;
    const uint16_t* wr;
    RouteView R;
    float* out;           // NULL: the output is not initialised here
    const float* resid;   // NULL: out starts at zero; else out starts as a copy of resid
    uint16_t* x_img;      // NULL, or x in bf16 as an operand image (tensor-core path)
    int img_rows;         // its rows (T rounded up to 16)
    // tensor-core path: only the per-expert assignment counts are produced here (added into these
    // zeroed words); the expert kernel derives offsets and builds each expert's permutation
    // segment itself, so no block of this grid waits for the others
    int* tc_counts;
};

// counts / offsets / active list / stable permutation of n = T*6 <= 64 entries, by one warp.
// Lane l owns experts 2l, 2l+1 and entries l, l+32.  An entry's place within its expert's
// segment = entries before it with the same expert: lanes holding equal experts find each
// other with __match_any_sync, and entries 32.. add the count among entries 0..31.
__device__ void dispatch_small(const RouterParams& p, const int* sidx, int* cnt) {
    const int lane = threadIdx.x & 31;
    const int n = p.T * K;
    const unsigned lt = (1u << lane) - 1u;
    const int ea = lane < n ? sidx[lane] : -1 - lane;            // distinct negatives never match
    const int eb = lane + 32 < n ? sidx[lane + 32] : -1 - lane;
    cnt[2 * lane] = 0;
    cnt[2 * lane + 1] = 0;
    const unsigned ma = __match_any_sync(0xffffffffu, ea);
    const unsigned mb = __match_any_sync(0xffffffffu, eb);
    __syncwarp();
    if (ea >= 0 && (ma & lt) == 0) cnt[ea] = __popc(ma);         // first lane of each group
    __syncwarp();
    const int ra = __popc(ma & lt);
    const int rb = (eb >= 0 ? cnt[eb] : 0) + __popc(mb & lt);    // entries 0..31 come first
    __syncwarp();
    if (eb >= 0 && (mb & lt) == 0) cnt[eb] += __popc(mb);
    __syncwarp();
    const int c0 = cnt[2 * lane], c1 = cnt[2 * lane + 1];
    int incl = c0 + c1;
    const int h0 = c0 > 0, h1 = c1 > 0;
    int hincl = h0 + h1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        const int hv = __shfl_up_sync(0xffffffffu, hincl, o);
        if (lane >= o) {
            incl += v;
            hincl += hv;
        }
    }
    const int ex0 = incl - c0 - c1;
    p.R.counts[2 * lane] = c0;
    p.R.counts[2 * lane + 1] = c1;
    p.R.offsets[2 * lane] = ex0;
    p.R.offsets[2 * lane + 1] = ex0 + c0;
    if (lane == 31) p.R.offsets[E] = incl;
    int pos = hincl - h0 - h1;
    if (h0) p.R.active[pos++] = 2 * lane;
    if (h1) p.R.active[pos] = 2 * lane + 1;
    if (lane == 31) p.R.active[E] = hincl;
    // offsets of the experts of this lane's entries, from their owning lanes
    const int sa = ea >= 0 ? ea : 0, sb = eb >= 0 ? eb : 0;
    const int oa0 = __shfl_sync(0xffffffffu, ex0, sa >> 1), oa1 = __shfl_sync(0xffffffffu, ex0 + c0, sa >> 1);
    const int ob0 = __shfl_sync(0xffffffffu, ex0, sb >> 1), ob1 = __shfl_sync(0xffffffffu, ex0 + c0, sb >> 1);
    if (ea >= 0) p.R.perm[((sa & 1) ? oa1 : oa0) + ra] = lane;
    if (eb >= 0) p.R.perm[((sb & 1) ? ob1 : ob0) + rb] = lane + 32;
}

// counts / offsets / active list / stable permutation of the T*6 entries (idx: shared or global)
template <bool FROM_SMEM>
__device__ void dispatch(const RouterParams& p, const int* sidx, int* cnt, int* cursor, int (*wc)[E]) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = p.T * K;
    if (tid < E) cnt[tid] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += RT_THREADS) atomicAdd(&cnt[FROM_SMEM ? sidx[i] : __ldcg(&p.R.topk_idx[i])], 1);
    __syncthreads();
    if (warp == 0) {
        // 64 experts, two per lane: exclusive scan and compaction of the experts with tokens
        const int c0 = cnt[2 * lane], c1 = cnt[2 * lane + 1];
        int incl = c0 + c1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const int ex0 = incl - c0 - c1;
        p.R.counts[2 * lane] = c0;
        p.R.counts[2 * lane + 1] = c1;
        p.R.offsets[2 * lane] = ex0;
        p.R.offsets[2 * lane + 1] = ex0 + c0;
        cursor[2 * lane] = ex0;
        cursor[2 * lane + 1] = ex0 + c0;
        if (lane == 31) p.R.offsets[E] = incl;
        const int h0 = c0 > 0, h1 = c1 > 0;
        int hincl = h0 + h1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, hincl, o);
            if (lane >= o) hincl += v;
        }
        int pos = hincl - h0 - h1;
        if (h0) p.R.active[pos++] = 2 * lane;
        if (h1) p.R.active[pos] = 2 * lane + 1;
        if (lane == 31) p.R.active[E] = hincl;
    }
    __syncthreads();
    // stable scatter in chunks of 256 entries: rank = cursor + earlier warps + earlier lanes
    for (int base = 0; base < n; base += RT_THREADS) {
        for (int i = tid; i < (RT_THREADS / 32) * E; i += RT_THREADS) (&wc[0][0])[i] = 0;
        __syncthreads();
        const int i = base + tid;
        const int ee = i < n ? (FROM_SMEM ? sidx[i] : __ldcg(&p.R.topk_idx[i])) : -1;
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

template <int TB>
__global__ void __cluster_dims__(RC, 1, 1) __launch_bounds__(RT_THREADS) router_kernel(RouterParams p) {
    cg::cluster_group cluster = cg::this_cluster();
    __shared__ double part_s[RC][TB][E];     // filled in CTA 0 by all CTAs of the cluster
    __shared__ __align__(8) uint64_t pbar;   // CTA 0: completes when the seven remote partials landed
    __shared__ __align__(16) double xs[TB][KCOLS];
    // ranking keys of the logits (CTA 0, after the GEMV): they reuse the x tile's space
    unsigned long long (*lk)[E] = reinterpret_cast<unsigned long long (*)[E]>(&xs[0][0]);
    static_assert(sizeof(double) * KCOLS >= sizeof(unsigned long long) * E, "key rows fit the x tile");
    __shared__ __align__(16) float lg[TB][E];
    __shared__ float smax[TB], sden[TB];
    __shared__ int sidx[TB * K];
    __shared__ int flag;
    __shared__ int cnt[E];
    __shared__ int cursor[E];
    __shared__ int wc[RT_THREADS / 32][E];

    const int tid = threadIdx.x;
    const int r = (int)cluster.block_rank();
    const int tb = blockIdx.x / RC;
    const int t0 = tb * TB;
    const int nt = min(TB, p.T - t0);
    const int k0 = r * KCOLS;

    // router weights are layer constants: fetch them before waiting on the previous kernel
    const int e = tid >> 2, part = tid & 3;
    const uint16_t* wrow = p.wr + (size_t)e * H + k0 + part * PART_COLS;
    // (kept in L2 with priority: 164 KB per layer, read by every forward)
    const uint64_t keep = policy_evict_last();
    uint4 wv[NVEC];
#pragma unroll
    for (int v = 0; v < NVEC; ++v) wv[v] = ldg_policy(wrow + 8 * v, keep);

    // CTA 0's partial-logit barrier is initialised and armed for the seven remote CTAs'
    // bytes before any of them can write (one cluster barrier, before the wait on the
    // previous kernel, so it is off the critical path)
    constexpr uint32_t REMOTE_BYTES = (RC - 1) * TB * E * sizeof(double);
    if (r == 0 && tid == 0) {
        mbar_init(&pbar, 1);
        mbar_arrive_expect_tx(&pbar, REMOTE_BYTES);
        fence_barrier_init();
    }
    cluster.sync();

    pdl_wait();                 // x may come from the previous kernel on the stream
    pdl_launch_dependents();    // let the expert kernel start its routing-free work

    bool out_of_range = false;   // a finite |x| the experts' f16 activation operands cannot hold
    for (int i = tid; i < TB * KCOLS; i += RT_THREADS) {
        const int t = i / KCOLS, c = i % KCOLS;
        const float v = t < nt ? p.x[(size_t)(t0 + t) * H + k0 + c] : 0.f;
        out_of_range |= f16_out_of_range(v);
        xs[t][c] = (double)v;
    }
    if (out_of_range) atomicExch(&p.R.ctrl[CTRL_ERROR], DEVERR_RANGE);
    __syncthreads();
    if (p.x_img) {
        // this CTA's 160 columns of its tokens, rounded to f16 (the tensor-core path's gate/up operand)
        for (int i = tid; i < TB * (KCOLS / 8); i += RT_THREADS) {
            const int t = i / (KCOLS / 8), kc = i % (KCOLS / 8);
            if (t < nt) {
                const double* v = &xs[t][kc * 8];
                uint4 o;
                o.x = pack_f16x2((float)v[0], (float)v[1]);
                o.y = pack_f16x2((float)v[2], (float)v[3]);
                o.z = pack_f16x2((float)v[4], (float)v[5]);
                o.w = pack_f16x2((float)v[6], (float)v[7]);
                *reinterpret_cast<uint4*>(p.x_img + img_index(p.img_rows, t0 + t, k0 + kc * 8)) = o;
            }
        }
    }

    // thread -> (expert e, quarter of the CTA's columns); products are exact in fp64.  With
    // few tokens each token's sum is split over NA interleaved chains (fixed order) so that
    // the fp64 FMAs overlap.
    constexpr int NA = TB >= 4 ? 1 : 4 / TB;
    double accp[TB][NA];
#pragma unroll
    for (int t = 0; t < TB; ++t)
#pragma unroll
        for (int k = 0; k < NA; ++k) accp[t][k] = 0.0;
#pragma unroll
    for (int v = 0; v < NVEC; ++v) {
        float w[8];
        bf16x2_to_f32(wv[v].x, w[0], w[1]);
        bf16x2_to_f32(wv[v].y, w[2], w[3]);
        bf16x2_to_f32(wv[v].z, w[4], w[5]);
        bf16x2_to_f32(wv[v].w, w[6], w[7]);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const double wd = (double)w[j];
#pragma unroll
            for (int t = 0; t < TB; ++t)
                accp[t][j % NA] = fma(xs[t][part * PART_COLS + 8 * v + j], wd, accp[t][j % NA]);
        }
    }
    double acc[TB];
#pragma unroll
    for (int t = 0; t < TB; ++t) {
        acc[t] = accp[t][0];
#pragma unroll
        for (int k = 1; k < NA; ++k) acc[t] += accp[t][k];
    }
#pragma unroll
    for (int t = 0; t < TB; ++t) {
        acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 1);
        acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 2);
    }
    // partials into CTA 0: local stores there, asynchronous remote stores (completing on CTA
    // 0's barrier) from the other seven
    if (part == 0) {
        if (r == 0) {
#pragma unroll
            for (int t = 0; t < TB; ++t) part_s[0][t][e] = acc[t];
        } else {
            const uint32_t rbar = mapa_shared(&pbar, 0);
#pragma unroll
            for (int t = 0; t < TB; ++t) st_async_f64(mapa_shared(&part_s[r][t][e], 0), acc[t], rbar);
        }
    }
    if (r != 0) {
        // CTAs 1..7 of every cluster initialise the layer output (the decode kernels add into
        // it after this grid completes)
        if (p.out) {
            const int nw = (gridDim.x / RC) * (RC - 1), w = tb * (RC - 1) + (r - 1);
            float4* o4 = reinterpret_cast<float4*>(p.out);
            const float4* r4 = reinterpret_cast<const float4*>(p.resid);
            const int n4 = p.T * H / 4;
            for (int i = w * RT_THREADS + tid; i < n4; i += nw * RT_THREADS)
                o4[i] = r4 ? r4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        return;
    }

    // ---- CTA 0: wait for the remote partials (bounded), then logits (fixed summation
    // order), softmax, top-6
    __syncthreads();   // CTA 0's own partials are in place
    if (!mbar_wait_bounded(&pbar, 0, WAIT_LIMIT_NS)) {
        if (tid == 0) atomicExch(&p.R.ctrl[CTRL_ERROR], DEVERR_FULL_WAIT);
        (void)mbar_wait_bounded(&pbar, 0, WAIT_LIMIT_NS);   // never exit with remote stores in flight
    }
    for (int i = tid; i < TB * E; i += RT_THREADS) {
        const int t = i / E, ee = i % E;
        if (t < nt) {
            double s = 0.0;
#pragma unroll
            for (int b = 0; b < RC; ++b) s += part_s[b][t][ee];
            const float l = (float)s;
            lg[t][ee] = l;
            p.R.logits[(size_t)(t0 + t) * E + ee] = l;
            // strict total order for the top-6: order-preserving bits of the logit (-0 folded into
            // +0, so equal logits tie), then the lower index; any logit vector, NaN included,
            // yields six distinct in-range experts
            uint32_t b = __float_as_uint(l + 0.0f);
            b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
            lk[t][ee] = ((unsigned long long)b << 32) | (unsigned long long)(E - 1 - ee);
        }
    }
    __syncthreads();

    const int warp = tid >> 5, lane = tid & 31;
    // softmax statistics: one warp per token (the highest warps), two logits per lane
    {
        const int t = RT_THREADS / 32 - 1 - warp;
        if (t < nt) {
            const float v0 = lg[t][lane], v1 = lg[t][lane + 32];
            float m = fmaxf(v0, v1);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            float den = expf(v0 - m) + expf(v1 - m);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
            if (lane == 0) {
                smax[t] = m;
                sden[t] = den;
            }
        }
    }
    // greedy top-6 by rank: candidate c of token t is ahead of `rank` experts, counted in
    // (logit descending, index ascending) order over the token's 64 keys (branch-free, the keys
    // read as broadcast 16-byte vectors); the six of rank < 6 are the top-6
    constexpr int RPT = (TB * E + RT_THREADS - 1) / RT_THREADS;   // candidates per thread
    int rank[RPT];
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
        const int i = tid + k * RT_THREADS, t = i / E, c = i % E;
        int rk = E;
        if (t < nt) {
            const unsigned long long kc = lk[t][c];
            const ulonglong2* row = reinterpret_cast<const ulonglong2*>(&lk[t][0]);
            rk = 0;
#pragma unroll
            for (int q = 0; q < E / 2; ++q) {
                const ulonglong2 f = row[q];
                rk += (int)(f.x > kc) + (int)(f.y > kc);
            }
        }
        rank[k] = rk;
    }
    __syncthreads();   // softmax statistics in place
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
        if (rank[k] < K) {
            const int i = tid + k * RT_THREADS, t = i / E, c = i % E;
            sidx[t * K + rank[k]] = c;
            p.R.topk_idx[(size_t)(t0 + t) * K + rank[k]] = c;
            p.R.topk_w[(size_t)(t0 + t) * K + rank[k]] = expf(lg[t][c] - smax[t]) / sden[t];
        }
    }
    __syncthreads();

    if (p.tc_counts) {
        // per-expert totals of this block's entries, one atomic per expert present
        if (tid < E) cnt[tid] = 0;
        __syncthreads();
        if (tid < nt * K) atomicAdd(&cnt[sidx[tid]], 1);
        __syncthreads();
        if (tid < E && cnt[tid] > 0) atomicAdd(&p.tc_counts[tid], cnt[tid]);
        return;
    }
    if (gridDim.x == RC) {     // one token block (T <= 8): one warp dispatches from shared memory
        if (warp == 0) dispatch_small(p, sidx, cnt);
        return;
    }
    // ---- several token blocks: the last one to finish dispatches
    __threadfence();
    __syncthreads();
    if (tid == 0) flag = (atomicAdd(&p.R.ctrl[CTRL_GLOBAL_TICKET], 1) == (int)(gridDim.x / RC) - 1);
    __syncthreads();
    if (!flag) return;
    __threadfence();
    if (tid == 0) p.R.ctrl[CTRL_GLOBAL_TICKET] = 0;
    dispatch<false>(p, sidx, cnt, cursor, wc);
}

}  // namespace

cudaError_t launch_router(const float* x, int T, int /*T_ws*/, const LayerView& L, const RouteView& R, float* out,
                          const float* resid, uint16_t* x_img, int img_rows, cudaStream_t st) {
    RouterParams p{x, T, L.router, R, out, resid, x_img, img_rows, x_img ? R.ctrl + CTRL_TC + TC_CNT : nullptr};
    const int TB = T <= 1 ? 1 : (T <= 2 ? 2 : (T <= 4 ? 4 : 8));
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(((T + TB - 1) / TB) * RC);
    cfg.blockDim = dim3(RT_THREADS);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // the same shared-memory carveout as the expert kernels
    const cudaError_t e0 = once_per_device((const void*)router_kernel<1>, [] {
        for (const void* f : {(const void*)router_kernel<1>, (const void*)router_kernel<2>, (const void*)router_kernel<4>,
                              (const void*)router_kernel<8>}) {
            const cudaError_t e =
                cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    });
    if (e0 != cudaSuccess) return e0;
    switch (TB) {
        case 1: return cudaLaunchKernelEx(&cfg, router_kernel<1>, p);
        case 2: return cudaLaunchKernelEx(&cfg, router_kernel<2>, p);
        case 4: return cudaLaunchKernelEx(&cfg, router_kernel<4>, p);
        default: return cudaLaunchKernelEx(&cfg, router_kernel<8>, p);
    }
}

}  // namespace focr
