// Grouped expert kernel for decode-sized batches: the shared expert and every
// selected routed expert, SwiGLU fused, weights dequantised in registers, fp32
// accumulation, combine by vector atomics into the zeroed layer output.
//
// Sources: frankenocr.pages.dev, "One forward pass", step 6 (64 routed experts + 2 fused
// shared experts, top-6 without renormalisation); franken_ocr README, "Architecture"
// (each expert 1280 -> 896 SiLU-gated); "Four bits, one shared scale" (int4 nibble +
// f32 group scale; int8 and bf16 formats).
//
// Work decomposition: an "item" is one slice of S intermediate rows of one expert
// (common.cuh: S = 32 int4 / 16 int8 / 8 bf16, ~60-75 KB of weights).  Items are
// numbered shared-expert slices first, then the slices of every expert that received
// tokens (ascending expert id), and CTA b of a persistent grid takes items b, b+G, ...
// A producer warp streams each item's block into a shared-memory ring with bulk async
// copies (cp.async.bulk + mbarrier); eight consumer warps compute, per batch of <= 8
// tokens routed to the item's expert:
//   phase 1: g = G_slice x, u = U_slice x   (quad rows x 8-column units, lane-strided,
//            warp transpose-reduce, shared-memory accumulation)
//   a = silu(g) * u                          (S values per token)
//   phase 2: y = D[:, slice] a, out[t] += w_t * y   (red.global.add.v4.f32)
// The shared-expert slices need no routing, so they run while the router kernel is
// still working (programmatic dependent launch); routed items start after
// griddepcontrol.wait.  Every mbarrier wait is bounded in time; on expiry the kernel
// records an error word in the workspace and stops.
#include "common.cuh"

namespace focr {
namespace {

constexpr int NCW = 8;                       // consumer warps
constexpr int NCT = NCW * 32;                // consumer threads
constexpr int NTHREADS = NCT + 32;           // + producer warp
constexpr int NSLOT = 2;
constexpr int TTMAX = 8;
constexpr uint32_t SLOT_BYTES = 76800;       // largest item (int4 g32) + its down scales
constexpr uint32_t DSC_BYTES = H * 4;        // one group's down scales
constexpr int SMAX = 32;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // 2 s

struct SmemLayout {
    static constexpr uint32_t slots = 0;
    static constexpr uint32_t xs = slots + NSLOT * SLOT_BYTES;          // [TTMAX][H] f32
    static constexpr uint32_t gu = xs + TTMAX * H * 4;                  // [2*SMAX][TTMAX] f32
    static constexpr uint32_t as = gu + 2 * SMAX * TTMAX * 4;           // [TTMAX][SMAX] f32
    static constexpr uint32_t tok = as + TTMAX * SMAX * 4;              // [TTMAX] i32
    static constexpr uint32_t wt = tok + TTMAX * 4;                     // [TTMAX] f32
    static constexpr uint32_t bars = wt + TTMAX * 4;                    // full[NSLOT], empty[NSLOT]
    static constexpr uint32_t misc = bars + 2 * NSLOT * 8;              // ok flag etc.
    static constexpr uint32_t total = misc + 16;
};

struct ExpertParams {
    const float* x;
    int T;
    float* out;
    LayerView L;
    RouteView R;
};

struct Item {
    const uint8_t* blk;   // item block (GU weights, GU scales, D weights)
    const float* dsc;     // this slice's down-scale group (nullptr for bf16)
    uint32_t blk_bytes;   // bytes of the block to copy
    int wtype, group, S;
    uint32_t gu_w_bytes, gu_s_bytes;
    int expert;           // -1 for the shared expert
};

__device__ __forceinline__ Item get_item(const ExpertParams& p, int item, int n_shared) {
    Item it;
    const ItemGeom* g;
    if (item < n_shared) {
        g = &p.L.sg;
        it.blk = p.L.shared_items + (size_t)item * g->item_bytes;
        it.dsc = is_quant(g->wtype) ? p.L.shared_dscale + (size_t)(item * g->S / g->group) * H : nullptr;
        it.expert = -1;
    } else {
        g = &p.L.rg;
        const int k = item - n_shared;
        const int a = k / g->slices, s = k % g->slices;
        const int e = p.R.active[a];
        it.blk = p.L.routed_items + ((size_t)e * g->slices + s) * g->item_bytes;
        it.dsc = is_quant(g->wtype)
                     ? p.L.routed_dscale + (size_t)e * g->dscale_expert_floats + (size_t)(s * g->S / g->group) * H
                     : nullptr;
        it.expert = e;
    }
    it.wtype = g->wtype;
    it.group = g->group;
    it.S = g->S;
    it.gu_w_bytes = g->gu_w_bytes;
    it.gu_s_bytes = g->gu_s_bytes;
    it.blk_bytes = g->gu_w_bytes + g->gu_s_bytes + g->d_w_bytes;
    return it;
}

// ------------------------------------------------------------------ warp transpose-reduce
// v[0..N) per lane; afterwards v[0] of lane l holds the warp total of element l >> (5 - log2 N).
template <int N, int O>
struct TR {
    static __device__ __forceinline__ void run(float* v, int lane) {
        if constexpr (O == 0) {
            return;
        } else if constexpr (N > 1) {
            const bool up = (lane & O) != 0;
#pragma unroll
            for (int i = 0; i < N / 2; ++i) {
                const float send = up ? v[i] : v[i + N / 2];
                const float keep = up ? v[i + N / 2] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
            }
            TR<N / 2, O / 2>::run(v, lane);
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], O);
            TR<1, O / 2>::run(v, lane);
        }
    }
};

template <int N>
__device__ __forceinline__ constexpr int log2i() {
    if constexpr (N <= 1) return 0;
    else return 1 + log2i<N / 2>();
}

// dequantise one unit row (8 columns) from shared memory
template <int W>
__device__ __forceinline__ void load_unit(const uint8_t* p, float (&w)[8]) {
    if constexpr (W == FOCR_W_INT4) {
        const uint32_t v = *reinterpret_cast<const uint32_t*>(p);
        dq_int4x8(v, w);
    } else if constexpr (W == FOCR_W_INT8) {
        const uint2 v = *reinterpret_cast<const uint2*>(p);
        float a[4], b[4];
        dq_int8x4(v.x, a);
        dq_int8x4(v.y, b);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            w[j] = a[j];
            w[4 + j] = b[j];
        }
    } else {
        const uint4 v = lds128(p);
        bf16x2_to_f32(v.x, w[0], w[1]);
        bf16x2_to_f32(v.y, w[2], w[3]);
        bf16x2_to_f32(v.z, w[4], w[5]);
        bf16x2_to_f32(v.w, w[6], w[7]);
    }
}

// ------------------------------------------------------------------ phase 1: gate/up
template <int W, int TT>
__device__ __forceinline__ void phase_gate_up(const Item& it, const uint8_t* slot, const float* xs, float* gu,
                                              int warp, int lane) {
    constexpr int UB = unit_row_bytes(W);
    constexpr int S = slice_rows(W);
    constexpr int NQ = S / 2;
    constexpr int KS = (W == FOCR_W_BF16) ? 2 : 1;
    constexpr int UPT = UNITS / KS;   // units per task
    constexpr int N = 4 * TT;
    const int ngk = is_quant(W) ? H / it.group : 1;
    const uint8_t* gw = slot;
    const float* gs = reinterpret_cast<const float*>(slot + it.gu_w_bytes);
    for (int task = warp; task < NQ * KS; task += NCW) {
        const int quad = task / KS, piece = task % KS;
        float acc[N];
#pragma unroll
        for (int i = 0; i < N; ++i) acc[i] = 0.f;
        for (int u = piece * UPT + lane; u < (piece + 1) * UPT; u += 32) {
            float xv[TT][8];
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                const float4 a = lds128f(xs + t * H + 8 * u);
                const float4 b = lds128f(xs + t * H + 8 * u + 4);
                xv[t][0] = a.x; xv[t][1] = a.y; xv[t][2] = a.z; xv[t][3] = a.w;
                xv[t][4] = b.x; xv[t][5] = b.y; xv[t][6] = b.z; xv[t][7] = b.w;
            }
            float4 sc = make_float4(1.f, 1.f, 1.f, 1.f);
            if constexpr (is_quant(W)) sc = lds128f(gs + ((size_t)quad * ngk + (8 * u) / it.group) * 4);
            const float scr[4] = {sc.x, sc.y, sc.z, sc.w};
            const uint8_t* up = gw + ((size_t)(quad * UNITS + u) * 4) * UB;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                float w[8];
                load_unit<W>(up + r * UB, w);
#pragma unroll
                for (int t = 0; t < TT; ++t) {
                    float s = 0.f;
#pragma unroll
                    for (int j = 0; j < 8; ++j) s = fmaf(w[j], xv[t][j], s);
                    if constexpr (is_quant(W)) acc[r * TT + t] = fmaf(scr[r], s, acc[r * TT + t]);
                    else acc[r * TT + t] += s;
                }
            }
        }
        TR<N, 16>::run(acc, lane);
        constexpr int SH = 5 - log2i<N>();
        if ((lane & ((1 << SH) - 1)) == 0) {
            const int e = lane >> SH;
            const int r = e / TT, t = e % TT;
            const int row = (r < 2) ? (2 * quad + r) : (S + 2 * quad + r - 2);
            atomicAdd(&gu[row * TTMAX + t], acc[0]);
        }
    }
}

// ------------------------------------------------------------------ phase 2: down + combine
// dequantise one 16-byte down-row slice (S codes)
template <int W>
__device__ __forceinline__ void load_down_row(const uint8_t* p, float (&w)[slice_rows(W)]) {
    const uint4 v = lds128(p);
    const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
    if constexpr (W == FOCR_W_INT4) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float q[8];
            dq_int4x8(vv[i], q);
#pragma unroll
            for (int j = 0; j < 8; ++j) w[8 * i + j] = q[j];
        }
    } else if constexpr (W == FOCR_W_INT8) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float q[4];
            dq_int8x4(vv[i], q);
#pragma unroll
            for (int j = 0; j < 4; ++j) w[4 * i + j] = q[j];
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) bf16x2_to_f32(vv[i], w[2 * i], w[2 * i + 1]);
    }
}

template <int W, int TT>
__device__ __forceinline__ void phase_down(const Item& it, const uint8_t* slot, const float* as, const int* tok,
                                           const float* wt, float* out, int ctid) {
    constexpr int S = slice_rows(W);
    constexpr int TC = TT < 4 ? TT : 4;   // tokens per pass (keeps y[][] in registers)
    const uint8_t* dw = slot + it.gu_w_bytes + it.gu_s_bytes;
    const float* dsc = reinterpret_cast<const float*>(slot + it.blk_bytes);
    for (int rq = ctid; rq < H / 4; rq += NCT) {
        float4 ds = make_float4(1.f, 1.f, 1.f, 1.f);
        if constexpr (is_quant(W)) ds = lds128f(dsc + 4 * rq);
        const float dsr[4] = {ds.x, ds.y, ds.z, ds.w};
#pragma unroll 1
        for (int t0 = 0; t0 < TT; t0 += TC) {
            float y[4][TC];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                float w[S];
                load_down_row<W>(dw + (size_t)(4 * rq + r) * 16, w);
#pragma unroll
                for (int t = 0; t < TC; ++t) {
                    float s = 0.f;
#pragma unroll
                    for (int k4 = 0; k4 < S; k4 += 4) {
                        const float4 a = lds128f(as + (t0 + t) * SMAX + k4);
                        s = fmaf(w[k4], a.x, s);
                        s = fmaf(w[k4 + 1], a.y, s);
                        s = fmaf(w[k4 + 2], a.z, s);
                        s = fmaf(w[k4 + 3], a.w, s);
                    }
                    y[r][t] = s * dsr[r];
                }
            }
#pragma unroll
            for (int t = 0; t < TC; ++t) {
                const int tk = tok[t0 + t];
                if (tk >= 0) {
                    const float ww = wt[t0 + t];
                    red_add_v4(out + (size_t)tk * H + 4 * rq, ww * y[0][t], ww * y[1][t], ww * y[2][t],
                               ww * y[3][t]);
                }
            }
        }
    }
}

template <int W>
__device__ __forceinline__ void run_batch(int TT, const Item& it, const uint8_t* slot, char* smem, float* out,
                                          int warp, int lane, int ctid, bool phase1) {
    const float* xs = reinterpret_cast<const float*>(smem + SmemLayout::xs);
    float* gu = reinterpret_cast<float*>(smem + SmemLayout::gu);
    const float* as = reinterpret_cast<const float*>(smem + SmemLayout::as);
    const int* tok = reinterpret_cast<const int*>(smem + SmemLayout::tok);
    const float* wt = reinterpret_cast<const float*>(smem + SmemLayout::wt);
    if (phase1) {
        switch (TT) {
            case 1: phase_gate_up<W, 1>(it, slot, xs, gu, warp, lane); break;
            case 2: phase_gate_up<W, 2>(it, slot, xs, gu, warp, lane); break;
            case 4: phase_gate_up<W, 4>(it, slot, xs, gu, warp, lane); break;
            default: phase_gate_up<W, 8>(it, slot, xs, gu, warp, lane); break;
        }
    } else {
        switch (TT) {
            case 1: phase_down<W, 1>(it, slot, as, tok, wt, out, ctid); break;
            case 2: phase_down<W, 2>(it, slot, as, tok, wt, out, ctid); break;
            case 4: phase_down<W, 4>(it, slot, as, tok, wt, out, ctid); break;
            default: phase_down<W, 8>(it, slot, as, tok, wt, out, ctid); break;
        }
    }
}

__device__ __forceinline__ void consumer_sync() { named_bar_sync(1, NCT); }

__global__ void __launch_bounds__(NTHREADS, 1) expert_decode_kernel(ExpertParams p) {
    extern __shared__ __align__(128) char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + SmemLayout::bars);
    uint64_t* empty = full + NSLOT;
    volatile int* okflag = reinterpret_cast<volatile int*>(smem + SmemLayout::misc);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_shared = p.L.sg.slices;

    if (tid == 0) {
        for (int s = 0; s < NSLOT; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        fence_barrier_init();
        okflag[0] = 1;   // consumer wait result
        okflag[1] = 0;   // abort
    }
    {
        float* gu = reinterpret_cast<float*>(smem + SmemLayout::gu);
        for (int i = tid; i < 2 * SMAX * TTMAX; i += NTHREADS) gu[i] = 0.f;
    }
    __syncthreads();

    if (warp == NCW) {
        // ------------------------------------------------------------ producer
        if (lane != 0) return;
        const uint64_t pol_w = policy_evict_first();
        int n_items = 0x7fffffff;
        bool waited = false;
        int issued = 0;
        for (int it = 0;; ++it) {
            const int item = blockIdx.x + it * gridDim.x;
            if (item >= n_shared && !waited) {
                pdl_wait();
                waited = true;
                n_items = n_shared + p.R.active[E] * p.L.rg.slices;
            }
            if (item >= n_items) break;
            const int slot = it % NSLOT;
            if (it >= NSLOT && !mbar_wait_bounded(&empty[slot], ((it / NSLOT) - 1) & 1, WAIT_LIMIT_NS)) {
                atomicExch(&p.R.ctrl[CTRL_ERROR], DEVERR_EMPTY_WAIT);
                okflag[1] = 1;
                break;
            }
            if (okflag[1]) break;
            const Item d = get_item(p, item, n_shared);
            uint8_t* dst = reinterpret_cast<uint8_t*>(smem + SmemLayout::slots + slot * SLOT_BYTES);
            const uint32_t bytes = d.blk_bytes + (d.dsc ? DSC_BYTES : 0u);
            mbar_arrive_expect_tx(&full[slot], bytes);
            bulk_g2s(dst, d.blk, d.blk_bytes, &full[slot], pol_w);
            if (d.dsc) bulk_g2s(dst + d.blk_bytes, d.dsc, DSC_BYTES, &full[slot], pol_w);
            issued = it + 1;
        }
        // never leave copies in flight: wait (bounded) for the last issued ones
        for (int it = max(0, issued - NSLOT); it < issued; ++it)
            (void)mbar_wait_bounded(&full[it % NSLOT], (it / NSLOT) & 1, WAIT_LIMIT_NS);
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int ctid = tid;
    int* tok = reinterpret_cast<int*>(smem + SmemLayout::tok);
    float* wtv = reinterpret_cast<float*>(smem + SmemLayout::wt);
    float* xs = reinterpret_cast<float*>(smem + SmemLayout::xs);
    float* gu = reinterpret_cast<float*>(smem + SmemLayout::gu);
    float* as = reinterpret_cast<float*>(smem + SmemLayout::as);
    int n_items = 0x7fffffff;
    bool waited = false;
    for (int it = 0;; ++it) {
        const int item = blockIdx.x + it * gridDim.x;
        if (item >= n_shared && !waited) {
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
        const Item d = get_item(p, item, n_shared);
        const uint8_t* sbuf = reinterpret_cast<const uint8_t*>(smem + SmemLayout::slots + slot * SLOT_BYTES);

        int ntok, seg = 0;
        if (d.expert < 0) {
            ntok = p.T;
        } else {
            ntok = p.R.counts[d.expert];
            seg = p.R.offsets[d.expert];
        }
        for (int b0 = 0; b0 < ntok; b0 += TTMAX) {
            const int nb = min(TTMAX, ntok - b0);
            const int TT = nb <= 1 ? 1 : (nb <= 2 ? 2 : (nb <= 4 ? 4 : 8));
            if (ctid < TTMAX) {
                int tk = -1;
                float ww = 0.f;
                if (ctid < nb) {
                    if (d.expert < 0) {
                        tk = b0 + ctid;
                        ww = 1.f;
                    } else {
                        const int e = p.R.perm[seg + b0 + ctid];
                        tk = e / K;
                        ww = p.R.topk_w[e];
                    }
                }
                tok[ctid] = tk;
                wtv[ctid] = ww;
            }
            consumer_sync();
            for (int i = ctid; i < TT * (H / 4); i += NCT) {
                const int t = i / (H / 4), c = (i % (H / 4)) * 4;
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (tok[t] >= 0) v = __ldg(reinterpret_cast<const float4*>(p.x + (size_t)tok[t] * H + c));
                *reinterpret_cast<float4*>(xs + t * H + c) = v;
            }
            consumer_sync();
            switch (d.wtype) {
                case FOCR_W_INT4: run_batch<FOCR_W_INT4>(TT, d, sbuf, smem, p.out, warp, lane, ctid, true); break;
                case FOCR_W_INT8: run_batch<FOCR_W_INT8>(TT, d, sbuf, smem, p.out, warp, lane, ctid, true); break;
                default: run_batch<FOCR_W_BF16>(TT, d, sbuf, smem, p.out, warp, lane, ctid, true); break;
            }
            consumer_sync();
            for (int i = ctid; i < d.S * TT; i += NCT) {
                const int r = i / TT, t = i % TT;
                const float g = gu[r * TTMAX + t], u = gu[(d.S + r) * TTMAX + t];
                as[t * SMAX + r] = g / (1.f + __expf(-g)) * u;
                gu[r * TTMAX + t] = 0.f;
                gu[(d.S + r) * TTMAX + t] = 0.f;
            }
            if (!waited) {
                // the router zeroes `out`: no contribution may land before it has finished
                pdl_wait();
                waited = true;
                n_items = n_shared + p.R.active[E] * p.L.rg.slices;
            }
            consumer_sync();
            switch (d.wtype) {
                case FOCR_W_INT4: run_batch<FOCR_W_INT4>(TT, d, sbuf, smem, p.out, warp, lane, ctid, false); break;
                case FOCR_W_INT8: run_batch<FOCR_W_INT8>(TT, d, sbuf, smem, p.out, warp, lane, ctid, false); break;
                default: run_batch<FOCR_W_BF16>(TT, d, sbuf, smem, p.out, warp, lane, ctid, false); break;
            }
            consumer_sync();
        }
        if (ctid == 0) mbar_arrive(&empty[slot]);
    }
}

int g_num_sms = 0;

}  // namespace

cudaError_t launch_expert_decode(const float* x, int T, const LayerView& L, const RouteView& R, float* out,
                                 cudaStream_t st) {
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(expert_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)SmemLayout::total);
        if (e != cudaSuccess) return e;
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
        configured = true;
    }
    ExpertParams p{x, T, out, L, R};
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(g_num_sms);
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = SmemLayout::total;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, expert_decode_kernel, p);
}

}  // namespace focr
