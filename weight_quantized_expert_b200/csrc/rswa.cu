// R-SWA decode attention: one decode step of one attention layer for B sequences.
//
// Source: franken_ocr README, "Design Philosophy" (bounded generated-token KV) and "Architecture"
// (R-SWA: each generated token attends to every reference token -- the visual prefill and the
// prompt, a frozen block that is never evicted -- plus the previous 128 generated tokens, held in
// a ring buffer); frankenocr.pages.dev, "One forward pass", step 6 (ten heads of dimension 128, a
// read-only reference block plus a 128-slot ring that slides).
// Readings where the pages are silent: scores are scaled by 1/sqrt(128); q and k arrive with any
// position encoding applied; the window counts the current token, so it is exactly the ring's 128
// slots (generated token p lives in slot p mod 128).
//
//   keys of sequence b, head h: reference rows r < ref_len[b], then the generated tokens
//   p in [max(0, n - 128), n) with n = n_gen[b] (the current token p = n - 1 from k_new / v_new);
//   out = sum_j softmax_j(q . k_j / sqrt(128)) v_j;   then slot (n - 1) mod 128 <- k_new, v_new.
//
// Kernels (HBM-bound: every key and value row is read once, 1 KB per key and head):
//   rswa_partial_kernel  grid (B x 10 heads, S key chunks), 128 threads.  Eight lanes share a key
//                        (16 of its 128 dims each, float4 loads), sixteen keys in flight per CTA;
//                        each lane group keeps an online softmax (running max, sum, 16 value dims),
//                        the CTA merges its 16 groups in shared memory and writes one partial
//                        (max, sum, 128 weighted value dims).  The chunk-0 CTA of each head stores
//                        the current k / v in the ring: no CTA reads that slot (the current token
//                        is taken from k_new / v_new), so the store races with nothing.
//   rswa_combine_kernel  one CTA per (sequence, head), one thread per dim: merges the S partials
//                        (programmatic dependent launch after the partial kernel).
// A sequence whose ref_len lies outside [0, Rcap] or whose n_gen < 1 gets NaN outputs and keeps its
// ring.
#include <math.h>
#include <stdio.h>

#include <algorithm>

#include "common.cuh"
#include "launch_state.h"
#include "rswa.h"

namespace focr {
namespace {

constexpr int RH = FOCR_RSWA_HEADS, RD = FOCR_RSWA_DIM, RW = FOCR_RSWA_RING;
constexpr int PT = 128;                 // threads of the partial kernel
constexpr int GROUPS = PT / 8;          // keys in flight per CTA (8 lanes each)
constexpr int PART = RD + 2;            // floats per partial: max, sum, 128 dims
constexpr float SCALE = 0.08838834764831845f;   // 1 / sqrt(128)

struct RswaParams {
    const float* q;
    const float* k_new;
    const float* v_new;
    const float* k_ref;
    const float* v_ref;
    const int32_t* ref_len;
    const int32_t* n_gen;
    float* k_ring;
    float* v_ring;
    float* out;
    float* part;     // [B * RH][S][PART]
    int Rcap, B, S, chunk;
};

__device__ __forceinline__ bool seq_valid(int R, int n, int Rcap) { return R >= 0 && R <= Rcap && n >= 1; }

__global__ void __launch_bounds__(PT) rswa_partial_kernel(RswaParams p) {
    __shared__ float sm_m[GROUPS], sm_l[GROUPS];
    __shared__ __align__(16) float sm_acc[GROUPS][RD];
    const int bh = blockIdx.x, s = blockIdx.y, b = bh / RH;
    const int tid = threadIdx.x, g = tid >> 3, sub = tid & 7;   // key group, lane within it
    pdl_wait();   // q, k_new, v_new and the lengths may come from the previous kernel
    const int R = __ldg(p.ref_len + b), n = __ldg(p.n_gen + b);
    if (!seq_valid(R, n, p.Rcap)) return;   // the combine kernel writes NaN
    const int win = min(n, RW), p0 = n - win, nk = R + win;
    const int cur = (n - 1) % RW;
    const size_t hrow = (size_t)bh * RD;
    const float* kref = p.k_ref + (size_t)bh * p.Rcap * RD;
    const float* vref = p.v_ref + (size_t)bh * p.Rcap * RD;
    const float* kring = p.k_ring + (size_t)bh * RW * RD;
    const float* vring = p.v_ring + (size_t)bh * RW * RD;

    float qv[16];
    {
        const float4* q4 = reinterpret_cast<const float4*>(p.q + hrow + 16 * sub);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 t = __ldg(q4 + i);
            qv[4 * i] = t.x;
            qv[4 * i + 1] = t.y;
            qv[4 * i + 2] = t.z;
            qv[4 * i + 3] = t.w;
        }
    }
    float m = -INFINITY, l = 0.f, acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0.f;
    const int j0 = s * p.chunk, j1 = min(nk, j0 + p.chunk);
    // the loop runs the same rounds in every lane (the shuffles need the whole warp); a group whose
    // key lies past the chunk computes nothing and updates nothing
    for (int jb = j0; jb < j1; jb += GROUPS) {
        const int j = jb + g;
        const bool live = j < j1;
        float4 kk[4], vv[4];
        if (live) {
            const float *kp, *vp;
            if (j < R) {
                kp = kref + (size_t)j * RD;
                vp = vref + (size_t)j * RD;
            } else {
                const int pos = p0 + (j - R);
                if (pos == n - 1) {
                    kp = p.k_new + hrow;
                    vp = p.v_new + hrow;
                } else {
                    kp = kring + (size_t)(pos % RW) * RD;
                    vp = vring + (size_t)(pos % RW) * RD;
                }
            }
            const float4* k4 = reinterpret_cast<const float4*>(kp + 16 * sub);
            const float4* v4 = reinterpret_cast<const float4*>(vp + 16 * sub);
#pragma unroll
            for (int i = 0; i < 4; ++i) kk[i] = __ldg(k4 + i);
#pragma unroll
            for (int i = 0; i < 4; ++i) vv[i] = __ldg(v4 + i);
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) kk[i] = vv[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float dot = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            dot = fmaf(qv[4 * i], kk[i].x, dot);
            dot = fmaf(qv[4 * i + 1], kk[i].y, dot);
            dot = fmaf(qv[4 * i + 2], kk[i].z, dot);
            dot = fmaf(qv[4 * i + 3], kk[i].w, dot);
        }
        dot += __shfl_xor_sync(0xffffffffu, dot, 1);
        dot += __shfl_xor_sync(0xffffffffu, dot, 2);
        dot += __shfl_xor_sync(0xffffffffu, dot, 4);
        if (!live) continue;
        const float sc = dot * SCALE;
        const float mn = fmaxf(m, sc);
        const float corr = expf(m - mn), w = expf(sc - mn);
        l = l * corr + w;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc[4 * i] = acc[4 * i] * corr + w * vv[i].x;
            acc[4 * i + 1] = acc[4 * i + 1] * corr + w * vv[i].y;
            acc[4 * i + 2] = acc[4 * i + 2] * corr + w * vv[i].z;
            acc[4 * i + 3] = acc[4 * i + 3] * corr + w * vv[i].w;
        }
        m = mn;
    }
    // merge the CTA's key groups
    if (sub == 0) {
        sm_m[g] = m;
        sm_l[g] = l;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) sm_acc[g][16 * sub + i] = acc[i];
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int k = 0; k < GROUPS; ++k) M = fmaxf(M, sm_m[k]);
    float L = 0.f, A = 0.f;
    if (M != -INFINITY) {
#pragma unroll
        for (int k = 0; k < GROUPS; ++k) {
            const float e = expf(sm_m[k] - M);   // 0 for an empty group
            L += sm_l[k] * e;
            A += sm_acc[k][tid] * e;
        }
    }
    float* out = p.part + ((size_t)bh * p.S + s) * PART;
    if (tid == 0) {
        out[0] = M;
        out[1] = L;
    }
    out[2 + tid] = A;
    if (s == 0) {   // store the current token in its ring slot
        p.k_ring[(size_t)bh * RW * RD + (size_t)cur * RD + tid] = __ldg(p.k_new + hrow + tid);
        p.v_ring[(size_t)bh * RW * RD + (size_t)cur * RD + tid] = __ldg(p.v_new + hrow + tid);
    }
}

__global__ void __launch_bounds__(RD) rswa_combine_kernel(RswaParams p) {
    const int bh = blockIdx.x, b = bh / RH, d = threadIdx.x;
    pdl_wait();   // the partials
    const int R = __ldg(p.ref_len + b), n = __ldg(p.n_gen + b);
    float* o = p.out + (size_t)bh * RD;
    if (!seq_valid(R, n, p.Rcap)) {
        o[d] = __int_as_float(0x7fc00000);   // NaN
        return;
    }
    const float* part = p.part + (size_t)bh * p.S * PART;
    float M = -INFINITY;
    for (int s = 0; s < p.S; ++s) M = fmaxf(M, __ldcg(part + (size_t)s * PART));
    float L = 0.f, A = 0.f;
    for (int s = 0; s < p.S; ++s) {
        const float ms = __ldcg(part + (size_t)s * PART);
        if (ms == -INFINITY) continue;   // an empty chunk
        const float e = expf(ms - M);
        L += __ldcg(part + (size_t)s * PART + 1) * e;
        A += __ldcg(part + (size_t)s * PART + 2 + d) * e;
    }
    o[d] = A / L;
}

cudaError_t launch_pdl(const void* fn, dim3 grid, dim3 block, void** args, cudaStream_t st) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace

RswaPlan rswa_plan(int B, int Rcap) {
    const int sms = device_sms() > 0 ? device_sms() : 148;
    const int keys = Rcap + RW;
    const int heads = B * RH;
    int S = (2 * sms + heads - 1) / heads;                 // about two CTAs per SM
    S = std::max(1, std::min(S, (keys + 63) / 64));       // at least 64 keys per chunk
    RswaPlan pl;
    pl.chunk = (keys + S - 1) / S;
    pl.S = (keys + pl.chunk - 1) / pl.chunk;
    return pl;
}

size_t rswa_part_bytes(int B, int Rcap) {
    return sizeof(float) * (size_t)B * RH * (size_t)rswa_plan(B, Rcap).S * PART;
}

cudaError_t launch_rswa(const float* q, const float* k_new, const float* v_new, const float* k_ref,
                        const float* v_ref, const int32_t* ref_len, int Rcap, float* k_ring, float* v_ring,
                        const int32_t* n_gen, int B, float* out, float* part, cudaStream_t st) {
    const RswaPlan pl = rswa_plan(B, Rcap);
    RswaParams p;
    p.q = q;
    p.k_new = k_new;
    p.v_new = v_new;
    p.k_ref = k_ref;
    p.v_ref = v_ref;
    p.ref_len = ref_len;
    p.n_gen = n_gen;
    p.k_ring = k_ring;
    p.v_ring = v_ring;
    p.out = out;
    p.part = part;
    p.Rcap = Rcap;
    p.B = B;
    p.S = pl.S;
    p.chunk = pl.chunk;
    void* args[] = {&p};
    cudaError_t e = launch_pdl((const void*)rswa_partial_kernel, dim3(B * RH, pl.S), dim3(PT), args, st);
    if (e != cudaSuccess) return e;
    return launch_pdl((const void*)rswa_combine_kernel, dim3(B * RH), dim3(RD), args, st);
}

}  // namespace focr

// ------------------------------------------------------------------ C ABI
namespace focr {
focr_status report_error(focr_status s, const char* msg);   // the library's focr_last_error() record
}  // namespace focr

extern "C" {

size_t focr_rswa_workspace_bytes(int32_t B, int32_t Rcap) {
    if (B < 1) B = 1;
    if (B > FOCR_RSWA_B_MAX) B = FOCR_RSWA_B_MAX;
    if (Rcap < 1) Rcap = 1;
    if (Rcap > FOCR_RSWA_RCAP_MAX) Rcap = FOCR_RSWA_RCAP_MAX;
    return (focr::rswa_part_bytes(B, Rcap) + 255) & ~(size_t)255;
}

focr_status focr_rswa_decode(const float* q, const float* k_new, const float* v_new, const float* k_ref,
                             const float* v_ref, const int32_t* ref_len, int32_t Rcap, float* k_ring, float* v_ring,
                             const int32_t* n_gen, int32_t B, float* out, void* workspace, size_t ws_bytes,
                             void* stream) {
    using focr::report_error;
    report_error(FOCR_OK, "");
    char msg[160];
    if (!q || !k_new || !v_new || !k_ref || !v_ref || !ref_len || !k_ring || !v_ring || !n_gen || !out || !workspace)
        return report_error(FOCR_ERR_INVALID_ARG, "NULL argument");
    if (B < 1 || B > FOCR_RSWA_B_MAX) {
        snprintf(msg, sizeof(msg), "B=%d outside [1, %d]", B, FOCR_RSWA_B_MAX);
        return report_error(FOCR_ERR_INVALID_ARG, msg);
    }
    if (Rcap < 1 || Rcap > FOCR_RSWA_RCAP_MAX) {
        snprintf(msg, sizeof(msg), "Rcap=%d outside [1, %d]", Rcap, FOCR_RSWA_RCAP_MAX);
        return report_error(FOCR_ERR_INVALID_ARG, msg);
    }
    const void* f[] = {q, k_new, v_new, k_ref, v_ref, k_ring, v_ring, out};
    for (const void* ptr : f)
        if ((uintptr_t)ptr % 16) return report_error(FOCR_ERR_INVALID_ARG, "float buffers must be 16-byte aligned");
    if ((uintptr_t)ref_len % 4 || (uintptr_t)n_gen % 4 || (uintptr_t)workspace % 256)
        return report_error(FOCR_ERR_INVALID_ARG, "misaligned lengths or workspace");
    const size_t need = focr_rswa_workspace_bytes(B, Rcap);
    if (ws_bytes < need) {
        snprintf(msg, sizeof(msg), "workspace of %zu bytes < %zu needed", ws_bytes, need);
        return report_error(FOCR_ERR_INVALID_ARG, msg);
    }
    const cudaError_t e = focr::launch_rswa(q, k_new, v_new, k_ref, v_ref, ref_len, Rcap, k_ring, v_ring, n_gen, B,
                                            out, reinterpret_cast<float*>(workspace), (cudaStream_t)stream);
    if (e != cudaSuccess) {
        snprintf(msg, sizeof(msg), "launch_rswa: %s (%s)", cudaGetErrorName(e), cudaGetErrorString(e));
        return report_error(FOCR_ERR_CUDA, msg);
    }
    return FOCR_OK;
}

}  // extern "C"
