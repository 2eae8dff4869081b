// C ABI of libfocr_moe: argument checks, packing, export, forward.  See include/focr_moe.h.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "common.cuh"
#include "lm_head.h"
#include "pack.h"
#include "w8a8.h"

using namespace focr;

struct focr_moe_layer {
    int32_t routed_type, shared_type, group;
    ItemGeom rg, sg;
    TcGeom rtg, stg;      // tensor-core layout of the routed and shared sets
    uint8_t* dev = nullptr;
    size_t bytes = 0;
    size_t off_router = 0, off_ritems = 0, off_rdsc = 0, off_sitems = 0, off_sdsc = 0;
    size_t off_tc_rgu = 0, off_tc_rdn = 0, off_tc_sgu = 0, off_tc_sdn = 0;
    TcView tc_view() const {
        TcView v{};
        v.r = TcSetView{dev + off_tc_rgu, dev + off_tc_rdn, rtg};
        v.s = TcSetView{dev + off_tc_sgu, dev + off_tc_sdn, stg};
        return v;
    }
    LayerView view() const {
        LayerView v{};
        v.router = reinterpret_cast<const uint16_t*>(dev + off_router);
        v.routed_items = dev + off_ritems;
        v.routed_dscale = reinterpret_cast<const float*>(dev + off_rdsc);
        v.shared_items = dev + off_sitems;
        v.shared_dscale = reinterpret_cast<const float*>(dev + off_sdsc);
        v.rg = rg;
        v.sg = sg;
        return v;
    }
};

namespace {

thread_local std::string g_err;

focr_status fail(focr_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
focr_status fail(focr_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_err = buf;
    return s;
}

focr_status cuda_fail(cudaError_t e, const char* what) {
    return fail(FOCR_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

#define CUDA_TRY(call)                                           \
    do {                                                         \
        cudaError_t e__ = (call);                                \
        if (e__ != cudaSuccess) return cuda_fail(e__, #call);    \
    } while (0)

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

focr_status check_types(int rt, int st, int g) {
    auto ok = [&](int wt) {
        if (wt == FOCR_W_BF16) return true;
        if (wt == FOCR_W_INT4) return g == 32 || g == 64 || g == 128;
        if (wt == FOCR_W_INT8) return g == 128;
        return false;
    };
    if (!ok(rt)) return fail(FOCR_ERR_UNSUPPORTED, "routed weight type %d with group %d is not supported", rt, g);
    if (!ok(st)) return fail(FOCR_ERR_UNSUPPORTED, "shared weight type %d with group %d is not supported", st, g);
    return FOCR_OK;
}

void plan(focr_moe_layer* L) {
    size_t o = 0;
    L->off_router = o;
    o = align_up(o + sizeof(uint16_t) * E * H, 256);
    L->off_ritems = o;
    o = align_up(o + (size_t)E * L->rg.slices * L->rg.item_bytes, 256);
    L->off_rdsc = o;
    o = align_up(o + sizeof(float) * (size_t)E * L->rg.dscale_expert_floats, 256);
    L->off_sitems = o;
    o = align_up(o + (size_t)L->sg.slices * L->sg.item_bytes, 256);
    L->off_sdsc = o;
    o = align_up(o + sizeof(float) * (size_t)L->sg.dscale_expert_floats, 256);
    L->off_tc_rgu = o;
    o = align_up(o + (size_t)E * L->rtg.gu_bytes, 256);
    L->off_tc_rdn = o;
    o = align_up(o + (size_t)E * L->rtg.dn_bytes, 256);
    L->off_tc_sgu = o;
    o = align_up(o + L->stg.gu_bytes, 256);
    L->off_tc_sdn = o;
    o = align_up(o + L->stg.dn_bytes, 256);
    L->bytes = o;
}

}  // namespace

namespace focr {
// Record a message for focr_last_error() from another translation unit of the library.
focr_status report_error(focr_status s, const char* msg) {
    g_err = msg;
    return s;
}
}  // namespace focr

extern "C" {

const char* focr_last_error(void) { return g_err.c_str(); }

const char* focr_version(void) {
    static char buf[128];
    snprintf(buf, sizeof(buf), "focr_moe sm_100a cuda %d.%d", CUDART_VERSION / 1000, (CUDART_VERSION % 1000) / 10);
    return buf;
}

focr_status focr_moe_pack_weights(const focr_moe_weights_desc* d, focr_moe_layer** out, void* stream) {
    g_err.clear();
    if (!d || !out) return fail(FOCR_ERR_INVALID_ARG, "desc and out must not be NULL");
    *out = nullptr;
    if (!d->w_gate || !d->w_up || !d->w_down || !d->ws_gate || !d->ws_up || !d->ws_down || !d->w_router_bf16)
        return fail(FOCR_ERR_INVALID_ARG, "a weight pointer is NULL");
    focr_status s = check_types(d->routed_type, d->shared_type, d->group_size);
    if (s != FOCR_OK) return s;
    focr_moe_layer* L = new (std::nothrow) focr_moe_layer();
    if (!L) return fail(FOCR_ERR_OOM, "host allocation failed");
    L->routed_type = d->routed_type;
    L->shared_type = d->shared_type;
    L->group = d->group_size;
    L->rg = make_geom(d->routed_type, d->group_size, I);
    L->sg = make_geom(d->shared_type, d->group_size, IS);
    L->rtg = make_tc_geom(d->routed_type, d->group_size, I, tc_tile_group(d->routed_type));
    L->stg = make_tc_geom(d->shared_type, d->group_size, IS, 1);
    plan(L);

    std::vector<uint8_t> host;
    try {
        host.assign(L->bytes, 0);
    } catch (...) {
        delete L;
        return fail(FOCR_ERR_OOM, "host staging of %zu bytes failed", L->bytes);
    }
    std::memcpy(host.data() + L->off_router, d->w_router_bf16, sizeof(uint16_t) * E * H);
    const ItemGeom rg = L->rg;
    uint8_t* ritems = host.data() + L->off_ritems;
    float* rdsc = reinterpret_cast<float*>(host.data() + L->off_rdsc);
    uint8_t* hb = host.data();
    parallel_for(E + 1, [&](int e) {
        if (e < E) {
            host_pack_set(d->w_gate + (size_t)e * I * H, d->w_up + (size_t)e * I * H, d->w_down + (size_t)e * H * I,
                          rg, ritems + (size_t)e * rg.slices * rg.item_bytes, rdsc + (size_t)e * rg.dscale_expert_floats,
                          hb + L->off_tc_rgu + (size_t)e * L->rtg.gu_bytes, hb + L->off_tc_rdn + (size_t)e * L->rtg.dn_bytes,
                          L->rtg.grp);
        } else {
            host_pack_set(d->ws_gate, d->ws_up, d->ws_down, L->sg, hb + L->off_sitems,
                          reinterpret_cast<float*>(hb + L->off_sdsc), hb + L->off_tc_sgu, hb + L->off_tc_sdn, L->stg.grp);
        }
    });

    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaMalloc(&L->dev, L->bytes);
    if (e != cudaSuccess) {
        delete L;
        return fail(e == cudaErrorMemoryAllocation ? FOCR_ERR_OOM : FOCR_ERR_CUDA, "cudaMalloc(%zu): %s", L->bytes,
                    cudaGetErrorString(e));
    }
    e = cudaMemcpyAsync(L->dev, host.data(), L->bytes, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) {
        cudaFree(L->dev);
        delete L;
        return cuda_fail(e, "upload of packed layer");
    }
    *out = L;
    return FOCR_OK;
}

focr_status focr_moe_layer_clone(const focr_moe_layer* src, focr_moe_layer** out, void* stream) {
    g_err.clear();
    if (!src || !out) return fail(FOCR_ERR_INVALID_ARG, "src and out must not be NULL");
    *out = nullptr;
    focr_moe_layer* L = new (std::nothrow) focr_moe_layer(*src);
    if (!L) return fail(FOCR_ERR_OOM, "host allocation failed");
    L->dev = nullptr;
    cudaError_t e = cudaMalloc(&L->dev, L->bytes);
    if (e != cudaSuccess) {
        delete L;
        return fail(e == cudaErrorMemoryAllocation ? FOCR_ERR_OOM : FOCR_ERR_CUDA, "cudaMalloc(%zu): %s", src->bytes,
                    cudaGetErrorString(e));
    }
    cudaStream_t st = (cudaStream_t)stream;
    e = cudaMemcpyAsync(L->dev, src->dev, L->bytes, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) {
        cudaFree(L->dev);
        delete L;
        return cuda_fail(e, "clone copy");
    }
    *out = L;
    return FOCR_OK;
}

void focr_moe_layer_free(focr_moe_layer* L) {
    if (!L) return;
    if (L->dev) cudaFree(L->dev);
    delete L;
}

size_t focr_moe_layer_device_bytes(const focr_moe_layer* L) { return L ? L->bytes : 0; }

static bool matrix_shape(const focr_moe_layer* L, int32_t m, int* wtype, int64_t* rows, int64_t* cols, int* group) {
    switch (m) {
        case FOCR_MAT_GATE: case FOCR_MAT_UP:
            *wtype = L->routed_type; *rows = I; *cols = H; break;
        case FOCR_MAT_DOWN:
            *wtype = L->routed_type; *rows = H; *cols = I; break;
        case FOCR_MAT_SHARED_GATE: case FOCR_MAT_SHARED_UP:
            *wtype = L->shared_type; *rows = IS; *cols = H; break;
        case FOCR_MAT_SHARED_DOWN:
            *wtype = L->shared_type; *rows = H; *cols = IS; break;
        case FOCR_MAT_ROUTER:
            *wtype = FOCR_W_BF16; *rows = E; *cols = H; break;
        default:
            return false;
    }
    *group = is_quant(*wtype) ? L->group : 0;
    return true;
}

focr_status focr_moe_export_sizes(const focr_moe_layer* L, int32_t matrix, size_t* code_bytes, size_t* n_scales) {
    g_err.clear();
    if (!L || !code_bytes || !n_scales) return fail(FOCR_ERR_INVALID_ARG, "NULL argument");
    int wt, g;
    int64_t rows, cols;
    if (!matrix_shape(L, matrix, &wt, &rows, &cols, &g)) return fail(FOCR_ERR_INVALID_ARG, "unknown matrix %d", matrix);
    const size_t n = (size_t)(rows * cols);
    *code_bytes = wt == FOCR_W_INT4 ? n / 2 : (wt == FOCR_W_INT8 ? n : 2 * n);
    *n_scales = is_quant(wt) ? (size_t)rows * (size_t)((cols + g - 1) / g) : 0;
    return FOCR_OK;
}

focr_status focr_moe_export_quantized(const focr_moe_layer* L, int32_t matrix, int32_t expert, void* codes,
                                      size_t code_bytes, float* scales, size_t n_scales) {
    size_t need_c, need_s;
    focr_status s = focr_moe_export_sizes(L, matrix, &need_c, &need_s);
    if (s != FOCR_OK) return s;
    const bool routed = matrix <= FOCR_MAT_DOWN;
    if (routed && (expert < 0 || expert >= E)) return fail(FOCR_ERR_INVALID_ARG, "expert %d out of range", expert);
    if (!codes || code_bytes < need_c) return fail(FOCR_ERR_INVALID_ARG, "codes buffer too small (need %zu)", need_c);
    if (need_s && (!scales || n_scales < need_s))
        return fail(FOCR_ERR_INVALID_ARG, "scales buffer too small (need %zu)", need_s);
    if (matrix == FOCR_MAT_ROUTER) {
        CUDA_TRY(cudaMemcpy(codes, L->dev + L->off_router, need_c, cudaMemcpyDeviceToHost));
        return FOCR_OK;
    }
    const ItemGeom& g = routed ? L->rg : L->sg;
    const size_t items_bytes = (size_t)g.slices * g.item_bytes;
    const size_t item_off = routed ? L->off_ritems + (size_t)expert * items_bytes : L->off_sitems;
    const size_t dsc_off = routed ? L->off_rdsc + sizeof(float) * (size_t)expert * g.dscale_expert_floats : L->off_sdsc;
    std::vector<uint8_t> items(items_bytes);
    std::vector<float> dsc(g.dscale_expert_floats);
    CUDA_TRY(cudaMemcpy(items.data(), L->dev + item_off, items_bytes, cudaMemcpyDeviceToHost));
    if (!dsc.empty())
        CUDA_TRY(cudaMemcpy(dsc.data(), L->dev + dsc_off, dsc.size() * sizeof(float), cudaMemcpyDeviceToHost));
    const int which = (matrix == FOCR_MAT_GATE || matrix == FOCR_MAT_SHARED_GATE) ? 0
                      : (matrix == FOCR_MAT_UP || matrix == FOCR_MAT_SHARED_UP) ? 1 : 2;
    int wt, grp;
    int64_t rows, cols;
    matrix_shape(L, matrix, &wt, &rows, &cols, &grp);
    const size_t n = (size_t)(rows * cols);
    if (wt == FOCR_W_BF16) {
        host_unpack_matrix(items.data(), nullptr, g, which, nullptr, reinterpret_cast<uint16_t*>(codes), nullptr);
    } else {
        std::vector<int8_t> q(n);
        host_unpack_matrix(items.data(), dsc.data(), g, which, q.data(), nullptr, scales);
        if (wt == FOCR_W_INT8) {
            std::memcpy(codes, q.data(), n);
        } else {
            uint8_t* c = reinterpret_cast<uint8_t*>(codes);
            for (size_t j = 0; j < n / 2; ++j)
                c[j] = (uint8_t)(((uint8_t)q[2 * j] & 0xFu) | (((uint8_t)q[2 * j + 1] & 0xFu) << 4));
        }
    }
    return FOCR_OK;
}

size_t focr_moe_workspace_bytes(int32_t T_max) {
    if (T_max < 1) T_max = 1;
    if (T_max > FOCR_T_MAX) T_max = FOCR_T_MAX;
    // sized for both the MoE layer and the dense layer (whose shared-set regions are larger)
    const size_t a = ws_layout(T_max, IS).total, b = ws_layout(T_max, IS_MAX).total;
    return a > b ? a : b;
}

size_t focr_moe_workspace_zero_bytes(void) { return ws_layout(1).gpart; }

focr_status focr_moe_layer_forward_ex(const focr_moe_layer* L, const float* hidden, int32_t T, float* out,
                                      void* workspace, size_t ws_bytes, const focr_moe_route_debug* dbg, int32_t flags,
                                      void* stream) {
    g_err.clear();
    if (!L || !L->dev) return fail(FOCR_ERR_INVALID_ARG, "layer is NULL");
    if (flags & ~(FOCR_FWD_RESIDUAL | FOCR_FWD_DETERMINISTIC)) return fail(FOCR_ERR_INVALID_ARG, "unknown flags 0x%x", (unsigned)flags);
    if (T < 1 || T > FOCR_T_MAX) return fail(FOCR_ERR_INVALID_ARG, "T=%d outside [1, %d]", T, FOCR_T_MAX);
    if (!hidden || !out || !workspace) return fail(FOCR_ERR_INVALID_ARG, "hidden, out and workspace must not be NULL");
    if (!aligned(hidden, 16) || !aligned(out, 16)) return fail(FOCR_ERR_INVALID_ARG, "hidden/out must be 16-byte aligned");
    if (!aligned(workspace, 256)) return fail(FOCR_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    const size_t need = ws_layout(T, IS).total;
    if (ws_bytes < need) return fail(FOCR_ERR_INVALID_ARG, "workspace of %zu bytes < %zu needed for T=%d", ws_bytes, need, T);
    {
        const char* h0 = (const char*)hidden;
        const char* o0 = (const char*)out;
        const size_t nb = (size_t)T * H * sizeof(float);
        if (h0 < o0 + nb && o0 < h0 + nb) return fail(FOCR_ERR_INVALID_ARG, "hidden and out overlap");
    }
    cudaStream_t st = (cudaStream_t)stream;
    const RouteView R = route_view(workspace, T, IS);
    const LayerView V = L->view();
    const bool resid = (flags & FOCR_FWD_RESIDUAL) != 0;
    if (T <= SMALL_T) {
        CUDA_TRY(launch_router(hidden, T, T, V, R, out, resid ? hidden : nullptr, nullptr, 0, st));
        CUDA_TRY(launch_decode_small(hidden, T, V, R, out, false, (flags & FOCR_FWD_DETERMINISTIC) != 0, st));
    } else if (T <= MID_T) {
        CUDA_TRY(launch_router(hidden, T, T, V, R, out, resid ? hidden : nullptr, nullptr, 0, st));
        CUDA_TRY(launch_expert_decode(hidden, T, V, R, out, false, st));
    } else {
        const TcWork W = tc_work(workspace, T, IS);
        CUDA_TRY(launch_router(hidden, T, T, V, R, nullptr, nullptr, W.x_img, W.tpad, st));
        CUDA_TRY(launch_expert_tc(hidden, T, L->tc_view(), R, W, out, resid, false, st));
    }
    if (dbg) {
        if (dbg->logits) CUDA_TRY(cudaMemcpyAsync(dbg->logits, R.logits, sizeof(float) * T * E, cudaMemcpyDeviceToDevice, st));
        if (dbg->topk_idx) CUDA_TRY(cudaMemcpyAsync(dbg->topk_idx, R.topk_idx, sizeof(int32_t) * T * K, cudaMemcpyDeviceToDevice, st));
        if (dbg->topk_w) CUDA_TRY(cudaMemcpyAsync(dbg->topk_w, R.topk_w, sizeof(float) * T * K, cudaMemcpyDeviceToDevice, st));
        if (dbg->counts) CUDA_TRY(cudaMemcpyAsync(dbg->counts, R.counts, sizeof(int32_t) * E, cudaMemcpyDeviceToDevice, st));
        if (dbg->offsets) CUDA_TRY(cudaMemcpyAsync(dbg->offsets, R.offsets, sizeof(int32_t) * (E + 1), cudaMemcpyDeviceToDevice, st));
        if (dbg->perm) CUDA_TRY(cudaMemcpyAsync(dbg->perm, R.perm, sizeof(int32_t) * T * K, cudaMemcpyDeviceToDevice, st));
    }
    return FOCR_OK;
}

// ------------------------------------------------------------------ lm_head + RMSNorm

struct focr_lm_head {
    uint8_t* dev = nullptr;   // codes (V * H bytes) then scales (V floats)
    size_t bytes = 0;
};

focr_status focr_lm_head_pack(const float* w, focr_lm_head** out, void* stream) {
    g_err.clear();
    if (!w || !out) return fail(FOCR_ERR_INVALID_ARG, "w and out must not be NULL");
    *out = nullptr;
    const size_t code_bytes = (size_t)FOCR_VOCAB * H, bytes = code_bytes + sizeof(float) * FOCR_VOCAB;
    std::vector<uint8_t> host;
    try {
        host.resize(bytes);
    } catch (...) {
        return fail(FOCR_ERR_OOM, "host staging of %zu bytes failed", bytes);
    }
    host_pack_lm_head(w, FOCR_VOCAB, host.data(), reinterpret_cast<float*>(host.data() + code_bytes));
    focr_lm_head* L = new (std::nothrow) focr_lm_head();
    if (!L) return fail(FOCR_ERR_OOM, "host allocation failed");
    cudaError_t e = cudaMalloc(&L->dev, bytes);
    if (e != cudaSuccess) {
        delete L;
        return fail(e == cudaErrorMemoryAllocation ? FOCR_ERR_OOM : FOCR_ERR_CUDA, "cudaMalloc(%zu): %s", bytes,
                    cudaGetErrorString(e));
    }
    L->bytes = bytes;
    cudaStream_t st = (cudaStream_t)stream;
    e = cudaMemcpyAsync(L->dev, host.data(), bytes, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) {
        cudaFree(L->dev);
        delete L;
        return cuda_fail(e, "upload of packed lm_head");
    }
    *out = L;
    return FOCR_OK;
}

void focr_lm_head_free(focr_lm_head* L) {
    if (!L) return;
    if (L->dev) cudaFree(L->dev);
    delete L;
}

focr_status focr_lm_head_export(const focr_lm_head* L, int8_t* codes, float* scales) {
    g_err.clear();
    if (!L || !codes || !scales) return fail(FOCR_ERR_INVALID_ARG, "NULL argument");
    const size_t code_bytes = (size_t)FOCR_VOCAB * H;
    std::vector<uint8_t> host(code_bytes);
    CUDA_TRY(cudaMemcpy(host.data(), L->dev, code_bytes, cudaMemcpyDeviceToHost));
    CUDA_TRY(cudaMemcpy(scales, L->dev + code_bytes, sizeof(float) * FOCR_VOCAB, cudaMemcpyDeviceToHost));
    host_unpack_lm_head(host.data(), FOCR_VOCAB, codes);
    return FOCR_OK;
}

size_t focr_lm_head_workspace_bytes(int32_t T_max) {
    if (T_max < 1) T_max = 1;
    if (T_max > FOCR_T_MAX) T_max = FOCR_T_MAX;
    int grid = 1024;   // upper bound on the CTAs of one launch (one per SM)
    return align_up(256 + sizeof(unsigned long long) * (size_t)grid * T_max, 256);
}

focr_status focr_lm_head_gemv(const focr_lm_head* L, const float* x, int32_t T, float* logits, int32_t* argmax,
                              void* workspace, size_t ws_bytes, void* stream) {
    g_err.clear();
    if (!L || !L->dev) return fail(FOCR_ERR_INVALID_ARG, "lm_head is NULL");
    if (T < 1 || T > FOCR_T_MAX) return fail(FOCR_ERR_INVALID_ARG, "T=%d outside [1, %d]", T, FOCR_T_MAX);
    if (!x || !argmax || !workspace) return fail(FOCR_ERR_INVALID_ARG, "x, argmax and workspace must not be NULL");
    if (!aligned(x, 16) || !aligned(workspace, 256)) return fail(FOCR_ERR_INVALID_ARG, "misaligned x or workspace");
    if (ws_bytes < focr_lm_head_workspace_bytes(T))
        return fail(FOCR_ERR_INVALID_ARG, "workspace of %zu bytes < %zu needed", ws_bytes, focr_lm_head_workspace_bytes(T));
    const int grid = lm_head_grid();
    if (grid > 1024) return fail(FOCR_ERR_UNSUPPORTED, "%d SMs exceed the workspace plan", grid);
    const uint4* codes = reinterpret_cast<const uint4*>(L->dev);
    const float* scales = reinterpret_cast<const float*>(L->dev + (size_t)FOCR_VOCAB * H);
    CUDA_TRY(launch_lm_head(codes, scales, x, T, logits, argmax, workspace, (cudaStream_t)stream));
    return FOCR_OK;
}

// ------------------------------------------------------------------ W8A8 linear

struct focr_w8a8 {
    uint8_t* dev = nullptr;   // codes (tiles * KS * 512 bytes) then scales (16 * tiles floats)
    int64_t N = 0;
    int32_t K = 0;
    int64_t tiles = 0;
    int64_t KS = 0;
    size_t code_bytes = 0;
};

namespace {

// workspace: [err word, 256 B][cnt: tiles u32][sx: FOCR_W8A8_T_MAX f32][qx fragments: KS x 8 groups x 256 B]
// [acc: T x 16 tiles i32]; every offset is independent of T, so calls with different T can share one workspace
struct W8a8Ws {
    size_t err = 0, cnt = 256, sx = 0, qxf = 0, acc = 0;
};

W8a8Ws w8a8_ws(const focr_w8a8* m) {
    W8a8Ws o;
    o.sx = align_up(o.cnt + sizeof(uint32_t) * (size_t)m->tiles, 256);
    o.qxf = align_up(o.sx + sizeof(float) * FOCR_W8A8_T_MAX, 256);
    o.acc = align_up(o.qxf + (size_t)m->KS * 256 * (FOCR_W8A8_T_MAX / 8), 256);
    return o;
}

}  // namespace

focr_status focr_w8a8_pack(const float* w, int64_t N, int32_t K, focr_w8a8** out, void* stream) {
    g_err.clear();
    if (!w || !out) return fail(FOCR_ERR_INVALID_ARG, "w and out must not be NULL");
    *out = nullptr;
    if (N < 1 || N > FOCR_W8A8_N_MAX) return fail(FOCR_ERR_INVALID_ARG, "N=%lld outside [1, %d]", (long long)N, FOCR_W8A8_N_MAX);
    if (K < 1 || K > FOCR_W8A8_K_MAX) return fail(FOCR_ERR_INVALID_ARG, "K=%d outside [1, %d]", K, FOCR_W8A8_K_MAX);
    const int64_t tiles = (N + 15) / 16, KS = ((int64_t)K + 31) / 32;
    const size_t code_bytes = (size_t)(tiles * KS * 512), bytes = code_bytes + sizeof(float) * (size_t)(16 * tiles);
    std::vector<uint8_t> host;
    try {
        host.resize(bytes);
    } catch (...) {
        return fail(FOCR_ERR_OOM, "host staging of %zu bytes failed", bytes);
    }
    host_pack_w8a8(w, N, K, host.data(), reinterpret_cast<float*>(host.data() + code_bytes));
    focr_w8a8* M = new (std::nothrow) focr_w8a8();
    if (!M) return fail(FOCR_ERR_OOM, "host allocation failed");
    M->N = N;
    M->K = K;
    M->tiles = tiles;
    M->KS = KS;
    M->code_bytes = code_bytes;
    cudaError_t e = cudaMalloc(&M->dev, bytes);
    if (e != cudaSuccess) {
        delete M;
        return fail(e == cudaErrorMemoryAllocation ? FOCR_ERR_OOM : FOCR_ERR_CUDA, "cudaMalloc(%zu): %s", bytes,
                    cudaGetErrorString(e));
    }
    cudaStream_t st = (cudaStream_t)stream;
    e = cudaMemcpyAsync(M->dev, host.data(), bytes, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) {
        cudaFree(M->dev);
        delete M;
        return cuda_fail(e, "upload of packed W8A8 matrix");
    }
    *out = M;
    return FOCR_OK;
}

void focr_w8a8_free(focr_w8a8* M) {
    if (!M) return;
    if (M->dev) cudaFree(M->dev);
    delete M;
}

focr_status focr_w8a8_export(const focr_w8a8* M, int8_t* codes, float* scales, int64_t* N, int32_t* K) {
    g_err.clear();
    if (!M || !M->dev) return fail(FOCR_ERR_INVALID_ARG, "matrix is NULL");
    if (N) *N = M->N;
    if (K) *K = M->K;
    if (!codes && !scales) return FOCR_OK;
    if (!codes || !scales) return fail(FOCR_ERR_INVALID_ARG, "codes and scales must both be given");
    std::vector<uint8_t> host(M->code_bytes);
    CUDA_TRY(cudaMemcpy(host.data(), M->dev, M->code_bytes, cudaMemcpyDeviceToHost));
    CUDA_TRY(cudaMemcpy(scales, M->dev + M->code_bytes, sizeof(float) * (size_t)M->N, cudaMemcpyDeviceToHost));
    host_unpack_w8a8(host.data(), M->N, M->K, codes);
    return FOCR_OK;
}

focr_status focr_w8a8_quantize_x(const float* x, int32_t T, int32_t K, int8_t* qx, float* sx, void* stream) {
    g_err.clear();
    if (!x || !qx || !sx) return fail(FOCR_ERR_INVALID_ARG, "x, qx and sx must not be NULL");
    if (T < 1 || T > FOCR_T_MAX) return fail(FOCR_ERR_INVALID_ARG, "T=%d outside [1, %d]", T, FOCR_T_MAX);
    if (K < 1 || K > FOCR_W8A8_K_MAX) return fail(FOCR_ERR_INVALID_ARG, "K=%d outside [1, %d]", K, FOCR_W8A8_K_MAX);
    if (!aligned(x, 4) || !aligned(sx, 4)) return fail(FOCR_ERR_INVALID_ARG, "x and sx must be 4-byte aligned");
    CUDA_TRY(launch_w8a8_quantize(x, T, K, qx, nullptr, sx, (cudaStream_t)stream));
    return FOCR_OK;
}

size_t focr_w8a8_workspace_bytes(const focr_w8a8* M, int32_t T_max) {
    if (!M) return 0;
    if (T_max < 1) T_max = 1;
    if (T_max > FOCR_W8A8_T_MAX) T_max = FOCR_W8A8_T_MAX;
    const W8a8Ws o = w8a8_ws(M);
    const W8a8Plan pl = w8a8_plan(M->tiles, (int)M->KS);
    const size_t acc = pl.S > 1 ? sizeof(int32_t) * (size_t)T_max * (size_t)(16 * M->tiles) : 0;
    return align_up(o.acc + acc, 256);
}

focr_status focr_w8a8_gemv(const focr_w8a8* M, const float* x, int32_t T, float* y, void* workspace,
                           size_t ws_bytes, void* stream) {
    g_err.clear();
    if (!M || !M->dev) return fail(FOCR_ERR_INVALID_ARG, "matrix is NULL");
    if (!x || !y || !workspace) return fail(FOCR_ERR_INVALID_ARG, "x, y and workspace must not be NULL");
    if (T < 1 || T > FOCR_W8A8_T_MAX) return fail(FOCR_ERR_INVALID_ARG, "T=%d outside [1, %d]", T, FOCR_W8A8_T_MAX);
    if (!aligned(x, 4) || !aligned(y, 4) || !aligned(workspace, 256))
        return fail(FOCR_ERR_INVALID_ARG, "misaligned x, y or workspace");
    const size_t need = focr_w8a8_workspace_bytes(M, T);
    if (ws_bytes < need) return fail(FOCR_ERR_INVALID_ARG, "workspace of %zu bytes < %zu needed", ws_bytes, need);
    const W8a8Ws o = w8a8_ws(M);
    char* ws = reinterpret_cast<char*>(workspace);
    uint32_t* cnt = reinterpret_cast<uint32_t*>(ws + o.cnt);
    float* sx = reinterpret_cast<float*>(ws + o.sx);
    uint32_t* qxf = reinterpret_cast<uint32_t*>(ws + o.qxf);
    int32_t* acc = reinterpret_cast<int32_t*>(ws + o.acc);
    uint32_t* err = reinterpret_cast<uint32_t*>(ws + o.err);
    cudaStream_t st = (cudaStream_t)stream;
    CUDA_TRY(launch_w8a8_quantize(x, T, M->K, nullptr, qxf, sx, st));
    const float* sw = reinterpret_cast<const float*>(M->dev + M->code_bytes);
    CUDA_TRY(launch_w8a8_gemv(M->dev, sw, M->N, M->K, qxf, sx, T, y, acc, cnt, err, st));
    return FOCR_OK;
}

focr_status focr_w8a8_check(void* workspace, void* stream) {
    g_err.clear();
    if (!workspace || !aligned(workspace, 256)) return fail(FOCR_ERR_INVALID_ARG, "workspace is NULL or misaligned");
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t word = 0;
    CUDA_TRY(cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st));
    CUDA_TRY(cudaStreamSynchronize(st));
    if (!word) return FOCR_OK;
    CUDA_TRY(cudaMemsetAsync(workspace, 0, sizeof(word), st));
    CUDA_TRY(cudaStreamSynchronize(st));
    return fail(FOCR_ERR_TIMEOUT, "a bounded wait of the W8A8 GEMV ran out; the outputs of that call are not valid");
}

focr_status focr_lm_head_check(void* workspace, void* stream) {
    g_err.clear();
    if (!workspace || !aligned(workspace, 256)) return fail(FOCR_ERR_INVALID_ARG, "workspace is NULL or misaligned");
    cudaStream_t st = (cudaStream_t)stream;
    int32_t* word = reinterpret_cast<int32_t*>(workspace) + 1;
    int32_t v = 0;
    CUDA_TRY(cudaMemcpyAsync(&v, word, sizeof(v), cudaMemcpyDeviceToHost, st));
    CUDA_TRY(cudaStreamSynchronize(st));
    if (!v) return FOCR_OK;
    CUDA_TRY(cudaMemsetAsync(word, 0, sizeof(v), st));
    CUDA_TRY(cudaStreamSynchronize(st));
    return fail(FOCR_ERR_TIMEOUT, "a bounded wait of the lm_head GEMV ran out; the outputs of that call are not valid");
}

focr_status focr_rmsnorm(const float* x, const float* gamma, int32_t T, float eps, float* out, void* stream) {
    g_err.clear();
    if (T < 1 || T > FOCR_T_MAX) return fail(FOCR_ERR_INVALID_ARG, "T=%d outside [1, %d]", T, FOCR_T_MAX);
    if (!x || !out) return fail(FOCR_ERR_INVALID_ARG, "x and out must not be NULL");
    if (!aligned(x, 16) || !aligned(out, 16) || (gamma && !aligned(gamma, 16)))
        return fail(FOCR_ERR_INVALID_ARG, "x, out and gamma must be 16-byte aligned");
    if (!(eps >= 0.f)) return fail(FOCR_ERR_INVALID_ARG, "eps must be >= 0");
    CUDA_TRY(launch_rmsnorm(x, gamma, T, eps, out, (cudaStream_t)stream));
    return FOCR_OK;
}

focr_status focr_moe_layer_forward(const focr_moe_layer* L, const float* hidden, int32_t T, float* out,
                                   void* workspace, size_t ws_bytes, const focr_moe_route_debug* dbg, void* stream) {
    return focr_moe_layer_forward_ex(L, hidden, T, out, workspace, ws_bytes, dbg, 0, stream);
}

// ------------------------------------------------------------------ dense SwiGLU MLP (layer 0)

struct focr_dense_mlp {
    int32_t wtype, group;
    ItemGeom g;
    TcGeom tg;
    uint8_t* dev = nullptr;
    size_t bytes = 0, off_items = 0, off_dsc = 0, off_tc_gu = 0, off_tc_dn = 0;
};

focr_status focr_dense_mlp_pack(const float* w_gate, const float* w_up, const float* w_down, int32_t wtype,
                                int32_t group, focr_dense_mlp** out, void* stream) {
    g_err.clear();
    if (!w_gate || !w_up || !w_down || !out) return fail(FOCR_ERR_INVALID_ARG, "NULL argument");
    *out = nullptr;
    focr_status s = check_types(wtype, wtype, group);
    if (s != FOCR_OK) return s;
    focr_dense_mlp* M = new (std::nothrow) focr_dense_mlp();
    if (!M) return fail(FOCR_ERR_OOM, "host allocation failed");
    M->wtype = wtype;
    M->group = is_quant(wtype) ? group : 0;
    M->g = make_geom(wtype, group, FOCR_DENSE_INTER);
    M->tg = make_tc_geom(wtype, group, FOCR_DENSE_INTER, 1);
    M->off_items = 0;
    M->off_dsc = align_up((size_t)M->g.slices * M->g.item_bytes, 256);
    M->off_tc_gu = align_up(M->off_dsc + sizeof(float) * (size_t)M->g.dscale_expert_floats, 256);
    M->off_tc_dn = align_up(M->off_tc_gu + M->tg.gu_bytes, 256);
    M->bytes = align_up(M->off_tc_dn + M->tg.dn_bytes, 256);
    std::vector<uint8_t> host;
    try {
        host.assign(M->bytes, 0);
    } catch (...) {
        delete M;
        return fail(FOCR_ERR_OOM, "host staging of %zu bytes failed", M->bytes);
    }
    host_pack_set(w_gate, w_up, w_down, M->g, host.data(), reinterpret_cast<float*>(host.data() + M->off_dsc),
                  host.data() + M->off_tc_gu, host.data() + M->off_tc_dn, M->tg.grp);
    cudaError_t e = cudaMalloc(&M->dev, M->bytes);
    if (e != cudaSuccess) {
        delete M;
        return fail(e == cudaErrorMemoryAllocation ? FOCR_ERR_OOM : FOCR_ERR_CUDA, "cudaMalloc(%zu): %s", M->bytes,
                    cudaGetErrorString(e));
    }
    cudaStream_t st = (cudaStream_t)stream;
    e = cudaMemcpyAsync(M->dev, host.data(), M->bytes, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) {
        cudaFree(M->dev);
        delete M;
        return cuda_fail(e, "upload of packed dense MLP");
    }
    *out = M;
    return FOCR_OK;
}

void focr_dense_mlp_free(focr_dense_mlp* M) {
    if (!M) return;
    if (M->dev) cudaFree(M->dev);
    delete M;
}

focr_status focr_dense_mlp_export_quantized(const focr_dense_mlp* M, int32_t matrix, void* codes, size_t code_bytes,
                                            float* scales, size_t n_scales) {
    g_err.clear();
    if (!M || !codes) return fail(FOCR_ERR_INVALID_ARG, "NULL argument");
    if (matrix < 0 || matrix > 2) return fail(FOCR_ERR_INVALID_ARG, "unknown matrix %d", matrix);
    const int64_t rows = matrix < 2 ? FOCR_DENSE_INTER : H, cols = matrix < 2 ? H : FOCR_DENSE_INTER;
    const size_t n = (size_t)(rows * cols);
    const int wt = M->wtype;
    const size_t need_c = wt == FOCR_W_INT4 ? n / 2 : (wt == FOCR_W_INT8 ? n : 2 * n);
    const size_t need_s = is_quant(wt) ? (size_t)rows * (size_t)((cols + M->group - 1) / M->group) : 0;
    if (code_bytes < need_c) return fail(FOCR_ERR_INVALID_ARG, "codes buffer too small (need %zu)", need_c);
    if (need_s && (!scales || n_scales < need_s))
        return fail(FOCR_ERR_INVALID_ARG, "scales buffer too small (need %zu)", need_s);
    std::vector<uint8_t> items((size_t)M->g.slices * M->g.item_bytes);
    std::vector<float> dsc(M->g.dscale_expert_floats);
    CUDA_TRY(cudaMemcpy(items.data(), M->dev + M->off_items, items.size(), cudaMemcpyDeviceToHost));
    if (!dsc.empty())
        CUDA_TRY(cudaMemcpy(dsc.data(), M->dev + M->off_dsc, dsc.size() * sizeof(float), cudaMemcpyDeviceToHost));
    if (wt == FOCR_W_BF16) {
        host_unpack_matrix(items.data(), nullptr, M->g, matrix, nullptr, reinterpret_cast<uint16_t*>(codes), nullptr);
    } else {
        std::vector<int8_t> q(n);
        host_unpack_matrix(items.data(), dsc.data(), M->g, matrix, q.data(), nullptr, scales);
        if (wt == FOCR_W_INT8) {
            std::memcpy(codes, q.data(), n);
        } else {
            uint8_t* c = reinterpret_cast<uint8_t*>(codes);
            for (size_t j = 0; j < n / 2; ++j)
                c[j] = (uint8_t)(((uint8_t)q[2 * j] & 0xFu) | (((uint8_t)q[2 * j + 1] & 0xFu) << 4));
        }
    }
    return FOCR_OK;
}

focr_status focr_dense_mlp_forward(const focr_dense_mlp* M, const float* x, int32_t T, float* out, void* workspace,
                                   size_t ws_bytes, int32_t flags, void* stream) {
    g_err.clear();
    if (!M || !M->dev) return fail(FOCR_ERR_INVALID_ARG, "dense MLP is NULL");
    if (flags & ~(FOCR_FWD_RESIDUAL | FOCR_FWD_DETERMINISTIC)) return fail(FOCR_ERR_INVALID_ARG, "unknown flags 0x%x", (unsigned)flags);
    if (T < 1 || T > FOCR_T_MAX) return fail(FOCR_ERR_INVALID_ARG, "T=%d outside [1, %d]", T, FOCR_T_MAX);
    if (!x || !out || !workspace) return fail(FOCR_ERR_INVALID_ARG, "x, out and workspace must not be NULL");
    if (!aligned(x, 16) || !aligned(out, 16) || !aligned(workspace, 256))
        return fail(FOCR_ERR_INVALID_ARG, "misaligned x, out or workspace");
    if (ws_bytes < ws_layout(T, IS_MAX).total)
        return fail(FOCR_ERR_INVALID_ARG, "workspace of %zu bytes < %zu needed", ws_bytes, ws_layout(T, IS_MAX).total);
    const size_t nb = (size_t)T * H * sizeof(float);
    {
        const char* a = (const char*)x;
        const char* b = (const char*)out;
        if (a < b + nb && b < a + nb) return fail(FOCR_ERR_INVALID_ARG, "x and out overlap");
    }
    cudaStream_t st = (cudaStream_t)stream;
    if (T <= SMALL_T) {
        if (flags & FOCR_FWD_RESIDUAL) CUDA_TRY(cudaMemcpyAsync(out, x, nb, cudaMemcpyDeviceToDevice, st));
        else CUDA_TRY(cudaMemsetAsync(out, 0, nb, st));
        LayerView v{};
        v.shared_items = M->dev + M->off_items;
        v.shared_dscale = reinterpret_cast<const float*>(M->dev + M->off_dsc);
        v.routed_items = v.shared_items;
        v.routed_dscale = v.shared_dscale;
        v.rg = M->g;
        v.sg = M->g;
        CUDA_TRY(launch_decode_small(x, T, v, route_view(workspace, T, IS_MAX), out, true,
                                     (flags & FOCR_FWD_DETERMINISTIC) != 0, st));
    } else {
        TcView v{};
        v.s = TcSetView{M->dev + M->off_tc_gu, M->dev + M->off_tc_dn, M->tg};
        v.r = v.s;
        CUDA_TRY(launch_expert_tc(x, T, v, route_view(workspace, T, IS_MAX), tc_work(workspace, T, IS_MAX), out,
                                  (flags & FOCR_FWD_RESIDUAL) != 0, true, st));
    }
    return FOCR_OK;
}

focr_status focr_moe_check(void* workspace, void* stream) {
    g_err.clear();
    if (!workspace) return fail(FOCR_ERR_INVALID_ARG, "workspace is NULL");
    cudaStream_t st = (cudaStream_t)stream;
    int32_t* ctrl = reinterpret_cast<int32_t*>((char*)workspace + ws_layout(1).ctrl);
    int32_t v = 0;
    CUDA_TRY(cudaMemcpyAsync(&v, ctrl + CTRL_ERROR, sizeof(v), cudaMemcpyDeviceToHost, st));
    CUDA_TRY(cudaStreamSynchronize(st));
    if (v != 0) {
        const int32_t zero = 0;
        CUDA_TRY(cudaMemcpyAsync(ctrl + CTRL_ERROR, &zero, sizeof(zero), cudaMemcpyHostToDevice, st));
        CUDA_TRY(cudaStreamSynchronize(st));
        if (v == DEVERR_RANGE)
            return fail(FOCR_ERR_RANGE, "activations beyond the f16 operand range (|v| > 65504) met by a forward");
        return fail(FOCR_ERR_TIMEOUT, "device wait ran out (code %d)", v);
    }
    return FOCR_OK;
}

// ------------------------------------------------------------------ decode step
// Workspace of one decode step: [lm_head ticket | MoE/dense workspace | lm_head keys | h0 | h1].
// The ticket and the MoE workspace's zero prefix sit at offsets that do not depend on T, so
// calls with different T may share one workspace.
namespace {
constexpr size_t kStepMoeOff = 256;
size_t step_keys_off(int T) { return align_up(kStepMoeOff + focr_moe_workspace_bytes(T), 256); }
size_t step_h0_off(int T) {
    return align_up(step_keys_off(T) + sizeof(unsigned long long) * 1024 * (size_t)T, 256);
}
size_t step_h1_off(int T) { return align_up(step_h0_off(T) + sizeof(float) * H * (size_t)T, 256); }
size_t step_bytes(int T) { return align_up(step_h1_off(T) + sizeof(float) * H * (size_t)T, 256); }
}  // namespace

size_t focr_decode_step_workspace_bytes(int32_t T_max) {
    if (T_max < 1) T_max = 1;
    if (T_max > FOCR_T_MAX) T_max = FOCR_T_MAX;
    return step_bytes(T_max);
}

focr_status focr_decode_step(const focr_decode_model* m, const float* x, int32_t T, float* logits, int32_t* argmax,
                             float* hidden_out, void* workspace, size_t ws_bytes, void* stream) {
    g_err.clear();
    if (!m || !m->dense || !m->head || m->n_moe < 0 || (m->n_moe > 0 && !m->moe))
        return fail(FOCR_ERR_INVALID_ARG, "incomplete decode model");
    for (int i = 0; i < m->n_moe; ++i)
        if (!m->moe[i]) return fail(FOCR_ERR_INVALID_ARG, "MoE layer %d is NULL", i);
    if (!(m->eps >= 0.f)) return fail(FOCR_ERR_INVALID_ARG, "eps must be >= 0");
    if (T < 1 || T > FOCR_T_MAX) return fail(FOCR_ERR_INVALID_ARG, "T=%d outside [1, %d]", T, FOCR_T_MAX);
    if (!x || !argmax || !workspace) return fail(FOCR_ERR_INVALID_ARG, "x, argmax and workspace must not be NULL");
    if (!aligned(x, 16) || !aligned(workspace, 256) || (hidden_out && !aligned(hidden_out, 16)))
        return fail(FOCR_ERR_INVALID_ARG, "misaligned x, hidden_out or workspace");
    if (ws_bytes < step_bytes(T))
        return fail(FOCR_ERR_INVALID_ARG, "workspace of %zu bytes < %zu needed for T=%d", ws_bytes, step_bytes(T), T);
    if (lm_head_grid() > 1024) return fail(FOCR_ERR_UNSUPPORTED, "more SMs than the workspace plan");
    char* w = static_cast<char*>(workspace);
    void* mws = w + kStepMoeOff;
    const size_t mws_bytes = focr_moe_workspace_bytes(T);
    float* h0 = reinterpret_cast<float*>(w + step_h0_off(T));
    float* h1 = reinterpret_cast<float*>(w + step_h1_off(T));
    cudaStream_t st = (cudaStream_t)stream;
    // h <- RMSNorm_l(h + FFN_l(h)) for the dense layer 0 and every MoE layer; the last norm feeds lm_head
    auto gamma = [&](int l) -> const float* { return m->gamma ? m->gamma[l] : nullptr; };
    focr_status s = focr_dense_mlp_forward(m->dense, x, T, h0, mws, mws_bytes, FOCR_FWD_RESIDUAL, stream);
    if (s != FOCR_OK) return s;
    float* last = (m->n_moe == 0 && hidden_out) ? hidden_out : h1;
    s = focr_rmsnorm(h0, gamma(0), T, m->eps, last, stream);
    if (s != FOCR_OK) return s;
    for (int l = 0; l < m->n_moe; ++l) {
        s = focr_moe_layer_forward_ex(m->moe[l], last, T, h0, mws, mws_bytes, nullptr, FOCR_FWD_RESIDUAL, stream);
        if (s != FOCR_OK) return s;
        float* dst = (l == m->n_moe - 1 && hidden_out) ? hidden_out : h1;
        s = focr_rmsnorm(h0, gamma(l + 1), T, m->eps, dst, stream);
        if (s != FOCR_OK) return s;
        last = dst;
    }
    const focr_lm_head* L = m->head;
    const uint4* codes = reinterpret_cast<const uint4*>(L->dev);
    const float* scales = reinterpret_cast<const float*>(L->dev + (size_t)FOCR_VOCAB * H);
    // a bounded wait of the lm_head that runs out is reported by focr_moe_check(workspace + 256)
    int32_t* err = reinterpret_cast<int32_t*>(w + kStepMoeOff + ws_layout(1).ctrl) + CTRL_ERROR;
    CUDA_TRY(launch_lm_head(codes, scales, last, T, logits, argmax, reinterpret_cast<int*>(w),
                            reinterpret_cast<unsigned long long*>(w + step_keys_off(T)), err, st));
    return FOCR_OK;
}

}  // extern "C"
