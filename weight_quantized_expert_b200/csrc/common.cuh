// Internal definitions shared by the kernels and the C ABI of libfocr_moe.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/focr_moe.h"

namespace focr {

constexpr int H = FOCR_HIDDEN;
constexpr int E = FOCR_EXPERTS;
constexpr int K = FOCR_TOPK;
constexpr int I = FOCR_INTER;
constexpr int IS = FOCR_SHARED_INTER;

// ---------------------------------------------------------------------------------------
// Device layout of a SwiGLU weight set ("item" = one slice of S intermediate rows).
//
// The decode kernel feeds 16x8x16 tensor-core fragments straight from registers, so the
// packer stores every weight where the lane that needs it will load it.  For a slice
// [i0, i0 + S) of the intermediate axis, tile t (of S/8) stacks 8 gate rows over the 8
// matching up rows: tile row g < 8 is gate row i0+8t+g, tile row g+8 is up row i0+8t+g.
// Lane L = 4*gr + c of a warp holds, for k-step q (input columns 16q .. 16q+15), the
// eight A-fragment elements
//   e0..e7 = (gr, k0) (gr, k0+1) (gr+8, k0) (gr+8, k0+1) (gr, k0+8) (gr, k0+9) (gr+8, k0+8) (gr+8, k0+9)
// with k0 = 16q + 2c.  The item block holds, contiguously:
//   GU weights : [tile][q / KPV][lane][KPV * FB bytes]   FB = 4 (int4), 8 (int8), 16 (bf16),
//                KPV = 16 / FB k-steps per 16-byte lane vector
//   GU scales  : [tile][1280/g groups][8 gr][2 (gate, up)] f32      (quantised types only)
//   D weights  : [80 output tiles][lane][8 bytes]  rows 16m+gr, 16m+gr+8 of down[:, i0 : i0+S]
//                (int4: two k-steps; int8: one k-step; bf16: one 16x8x8 step, elements
//                (gr, 2c) (gr, 2c+1) (gr+8, 2c) (gr+8, 2c+1))
// and, outside the item block, the down scales of the whole expert:
//   D scales   : [ceil(inter/g) groups][1280 rows] f32               (quantised types only)
// Codes are offset-binary: int4 q+8 with e0..e7 in nibble slots 0,4,1,5,2,6,3,7 of a
// 32-bit word (so one mask pulls a register pair); int8 q+128 in bytes e0..e7; bf16 as
// bit patterns.  S is 32 (int4), 16 (int8), 8 (bf16): a down row slice is always 16 bytes.
// ---------------------------------------------------------------------------------------
constexpr int UNITS = H / 8;  // 160 units of 8 input columns (item size bookkeeping)
constexpr int KSTEPS = H / 16;  // 80 k-steps of 16 input columns
constexpr int OTILES = H / 16;  // 80 output tiles of 16 rows

__host__ __device__ constexpr int slice_rows(int wtype) {
    return wtype == FOCR_W_INT4 ? 32 : (wtype == FOCR_W_INT8 ? 16 : 8);
}
__host__ __device__ constexpr int unit_row_bytes(int wtype) {
    return wtype == FOCR_W_INT4 ? 4 : (wtype == FOCR_W_INT8 ? 8 : 16);
}
__host__ __device__ constexpr int frag_bytes(int wtype) { return unit_row_bytes(wtype); }
__host__ __device__ constexpr int ksteps_per_vec(int wtype) { return 16 / frag_bytes(wtype); }
__host__ __device__ constexpr bool is_quant(int wtype) { return wtype != FOCR_W_BF16; }
// nibble slot of A-fragment element j (int4)
__host__ __device__ constexpr int nibble_slot(int j) { return (j >> 1) | ((j & 1) << 2); }

// compile-time sizes of an item block (G = group size; ignored for bf16)
__host__ __device__ constexpr uint32_t gu_w_bytes_of(int wtype) {
    return (uint32_t)(slice_rows(wtype) / 8) * KSTEPS * 32 * frag_bytes(wtype);
}
__host__ __device__ constexpr uint32_t gu_s_bytes_of(int wtype, int G) {
    return is_quant(wtype) ? (uint32_t)(slice_rows(wtype) / 8) * (H / G) * 16 * 4 : 0u;
}
__host__ __device__ constexpr uint32_t d_w_bytes_of() { return (uint32_t)OTILES * 32 * 8; }
__host__ __device__ constexpr uint32_t blk_bytes_of(int wtype, int G) {
    return gu_w_bytes_of(wtype) + gu_s_bytes_of(wtype, G) + d_w_bytes_of();
}

struct ItemGeom {
    int wtype, group, S, inter, slices;
    uint32_t gu_w_bytes, gu_s_bytes, d_w_bytes, item_bytes;  // item_bytes: 128-byte multiple
    uint32_t dscale_expert_floats;                           // ceil(inter/g) * 1280 (0 for bf16)
};

__host__ __device__ inline ItemGeom make_geom(int wtype, int group, int inter) {
    ItemGeom g{};
    g.wtype = wtype;
    g.group = is_quant(wtype) ? group : 0;
    g.S = slice_rows(wtype);
    g.inter = inter;
    g.slices = inter / g.S;
    g.gu_w_bytes = gu_w_bytes_of(wtype);
    g.gu_s_bytes = is_quant(wtype) ? gu_s_bytes_of(wtype, group) : 0u;
    g.d_w_bytes = d_w_bytes_of();
    uint32_t raw = g.gu_w_bytes + g.gu_s_bytes + g.d_w_bytes;
    g.item_bytes = (raw + 127u) & ~127u;
    g.dscale_expert_floats = is_quant(wtype) ? (uint32_t)((inter + group - 1) / group) * H : 0u;
    return g;
}

// Device-side view of a packed layer (passed by value to kernels).
struct LayerView {
    const uint16_t* router;        // [64][1280] bf16
    const uint8_t* routed_items;   // [64][slices][item_bytes]
    const float* routed_dscale;    // [64][ceil(inter/g)][1280]
    const uint8_t* shared_items;   // [slices][item_bytes]
    const float* shared_dscale;    // [1792/g][1280]
    ItemGeom rg, sg;
};

// ---------------------------------------------------------------------------------------
// Second device layout of a weight set, read by the tensor-core (tcgen05) grouped kernel
// for batches of more than 8 tokens.  Every matrix is cut into blocks of 128 rows x 64
// input columns (one "K-block").  Tiles come in groups of `grp` (routed experts: the most tiles a
// work unit covers, tc_tile_group; the shared set: 1); within a group the blocks of one K-block
// are adjacent, so a unit covering several tiles streams each of its K-blocks with one copy, and
// with grp = 1 the K-blocks of a tile are adjacent instead (tc_block_index):
//   gate/up : tiles p of 64 intermediates x 20 K-blocks; block row r = 16 j + 8 h + r' is gate
//             (h = 0) or up (h = 1) row 64 p + 8 j + r' (so a gate row and its up row sit 8 TMEM
//             lanes apart, inside one warp's quarter of the accumulator)
//   down    : m-tiles of 128 output rows x inter / 64 K-blocks; block row r is output row 128 m + r
// Quantised blocks: codes [128 rows][RB bytes] then f32 scales [128 rows][SPK].  A row's
// codes come in four pairs (k-core c, k-core c + 4) of 8-element k-cores (one k-core per
// 16-byte row of the tensor core's shared-memory operand):
//   int4 (RB = 32): pair c = 8 bytes = two 32-bit words, word 0 k-core c, word 1 k-core c+4;
//                   element 2m of a k-core in nibble m, element 2m+1 in nibble m+4, q + 8
//   int8 (RB = 64): pair c = 16 bytes, bytes 0-7 k-core c, bytes 8-15 k-core c+4, q + 128
// SPK = 64 / g scales per row for g = 32 (k-cores 0-3 use the first, 4-7 the second), one
// otherwise (for g = 128 each scale is stored with both K-blocks of its group).
// bf16 blocks: the operand image itself, [16 row groups][8 k-cores][8 rows][8 bf16] (16 KB):
// the K-major, unswizzled core-matrix layout tcgen05.mma reads from shared memory.
// ---------------------------------------------------------------------------------------
constexpr int TC_KB = 64;                  // input columns per K-block
constexpr int TC_M = 128;                  // rows per block (the MMA's M)
constexpr int TC_KBH = H / TC_KB;          // 20 K-blocks of a gate/up row
constexpr int TC_MT = H / TC_M;            // 10 output tiles of a down projection

__host__ __device__ constexpr int tc_spk(int G) { return G >= 64 ? 1 : 64 / G; }
__host__ __device__ constexpr uint32_t tc_row_bytes(int wtype) { return wtype == FOCR_W_INT4 ? 32u : 64u; }
__host__ __device__ constexpr uint32_t tc_block_bytes(int wtype, int G) {
    return is_quant(wtype) ? (uint32_t)TC_M * tc_row_bytes(wtype) + (uint32_t)TC_M * 4u * (uint32_t)tc_spk(G)
                           : (uint32_t)TC_M * TC_KB * 2u;
}

// Tiles of one routed work unit at most (and the routed tile group) by weight type, so that one
// K-block of a unit's tiles is 16-18 KB: int4 4, int8 2, bf16 1.
__host__ __device__ constexpr int tc_tile_group(int wtype) {
    return wtype == FOCR_W_INT4 ? 4 : (wtype == FOCR_W_INT8 ? 2 : 1);
}

// Block index of (tile, K-block) in a matrix of `tiles` tiles x `nkb` K-blocks with tile groups
// of `grp`: the group starting at tile t0 = grp * (tile / grp) holds gs = min(grp, tiles - t0)
// tiles, stored as [K-block][tile in group] after the t0 * nkb blocks of the groups before it.
__host__ __device__ constexpr size_t tc_block_index(int tiles, int nkb, int tile, int kb, int grp) {
    return (size_t)(tile - tile % grp) * nkb +
           (size_t)kb * (tiles - (tile - tile % grp) < grp ? tiles - (tile - tile % grp) : grp) + tile % grp;
}

struct TcGeom {
    int wtype, group, inter;
    int tiles;            // inter / 64 gate/up tiles (= K-blocks of the down projection)
    int grp;              // tile group of the layout (tc_block_index)
    uint32_t blk;         // bytes of one block
    size_t gu_bytes;      // tiles * 20 blocks
    size_t dn_bytes;      // 10 m-tiles * tiles blocks
};

__host__ __device__ inline TcGeom make_tc_geom(int wtype, int group, int inter, int grp) {
    TcGeom g{};
    g.grp = grp;
    g.wtype = wtype;
    g.group = is_quant(wtype) ? group : 0;
    g.inter = inter;
    g.tiles = inter / TC_KB;
    g.blk = tc_block_bytes(wtype, is_quant(wtype) ? group : 64);
    g.gu_bytes = (size_t)g.tiles * TC_KBH * g.blk;
    g.dn_bytes = (size_t)TC_MT * g.tiles * g.blk;
    return g;
}

struct TcSetView {
    const uint8_t* gu;    // routed: [64 experts][gu_bytes]; shared: [gu_bytes]
    const uint8_t* dn;    // routed: [64 experts][dn_bytes]; shared: [dn_bytes]
    TcGeom g;
};

struct TcView {
    TcSetView r, s;       // routed experts, shared (or dense) set
};

// ---------------------------------------------------------------------------------------
// Workspace layout (bytes from the workspace base).  Control words first; they are
// zero on entry and every forward returns them to zero.
// ---------------------------------------------------------------------------------------
constexpr int ROUTER_KSPLIT = 8;          // 1280 = 8 x 160 input columns: one CTA each of a cluster
constexpr int ROUTER_TB = 8;              // tokens per router CTA
constexpr int MAX_TB = (FOCR_T_MAX + ROUTER_TB - 1) / ROUTER_TB;

struct WsLayout {
    // regions that are zero on entry and that every forward leaves zero; their offsets do
    // not depend on T_max, so calls with different T may share one workspace
    size_t ctrl;          // int32 [MAX_TB tickets][1 global ticket][1 error word][pad][CTRL_TC_WORDS]
    size_t tcnt;          // i32 [GU_TILES]               arrival counters of the k-split gate/up tiles (T <= 8)
    size_t dacc;          // i64 [8][1280]                the down projections' output sums (T <= 8), fixed point
    size_t dflag;         // i32 [8][1280]                1: a non-finite or out-of-range part
    size_t dcnt;          // i32 [80]                     units finished per 16-row output tile
    // regions every forward writes before reading
    size_t gpart;         // f32 [GU_TILES][4 parts][32][4]  the k-split gate/up tiles' part sums (T <= 8)
    size_t a16;           // uint2 [A16_STEPS][32]   f16 a fragments (int4 / int8 down, T <= 8)
    size_t abf;           // uint2 [ABF_STEPS][32]   bf16 a hi, lo fragments (bf16 down, T <= 8)
    size_t logits;        // f32 [T_max][64]
    size_t topk_idx;      // i32 [T_max][6]
    size_t topk_w;        // f32 [T_max][6]
    size_t counts;        // i32 [64]
    size_t offsets;       // i32 [65]
    size_t active;        // i32 [64] experts with tokens, ascending; [64] = U
    size_t perm;          // i32 [T_max*6]
    // tensor-core grouped path (T > 8 only; size 0 otherwise)
    size_t x_img;         // bf16 [20][T_pad][64]               x in token order, operand image per K-block
    size_t x_img_r;       // bf16 [20][TC_AROWS(T_max)][64]     x in dispatch order (each expert's rows)
    size_t a_img;         // bf16 [14][TC_AROWS(T_max)][64]     routed a, operand image per K-block
    size_t a_sh;          // bf16 [shared K-blocks][T_pad][64]  shared-set a, operand image
    size_t y_slot;        // f32 [T_max*6][1280]                each (token, slot) expert output
    size_t y_sh;          // f32 [parts][T_max][1280]           shared-set output, per K part
    size_t total;
};

// gate/up tiles of 8 intermediates: a shared set of up to IS_MAX intermediates, then 64
// routed experts (896/8 each); a set of IS_MAX = 6848 covers the dense layer
constexpr int IS_MAX = FOCR_DENSE_INTER;
constexpr int GU_TILES = IS_MAX / 8 + E * (I / 8);
constexpr int A16_STEPS = IS_MAX / 16 + E * (I / 16);   // k-steps of 16 intermediates
constexpr int ABF_STEPS = IS_MAX / 8 + E * (I / 8);     // k-steps of 8 intermediates

constexpr size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// K parts of the shared (or dense) set's down projection in the tensor-core path: the parts'
// partial outputs are separate and summed by the combine in a fixed order
__host__ __device__ constexpr int tc_parts(int inter) {
    return inter / TC_KB / 7 < 1 ? 1 : (inter / TC_KB / 7 > 8 ? 8 : inter / TC_KB / 7);
}
__host__ __device__ constexpr int tc_kpp(int inter) {   // K-blocks per part
    return (inter / TC_KB + tc_parts(inter) - 1) / tc_parts(inter);
}
// rows of the routed a image: every expert's segment is padded to a multiple of 16 rows
__host__ __device__ constexpr size_t tc_arows(int T) { return align_up((size_t)T * K + (size_t)E * 15, 16); }

// `shared_inter`: intermediate width of the shared set the call runs (1792 for the MoE
// layer, 6848 for the dense layer); it sizes the tensor-core path's shared-set regions
constexpr WsLayout ws_layout(int T_max, int shared_inter = IS) {
    WsLayout w{};
    size_t o = 0;
    w.ctrl = o;      o = align_up(o + sizeof(int32_t) * (MAX_TB + 256), 256);
    w.tcnt = o;      o = align_up(o + sizeof(int32_t) * (size_t)GU_TILES, 256);
    w.dacc = o;      o = align_up(o + sizeof(int64_t) * 8 * H, 256);
    w.dflag = o;     o = align_up(o + sizeof(int32_t) * 8 * H, 256);
    w.dcnt = o;      o = align_up(o + sizeof(int32_t) * (H / 16), 256);
    w.gpart = o;     o = align_up(o + sizeof(float) * 4 * 4 * 32 * (size_t)GU_TILES, 256);
    w.a16 = o;       o = align_up(o + 8 * 32 * (size_t)A16_STEPS, 256);
    w.abf = o;       o = align_up(o + 8 * 32 * (size_t)ABF_STEPS, 256);
    w.logits = o;    o = align_up(o + sizeof(float) * (size_t)T_max * E, 256);
    w.topk_idx = o;  o = align_up(o + sizeof(int32_t) * (size_t)T_max * K, 256);
    w.topk_w = o;    o = align_up(o + sizeof(float) * (size_t)T_max * K, 256);
    w.counts = o;    o = align_up(o + sizeof(int32_t) * E, 256);
    w.offsets = o;   o = align_up(o + sizeof(int32_t) * (E + 1), 256);
    w.active = o;    o = align_up(o + sizeof(int32_t) * (E + 1), 256);
    w.perm = o;      o = align_up(o + sizeof(int32_t) * (size_t)T_max * K, 256);
    const bool tc = T_max > 8;
    const size_t tpad = align_up((size_t)T_max, 16);
    w.x_img = o;     o = align_up(o + (tc ? 2 * tpad * H : 0), 256);
    w.x_img_r = o;   o = align_up(o + (tc ? (size_t)TC_KBH * tc_arows(T_max) * TC_KB * 2 : 0), 256);
    w.a_img = o;     o = align_up(o + (tc ? (size_t)(I / TC_KB) * tc_arows(T_max) * TC_KB * 2 : 0), 256);
    w.a_sh = o;      o = align_up(o + (tc ? (size_t)(shared_inter / TC_KB) * tpad * TC_KB * 2 : 0), 256);
    w.y_slot = o;    o = align_up(o + (tc ? sizeof(float) * (size_t)T_max * K * H : 0), 256);
    w.y_sh = o;      o = align_up(o + (tc ? sizeof(float) * (size_t)tc_parts(shared_inter) * T_max * H : 0), 256);
    w.total = o;
    return w;
}

// control-word indices (int32) inside ws.ctrl
constexpr int CTRL_GLOBAL_TICKET = MAX_TB;
constexpr int CTRL_ERROR = MAX_TB + 1;
// counters of the tensor-core grouped kernel (reset by its last CTA)
constexpr int CTRL_TC = MAX_TB + 8;
constexpr int TC_WORK = 0;        // next work unit (dynamic scheduler)
constexpr int TC_EXIT = 1;        // CTAs finished
constexpr int TC_DN_DONE = 2;     // down-projection units finished
constexpr int TC_DEP_R = 3;       // [64] gate/up units finished per routed expert
constexpr int TC_DEP_S = 67;      // [8] gate/up units finished per K part of the shared set
constexpr int TC_DEP_X = 75;      // [64] token rows of each routed expert gathered
constexpr int TC_CNT = 139;       // [64] assignments per routed expert, added by the router
constexpr int TC_WORDS = 203;
static_assert(CTRL_TC + TC_WORDS <= MAX_TB + 256, "control words fit the ctrl region");

struct RouteView {   // device pointers into the workspace
    int32_t* ctrl;
    float* logits;
    int32_t* topk_idx;
    float* topk_w;
    int32_t* counts;
    int32_t* offsets;
    int32_t* active;
    int32_t* perm;
    int32_t* tcnt;
    unsigned long long* dacc;
    int32_t* dflag;
    int32_t* dcnt;
    float* gpart;
    uint2* a16;
    uint2* abf;
};

inline RouteView route_view(void* ws, int T_max, int shared_inter = IS) {
    WsLayout L = ws_layout(T_max, shared_inter);
    char* b = (char*)ws;
    return RouteView{(int32_t*)(b + L.ctrl), (float*)(b + L.logits),
                     (int32_t*)(b + L.topk_idx), (float*)(b + L.topk_w), (int32_t*)(b + L.counts),
                     (int32_t*)(b + L.offsets), (int32_t*)(b + L.active), (int32_t*)(b + L.perm),
                     (int32_t*)(b + L.tcnt), (unsigned long long*)(b + L.dacc), (int32_t*)(b + L.dflag),
                     (int32_t*)(b + L.dcnt), (float*)(b + L.gpart), (uint2*)(b + L.a16), (uint2*)(b + L.abf)};
}

// workspace regions of the tensor-core grouped path
// Operand images (bf16, K-major core-matrix layout of the tensor core's shared-memory operand):
// element (row r, k) of K-block kb sits at [kb][r / 8][(k % 64) / 8][r % 8][k % 8], so the rows
// [r0, r0 + N) of one K-block (r0 a multiple of 8) are N * 128 contiguous bytes.
__host__ __device__ inline size_t img_index(int rows, int r, int k) {
    return ((size_t)(k / TC_KB) * rows + (size_t)(r & ~7)) * TC_KB + (size_t)((k % TC_KB) / 8) * 64 + (r & 7) * 8 +
           (k & 7);
}

struct TcWork {
    uint16_t* x_img;      // x in token order (tpad rows)
    uint16_t* x_img_r;    // x rows in dispatch order (arows rows)
    uint16_t* a_img;      // routed a image
    uint16_t* a_sh;       // shared a image
    float* y_slot;
    float* y_sh;
    int arows;            // rows of the routed a image
    int tpad;             // T rounded up to 16 (rows of the shared a image)
};

inline TcWork tc_work(void* ws, int T, int shared_inter) {
    WsLayout L = ws_layout(T, shared_inter);
    char* b = (char*)ws;
    return TcWork{(uint16_t*)(b + L.x_img), (uint16_t*)(b + L.x_img_r), (uint16_t*)(b + L.a_img), (uint16_t*)(b + L.a_sh),
                  (float*)(b + L.y_slot), (float*)(b + L.y_sh), (int)tc_arows(T), (int)align_up((size_t)T, 16)};
}

// error codes a kernel may store in the error word
// activations outside the f16 operand range (finite |v| > 65504) met by a kernel; the
// forward completes, and focr_moe_check reports FOCR_ERR_RANGE
constexpr int DEVERR_RANGE = 8;
__device__ __forceinline__ bool f16_out_of_range(float v) { return fabsf(v) > 65504.f && fabsf(v) <= 3.402823466e38f; }
constexpr int DEVERR_FULL_WAIT = 1;
constexpr int DEVERR_EMPTY_WAIT = 2;

// ------------------------------------------------------------------ launchers (per .cu)
// out: NULL leaves the layer output alone (the tensor-core path's combine writes all of it);
// otherwise resid NULL zeroes `out` before the experts add into it, and a non-NULL resid
// makes `out` start as a copy of resid.
cudaError_t launch_router(const float* x, int T, int T_ws, const LayerView& L, const RouteView& R, float* out,
                          const float* resid, uint16_t* x_img, int img_rows, cudaStream_t st);
// Tensor-core grouped path (expert_tc.cu), T > 8: the shared set and the selected experts
// as tcgen05 GEMMs, then the combine out = resid + shared + sum_j w_j expert_j (fixed
// order).  shared_only: the dense layer (one always-on set, no routing); it then also
// writes the x image itself.
cudaError_t launch_expert_tc(const float* x, int T, const TcView& V, const RouteView& R, const TcWork& W,
                             float* out, bool resid, bool shared_only, cudaStream_t st);
// T <= SMALL_T: gate/up + swiglu kernel, then the down kernel (decode_small.cu)
constexpr int SMALL_T = 8;
// SMALL_T < T <= MID_T: the grouped mma.sync kernel (expert_decode.cu), behind the router's own
// dispatch; larger batches take the tensor-core kernel (expert_tc.cu), which measured slower than
// it up to 64 tokens (batch 32: 164 vs 122 us; batch 64: 180 vs 171 us)
constexpr int MID_T = 64;
cudaError_t launch_expert_decode(const float* x, int T, const LayerView& L, const RouteView& R, float* out,
                                 bool shared_only, cudaStream_t st);
cudaError_t launch_decode_small(const float* x, int T, const LayerView& L, const RouteView& R, float* out,
                                bool shared_only, bool deterministic, cudaStream_t st);

}  // namespace focr

// ---------------------------------------------------------------------------------------
// PTX helpers (device only)
// ---------------------------------------------------------------------------------------
#ifdef __CUDACC__
namespace focr {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// try_wait that may suspend the thread for up to `hint_ns` while the phase is pending
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete; give up after ~limit_ns.
// Slow path of mbar_wait_bounded, kept out of line so that the common case (the phase has
// already completed) costs one try_wait and a branch in the caller's loop.
static __device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait_hint(bar, parity, 20000u)) return true;
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
}

__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    if (__builtin_expect(mbar_try_wait(bar, parity), 1)) return true;
    return mbar_wait_slow(bar, parity, limit_ns);
}

// Bulk (non-tensor) async copy global -> own shared memory, completing on an mbarrier.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], "
        "%4;" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// Address of the same shared variable in CTA `rank` of the cluster (shared::cluster window).
__device__ __forceinline__ uint32_t mapa_shared(const void* p, uint32_t rank) {
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
    return a;
}

// Asynchronous 8-byte store into another CTA's shared memory; its bytes complete on that
// CTA's mbarrier (both addresses in the shared::cluster window).
__device__ __forceinline__ void st_async_f64(uint32_t remote_addr, double v, uint32_t remote_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b64 [%0], %1, [%2];" ::"r"(remote_addr),
                 "l"(__double_as_longlong(v)), "r"(remote_bar)
                 : "memory");
}

// Bulk prefetch of global memory into L2 (no shared memory involved).
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// 16-byte read-only load with an L2 cache-eviction policy (createpolicy)
__device__ __forceinline__ uint4 ldg_policy(const void* p, uint64_t policy) {
    uint4 v;
    asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(policy));
    return v;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Programmatic dependent launch controls.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Named barrier over `count` threads (id != 0).
__device__ __forceinline__ void named_bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Fixed-point accumulation, for sums whose value must not depend on the order in which their
// parts arrive: each part is rounded once to a multiple of 2^-32 (|part| < 2^30), the parts add
// exactly as 64-bit integers (any order gives the same total), and the total converts back to
// fp32 once.  A part that is not finite or out of that range is recorded by the caller in a flag
// instead, and the total then reads as NaN.
constexpr double FX_ONE = 4294967296.0;   // 2^32
__device__ __forceinline__ bool fx_ok(float v) { return fabsf(v) < 1073741824.f; }   // false for NaN / inf
__device__ __forceinline__ unsigned long long fx_of(float v) {
    return (unsigned long long)__double2ll_rn((double)v * FX_ONE);
}
__device__ __forceinline__ float fx_to_float(unsigned long long a) { return (float)((double)(long long)a * (1.0 / FX_ONE)); }
__device__ __forceinline__ void red_add_u64(unsigned long long* addr, unsigned long long v) {
    asm volatile("red.global.add.u64 [%0], %1;" ::"l"(addr), "l"(v) : "memory");
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

__device__ __forceinline__ uint4 lds128(const void* p) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

__device__ __forceinline__ float4 lds128f(const void* p) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

// ------------------------------------------------------------------ dequantisation
// A float whose bits are 0x4B0000vv equals 2^23 + vv exactly; subtracting 2^23 + bias
// recovers the signed code.  __byte_perm places byte j of `src` under the exponent.
__device__ __forceinline__ float byte_to_float(uint32_t src, int j) {
    return __uint_as_float(__byte_perm(src, 0x4B000000u, 0x7440u | (uint32_t)j));
}

// 8 int4 codes (offset-binary, columns c..c+7 of one row) -> 8 floats q in [-8, 7]
__device__ __forceinline__ void dq_int4x8(uint32_t w, float (&q)[8]) {
    const uint32_t lo = w & 0x0F0F0F0Fu;          // columns c, c+2, c+4, c+6
    const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;   // columns c+1, c+3, c+5, c+7
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        q[2 * b] = byte_to_float(lo, b) - 8388616.0f;
        q[2 * b + 1] = byte_to_float(hi, b) - 8388616.0f;
    }
}

// 4 int8 codes (offset-binary) -> 4 floats q in [-127, 127]
__device__ __forceinline__ void dq_int8x4(uint32_t w, float (&q)[4]) {
#pragma unroll
    for (int b = 0; b < 4; ++b) q[b] = byte_to_float(w, b) - 8388736.0f;
}

// 2 bf16 -> 2 floats
__device__ __forceinline__ void bf16x2_to_f32(uint32_t w, float& a, float& b) {
    a = __uint_as_float(w << 16);
    b = __uint_as_float(w & 0xFFFF0000u);
}

}  // namespace focr
#endif
