/*
 * focr_moe -- one mixture-of-experts layer forward with group-quantised experts,
 * for NVIDIA B200 (sm_100a).  C ABI: plain pointers and sizes, no framework types.
 *
 * The layer (frankenocr.pages.dev, "One forward pass", step 6; franken_ocr
 * README, "Architecture" and "Design Philosophy"):
 *   hidden H = 1280; a softmax router over E = 64 routed experts picks the top
 *   k = 6 greedily and does NOT renormalise the chosen probabilities; 2 shared
 *   experts, fused into one SwiGLU of width 1792, always contribute with weight 1;
 *   each routed expert is a SwiGLU FFN 1280 -> 896 -> 1280:
 *       expert(x) = D (silu(G x) * (U x)),  silu(v) = v / (1 + exp(-v))
 *       out[t]    = sum_j p[t, idx_j] * expert_{idx_j}(x_t) + shared(x_t)
 *   (the layer output has no residual added).
 * Weight storage (frankenocr.pages.dev, "Four bits, one shared scale"): an int4
 * weight is a two's-complement nibble sharing one f32 scale with its group; int8
 * and bf16 are the other formats of the pages' quantisation recipe.
 *
 * Conventions for every call:
 *   - All dimensions are fixed at compile time (the FOCR_* constants below);
 *     anything else is FOCR_ERR_UNSUPPORTED.
 *   - Weights are given as HOST fp32 arrays in nn.Linear orientation [out, in],
 *     row-major, owned by the caller and only read during the call.
 *   - Activations are DEVICE pointers owned by the caller, fp32 row-major,
 *     16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Forward calls are asynchronous on that stream; pack/export/clone calls
 *     synchronise before returning.
 *   - Arguments are checked before anything is launched; on error nothing is
 *     launched and focr_last_error() (thread-local) says why.
 */
#ifndef FOCR_MOE_H
#define FOCR_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FOCR_HIDDEN 1280        /* hidden size */
#define FOCR_EXPERTS 64         /* routed experts */
#define FOCR_TOPK 6             /* experts per token */
#define FOCR_INTER 896          /* routed-expert intermediate */
#define FOCR_SHARED_INTER 1792  /* fused shared experts (2 x 896) */
#define FOCR_VOCAB 129280       /* lm_head rows */
#define FOCR_DENSE_INTER 6848   /* dense layer-0 intermediate */
#define FOCR_T_MAX 8192         /* most tokens one forward call accepts */

typedef enum {
    FOCR_OK = 0,
    FOCR_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, T out of range, short workspace */
    FOCR_ERR_UNSUPPORTED = 2,  /* weight type / group size / dimension not supported */
    FOCR_ERR_CUDA = 3,         /* a CUDA runtime call failed (message has the CUDA error) */
    FOCR_ERR_OOM = 4,          /* device or host allocation failed */
    FOCR_ERR_TIMEOUT = 5,      /* a bounded device-side wait ran out (see focr_moe_check) */
    FOCR_ERR_RANGE = 6         /* an activation the f16 operands cannot hold (finite |v| > 65504) was met;
                                  reported after the fact by focr_moe_check (see there) */
} focr_status;

typedef enum { FOCR_W_BF16 = 0, FOCR_W_INT8 = 1, FOCR_W_INT4 = 2 } focr_wtype;

/* Which matrix of a packed layer focr_moe_export_quantized() returns. */
typedef enum {
    FOCR_MAT_GATE = 0, FOCR_MAT_UP = 1, FOCR_MAT_DOWN = 2,          /* routed expert `expert` */
    FOCR_MAT_SHARED_GATE = 3, FOCR_MAT_SHARED_UP = 4, FOCR_MAT_SHARED_DOWN = 5,
    FOCR_MAT_ROUTER = 6
} focr_matrix;

/* Host-side description of one layer's weights (all fp32 except the router). */
typedef struct {
    const float* w_gate;          /* [64, 896, 1280] */
    const float* w_up;            /* [64, 896, 1280] */
    const float* w_down;          /* [64, 1280, 896] */
    const float* ws_gate;         /* [1792, 1280]    */
    const float* ws_up;           /* [1792, 1280]    */
    const float* ws_down;         /* [1280, 1792]    */
    const uint16_t* w_router_bf16;/* [64, 1280] bf16 bit patterns */
    int32_t routed_type;          /* focr_wtype of the routed experts */
    int32_t shared_type;          /* focr_wtype of the shared expert  */
    int32_t group_size;           /* 32, 64 or 128 (int4); 128 (int8); ignored for bf16 */
} focr_moe_weights_desc;

typedef struct focr_moe_layer focr_moe_layer;   /* opaque, device-resident, library-owned */

/* Optional routing outputs of a forward call (each pointer may be NULL; DEVICE memory). */
typedef struct {
    float* logits;       /* [T, 64] fp32 router logits                               */
    int32_t* topk_idx;   /* [T, 6]  chosen experts, best first (ties: lower index)   */
    float* topk_w;       /* [T, 6]  their softmax probabilities (not renormalised)   */
    int32_t* counts;     /* [64]    tokens routed to each expert                     */
    int32_t* offsets;    /* [65]    exclusive prefix sum of counts                   */
    int32_t* perm;       /* [T*6]   entries t*6+j grouped by expert, token-ascending */
} focr_moe_route_debug;

/*
 * focr_moe_pack_weights -- quantise and lay out one layer on the device.
 * Quantisation ("Four bits, one shared scale"): for every group of g consecutive
 * input-axis elements of one output row, s = max|w| / Q as one fp32 division
 * (Q = 7 for int4, 127 for int8), q = round-half-even(w / s) clamped to [-8, 7]
 * or [-127, 127]; an all-zero group has s = 0, q = 0.  bf16 weights are rounded
 * to nearest-even; the router is taken as given (bf16).
 * The device layout is private (tiled for 16-byte loads and bulk copies); use
 * focr_moe_export_quantized() to read back the canonical codes.
 * On success *out owns device memory until focr_moe_layer_free().  Synchronises.
 */
focr_status focr_moe_pack_weights(const focr_moe_weights_desc* desc, focr_moe_layer** out, void* stream);

/* Device copy of a packed layer (same codes, new memory).  Synchronises. */
focr_status focr_moe_layer_clone(const focr_moe_layer* src, focr_moe_layer** out, void* stream);

void focr_moe_layer_free(focr_moe_layer* layer);

/* Device bytes held by a packed layer. */
size_t focr_moe_layer_device_bytes(const focr_moe_layer* layer);

/*
 * focr_moe_export_sizes / focr_moe_export_quantized -- canonical quantised form of
 * one matrix (for bit-exact checks).  Canonical codes: int4 as two's-complement
 * nibbles, element 2j in bits 0-3 and 2j+1 in bits 4-7 of byte j, row-major;
 * int8 as int8 row-major; bf16 as uint16 bit patterns row-major.  Scales: f32
 * [rows, ceil(cols / g)] row-major (none for bf16).  `expert` is ignored for the
 * shared matrices and the router.  Buffers are HOST memory of at least the sizes
 * focr_moe_export_sizes() reports.  Synchronises.
 */
focr_status focr_moe_export_sizes(const focr_moe_layer* layer, int32_t matrix, size_t* code_bytes,
                                  size_t* n_scales);
focr_status focr_moe_export_quantized(const focr_moe_layer* layer, int32_t matrix, int32_t expert,
                                      void* codes_host, size_t code_bytes, float* scales_host,
                                      size_t n_scales);

/* Workspace a forward call with up to T_max tokens needs (bytes). */
size_t focr_moe_workspace_bytes(int32_t T_max);

/* Length of the workspace prefix (control words, k-split partial sums and their arrival
 * counters) that must be zero when a forward starts and that every forward leaves zero.
 * It does not depend on T_max.  Zeroing these bytes makes a workspace usable again after
 * focr_moe_check reported a device error. */
size_t focr_moe_workspace_zero_bytes(void);

/*
 * focr_moe_layer_forward -- out[T, 1280] = MoE(hidden[T, 1280]).
 *   hidden, out : DEVICE fp32, 16-byte aligned, caller-owned; must not overlap.
 *   1 <= T <= FOCR_T_MAX.
 *   workspace   : DEVICE scratch of ws_bytes >= focr_moe_workspace_bytes(T), 256-byte
 *                 aligned.  It must be zero-filled before its first use; every forward
 *                 leaves its first focr_moe_workspace_zero_bytes() bytes zero again, so
 *                 calls with different T may share it.  Calls that share a workspace
 *                 must be ordered on one stream.
 *   dbg         : optional routing outputs (NULL for none).
 * Steps, all on `stream`: router GEMV (fp64 accumulation of exact products,
 * rounded to fp32) + softmax + greedy top-6 (rank by fp32 logit, ties to the
 * lower index) + dispatch (counting sort of t*6+j by expert, stable), then the
 * shared expert and the selected experts (codes dequantised in registers, fp32
 * accumulation), which add w * expert(x) into out: for T <= 8 a gate/up kernel
 * and a down kernel, for larger T one grouped expert kernel.
 */
focr_status focr_moe_layer_forward(const focr_moe_layer* layer, const float* hidden, int32_t T, float* out,
                                   void* workspace, size_t ws_bytes, const focr_moe_route_debug* dbg,
                                   void* stream);

/*
 * focr_moe_layer_forward_noalloc -- the same forward as focr_moe_layer_forward, for
 * callers that cannot allocate device memory where they run the layer (a plug-in or
 * callback inside an application that owns the device memory budget, or
 * latency-critical code that must not call cudaMalloc, which can block and
 * synchronise the device).  The pages have no counterpart of this entry point.
 *   - Allocates nothing: no cudaMalloc/cudaFree and no allocating library routine.
 *     Its scratch is a fixed array of FOCR_NOALLOC_SCRATCH_BYTES in the library's
 *     device image, held by every GPU that loads the library until process exit.
 *   - 1 <= T <= FOCR_NOALLOC_T_MAX; a larger T is rejected with FOCR_ERR_INVALID_ARG.
 *   - hidden, out, dbg, stream: as for focr_moe_layer_forward (caller-owned buffers).
 *   - The first call on a device looks up the array's device address and zero-fills
 *     it synchronously; make that first call before any stream capture.  Later calls
 *     launch only the forward: its control words and partial sums start at zero because
 *     every forward that completes leaves them zero.
 *   - All calls share the one array and it keeps the last call's contents: calls that
 *     overlap on the GPU (other streams, other host threads) race and give wrong
 *     results.  Serialise them on one stream.
 *   - A bounded device wait that runs out is not reported by the call itself (the call
 *     returns before the GPU runs it): focr_moe_check_noalloc reports it.
 */
#define FOCR_NOALLOC_T_MAX 320
#define FOCR_NOALLOC_SCRATCH_BYTES 50665216
focr_status focr_moe_layer_forward_noalloc(const focr_moe_layer* layer, const float* hidden, int32_t T, float* out,
                                           const focr_moe_route_debug* dbg, void* stream);

/*
 * focr_moe_check_noalloc -- focr_moe_check for the allocation-free forward's fixed array on
 * the current device: synchronises `stream` and returns FOCR_OK, or FOCR_ERR_TIMEOUT if a
 * bounded device wait of an earlier call ran out.  In that case it also zero-fills the
 * array's control words and partial sums (which that call may have left behind), so the
 * next call starts clean.  Allocates nothing.
 */
focr_status focr_moe_check_noalloc(void* stream);

/* Flags of the *_ex / dense forwards. */
#define FOCR_FWD_RESIDUAL 1   /* out = hidden + layer(hidden) instead of layer(hidden) */
/* Bit-identical results for identical calls on every path: T <= 8 then sums its parts as 64-bit
 * fixed-point integers (each part rounded once to a multiple of 2^-32) instead of fp32 atomics.
 * The tensor-core path (T > 64) always sums in a fixed order; 9 <= T <= 64 is not covered. */
#define FOCR_FWD_DETERMINISTIC 2

/*
 * focr_moe_layer_forward_ex -- focr_moe_layer_forward with flags (0 or FOCR_FWD_RESIDUAL).
 * With FOCR_FWD_RESIDUAL the output starts as a copy of `hidden` (the decoder's residual
 * stream h <- h + MoE(h)); arguments and workspace rules are otherwise the same.
 */
focr_status focr_moe_layer_forward_ex(const focr_moe_layer* layer, const float* hidden, int32_t T, float* out,
                                      void* workspace, size_t ws_bytes, const focr_moe_route_debug* dbg,
                                      int32_t flags, void* stream);

/*
 * Dense SwiGLU MLP of decoder layer 0 (frankenocr.pages.dev, "One forward pass", step 6:
 * layer 0 is a dense SwiGLU MLP): out = D (silu(G x) * (U x)) with G, U [6848, 1280] and
 * D [1280, 6848] (HOST fp32, [out, in] row-major).  Quantisation as focr_moe_pack_weights
 * (int8 with group 128 in the decode recipe; 6848 = 53 x 128 + 64, so the last group of
 * a down row has 64 elements and its own scale).  The forward runs on the MoE layer's
 * expert kernels as a single always-on weight set (the decode kernels for T <= 8, the
 * grouped kernel for larger T).
 */
typedef struct focr_dense_mlp focr_dense_mlp;
focr_status focr_dense_mlp_pack(const float* w_gate, const float* w_up, const float* w_down, int32_t wtype,
                                int32_t group, focr_dense_mlp** out, void* stream);
void focr_dense_mlp_free(focr_dense_mlp* mlp);
/* Canonical codes/scales of matrix 0 (gate), 1 (up) or 2 (down), formats as focr_moe_export_quantized;
 * codes: rows*cols (int8), rows*cols/2 (int4) or 2*rows*cols (bf16) bytes, scales rows*ceil(cols/g). */
focr_status focr_dense_mlp_export_quantized(const focr_dense_mlp* mlp, int32_t matrix, void* codes_host,
                                            size_t code_bytes, float* scales_host, size_t n_scales);
/* x, out: DEVICE fp32 [T, 1280], 16-byte aligned, not overlapping; workspace as for
 * focr_moe_layer_forward (focr_moe_workspace_bytes(T)); flags 0 or FOCR_FWD_RESIDUAL. */
focr_status focr_dense_mlp_forward(const focr_dense_mlp* mlp, const float* x, int32_t T, float* out,
                                   void* workspace, size_t ws_bytes, int32_t flags, void* stream);

/*
 * focr_moe_check -- read the device error word a forward may have set in `workspace`.
 * Synchronises `stream`.  Returns FOCR_OK, FOCR_ERR_TIMEOUT (a bounded device wait ran out;
 * that forward's output is not valid), or FOCR_ERR_RANGE (an activation fed to the f16 operands
 * -- the layer input x, or on the small-batch kernels the SwiGLU output -- had a finite
 * magnitude above 65504, the largest f16; the forward completed but the affected tokens'
 * outputs are not valid), and clears the word.
 */
focr_status focr_moe_check(void* workspace, void* stream);

/* ------------------------------------------------------------------ decode-step companions
 * Source: frankenocr.pages.dev, "One forward pass", step 7 -- the final RMSNorm feeds an
 * lm_head GEMV from 1,280 to 129,280 logits, and greedy decoding picks the argmax;
 * "Four bits, one shared scale" -- int8 on lm_head.
 */

typedef struct focr_lm_head focr_lm_head;   /* opaque, device-resident, library-owned */

/*
 * focr_lm_head_pack -- quantise the lm_head [129280, 1280] (HOST fp32, row-major) to int8
 * with one scale per row (s = max|w_row| / 127 in fp32, q = round-half-even(w / s)
 * clamped to [-127, 127]; an all-zero row has s = 0) and lay it out on the device.
 * Synchronises.
 */
focr_status focr_lm_head_pack(const float* w, focr_lm_head** out, void* stream);
void focr_lm_head_free(focr_lm_head* head);

/* Canonical codes (int8 [129280, 1280] row-major) and row scales (f32 [129280]) to HOST memory. */
focr_status focr_lm_head_export(const focr_lm_head* head, int8_t* codes_host, float* scales_host);

/* Workspace a focr_lm_head_gemv call with up to T_max tokens needs (bytes). */
size_t focr_lm_head_workspace_bytes(int32_t T_max);

/*
 * focr_lm_head_gemv -- logits[t, n] = s_n * sum_k q_nk x[t, k] and argmax[t] (ties to the
 * lowest row).  x: DEVICE fp32 [T, 1280], 16-byte aligned; logits: DEVICE fp32 [T, 129280]
 * or NULL; argmax: DEVICE int32 [T].  1 <= T <= FOCR_T_MAX.  workspace: DEVICE, 256-byte
 * aligned, >= focr_lm_head_workspace_bytes(T), zero-filled before first use (left with its
 * control word zero).  Asynchronous on `stream`.
 */
focr_status focr_lm_head_gemv(const focr_lm_head* head, const float* x, int32_t T, float* logits,
                              int32_t* argmax, void* workspace, size_t ws_bytes, void* stream);

/*
 * focr_lm_head_check -- synchronises `stream` and reports whether a focr_lm_head_gemv call on this
 * workspace met a device wait that ran out (the T <= 8 kernel's shared-memory pipeline waits are
 * bounded): FOCR_ERR_TIMEOUT (that call's outputs are not valid; the word is cleared) or FOCR_OK.
 */
focr_status focr_lm_head_check(void* workspace, void* stream);

/*
 * focr_rmsnorm -- out[t] = x[t] / sqrt(mean(x[t]^2) + eps) * gamma (gamma NULL: 1).
 * x, out: DEVICE fp32 [T, 1280], 16-byte aligned (may be the same buffer); gamma: DEVICE
 * fp32 [1280] or NULL.  Asynchronous on `stream`.
 */
focr_status focr_rmsnorm(const float* x, const float* gamma, int32_t T, float eps, float* out, void* stream);

/*
 * focr_decode_step -- one decode step of the decoder stack (frankenocr.pages.dev, "One forward
 * pass", steps 6-7: layer 0 is the dense SwiGLU MLP, the other decoder layers are MoE layers,
 * a final RMSNorm feeds the lm_head GEMV and greedy decoding takes the argmax):
 *     h = RMSNorm_0(x + Dense(x));   h = RMSNorm_l(h + MoE_l(h)) for l = 1 .. n_moe;
 *     logits = lm_head(h);           argmax[t] = index of the largest logit (ties: lowest row)
 * The attention sub-layers of the decoder are outside this library; callers that run them
 * chain their own kernels between steps on the same stream.  Every stage is an asynchronous
 * launch on `stream` (programmatic dependent launch between the library's kernels), so the
 * whole step can be captured into one CUDA graph.
 *   m:          the model; layers and lm_head are packed handles, gamma[l] (l = 0 .. n_moe) the
 *               RMSNorm weights (DEVICE fp32 [1280], 16-byte aligned) or gamma == NULL for all
 *               ones; eps >= 0.  The library does not take ownership of anything in m.
 *   x:          DEVICE fp32 [T, 1280], 16-byte aligned, 1 <= T <= FOCR_T_MAX.
 *   logits:     DEVICE fp32 [T, 129280] or NULL;  argmax: DEVICE int32 [T].
 *   hidden_out: DEVICE fp32 [T, 1280] (the final normed hidden state) or NULL.
 *   workspace:  DEVICE, 256-byte aligned, >= focr_decode_step_workspace_bytes(T) bytes,
 *               zero-filled once before its first use (every step that completes leaves its
 *               control words zero; calls with different T may share it; calls on one
 *               workspace must not overlap).  focr_moe_check on (workspace + 256) reports a
 *               bounded device wait that ran out.
 * Errors: FOCR_ERR_INVALID_ARG for a NULL or incomplete model, T out of range, misaligned or
 * too small buffers; FOCR_ERR_CUDA if a launch fails (stages before it stay queued).
 */
typedef struct focr_decode_model {
    const focr_dense_mlp* dense;        /* decoder layer 0 */
    const focr_moe_layer* const* moe;   /* decoder layers 1 .. n_moe */
    int32_t n_moe;
    const float* const* gamma;          /* n_moe + 1 RMSNorm weights, or NULL */
    float eps;
    const focr_lm_head* head;
} focr_decode_model;
size_t focr_decode_step_workspace_bytes(int32_t T_max);
focr_status focr_decode_step(const focr_decode_model* m, const float* x, int32_t T, float* logits, int32_t* argmax,
                             float* hidden_out, void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ W8A8 linear
 * Source: franken_ocr README, "CPU Backend and Optimizations" -- the int8 decode linears run
 * one quantise-plus-GEMV pass per token: the activation is quantised to int8, integer dot
 * products accumulate exactly in i32 (no saturation) and the two scales are applied at the end;
 * "Command Reference", `focr robot` -- K = 6848 is the worst case of that accumulation.
 * Readings (the pages fix no formula): weights int8 with one scale per row and activations
 * int8 with one scale per token, both symmetric:
 *     s = fp32(max|v|) / 127 (one fp32 division), q = round-half-even(v / s) clamped to
 *     [-127, 127]; an all-zero row or token has s = 0 and q = 0;
 *     acc[t, n] = sum_k q_w[n, k] * q_x[t, k]    (exact: |acc| <= K * 127^2 < 2^31);
 *     y[t, n]   = fp32((fp64(s_w[n]) * fp64(s_x[t])) * fp64(acc[t, n])).
 * Every step is exact integer arithmetic or one correctly rounded IEEE operation, so results
 * are bit-identical to any implementation of the same formula.  Inputs must be finite.
 */
#define FOCR_W8A8_T_MAX 64         /* most tokens one focr_w8a8_gemv call accepts */
#define FOCR_W8A8_K_MAX 133143     /* largest K with K * 127^2 < 2^31 */
#define FOCR_W8A8_N_MAX 67108864   /* most rows of one matrix */

typedef struct focr_w8a8 focr_w8a8;   /* opaque, device-resident, library-owned */

/*
 * focr_w8a8_pack -- quantise w (HOST fp32 [N, K], row-major) to int8 with one scale per row
 * and lay it out on the device (row tiles of 16, k-steps of 32, zero-padded; N * K bytes of
 * codes after padding).  1 <= N <= FOCR_W8A8_N_MAX, 1 <= K <= FOCR_W8A8_K_MAX.  Synchronises.
 * Errors: FOCR_ERR_INVALID_ARG (NULL, sizes out of range), FOCR_ERR_OOM, FOCR_ERR_CUDA.
 */
focr_status focr_w8a8_pack(const float* w, int64_t N, int32_t K, focr_w8a8** out, void* stream);
void focr_w8a8_free(focr_w8a8* m);

/* Canonical codes (int8 [N, K] row-major) and row scales (f32 [N]) to HOST memory; N and K of m. */
focr_status focr_w8a8_export(const focr_w8a8* m, int8_t* codes_host, float* scales_host, int64_t* N, int32_t* K);

/*
 * focr_w8a8_quantize_x -- the activation quantiser alone: x (DEVICE fp32 [T, K], row-major) to
 * qx (DEVICE int8 [T, K]) and sx (DEVICE fp32 [T]).  1 <= T <= FOCR_T_MAX, 1 <= K <=
 * FOCR_W8A8_K_MAX.  Asynchronous on `stream`.
 */
focr_status focr_w8a8_quantize_x(const float* x, int32_t T, int32_t K, int8_t* qx, float* sx, void* stream);

/* Workspace a focr_w8a8_gemv call on m with up to T_max tokens needs (bytes). */
size_t focr_w8a8_workspace_bytes(const focr_w8a8* m, int32_t T_max);

/*
 * focr_w8a8_gemv -- y = W8A8(m, x): quantises x per token, then the integer GEMV and the
 * scales (two launches, chained by programmatic dependent launch).
 *   x: DEVICE fp32 [T, K] row-major (K of m), 1 <= T <= FOCR_W8A8_T_MAX;  y: DEVICE fp32 [T, N].
 *   workspace: DEVICE, 256-byte aligned, >= focr_w8a8_workspace_bytes(m, T) bytes, zero-filled
 *   once before its first use (every completed call leaves its sums and counters zero; calls
 *   on one workspace must not overlap).  Asynchronous on `stream`; focr_w8a8_check reports a
 *   device wait that ran out.
 * Errors: FOCR_ERR_INVALID_ARG (NULL, T out of range, misaligned or short workspace),
 * FOCR_ERR_CUDA (a launch failed).
 */
focr_status focr_w8a8_gemv(const focr_w8a8* m, const float* x, int32_t T, float* y, void* workspace,
                           size_t ws_bytes, void* stream);

/*
 * focr_w8a8_check -- synchronises `stream` and reports whether a focr_w8a8_gemv call on this
 * workspace met a device wait that ran out (its shared-memory pipeline waits are bounded):
 * FOCR_ERR_TIMEOUT (the outputs of that call are not valid; the word is cleared) or FOCR_OK.
 */
focr_status focr_w8a8_check(void* workspace, void* stream);

/* ------------------------------------------------------------------ R-SWA decode attention
 * Source: franken_ocr README, "Design Philosophy" (bounded generated-token KV) and "Architecture"
 * (R-SWA: each generated token attends to every reference token -- visual prefill plus prompt, a
 * frozen block never evicted -- plus the previous 128 generated tokens through a ring buffer);
 * frankenocr.pages.dev, "One forward pass", step 6 (10 heads of dimension 128, a 128-slot ring).
 * Readings (the pages fix no formula): scores are scaled by 1/sqrt(128); q and k arrive with any
 * position encoding applied; the window counts the current token, so it is the ring's 128 slots;
 * generated token p lives in slot p mod 128.  For sequence b with R = ref_len[b] and n = n_gen[b]
 * (generated tokens so far, the current one included):
 *     keys: reference rows 0 .. R-1, generated tokens max(0, n-128) .. n-1 (the current one from
 *     k_new / v_new);  out = sum_j softmax_j(q . k_j / sqrt(128)) v_j, per head;
 *     afterwards slot (n-1) mod 128 of the ring holds k_new / v_new.
 */
#define FOCR_RSWA_HEADS 10
#define FOCR_RSWA_DIM 128
#define FOCR_RSWA_RING 128
#define FOCR_RSWA_RCAP_MAX 32768   /* most reference rows per sequence */
#define FOCR_RSWA_B_MAX 4096       /* most sequences per call */

/* Workspace a focr_rswa_decode call with B sequences and capacity Rcap needs (bytes). */
size_t focr_rswa_workspace_bytes(int32_t B, int32_t Rcap);

/*
 * focr_rswa_decode -- one decode step of one R-SWA attention layer for B sequences.
 *   q, k_new, v_new, out: DEVICE fp32 [B][10][128].
 *   k_ref, v_ref: DEVICE fp32 [B][10][Rcap][128] (row r of sequence b, head h at ((b*10+h)*Rcap+r)*128);
 *     read only.  1 <= Rcap <= FOCR_RSWA_RCAP_MAX.
 *   k_ring, v_ring: DEVICE fp32 [B][10][128][128], read, and slot (n_gen[b]-1) mod 128 written.
 *   ref_len, n_gen: DEVICE int32 [B].  A sequence with ref_len outside [0, Rcap] or n_gen < 1 gets
 *     NaN outputs and keeps its ring.
 *   workspace: DEVICE, 256-byte aligned, >= focr_rswa_workspace_bytes(B, Rcap) bytes (no zero fill
 *     needed).  Every float pointer 16-byte aligned; inputs finite.  1 <= B <= FOCR_RSWA_B_MAX.
 *   Two launches on `stream` (programmatic dependent launch between them); asynchronous.
 * Errors: FOCR_ERR_INVALID_ARG (NULL, misaligned, sizes out of range, short workspace);
 * FOCR_ERR_CUDA (a launch failed).
 */
focr_status focr_rswa_decode(const float* q, const float* k_new, const float* v_new, const float* k_ref,
                             const float* v_ref, const int32_t* ref_len, int32_t Rcap, float* k_ring, float* v_ring,
                             const int32_t* n_gen, int32_t B, float* out, void* workspace, size_t ws_bytes,
                             void* stream);

/*
 * focr_tc_selftest -- diagnostic: one tensor-core tile through the library's tcgen05 primitives
 * (the ones the T > 8 grouped kernel uses), to check them against a host GEMM.
 * D[128, n] = A[128, k] * B[n, k]^T with A, B bf16 bit patterns (DEVICE, row-major, 16-byte
 * aligned) and D fp32 (DEVICE); the MMA reads A from shared memory (a_from_tmem = 0) or from
 * tensor memory after tcgen05.st (a_from_tmem = 1).  n: multiple of 16 in [16, 256]; k: multiple
 * of 64 in [64, 256].  *err (DEVICE int32) is set to 1 if the kernel's bounded wait ran out.
 * Asynchronous on `stream`.  (A check of the hardware path, not part of the layer.)
 */
focr_status focr_tc_selftest(const uint16_t* a, const uint16_t* b, int32_t n, int32_t k, int32_t a_from_tmem,
                             float* d, int32_t* err, void* stream);

/* Thread-local description of the last error (empty string if none). */
const char* focr_last_error(void);

/* Library build string (compiler, arch). */
const char* focr_version(void);

#ifdef __cplusplus
}
#endif
#endif /* FOCR_MOE_H */
