/*
 * CPU oracle for the group-quantised MoE layer and its decode-stack companions.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code with
 * the CUDA path: quantiser, nibble packing, router, softmax/top-k, dispatch,
 * SwiGLU experts, shared expert, combine, RMSNorm and lm_head are all written
 * out here in plain loops with fp64 accumulation, for a reader to check
 * against the pages by eye.  Nothing here is blocked, fused or reordered.
 *
 * Sources (page title, section):
 *   [P1-fwd]  frankenocr.pages.dev, "One forward pass", step 6 (MoE decoder:
 *             64 routed experts + 2 fused shared experts, softmax router,
 *             top 6 picked greedily, no renormalisation) and step 7 (final
 *             RMSNorm, lm_head 1280 -> 129280, greedy decoding).
 *   [P1-q4]   frankenocr.pages.dev, "Four bits, one shared scale" (an int4
 *             weight is a two's-complement nibble sharing one f32 scale with
 *             its group; int4 on the expert bulk, int8 on lm_head, bf16 router).
 *   [P4-dim]  franken_ocr README, "Design Philosophy" (hidden 1280, 64 experts,
 *             top-6, MoE intermediate 896, vocab 129280).
 *   [P4-arch] franken_ocr README, "Architecture" (each expert 1280 -> 896
 *             SiLU-gated, 2 always-on shared experts, final RMSNorm, lm_head).
 *   [P4-rswa] franken_ocr README, "Design Philosophy", bounded generated-token
 *             KV, and "Architecture", R-SWA (every decoder attention layer:
 *             each generated token attends to all reference tokens, a frozen
 *             never-evicted block, plus the previous 128 generated tokens held
 *             in a ring buffer); frankenocr.pages.dev, "One forward pass",
 *             step 6 (ten heads of dimension 128; a read-only reference block
 *             plus a 128-slot sliding ring).
 *   [P4-cpu]  franken_ocr README, "CPU Backend and Optimizations" (int8 decode
 *             linears as a quantise-plus-GEMV pass per token on integer dot
 *             products with exact, non-saturating i32 accumulation) and
 *             "Command Reference", `focr robot` (the selftest's worst-case
 *             K = 6848 i32-accumulation case against a bit-identical scalar
 *             oracle).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - scale s = fp32(max|w|) / Q as one fp32 division (Q = 7 int4, 127 int8);
 *     q = clamp(round_half_even(w / s)) with the fp32 quotient; an all-zero
 *     group has s = 0 and q = 0;
 *   - a group is g consecutive elements along the input (K) axis of one output
 *     row; a row whose length is not a multiple of g ends in a short group whose
 *     scale is taken over that short group;
 *   - nibble order: element 2j in bits 0-3, element 2j+1 in bits 4-7;
 *   - router logits: fp64 sum of exact fp64 products, rounded to fp32; experts
 *     ranked by (fp32 logit descending, index ascending); weights are the fp64
 *     softmax probabilities of the chosen experts, not renormalised;
 *   - the two shared experts are one SwiGLU of width 1792 with weight 1;
 *   - layer output = sum_j w_j * expert_j(x) + shared(x), without a residual.
 *
 * Parity pins: every function here is checked by the CPU tests against hand
 * values, closed forms, brute force or an independent numpy routine.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_DENSE 0   /* plain fp32 values (bf16-exact for bf16 weights) */
#define ORC_QUANT 1   /* int8 codes (int4 codes lie in [-8, 7]) + f32 group scales */

typedef struct {
    int32_t kind;
    int32_t group;      /* elements per scale group along cols (ORC_QUANT) */
    int64_t rows, cols;
    const float* f;     /* [rows, cols] when ORC_DENSE */
    const int8_t* q;    /* [rows, cols] when ORC_QUANT */
    const float* s;     /* [rows, ceil(cols / group)] when ORC_QUANT */
} orc_mat;

typedef struct {
    int32_t E, H, I, Is, topk;
    const uint16_t* router;      /* [E, H] bf16 bit patterns */
    orc_mat gate, up, down;      /* experts stacked along rows: gate/up [E*I, H], down [E*H, I] */
    orc_mat sgate, sup, sdown;   /* shared: [Is, H], [Is, H], [H, Is] */
} orc_moe;

/* ------------------------------------------------------------ bf16 format */

float orc_bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* round to nearest, ties to even (finite inputs) */
uint16_t orc_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lsb = (u >> 16) & 1u;
    return (uint16_t)((u + 0x7FFFu + lsb) >> 16);
}

void orc_round_bf16_array(const float* in, int64_t n, float* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_to_f32(orc_f32_to_bf16(in[i]));
}

/* ------------------------------------------------------------ quantiser [P1-q4] */

int64_t orc_num_groups(int64_t cols, int group) { return (cols + group - 1) / group; }

void orc_quantize_rows(const float* w, int64_t rows, int64_t cols, int group, int bits,
                       int8_t* q, float* s) {
    const int qmax = (bits == 4) ? 7 : 127;
    const int qmin = (bits == 4) ? -8 : -127;
    const int64_t ng = orc_num_groups(cols, group);
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < ng; ++g) {
            const int64_t c0 = g * group;
            const int64_t len = (cols - c0 < group) ? (cols - c0) : group;
            const float* wg = w + r * cols + c0;
            float m = 0.0f;
            for (int64_t i = 0; i < len; ++i) {
                float a = fabsf(wg[i]);
                if (a > m) m = a;
            }
            const float sc = m / (float)qmax;          /* one fp32 division */
            s[r * ng + g] = sc;
            for (int64_t i = 0; i < len; ++i) {
                int v = 0;
                if (sc != 0.0f) {
                    float ratio = wg[i] / sc;           /* fp32 quotient */
                    float rn = nearbyintf(ratio);       /* default mode: half to even */
                    if (rn > (float)qmax) rn = (float)qmax;
                    if (rn < (float)qmin) rn = (float)qmin;
                    v = (int)rn;
                }
                q[r * cols + c0 + i] = (int8_t)v;
            }
        }
    }
}

/* element 2j -> low nibble, 2j+1 -> high nibble; two's complement */
void orc_nibble_pack(const int8_t* q, int64_t n, uint8_t* out) {
    for (int64_t j = 0; j < n / 2; ++j) {
        uint8_t lo = (uint8_t)q[2 * j] & 0x0Fu;
        uint8_t hi = (uint8_t)q[2 * j + 1] & 0x0Fu;
        out[j] = (uint8_t)(lo | (hi << 4));
    }
}

static int8_t nibble_value(uint8_t nib) {
    /* 4-bit two's complement: 0..7 stay, 8..15 mean -8..-1 */
    return (int8_t)(nib >= 8 ? (int)nib - 16 : (int)nib);
}

void orc_nibble_unpack(const uint8_t* packed, int64_t n, int8_t* q) {
    for (int64_t j = 0; j < n / 2; ++j) {
        q[2 * j] = nibble_value(packed[j] & 0x0Fu);
        q[2 * j + 1] = nibble_value((packed[j] >> 4) & 0x0Fu);
    }
}

/* ------------------------------------------------------------ matrices */

static double mat_at(const orc_mat* m, int64_t r, int64_t c) {
    if (m->kind == ORC_DENSE) return (double)m->f[r * m->cols + c];
    const int64_t ng = orc_num_groups(m->cols, m->group);
    return (double)m->q[r * m->cols + c] * (double)m->s[r * ng + c / m->group];
}

/* y[i] = sum_c M[row0 + i, c] * x[c], i < n */
static void gemv_rows(const orc_mat* m, int64_t row0, int64_t n, const double* x, double* y) {
    for (int64_t i = 0; i < n; ++i) {
        double acc = 0.0;
        for (int64_t c = 0; c < m->cols; ++c) acc += mat_at(m, row0 + i, c) * x[c];
        y[i] = acc;
    }
}

void orc_gemv(const orc_mat* m, const double* x, double* y) { gemv_rows(m, 0, m->rows, x, y); }

static double silu(double v) { return v / (1.0 + exp(-v)); }

/* SwiGLU FFN [P4-arch]: y = D (silu(G x) * (U x)); G, U rows [g0, g0+inter), D rows [d0, d0+hid) */
static void swiglu(const orc_mat* G, const orc_mat* U, const orc_mat* D, int64_t g0, int64_t d0,
                   int64_t inter, int64_t hid, const double* x, double* y) {
    double* g = (double*)malloc(sizeof(double) * (size_t)inter);
    double* u = (double*)malloc(sizeof(double) * (size_t)inter);
    gemv_rows(G, g0, inter, x, g);
    gemv_rows(U, g0, inter, x, u);
    for (int64_t i = 0; i < inter; ++i) g[i] = silu(g[i]) * u[i];
    gemv_rows(D, d0, hid, g, y);
    free(g);
    free(u);
}

void orc_swiglu(const orc_mat* G, const orc_mat* U, const orc_mat* D, const double* x, double* y) {
    swiglu(G, U, D, 0, 0, G->rows, D->rows, x, y);
}

/* ------------------------------------------------------------ router [P1-fwd] */

void orc_router_logits(const float* x, const uint16_t* wr, int T, int H, int E, float* logits) {
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int k = 0; k < H; ++k)
                acc += (double)x[(int64_t)t * H + k] * (double)orc_bf16_to_f32(wr[(int64_t)e * H + k]);
            logits[(int64_t)t * E + e] = (float)acc;
        }
}

/* softmax over all E experts, then greedy top-k by (logit desc, index asc);
 * the chosen probabilities are returned as they are (no renormalisation). */
void orc_softmax_topk(const float* logits, int T, int E, int k, int32_t* idx, double* w,
                      double* probs /* nullable [T, E] */) {
    double* p = (double*)malloc(sizeof(double) * (size_t)E);
    char* taken = (char*)malloc((size_t)E);
    for (int t = 0; t < T; ++t) {
        const float* l = logits + (int64_t)t * E;
        double m = (double)l[0];
        for (int e = 1; e < E; ++e) if ((double)l[e] > m) m = (double)l[e];
        double den = 0.0;
        for (int e = 0; e < E; ++e) { p[e] = exp((double)l[e] - m); den += p[e]; }
        for (int e = 0; e < E; ++e) p[e] /= den;
        if (probs) for (int e = 0; e < E; ++e) probs[(int64_t)t * E + e] = p[e];
        memset(taken, 0, (size_t)E);
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e;   /* strict: ties keep the lower index */
            }
            taken[best] = 1;
            idx[(int64_t)t * k + j] = best;
            w[(int64_t)t * k + j] = p[best];
        }
    }
    free(p);
    free(taken);
}

/* stable counting sort of the flat (token, slot) entries t*k + j by expert id */
void orc_dispatch(const int32_t* idx, int T, int k, int E, int32_t* counts, int32_t* offsets,
                  int32_t* perm) {
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t i = 0; i < (int64_t)T * k; ++i) counts[idx[i]]++;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t* cursor = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    for (int e = 0; e < E; ++e) cursor[e] = offsets[e];
    for (int64_t i = 0; i < (int64_t)T * k; ++i) perm[cursor[idx[i]]++] = (int32_t)i;
    free(cursor);
}

/* ------------------------------------------------------------ MoE layer [P1-fwd] */

void orc_moe_forward(const orc_moe* L, const float* x, int T, float* out, float* logits,
                     int32_t* idx, double* w, int32_t* counts, int32_t* offsets, int32_t* perm,
                     int nthreads) {
    orc_router_logits(x, L->router, T, L->H, L->E, logits);
    orc_softmax_topk(logits, T, L->E, L->topk, idx, w, NULL);
    orc_dispatch(idx, T, L->topk, L->E, counts, offsets, perm);
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (int t = 0; t < T; ++t) {
        const int64_t H = L->H;
        double* xd = (double*)malloc(sizeof(double) * (size_t)H);
        double* y = (double*)malloc(sizeof(double) * (size_t)H);
        double* acc = (double*)calloc((size_t)H, sizeof(double));
        for (int64_t c = 0; c < H; ++c) xd[c] = (double)x[(int64_t)t * H + c];
        for (int j = 0; j < L->topk; ++j) {
            const int64_t e = idx[(int64_t)t * L->topk + j];
            const double wj = w[(int64_t)t * L->topk + j];
            swiglu(&L->gate, &L->up, &L->down, e * L->I, e * H, L->I, H, xd, y);
            for (int64_t c = 0; c < H; ++c) acc[c] += wj * y[c];
        }
        swiglu(&L->sgate, &L->sup, &L->sdown, 0, 0, L->Is, H, xd, y);   /* weight 1, always on */
        for (int64_t c = 0; c < H; ++c) out[(int64_t)t * H + c] = (float)(acc[c] + y[c]);
        free(xd);
        free(y);
        free(acc);
    }
    (void)nthreads;
}

/* ------------------------------------------------------------ companions [P1-fwd step 7] */

/* dense SwiGLU MLP (layer 0): out[t] = D (silu(G x_t) * (U x_t)) */
void orc_dense_mlp(const orc_mat* G, const orc_mat* U, const orc_mat* D, const float* x, int T,
                   float* out, int nthreads) {
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (int t = 0; t < T; ++t) {
        const int64_t H = D->rows;
        double* xd = (double*)malloc(sizeof(double) * (size_t)G->cols);
        double* y = (double*)malloc(sizeof(double) * (size_t)H);
        for (int64_t c = 0; c < G->cols; ++c) xd[c] = (double)x[(int64_t)t * G->cols + c];
        swiglu(G, U, D, 0, 0, G->rows, H, xd, y);
        for (int64_t c = 0; c < H; ++c) out[(int64_t)t * H + c] = (float)y[c];
        free(xd);
        free(y);
    }
    (void)nthreads;
}

/* y = x / sqrt(mean(x^2) + eps) * gamma  (gamma == NULL means 1) */
void orc_rmsnorm(const float* x, int T, int H, const float* gamma, double eps, float* out) {
    for (int t = 0; t < T; ++t) {
        double ss = 0.0;
        for (int c = 0; c < H; ++c) ss += (double)x[(int64_t)t * H + c] * (double)x[(int64_t)t * H + c];
        const double inv = 1.0 / sqrt(ss / (double)H + eps);
        for (int c = 0; c < H; ++c) {
            double g = gamma ? (double)gamma[c] : 1.0;
            out[(int64_t)t * H + c] = (float)((double)x[(int64_t)t * H + c] * inv * g);
        }
    }
}

/* lm_head with one int8 scale per row: logit_n = s_n * sum_k q_nk x_k; argmax with
 * ties to the lowest index, taken over the fp32-rounded logits. */
void orc_lm_head(const int8_t* q, const float* s, const float* x, int T, int64_t V, int H,
                 float* logits /* nullable [T, V] */, int32_t* argmax, int nthreads) {
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(static) num_threads(nthreads)
#endif
    for (int t = 0; t < T; ++t) {
        float best = 0.0f;
        int64_t bi = -1;
        for (int64_t n = 0; n < V; ++n) {
            double acc = 0.0;
            for (int k = 0; k < H; ++k) acc += (double)q[n * H + k] * (double)x[(int64_t)t * H + k];
            const float lg = (float)((double)s[n] * acc);
            if (logits) logits[(int64_t)t * V + n] = lg;
            if (bi < 0 || lg > best) { best = lg; bi = n; }
        }
        argmax[t] = (int32_t)bi;
    }
    (void)nthreads;
}

/* ------------------------------------------------------------ W8A8 GEMV [P4-cpu] */
/*
 * Per-token activation quantisation (reading: symmetric, like the weights, one fp32
 * scale per token): s_x = fp32(max_k |x_k|) / 127 as one fp32 division, q_k =
 * clamp(round_half_even(x_k / s_x)) to [-127, 127] with the fp32 quotient; s_x = 0
 * gives q = 0.
 */
void orc_w8a8_quantize_x(const float* x, int T, int K, int8_t* qx, float* sx) {
    for (int t = 0; t < T; ++t) {
        const float* xt = x + (int64_t)t * K;
        float m = 0.0f;
        for (int k = 0; k < K; ++k) {
            float a = fabsf(xt[k]);
            if (a > m) m = a;
        }
        const float sc = m / 127.0f;
        sx[t] = sc;
        for (int k = 0; k < K; ++k) {
            int v = 0;
            if (sc != 0.0f) {
                float rn = nearbyintf(xt[k] / sc);
                if (rn > 127.0f) rn = 127.0f;
                if (rn < -127.0f) rn = -127.0f;
                v = (int)rn;
            }
            qx[(int64_t)t * K + k] = (int8_t)v;
        }
    }
}

/*
 * y[t, n] = s_w[n] * s_x[t] * acc with acc = sum_k q_w[n, k] * q_x[t, k] over the
 * whole row (exact integer; the pages' kernels accumulate it in i32, which holds for
 * K <= 133143 at |q| <= 127), evaluated as fp32( (fp64(s_w) * fp64(s_x)) * fp64(acc) ).
 * The sum is formed in int64 here and returned through acc_out (nullable) so that
 * the tests can check the i32 bound.
 */
void orc_w8a8_gemv(const int8_t* qw, const float* sw, int64_t N, int K, const int8_t* qx, const float* sx,
                   int T, float* y, int64_t* acc_out) {
    for (int t = 0; t < T; ++t)
        for (int64_t n = 0; n < N; ++n) {
            int64_t acc = 0;
            for (int k = 0; k < K; ++k) acc += (int64_t)qw[n * K + k] * (int64_t)qx[(int64_t)t * K + k];
            if (acc_out) acc_out[(int64_t)t * N + n] = acc;
            y[(int64_t)t * N + n] = (float)(((double)sw[n] * (double)sx[t]) * (double)acc);
        }
}

/* ------------------------------------------------------------ R-SWA decode attention [P4-rswa] */
/*
 * One decode step of one attention layer for B sequences, H heads of dimension D, ring of W slots.
 * Sequence b holds ref_len[b] reference rows (row stride D, head stride Rcap * D) and has generated
 * n_gen[b] >= 1 tokens, the current one included; generated token p lives in ring slot p mod W.
 * The current token attends to every reference row and to the last min(n_gen, W) generated
 * tokens, itself included:
 *     s_j = (q . k_j) / sqrt(D),  a_j = exp(s_j - max_i s_i) / sum_i exp(s_i - max_i s_i),
 *     out = sum_j a_j v_j.
 * Its own k and v come from k_new / v_new; afterwards they are stored in slot (n_gen - 1) mod W.
 * Readings where the pages are silent: the scale is 1/sqrt(head dim); q and k arrive with any
 * position encoding already applied; "the previous 128 generated tokens" counts the current one,
 * so the window is exactly the ring's W slots.  A sequence with ref_len outside [0, Rcap] or
 * n_gen < 1 gets NaN outputs and leaves its ring unchanged.
 */
void orc_rswa_decode(const float* q, const float* k_new, const float* v_new, const float* k_ref,
                     const float* v_ref, const int32_t* ref_len, int Rcap, float* k_ring, float* v_ring,
                     const int32_t* n_gen, int B, int H, int D, int W, float* out) {
    double* sc = (double*)malloc(sizeof(double) * ((size_t)Rcap + (size_t)W));
    const double inv = 1.0 / sqrt((double)D);
    for (int b = 0; b < B; ++b) {
        const int R = ref_len[b], n = n_gen[b];
        const int valid = R >= 0 && R <= Rcap && n >= 1;
        const int p0 = n > W ? n - W : 0;   /* oldest generated token in the window */
        for (int h = 0; h < H; ++h) {
            const size_t bh = (size_t)b * H + h;
            const float* qv = q + bh * D;
            const float* kr = k_ref + bh * (size_t)Rcap * D;
            const float* vr = v_ref + bh * (size_t)Rcap * D;
            float* kg = k_ring + bh * (size_t)W * D;
            float* vg = v_ring + bh * (size_t)W * D;
            float* o = out + bh * D;
            if (!valid) {
                for (int d = 0; d < D; ++d) o[d] = NAN;
                continue;
            }
            /* keys in order: reference rows, then generated tokens oldest to newest */
            int nk = 0;
            for (int r = 0; r < R; ++r) {
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += (double)qv[d] * (double)kr[(size_t)r * D + d];
                sc[nk++] = acc * inv;
            }
            for (int p = p0; p < n; ++p) {
                const float* kp = p == n - 1 ? k_new + bh * D : kg + (size_t)(p % W) * D;
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += (double)qv[d] * (double)kp[d];
                sc[nk++] = acc * inv;
            }
            double m = sc[0];
            for (int j = 1; j < nk; ++j)
                if (sc[j] > m) m = sc[j];
            double den = 0.0;
            for (int j = 0; j < nk; ++j) den += exp(sc[j] - m);
            for (int d = 0; d < D; ++d) {
                double acc = 0.0;
                int j = 0;
                for (int r = 0; r < R; ++r, ++j) acc += exp(sc[j] - m) * (double)vr[(size_t)r * D + d];
                for (int p = p0; p < n; ++p, ++j) {
                    const float* vp = p == n - 1 ? v_new + bh * D : vg + (size_t)(p % W) * D;
                    acc += exp(sc[j] - m) * (double)vp[d];
                }
                o[d] = (float)(acc / den);
            }
            const int slot = (n - 1) % W;
            for (int d = 0; d < D; ++d) {
                kg[(size_t)slot * D + d] = k_new[bh * D + d];
                vg[(size_t)slot * D + d] = v_new[bh * D + d];
            }
        }
    }
    free(sc);
}

int orc_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
