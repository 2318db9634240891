/*
 * moe_oracle.c -- plain, slow, single-threaded CPU reference of the fused MoE layer
 * forward.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the bench's CPU
 * baseline call it; the product (the CUDA library) never does, and the two share no
 * code, header, table or helper.
 *
 * Arithmetic: FP64 everywhere, with these rounding points and nothing else:
 *   - BF16 inputs are widened exactly (bit pattern << 16).
 *   - router logits are FP32: one rounding of the FP64 dot product.
 *   - sigmoid scores are FP32: one rounding of the FP64 value 1/(1+exp(-l)).
 *   - selection keys are FP32: score + bias in FP32 arithmetic.
 *   - routing weights are FP32: one rounding of the FP64 ratio.
 *   - the expert activation h is rounded to BF16 (it feeds a BF16 GEMM).
 *   - the routed sum is rounded to BF16, the shared-expert output is rounded to
 *     BF16, and their sum is rounded to BF16.
 *   - optional routed scale: the routed sum is multiplied by it before its BF16
 *     rounding.
 *   - optional shared-expert gate: an FP32 logit (one rounding of the FP64 dot product
 *     of x with the gate row) through the same FP32 sigmoid as the router; the shared
 *     expert's FP64 output is multiplied by it before its BF16 rounding.
 *   - optional caller-computed shared output (BF16): added in place of the shared
 *     expert's own output, in the same order.
 *
 * Sources (page title, section):
 *   [P4] "Laguna exact M=8 BF16-input router top-k preregistration",
 *        "Question and arithmetic contract" and "Four-card component gate".
 *   [P2] "MTP1 isolated gather/shared-add closure" (b70-optimization-lab, 2026-07-16),
 *        description of moe_gather_shared_add_m2 and its route classes.
 *   [P5] FlashInfer PR #4646 "add cuTile fused MoE backend for BF16 and NVFP4 Unified
 *        MoE", description (SwiGLU gated / ReLU2 ungated) and walkthrough (routing
 *        permutation, grouped BF16 GEMM, weighted output combination).
 *   [P3] vLLM PR #64636 "SM80 skinny GEMM plans", cold-L2 table: the shared-expert gate,
 *        a (1, H) linear of the decode step.
 * The routed scale follows [P4] "Question and arithmetic contract" (the router's own
 * scale is 1.0; the configured routed scale is applied later to the routed output).  The
 * caller-computed shared output, optionally aliased by the layer output, follows [P2]
 * (the fused gather takes the completed shared-expert output; separate-output and
 * shared-output-alias forms).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_SCORE_SOFTMAX 0
#define ORACLE_SCORE_SIGMOID 1
#define ORACLE_ACT_SWIGLU 0
#define ORACLE_ACT_RELU2 1

/* ---- number formats -------------------------------------------------------------- */

/* BF16 -> double: a BF16 value is the upper half of an FP32 bit pattern. */
double oracle_bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* double -> BF16, round to nearest, ties to even, in one step from the double.
 * BF16 keeps 8 significant bits and FP32's exponent range: the quantum of a normal
 * value a in [2^(e-1), 2^e) is 2^(e-8); below 2^-126 the quantum is 2^-133. */
uint16_t oracle_double_to_bf16(double v) {
    if (isnan(v)) return 0x7fc0;
    int neg = signbit(v) ? 1 : 0;
    double a = fabs(v);
    uint16_t sign = neg ? 0x8000 : 0;
    if (a == 0.0) return sign;
    if (isinf(a)) return sign | 0x7f80;
    int e;
    (void)frexp(a, &e);                 /* a = m * 2^e, m in [0.5, 1) */
    int q = e - 8;
    if (e - 1 < -126) q = -133;
    double r = nearbyint(ldexp(a, -q)); /* default mode: nearest, ties to even */
    double res = ldexp(r, q);
    if (res >= ldexp(1.0, 128)) return sign | 0x7f80;
    float f = (float)res;               /* exact: at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return sign | (uint16_t)(u >> 16);
}

static double bf16_round(double v) { return oracle_bf16_to_double(oracle_double_to_bf16(v)); }

/* ---- router --------------------------------------------------------------------- */

/* l[t,e] = fp32( sum_h x[t,h] * Wr[e,h] ), the sum taken in FP64. */
void oracle_router_logits(const uint16_t* x, const uint16_t* wr, int T, int H, int E,
                          float* logits) {
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            double s = 0.0;
            for (int h = 0; h < H; ++h)
                s += oracle_bf16_to_double(x[(size_t)t * H + h]) *
                     oracle_bf16_to_double(wr[(size_t)e * H + h]);
            logits[(size_t)t * E + e] = (float)s;
        }
}

/* FP32 sigmoid, correctly rounded from the FP64 value [P4: "FP32 sigmoid"]. */
float oracle_sigmoid_f32(float l) { return (float)(1.0 / (1.0 + exp(-(double)l))); }

/* One row of the router contract [P4]: score, biased key for selection only, top-K by
 * (key descending, expert id ascending), weights from the unbiased scores.
 *   sigmoid: s_e = sigmoid(l_e) in FP32; key_e = s_e + b_e in FP32.
 *   softmax: key_e = l_e (softmax is monotone in the logit).
 *   weights, renorm: sigmoid -> s_k / sum_j s_j ; softmax -> exp(l_k-l_max)/sum_j exp(l_j-l_max),
 *   sums over the selected experts in slot order; without renorm, sigmoid -> s_k and
 *   softmax -> the full softmax probability over all E experts. */
static void topk_row(const float* l, int E, int K, int score, const float* bias, int renorm,
                     float* w_out, int32_t* id_out, unsigned char* taken, float* key) {
    for (int e = 0; e < E; ++e) {
        if (score == ORACLE_SCORE_SIGMOID) {
            float s = oracle_sigmoid_f32(l[e]);
            float b = bias ? bias[e] : 0.0f;
            key[e] = s + b; /* FP32 addition */
        } else {
            key[e] = bias ? l[e] + bias[e] : l[e];
        }
        taken[e] = 0;
    }
    for (int k = 0; k < K; ++k) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e]) continue;
            if (best < 0 || key[e] > key[best]) best = e; /* equal keys: keep lower id */
        }
        taken[best] = 1;
        id_out[k] = best;
    }
    if (score == ORACLE_SCORE_SIGMOID) {
        double sum = 0.0;
        for (int k = 0; k < K; ++k) sum += (double)oracle_sigmoid_f32(l[id_out[k]]);
        for (int k = 0; k < K; ++k) {
            double s = (double)oracle_sigmoid_f32(l[id_out[k]]);
            w_out[k] = renorm ? (float)(s / sum) : (float)s;
        }
    } else {
        double lmax = (double)l[0];
        for (int e = 1; e < E; ++e)
            if ((double)l[e] > lmax) lmax = (double)l[e];
        double sum = 0.0;
        if (renorm) {
            for (int k = 0; k < K; ++k) sum += exp((double)l[id_out[k]] - lmax);
        } else {
            for (int e = 0; e < E; ++e) sum += exp((double)l[e] - lmax);
        }
        for (int k = 0; k < K; ++k) w_out[k] = (float)(exp((double)l[id_out[k]] - lmax) / sum);
    }
}

/* Router top-k over M rows of logits.  logits_is_bf16: logits are BF16 bit patterns
 * widened exactly to FP32 [P4: "exact widening to FP32"]; else FP32.
 * Outputs per row m and slot k: weight w[m,k], expert id[m,k], source index
 * src[m,k] = k*M + m [P4 gate: "slot * 8 + row" at M = 8]. */
int oracle_topk(const void* logits, int logits_is_bf16, int M, int E, int K, int score,
                const float* bias, int renorm, float* w, int32_t* ids, int32_t* src) {
    if (M < 0 || E < 1 || K < 1 || K > E) return -1;
    float* row = (float*)malloc(sizeof(float) * (size_t)E);
    float* key = (float*)malloc(sizeof(float) * (size_t)E);
    unsigned char* taken = (unsigned char*)malloc((size_t)E);
    for (int m = 0; m < M; ++m) {
        for (int e = 0; e < E; ++e) {
            if (logits_is_bf16)
                row[e] = (float)oracle_bf16_to_double(((const uint16_t*)logits)[(size_t)m * E + e]);
            else
                row[e] = ((const float*)logits)[(size_t)m * E + e];
        }
        topk_row(row, E, K, score, bias, renorm, w + (size_t)m * K, ids + (size_t)m * K, taken, key);
        for (int k = 0; k < K; ++k) src[(size_t)m * K + k] = k * M + m;
    }
    free(row);
    free(key);
    free(taken);
    return 0;
}

/* ---- permutation [P5: routing permutation scan] ------------------------------------ */

/* counts per expert; offsets = exclusive prefix sum (offsets[E] = M*K); perm lists the
 * source indices k*M + m grouped by expert in ascending expert order and, within an
 * expert, in ascending token m (unpadded); inv[src] = position of src in perm.
 * Returns -1 (and writes nothing further) if an id is outside [0, E). */
int oracle_permute(const int32_t* ids, int M, int K, int E, int32_t* offsets, int32_t* perm,
                   int32_t* inv) {
    for (size_t i = 0; i < (size_t)M * K; ++i)
        if (ids[i] < 0 || ids[i] >= E) return -1;
    int pos = 0;
    for (int e = 0; e < E; ++e) {
        offsets[e] = pos;
        for (int m = 0; m < M; ++m)
            for (int k = 0; k < K; ++k)
                if (ids[(size_t)m * K + k] == e) {
                    int s = k * M + m;
                    perm[pos] = s;
                    inv[s] = pos;
                    ++pos;
                }
    }
    offsets[E] = pos;
    return 0;
}

/* ---- expert feed-forward [P5: SwiGLU (gated) / ReLU2 (ungated)] -------------------- */

/* One expert applied to one token.  w1 rows: SwiGLU -> [0,I) gate, [I,2I) up; ReLU2 ->
 * [0,I).  h_i = silu(gate_i) * up_i with silu(z) = z / (1 + exp(-z)), or max(g_i,0)^2;
 * h is rounded to BF16 (the operand of the second BF16 GEMM).  y = W2 . h in FP64. */
static void expert_ffn(const uint16_t* w1, const uint16_t* w2, int act, int H, int I,
                       const double* x, double* h, double* y) {
    for (int i = 0; i < I; ++i) {
        double g = 0.0;
        for (int c = 0; c < H; ++c) g += oracle_bf16_to_double(w1[(size_t)i * H + c]) * x[c];
        double a;
        if (act == ORACLE_ACT_SWIGLU) {
            double u = 0.0;
            for (int c = 0; c < H; ++c) u += oracle_bf16_to_double(w1[(size_t)(I + i) * H + c]) * x[c];
            a = g / (1.0 + exp(-g)) * u;
        } else {
            a = g > 0.0 ? g * g : 0.0;
        }
        h[i] = bf16_round(a);
    }
    for (int f = 0; f < H; ++f) {
        double s = 0.0;
        for (int i = 0; i < I; ++i) s += oracle_bf16_to_double(w2[(size_t)f * I + i]) * h[i];
        y[f] = s;
    }
}

/* Layer description shared with the Python wrapper (ctypes mirrors this layout). */
typedef struct {
    int T, H, I, E, K, act, score, renorm, I_shared;
    const uint16_t* router_w;    /* [E,H] or NULL when router_logits is given */
    const float* router_logits;  /* [T,E] FP32 or NULL */
    const float* bias;           /* [E] or NULL */
    const uint16_t* w13;         /* [E, 2I or I, H] */
    const uint16_t* w2;          /* [E, H, I] */
    const uint16_t* ws13;        /* [2I_s or I_s, H] or NULL */
    const uint16_t* ws2;         /* [H, I_s] or NULL */
    double routed_scale;         /* multiplies the routed sum before its BF16 rounding */
    const uint16_t* shared_gate; /* [H] gate row of the shared expert, or NULL */
    const uint16_t* shared_out;  /* [T,H] caller-computed shared output (BF16), or NULL */
} oracle_layer;

/* Forward for a subset of tokens rows[0..nrows) of a T-token batch (tokens are
 * independent, so a subset is exact).  x is the full [T,H] input.  Outputs, per listed
 * row r: out[r,H] BF16 bits; optional logits[r,E], w[r,K], ids[r,K].
 * Combine order [P2]: routed FP32 (here FP64) accumulation over the slots in slot
 * order -> (times the routed scale) -> BF16 -> add the BF16 shared-expert output (gated,
 * or the caller's) -> BF16. */
int oracle_forward_rows(const oracle_layer* L, const uint16_t* x, const int32_t* rows, int nrows,
                        uint16_t* out, float* logits_out, float* w_out, int32_t* ids_out) {
    const int H = L->H, I = L->I, E = L->E, K = L->K, T = L->T;
    if (K < 1 || K > E || K > 1024) return -1;
    for (int r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= T) return -2;
    const size_t rows1 = (size_t)(L->act == ORACLE_ACT_SWIGLU ? 2 * I : I);
    const int Is = L->I_shared;
    double* xd = (double*)malloc(sizeof(double) * (size_t)H);
    double* acc = (double*)malloc(sizeof(double) * (size_t)H);
    double* y = (double*)malloc(sizeof(double) * (size_t)H);
    int hmax = I > Is ? I : Is;
    double* h = (double*)malloc(sizeof(double) * (size_t)(hmax > 0 ? hmax : 1));
    float* l = (float*)malloc(sizeof(float) * (size_t)E);
    float* key = (float*)malloc(sizeof(float) * (size_t)E);
    unsigned char* taken = (unsigned char*)malloc((size_t)E);
    float w[1024];
    int32_t id[1024];
    for (int r = 0; r < nrows; ++r) {
        const int t = rows[r];
        for (int c = 0; c < H; ++c) xd[c] = oracle_bf16_to_double(x[(size_t)t * H + c]);
        if (L->router_logits) {
            for (int e = 0; e < E; ++e) l[e] = L->router_logits[(size_t)t * E + e];
        } else {
            oracle_router_logits(x + (size_t)t * H, L->router_w, 1, H, E, l);
        }
        topk_row(l, E, K, L->score, L->bias, L->renorm, w, id, taken, key);
        for (int c = 0; c < H; ++c) acc[c] = 0.0;
        for (int k = 0; k < K; ++k) {
            const int e = id[k];
            expert_ffn(L->w13 + (size_t)e * rows1 * H, L->w2 + (size_t)e * H * I, L->act, H, I, xd, h, y);
            for (int c = 0; c < H; ++c) acc[c] += (double)w[k] * y[c];
        }
        for (int c = 0; c < H; ++c) {
            double routed = bf16_round(L->routed_scale * acc[c]);
            acc[c] = routed;
        }
        if (Is > 0) {
            expert_ffn(L->ws13, L->ws2, L->act, H, Is, xd, h, y);
            double gate = 1.0;
            if (L->shared_gate) {
                float lg;
                oracle_router_logits(x + (size_t)t * H, L->shared_gate, 1, H, 1, &lg);
                gate = (double)oracle_sigmoid_f32(lg);
            }
            for (int c = 0; c < H; ++c) acc[c] = acc[c] + bf16_round(gate * y[c]);
        } else if (L->shared_out) {
            for (int c = 0; c < H; ++c) acc[c] = acc[c] + oracle_bf16_to_double(L->shared_out[(size_t)t * H + c]);
        }
        for (int c = 0; c < H; ++c) out[(size_t)r * H + c] = oracle_double_to_bf16(acc[c]);
        if (logits_out) memcpy(logits_out + (size_t)r * E, l, sizeof(float) * (size_t)E);
        if (w_out) memcpy(w_out + (size_t)r * K, w, sizeof(float) * (size_t)K);
        if (ids_out) memcpy(ids_out + (size_t)r * K, id, sizeof(int32_t) * (size_t)K);
    }
    free(xd);
    free(acc);
    free(y);
    free(h);
    free(l);
    free(key);
    free(taken);
    return 0;
}
