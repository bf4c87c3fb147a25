/*
 * moe_oracle.c -- CPU oracle of the dots-style fine-grained MoE FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain, obviously
 * correct restatement of what the layer computes.  Only the test suite, the
 * smoke check and the bench's CPU-baseline leg load it.  It shares no code,
 * header, table or helper with the CUDA library, and the CUDA library never
 * calls it.
 *
 * Sources (web pages; cited by title and section):
 *  [MLQM]  "dots3-note 架构深度解析：16B 激活参数的 280B MoE 如何实现高效推理"
 *          (mlqm.cn), section "稀疏激活：Top-8 路由如何把计算量压缩 17 倍" and
 *          the table "核心架构参数一览": sigmoid scoring, noaux_tc routing,
 *          top-8 of 256 routed experts + 1 shared expert, norm_topk_prob,
 *          hidden 5120, moe_intermediate_size 1536, BF16/FP8.
 *  [DEEP]  "Xiaohongshu dots3 note Open Source Deep Dive: 280B MoE Multimodal
 *          Model" (happyrock.cloud), §3.1 Expert Routing Mechanism (layer
 *          sketch: gate -> scores -> top-k -> renormalise -> shared + weighted
 *          routed sum), §3.3 layer diagram ("Weighted sum", shared "add"),
 *          §8.2 Ascend Adaptation Architecture (FUSED_MC2:
 *          dispatch -> gmm1 -> swiglu -> gmm2 -> combine).
 *  [DOTS1] "🤗 Transformers 中的 dots.llm1（Dots1）模型" (blog.gitcode.com),
 *          table "MoE 路由与专家相关字段" (n_group, topk_group, norm_topk_prob,
 *          routed_scaling_factor, moe_intermediate_size) and the parallel-plan
 *          paragraph (packed gate_up_proj; hidden_act silu in the config table).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - scores are sigmoid, not the sketch's softmax ([MLQM] states sigmoid);
 *  - noaux_tc: choice key c = sigmoid(logit) + bias; weights use the unbiased
 *    sigmoid; the bias is an input;
 *  - group score = sum of the top `group_topn` (2) choice keys in a group of
 *    E/n_group contiguous experts; keep the top `topk_group` groups;
 *  - ties in every top-k: larger key first, equal keys -> lower index first;
 *    a NaN key (NaN logit or bias) counts as -infinity;
 *  - weights: s_j / (s_0 + s_1 + ... + s_{k-1}) summed in slot order in fp32,
 *    then times routed_scaling_factor;
 *  - expert FFN is SwiGLU: down(SiLU(gate x) * up x), gate rows 0..I-1 and up
 *    rows I..2I-1 of a packed [2I, H] matrix; the shared expert is one SwiGLU
 *    of width n_shared*I;
 *  - routing decisions are taken in fp32 with the exp below, so that the CUDA
 *    router can reach the same bits; everything else is fp64.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int32_t T, H, E, k, I, n_shared;
    int32_t n_group, topk_group, group_topn;
    int32_t norm_topk_prob;
    float routed_scaling_factor;
    int32_t fp8; /* 0: bf16 operands; 1: e4m3 operands with 128-blocks */
} orc_config;

/* ------------------------------------------------------------------------ */
/* Number formats                                                           */
/* ------------------------------------------------------------------------ */

/* bf16 is the top 16 bits of an IEEE binary32: exact widening. */
float orc_bf16_to_f32(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* binary32 -> bf16, round to nearest even (NaN kept quiet). */
uint16_t orc_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* OCP FP8 E4M3 ("e4m3fn"): 1 sign, 4 exponent bits (bias 7), 3 mantissa
 * bits; no infinities; S.1111.111 is NaN; largest finite 448. */
float orc_e4m3_to_f32(uint8_t q) {
    int sign = q >> 7;
    int ex = (q >> 3) & 15;
    int man = q & 7;
    double v;
    if (ex == 15 && man == 7) return NAN;
    if (ex == 0)
        v = ldexp((double)man, -9); /* subnormal: man/8 * 2^(1-7) */
    else
        v = ldexp(1.0 + man / 8.0, ex - 7);
    return (float)(sign ? -v : v);
}

/* binary32 -> E4M3 by round-to-nearest-even with saturation to +-448
 * (values beyond the largest finite code clamp to it).  Written as a search
 * over the 127 non-negative finite codes, which is the definition itself:
 * pick the nearest representable magnitude, ties to the even code. */
uint8_t orc_f32_to_e4m3(float f) {
    if (f != f) return 0x7f;
    uint8_t sign = (f < 0.0f || (f == 0.0f && signbit(f))) ? 0x80 : 0x00;
    double a = fabs((double)f);
    if (a >= 448.0) return (uint8_t)(sign | 0x7e);
    int best = 0;
    double best_err = a;
    for (int c = 1; c <= 0x7e; ++c) {
        double v = (double)orc_e4m3_to_f32((uint8_t)c);
        double err = fabs(v - a);
        if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_err = err;
        }
    }
    return (uint8_t)(sign | best);
}

/* ------------------------------------------------------------------------ */
/* Router arithmetic in fp32 (a decision is an integer, so both sides must   */
/* take it in the same precision with the same operations)                   */
/* ------------------------------------------------------------------------ */

/* e^x in binary32 by Cody & Waite argument reduction (x = n ln2 + r with ln2
 * split into a 16-bit head and a binary32 tail, so n*LN2_HI is exact for
 * |n| < 2^8) followed by the degree-7 Taylor polynomial of e^r on
 * |r| <= ln2/2, evaluated by Horner's rule with fused multiply-adds, and an
 * exact scaling by 2^n.  The argument is clamped to [-86, 86] so that every
 * intermediate and the result stay normal binary32 numbers.
 * Every operation is an IEEE-754 correctly rounded +, *, fma or
 * round-to-integral, so any IEEE machine evaluating the same sequence gets
 * the same bits. */
#define ORC_LN2_HI 0x1.62e4p-1f        /* ln 2 to 16 significant bits  */
#define ORC_LN2_LO 0x1.7f7d1cp-20f     /* ln 2 - ORC_LN2_HI            */
#define ORC_INV_LN2 0x1.715476p+0f     /* 1/ln 2                       */
float orc_exp(float x) {
    if (x > 86.0f) x = 86.0f;
    if (x < -86.0f) x = -86.0f;
    float nf = rintf(x * ORC_INV_LN2);
    float r = fmaf(-nf, ORC_LN2_HI, x);
    r = fmaf(-nf, ORC_LN2_LO, r);
    /* Taylor coefficients 1/j!, j = 7..0, each rounded to binary32 */
    float p = 0x1.a01a02p-13f;        /* 1/5040 */
    p = fmaf(p, r, 0x1.6c16c2p-10f);  /* 1/720  */
    p = fmaf(p, r, 0x1.111112p-7f);   /* 1/120  */
    p = fmaf(p, r, 0x1.555556p-5f);   /* 1/24   */
    p = fmaf(p, r, 0x1.555556p-3f);   /* 1/6    */
    p = fmaf(p, r, 0x1.0p-1f);        /* 1/2    */
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    int n = (int)nf;
    uint32_t bits = (uint32_t)(n + 127) << 23; /* 2^n, n in [-125, 125] */
    float scale;
    memcpy(&scale, &bits, 4);
    return p * scale;
}

/* Sigmoid score of a router logit ([MLQM] "sigmoid评分函数"):
 * s = 1 / (1 + e^{-l}), one binary32 add and one correctly rounded divide. */
float orc_sigmoid(float l) {
    float e = orc_exp(-l);
    return 1.0f / (1.0f + e);
}

/* ------------------------------------------------------------------------ */
/* Step a1: router logits L = x W_g^T ([DEEP] §3.1 gate; §3.3 "Gate (Linear  */
/* 5120->256)").  Reference value in fp64 from the bf16 operands.            */
/* ------------------------------------------------------------------------ */
void orc_router_logits(const orc_config* cfg, const uint16_t* x, const uint16_t* wg,
                       double* logits) {
    const int T = cfg->T, H = cfg->H, E = cfg->E;
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int h = 0; h < H; ++h)
                acc += (double)orc_bf16_to_f32(x[(size_t)t * H + h]) *
                       (double)orc_bf16_to_f32(wg[(size_t)e * H + h]);
            logits[(size_t)t * E + e] = acc;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Steps a2-a4: sigmoid scores, noaux_tc biased (optionally group-limited)   */
/* top-k, renormalised unbiased weights.                                     */
/*   [MLQM] sigmoid scoring + noaux_tc + norm_topk_prob, top-8 of 256;        */
/*   [DOTS1] n_group / topk_group (choose groups by group score, then the    */
/*   top-k inside them), routed_scaling_factor;                              */
/*   [DEEP] §3.1 sketch: top-k then scores / sum(scores).                     */
/* logits: fp32 [T,E]; bias: fp32 [E]; idx: [T,k] slot order (key           */
/* descending, lower expert first on ties); w: [T,k]; gap (optional): per    */
/* token, key of the k-th choice minus key of the best unchosen eligible     */
/* expert (INFINITY when none is left).  Returns 0, or -1 on a bad config.   */
/* ------------------------------------------------------------------------ */
int orc_route(const orc_config* cfg, const float* logits, const float* bias, int32_t* idx,
              float* w, float* gap) {
    const int T = cfg->T, E = cfg->E, k = cfg->k;
    const int G = cfg->n_group < 1 ? 1 : cfg->n_group;
    const int tg = cfg->topk_group < 1 ? 1 : cfg->topk_group;
    const int tn = cfg->group_topn < 1 ? 1 : cfg->group_topn;
    if (k < 1 || k > E || E % G != 0 || tg > G || tn > E / G || k > tg * (E / G)) return -1;
    const int gsize = E / G;
    int status = 0;
#pragma omp parallel
    {
        float* s = (float*)malloc(sizeof(float) * E);
        float* c = (float*)malloc(sizeof(float) * E);
        char* eligible = (char*)malloc(E);
        char* taken = (char*)malloc(E);
        float* gscore = (float*)malloc(sizeof(float) * G);
        char* gkeep = (char*)malloc(G);
        float* top = (float*)malloc(sizeof(float) * tn);
#pragma omp for schedule(static)
        for (int t = 0; t < T; ++t) {
            for (int e = 0; e < E; ++e) {
                s[e] = orc_sigmoid(logits[(size_t)t * E + e]);
                c[e] = s[e] + bias[e]; /* the bias only steers the choice */
                if (c[e] != c[e]) c[e] = -INFINITY; /* NaN ranks below numbers */
                eligible[e] = 1;
                taken[e] = 0;
            }
            if (G > 1) {
                /* group score: the tn largest keys of the group, added from
                 * the largest down */
                for (int g = 0; g < G; ++g) {
                    char* used = taken; /* scratch, reset below */
                    for (int j = 0; j < tn; ++j) {
                        int best = -1;
                        for (int e = g * gsize; e < (g + 1) * gsize; ++e)
                            if (!used[e] && (best < 0 || c[e] > c[best])) best = e;
                        top[j] = c[best];
                        used[best] = 1;
                    }
                    float acc = top[0];
                    for (int j = 1; j < tn; ++j) acc = acc + top[j];
                    gscore[g] = acc != acc ? -INFINITY : acc;
                    for (int e = g * gsize; e < (g + 1) * gsize; ++e) used[e] = 0;
                }
                for (int g = 0; g < G; ++g) gkeep[g] = 0;
                for (int j = 0; j < tg; ++j) {
                    int best = -1;
                    for (int g = 0; g < G; ++g)
                        if (!gkeep[g] && (best < 0 || gscore[g] > gscore[best])) best = g;
                    gkeep[best] = 1;
                }
                for (int e = 0; e < E; ++e) eligible[e] = gkeep[e / gsize];
            }
            for (int j = 0; j < k; ++j) {
                int best = -1;
                for (int e = 0; e < E; ++e)
                    if (eligible[e] && !taken[e] && (best < 0 || c[e] > c[best])) best = e;
                taken[best] = 1;
                idx[(size_t)t * k + j] = best;
            }
            if (gap) {
                int next = -1;
                for (int e = 0; e < E; ++e)
                    if (eligible[e] && !taken[e] && (next < 0 || c[e] > c[next])) next = e;
                gap[t] = next < 0 ? INFINITY : c[idx[(size_t)t * k + k - 1]] - c[next];
            }
            float sum = 0.0f;
            for (int j = 0; j < k; ++j) sum = sum + s[idx[(size_t)t * k + j]];
            for (int j = 0; j < k; ++j) {
                float v = s[idx[(size_t)t * k + j]];
                if (cfg->norm_topk_prob) v = v / sum;
                w[(size_t)t * k + j] = v * cfg->routed_scaling_factor;
            }
        }
        free(s); free(c); free(eligible); free(taken); free(gscore); free(gkeep); free(top);
    }
    return status;
}

/* ------------------------------------------------------------------------ */
/* Step a5: dispatch order ([DEEP] §8.2 "dispatch"; grouped GEMM needs the   */
/* tokens of one expert contiguous).  Counting sort of the flattened slots   */
/* s = t*k + j by expert, stable in s, so rows of one expert are in token    */
/* order.  offsets [E+1], rows [T*k] = source token of each sorted row,      */
/* pos [T*k] = sorted row of each slot.                                      */
/* ------------------------------------------------------------------------ */
void orc_permute(const orc_config* cfg, const int32_t* idx, int32_t* offsets, int32_t* rows,
                 int32_t* pos) {
    const int E = cfg->E, n = cfg->T * cfg->k;
    int32_t* fill = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    for (int e = 0; e <= E; ++e) offsets[e] = 0;
    for (int s = 0; s < n; ++s) offsets[idx[s] + 1] += 1;
    for (int e = 0; e < E; ++e) offsets[e + 1] += offsets[e];
    for (int s = 0; s < n; ++s) {
        int e = idx[s];
        int r = offsets[e] + fill[e]++;
        rows[r] = s / cfg->k;
        pos[s] = r;
    }
    free(fill);
}

/* ------------------------------------------------------------------------ */
/* FP8 activation recipe (per token, per 128 columns): scale = amax / 448,   */
/* q = E4M3_RNE_satfinite(v / scale); an all-zero block gets scale 1.        */
/* Decided in binary32, like the device, because it produces integer codes.  */
/* ------------------------------------------------------------------------ */
void orc_quant_act_e4m3(int rows, int cols, const float* v, uint8_t* q, float* scale) {
    const int nb = (cols + 127) / 128;
    for (int r = 0; r < rows; ++r) {
        for (int b = 0; b < nb; ++b) {
            int c0 = b * 128, c1 = c0 + 128 < cols ? c0 + 128 : cols;
            float amax = 0.0f;
            for (int c = c0; c < c1; ++c) {
                float a = fabsf(v[(size_t)r * cols + c]);
                if (a > amax) amax = a;
            }
            float s = amax > 0.0f ? amax / 448.0f : 1.0f;
            scale[(size_t)r * nb + b] = s;
            for (int c = c0; c < c1; ++c)
                q[(size_t)r * cols + c] = orc_f32_to_e4m3(v[(size_t)r * cols + c] / s);
        }
    }
}

/* A weight matrix [rows, cols] either bf16, or e4m3 codes with one binary32
 * scale per 128x128 block (block (r/128, c/128), row-major over blocks). */
typedef struct {
    const void* data;
    const float* scale;
    int32_t rows, cols;
} orc_weight;

static void weight_row(const orc_weight* w, int fp8, int r, double* out) {
    if (!fp8) {
        const uint16_t* p = (const uint16_t*)w->data + (size_t)r * w->cols;
        for (int c = 0; c < w->cols; ++c) out[c] = (double)orc_bf16_to_f32(p[c]);
    } else {
        const uint8_t* p = (const uint8_t*)w->data + (size_t)r * w->cols;
        const int nbc = (w->cols + 127) / 128;
        for (int c = 0; c < w->cols; ++c)
            out[c] = (double)orc_e4m3_to_f32(p[c]) *
                     (double)w->scale[(size_t)(r / 128) * nbc + c / 128];
    }
}

/* Operand values as the expert GEMMs see them: in fp8 mode an activation row
 * is first quantised by the recipe above and dequantised. */
static void act_operand(int fp8, int n, const double* v, double* out, uint8_t* qbuf,
                        float* fbuf, float* sbuf) {
    if (!fp8) {
        for (int i = 0; i < n; ++i) out[i] = v[i];
        return;
    }
    for (int i = 0; i < n; ++i) fbuf[i] = (float)v[i];
    orc_quant_act_e4m3(1, n, fbuf, qbuf, sbuf);
    for (int i = 0; i < n; ++i)
        out[i] = (double)orc_e4m3_to_f32(qbuf[i]) * (double)sbuf[i / 128];
}

/* SiLU(g) = g * sigmoid(g) = g / (1 + e^{-g}) ([DOTS1] hidden_act "silu"). */
static double silu(double g) { return g / (1.0 + exp(-g)); }

/* One SwiGLU expert on one token ([DEEP] §8.2 "gmm1 -> swiglu -> gmm2";
 * [DOTS1] packed gate_up_proj):  a_i = SiLU(gate_i . x) * (up_i . x),
 * y_h = sum_i a_i * W2[h, i].  w13 is [2*Iw, H] (gate rows 0..Iw-1, up rows
 * Iw..2Iw-1), w2 is [H, Iw].  xop is the GEMM1 operand row, y is [H]. */
static void swiglu_expert(int H, int Iw, int fp8, const orc_weight* w13, const orc_weight* w2,
                          const double* xop, double* y, double* wrow, double* a, double* aop,
                          uint8_t* qbuf, float* fbuf, float* sbuf) {
    for (int i = 0; i < Iw; ++i) {
        double g = 0.0, u = 0.0;
        weight_row(w13, fp8, i, wrow);
        for (int h = 0; h < H; ++h) g += wrow[h] * xop[h];
        weight_row(w13, fp8, Iw + i, wrow);
        for (int h = 0; h < H; ++h) u += wrow[h] * xop[h];
        a[i] = silu(g) * u;
    }
    act_operand(fp8, Iw, a, aop, qbuf, fbuf, sbuf);
    for (int h = 0; h < H; ++h) {
        double acc = 0.0;
        weight_row(w2, fp8, h, wrow);
        for (int i = 0; i < Iw; ++i) acc += wrow[i] * aop[i];
        y[h] = acc;
    }
}

/* ------------------------------------------------------------------------ */
/* Steps a6-a9 for a list of tokens: out_t = SwiGLU_shared(x_t)              */
/*   + sum_j w[t,j] * SwiGLU_{idx[t,j]}(x_t)                                 */
/* ([DEEP] §3.1 "shared_out + routed_output", §3.3 "Weighted sum" + "add").  */
/* x: bf16 [T,H].  w13: [E*2I, H], w2: [E*H, I] (expert e owns row blocks e), */
/* w13s: [2*Is, H], w2s: [H, Is] with Is = n_shared*I.  In fp8 mode the      */
/* *_scale arrays hold the 128x128 block scales of each expert's matrices    */
/* (expert e's blocks follow expert e-1's).  tokens: ntok token ids; out:    */
/* [ntok, H] fp64.                                                            */
/* ------------------------------------------------------------------------ */
void orc_layer(const orc_config* cfg, const uint16_t* x, const int32_t* idx, const float* w,
               const void* w13, const float* w13_scale, const void* w2, const float* w2_scale,
               const void* w13s, const float* w13s_scale, const void* w2s,
               const float* w2s_scale, const int32_t* tokens, int ntok, double* out) {
    const int H = cfg->H, I = cfg->I, k = cfg->k, fp8 = cfg->fp8;
    const int Is = cfg->n_shared * I;
    const int Imax = Is > I ? Is : I;
    const int wmax = (H > Imax ? H : Imax);
    const size_t esz = fp8 ? 1 : 2;
    const size_t n13 = (size_t)2 * I * H, n2 = (size_t)H * I;
    const size_t nb13 = (size_t)((2 * I + 127) / 128) * ((H + 127) / 128);
    const size_t nb2 = (size_t)((H + 127) / 128) * ((I + 127) / 128);
#pragma omp parallel
    {
        double* xv = (double*)malloc(sizeof(double) * H);
        double* xop = (double*)malloc(sizeof(double) * H);
        double* y = (double*)malloc(sizeof(double) * H);
        double* wrow = (double*)malloc(sizeof(double) * wmax);
        double* a = (double*)malloc(sizeof(double) * Imax);
        double* aop = (double*)malloc(sizeof(double) * Imax);
        uint8_t* qbuf = (uint8_t*)malloc(wmax);
        float* fbuf = (float*)malloc(sizeof(float) * wmax);
        float* sbuf = (float*)malloc(sizeof(float) * (wmax / 128 + 2));
#pragma omp for schedule(dynamic, 1)
        for (int n = 0; n < ntok; ++n) {
            const int t = tokens[n];
            double* o = out + (size_t)n * H;
            for (int h = 0; h < H; ++h) xv[h] = (double)orc_bf16_to_f32(x[(size_t)t * H + h]);
            act_operand(fp8, H, xv, xop, qbuf, fbuf, sbuf);
            /* shared expert, weight 1, applied to every token */
            for (int h = 0; h < H; ++h) o[h] = 0.0;
            if (Is > 0) {
                orc_weight ws13 = {w13s, w13s_scale, 2 * Is, H};
                orc_weight ws2 = {w2s, w2s_scale, H, Is};
                swiglu_expert(H, Is, fp8, &ws13, &ws2, xop, y, wrow, a, aop, qbuf, fbuf, sbuf);
                for (int h = 0; h < H; ++h) o[h] += y[h];
            }
            /* routed experts, weighted */
            for (int j = 0; j < k; ++j) {
                const int e = idx[(size_t)t * k + j];
                const double wj = (double)w[(size_t)t * k + j];
                orc_weight we13 = {(const char*)w13 + (size_t)e * n13 * esz,
                                   fp8 ? w13_scale + (size_t)e * nb13 : NULL, 2 * I, H};
                orc_weight we2 = {(const char*)w2 + (size_t)e * n2 * esz,
                                  fp8 ? w2_scale + (size_t)e * nb2 : NULL, H, I};
                swiglu_expert(H, I, fp8, &we13, &we2, xop, y, wrow, a, aop, qbuf, fbuf, sbuf);
                for (int h = 0; h < H; ++h) o[h] += wj * y[h];
            }
        }
        free(xv); free(xop); free(y); free(wrow); free(a); free(aop);
        free(qbuf); free(fbuf); free(sbuf);
    }
}

/* ------------------------------------------------------------------------ */
/* Pre-norm around the layer (next to the layer, not inside it):            */
/*   [DEEP] §3.3 layer diagram: "Residual + RMSNorm" feeds the MoE FFN and   */
/*   "Residual + Output" follows it;                                         */
/*   [DOTS1] config table: rms_norm_eps = 1e-6; source-notes paragraph: the  */
/*   variance is taken in fp32, the row is scaled by its reciprocal square   */
/*   root, then multiplied by the weight.                                    */
/* Reading: u[t,h] = gamma[h] * h[t,h] / sqrt(mean_h h[t,h]^2 + eps), here   */
/* in fp64 from the bf16 operands and rounded once to bf16 (RNE).            */
/* ------------------------------------------------------------------------ */

/* binary64 -> bf16, round to nearest even, in one step (no detour through
 * binary32, which would round twice).  bf16 keeps 8 significant bits;
 * below 2^-126 its grid is the subnormal spacing 2^-133. */
uint16_t orc_f64_to_bf16(double d) {
    if (isnan(d)) return 0x7FC0u;
    const uint16_t sign = signbit(d) ? 0x8000u : 0u;
    const double a = fabs(d);
    if (a == 0.0) return sign;
    int e;
    (void)frexp(a, &e); /* a = m * 2^e, m in [0.5, 1): leading bit has weight 2^(e-1) */
    double q;
    if (e - 1 < -126)
        q = ldexp(rint(ldexp(a, 133)), -133);
    else
        q = ldexp(rint(ldexp(a, 8 - e)), e - 8);
    if (q >= ldexp(1.0, 128)) return sign | 0x7F80u; /* overflow to infinity */
    float f = (float)q; /* exact: q has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return sign | (uint16_t)(u >> 16);
}

/* h, u: bf16 [T,H]; gamma: bf16 [H]; r (optional): per row 1/sqrt(ms + eps). */
void orc_rmsnorm(int T, int H, const uint16_t* h, const uint16_t* gamma, double eps, uint16_t* u,
                 double* r) {
    for (int t = 0; t < T; ++t) {
        const uint16_t* row = h + (size_t)t * H;
        double ss = 0.0;
        for (int i = 0; i < H; ++i) {
            const double v = (double)orc_bf16_to_f32(row[i]);
            ss += v * v;
        }
        const double rt = 1.0 / sqrt(ss / H + eps);
        if (r) r[t] = rt;
        for (int i = 0; i < H; ++i)
            u[(size_t)t * H + i] = orc_f64_to_bf16((double)orc_bf16_to_f32(gamma[i]) *
                                                   ((double)orc_bf16_to_f32(row[i]) * rt));
    }
}

/* Element-wise binary64 -> bf16 (for the rounding pins). */
void orc_f64_to_bf16_n(const double* x, uint16_t* y, int64_t n) {
    for (int64_t i = 0; i < n; ++i) y[i] = orc_f64_to_bf16(x[i]);
}

/* Thread count for the OpenMP loops above (returns the count in effect). */
int orc_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* Element-wise helpers so that tests can sweep the scalar functions above. */
void orc_exp_n(const float* x, float* y, int64_t n) {
    for (int64_t i = 0; i < n; ++i) y[i] = orc_exp(x[i]);
}
void orc_sigmoid_n(const float* x, float* y, int64_t n) {
    for (int64_t i = 0; i < n; ++i) y[i] = orc_sigmoid(x[i]);
}
void orc_e4m3_encode_n(const float* x, uint8_t* q, int64_t n) {
    for (int64_t i = 0; i < n; ++i) q[i] = orc_f32_to_e4m3(x[i]);
}

/* ------------------------------------------------------------------------ */
/* DSA indexer (a second top-k workload next to the layer):                  */
/*   [DEEP] §4.2 "How DSA Works" and its indexer listing: per index head h, */
/*   ReLU(q_h . k_h), weighted by a per-query head weight and summed over    */
/*   heads, then the top-k keys per query;                                   */
/*   [MLQM] 混合注意力 paragraph: index_topk = 2048 with 64 index heads.      */
/* Readings: no 1/sqrt(d) scale (the listing has none); an optional causal   */
/* mask (query t at absolute position q_offset + t sees keys s <= q_offset + */
/* t); masked scores are -infinity and never selected; the top-k order is    */
/* score descending, equal scores by lower key index; rows with fewer valid  */
/* keys than topk are padded with -1.                                        */
/* q: bf16 [Sq, nh, D]; k: bf16 [Sk, nh, D]; w: bf16 [Sq, nh].               */
/* ------------------------------------------------------------------------ */
void orc_dsa_scores(int Sq, int Sk, int nh, int D, const uint16_t* q, const uint16_t* k,
                    const uint16_t* w, int causal, int q_offset, double* out) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < Sq; ++t) {
        for (int s = 0; s < Sk; ++s) {
            if (causal && s > q_offset + t) {
                out[(size_t)t * Sk + s] = -INFINITY;
                continue;
            }
            double acc = 0.0;
            for (int h = 0; h < nh; ++h) {
                const uint16_t* qv = q + ((size_t)t * nh + h) * D;
                const uint16_t* kv = k + ((size_t)s * nh + h) * D;
                double dot = 0.0;
                for (int d = 0; d < D; ++d)
                    dot += (double)orc_bf16_to_f32(qv[d]) * (double)orc_bf16_to_f32(kv[d]);
                if (dot > 0.0) acc += (double)orc_bf16_to_f32(w[(size_t)t * nh + h]) * dot;
            }
            out[(size_t)t * Sk + s] = acc;
        }
    }
}

/* Top-k of each row of binary32 scores [Sq, Sk] -> idx [Sq, topk]: a stable
 * selection by repeated maximum over the not-yet-chosen keys (plain, O(k Sk)).
 * -infinity and NaN scores are never chosen. */
void orc_dsa_topk(int Sq, int Sk, int topk, const float* scores, int32_t* idx) {
#pragma omp parallel
    {
        unsigned char* taken = (unsigned char*)calloc((size_t)Sk, 1);
#pragma omp for schedule(dynamic, 1)
        for (int t = 0; t < Sq; ++t) {
            const float* row = scores + (size_t)t * Sk;
            memset(taken, 0, (size_t)Sk);
            for (int j = 0; j < topk; ++j) {
                int best = -1;
                for (int s = 0; s < Sk; ++s) {
                    const float v = row[s];
                    if (taken[s] || !(v > -INFINITY)) continue;  /* skips NaN and -inf */
                    if (best < 0 || v > row[best]) best = s;       /* strict: lower index wins ties */
                }
                idx[(size_t)t * topk + j] = best;
                if (best >= 0) taken[best] = 1;
            }
        }
        free(taken);
    }
}
