/*
 * CPU oracle for the decoder-only transformer layer forward.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path links, loads or calls
 * this file; only tests/, the smoke check and the bench's CPU-baseline leg do.
 *
 * It is the plain definition of what the layer stack computes, written from
 * the three source pages:
 *   [ANEDVD]  ANEDVD src/engine.zig  (Engine.forward, Engine.prefill,
 *             rmsnormColumn, applyHeadNorm, ropeAndCache, runHead, tests)
 *   [frink]   frink_models decoder.rs (gqa_attention, route_top_k call,
 *             shared-expert gate, MultiSeqKv)
 *   [cortiq]  cortiq_engine pipeline.rs (rope_inv_freq, attn_scale,
 *             add_rmsnorm_fused_into, prefill/decode contract)
 *
 * Precision: every sum and every transcendental is fp64, summed in index
 * order by one thread. Values are rounded to bf16 (nearest-even) at exactly
 * the points where the pages store reduced precision, and nowhere else:
 *   R1  the RMSNorm output that feeds a projection  (rmsnormColumn writes f16)
 *   R2  q after bias/QK-norm/RoPE; k and v as stored in the KV cache
 *       (ropeAndCache stores the cache row in reduced precision)
 *   R3  the attention output that feeds o_proj      (Engine.forward, o input)
 *   R4  silu(gate) * up that feeds the down projection (split FFN path)
 * Weights arrive already bf16. OpenMP is used only over independent output
 * elements; each element is summed by one thread in index order, so results
 * do not depend on the thread count.
 *
 * Readings taken where the pages are silent:
 *   - RoPE pairing is half-split: element i pairs with i + d/2, angle
 *     pos * base^(-2i/d) ("rope" vs "ropeAdjacent" in ANEDVD; inv_freq from
 *     (head_dim, base) in cortiq).
 *   - GQA head h reads kv head h / (nq / nkv) (contiguous groups).
 *   - Router: softmax over all experts, top-k by probability, lower expert
 *     index first on ties, optional renormalisation of the k weights.
 *   - MoE output joins the residual as (routed + shared).
 *   - Greedy argmax picks the lowest index on ties.
 *   - Sliding window W: the query at position p attends keys p-W+1 .. p (the
 *     last W positions, itself included); a layer l is windowed when
 *     (l + 1) % max(pattern, 1) != 0 (cortiq layer_is_local / layer_window;
 *     ANEDVD passes `.window` to attentionDecode for sliding layers).
 *   - Attention logit softcap c: each scaled score s becomes c * tanh(s / c)
 *     before the softmax (ANEDVD `.logit_softcap`); the final logit softcap
 *     maps every logit the same way after the LM head (ANEDVD runHead).
 *   - Sandwich norms: the o_proj output and the dense FFN output are each
 *     RMS-normalised with their own gain before they join the residual
 *     (ANEDVD forward: post_attn / post_ffw through rmsnormFlat), no rounding.
 *   - q8_row weights: an int8 matrix with one fp32 scale per row stands for
 *     the matrix W[n][k] = scale[n] * q[n][k], dequantised exactly in fp64
 *     (cortiq's q8_row_parts of the projections).
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- bf16 */

/* Round an fp64 value to the nearest bf16 value (ties to even); returned as fp64. */
double orc_bf16(double v) {
    if (v == 0.0 || !isfinite(v)) return v;
    int e;
    frexp(fabs(v), &e);              /* |v| = m * 2^e, m in [0.5, 1) */
    int q = e - 8;                   /* 8 significant bits */
    if (q < -133) q = -133;          /* subnormal quantum */
    double r = nearbyint(ldexp(fabs(v), -q));
    double a = ldexp(r, q);
    return v < 0 ? -a : a;
}

static inline double bf(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static inline uint16_t to_bits(double v) { /* v must already be bf16-representable */
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

/* ---------------------------------------------------------------- pieces */

/* y[n] = sum_k W[n][k] * x[k]; W bf16 row-major [N][K]. */
void orc_matvec(const uint16_t* W, int64_t N, int64_t K, const double* x, double* y) {
#pragma omp parallel for schedule(static) if (N * K > 65536)
    for (int64_t n = 0; n < N; ++n) {
        const uint16_t* w = W + n * K;
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k) acc += bf(w[k]) * x[k];
        y[n] = acc;
    }
}

/* q8_row: y[n] = sum_k (S[n] * Q[n][k]) * x[k], the int8 row dequantised exactly. */
void orc_matvec_q8(const int8_t* Q, const float* S, int64_t N, int64_t K, const double* x, double* y) {
#pragma omp parallel for schedule(static) if (N * K > 65536)
    for (int64_t n = 0; n < N; ++n) {
        const int8_t* q = Q + n * K;
        const double sc = (double)S[n];
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k) acc += (sc * (double)q[k]) * x[k];
        y[n] = acc;
    }
}

/* out = x * (1 / sqrt(mean(x^2) + eps)) * g, unrounded (rmsnormColumn / rmsnormFlat). */
void orc_rmsnorm(const double* x, const float* g, int n, double eps, double* out) {
    double acc = 0.0;
    for (int i = 0; i < n; ++i) acc += x[i] * x[i];
    double inv = 1.0 / sqrt(acc / (double)n + eps);
    for (int i = 0; i < n; ++i) out[i] = x[i] * inv * (double)g[i];
}

/* QK-norm (ANEDVD applyHeadNorm): each d-wide head of v [heads][d] is normalised by
 * its own mean square and scaled by the [d] gain g, in place. */
void orc_head_rmsnorm(double* v, int heads, int d, const float* g, double eps) {
    for (int hh = 0; hh < heads; ++hh) orc_rmsnorm(v + (int64_t)hh * d, g, d, eps, v + (int64_t)hh * d);
}

/* Rotate every head of v ([heads][d]) to position pos, half-split pairing. */
void orc_rope(double* v, int heads, int d, int64_t pos, double base) {
    int half = d / 2;
    for (int i = 0; i < half; ++i) {
        double theta = pow(base, -2.0 * (double)i / (double)d);
        double a = (double)pos * theta;
        double c = cos(a), s = sin(a);
        for (int h = 0; h < heads; ++h) {
            double* x = v + (int64_t)h * d;
            double x0 = x[i], x1 = x[i + half];
            x[i] = x0 * c - x1 * s;
            x[i + half] = x0 * s + x1 * c;
        }
    }
}

/* One query head against cached rows first .. n-1 of one kv head:
 * s_j = q . K_j * scale, then c * tanh(s_j / c) when softcap c > 0;
 * out = sum_j softmax_j(s) V_j, max subtracted, sums in j order.
 * K, V rows are bf16 with row stride `stride` elements. */
void orc_attend_window(const double* q, const uint16_t* K, const uint16_t* V, int64_t stride, int d, int64_t first,
                       int64_t n, double scale, double softcap, double* out) {
    double* s = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double m = -INFINITY;
    for (int64_t j = first; j < n; ++j) {
        const uint16_t* k = K + j * stride;
        double acc = 0.0;
        for (int i = 0; i < d; ++i) acc += q[i] * bf(k[i]);
        s[j] = acc * scale;
        if (softcap > 0.0) s[j] = softcap * tanh(s[j] / softcap);
        if (s[j] > m) m = s[j];
    }
    double den = 0.0;
    for (int64_t j = first; j < n; ++j) {
        s[j] = exp(s[j] - m);
        den += s[j];
    }
    for (int i = 0; i < d; ++i) out[i] = 0.0;
    for (int64_t j = first; j < n; ++j) {
        const uint16_t* v = V + j * stride;
        for (int i = 0; i < d; ++i) out[i] += s[j] * bf(v[i]);
    }
    for (int i = 0; i < d; ++i) out[i] /= den;
    free(s);
}

/* Full causal attention over rows 0 .. n-1, no softcap. */
void orc_attend(const double* q, const uint16_t* K, const uint16_t* V, int64_t stride, int d, int64_t n,
                double scale, double* out) {
    orc_attend_window(q, K, V, stride, d, 0, n, scale, 0.0, out);
}

/* Attention window of layer `layer`: sliding_window on local layers, 0 (whole context) on
 * global ones; every max(swa_pattern, 1)-th layer is global. */
int orc_layer_window(const orc_config* c, int layer) {
    if (c->sliding_window <= 0) return 0;
    const int pattern = c->swa_pattern > 1 ? c->swa_pattern : 1;
    return (layer + 1) % pattern != 0 ? c->sliding_window : 0;
}

/* Softmax over all E logits, then the k most probable experts (lower index first on
 * equal probability), in descending order. w = P, or P / sum_topk P when renorm.
 * gap (optional) = smallest difference between consecutive sorted logits among the
 * first min(k+1, E) entries: the distance of the decision from a tie. */
void orc_route_topk(const double* logits, int E, int k, int renorm, int32_t* idx, double* w, double* gap) {
    double* p = (double*)malloc(sizeof(double) * (size_t)E);
    char* taken = (char*)calloc((size_t)E, 1);
    double m = -INFINITY;
    for (int e = 0; e < E; ++e)
        if (logits[e] > m) m = logits[e];
    double den = 0.0;
    for (int e = 0; e < E; ++e) {
        p[e] = exp(logits[e] - m);
        den += p[e];
    }
    for (int e = 0; e < E; ++e) p[e] /= den;
    int depth = k + 1 < E ? k + 1 : E;
    int32_t order[1024];
    for (int r = 0; r < depth && r < 1024; ++r) {
        int best = -1;
        for (int e = 0; e < E; ++e)
            if (!taken[e] && (best < 0 || p[e] > p[best])) best = e;
        taken[best] = 1;
        order[r] = best;
    }
    double sum = 0.0;
    for (int r = 0; r < k; ++r) sum += p[order[r]];
    for (int r = 0; r < k; ++r) {
        idx[r] = order[r];
        w[r] = renorm ? p[order[r]] / sum : p[order[r]];
    }
    if (gap) {
        double g = INFINITY;
        for (int r = 0; r + 1 < depth; ++r) {
            double d = logits[order[r]] - logits[order[r + 1]];
            if (d < g) g = d;
        }
        *gap = g;
    }
    free(p);
    free(taken);
}

static double silu(double z) { return z * (1.0 / (1.0 + exp(-z))); }
static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* y = W x with W either bf16 (W) or q8_row (Q, S). */
static void matvec_w(const uint16_t* W, const int8_t* Q, const float* S, int64_t N, int64_t K, const double* x,
                     double* y) {
    if (Q)
        orc_matvec_q8(Q, S, N, K, x, y);
    else
        orc_matvec(W, N, K, x, y);
}

/* The SwiGLU activation a = R4(silu(Wg x) * (Wu x)) [I]; u is scratch [I]. */
static void swiglu_act_w(const double* x, const uint16_t* Wg, const int8_t* Qg, const float* Sg, const uint16_t* Wu,
                         const int8_t* Qu, const float* Su, int I, int h, double* g, double* u) {
    matvec_w(Wg, Qg, Sg, I, h, x, g);
    matvec_w(Wu, Qu, Su, I, h, x, u);
    for (int i = 0; i < I; ++i) g[i] = orc_bf16(silu(g[i]) * u[i]);
}

/* SwiGLU with each of the three matrices bf16 or q8_row. */
static void swiglu_w(const double* x, const uint16_t* Wg, const int8_t* Qg, const float* Sg, const uint16_t* Wu,
                     const int8_t* Qu, const float* Su, const uint16_t* Wd, const int8_t* Qd, const float* Sd, int I,
                     int h, double* out) {
    double* g = (double*)malloc(sizeof(double) * (size_t)I);
    double* u = (double*)malloc(sizeof(double) * (size_t)I);
    swiglu_act_w(x, Wg, Qg, Sg, Wu, Qu, Su, I, h, g, u);
    matvec_w(Wd, Qd, Sd, h, I, g, out);
    free(g);
    free(u);
}

/* The activation alone: act = R4(silu(Wg x) * (Wu x)); Wg, Wu [I][h]. */
void orc_swiglu_act(const double* x, const uint16_t* Wg, const uint16_t* Wu, int I, int h, double* act) {
    double* u = (double*)malloc(sizeof(double) * (size_t)I);
    swiglu_act_w(x, Wg, NULL, NULL, Wu, NULL, NULL, I, h, act, u);
    free(u);
}

/* out = Wd * R4(silu(Wg x) * (Wu x)); Wg, Wu [I][h], Wd [h][I]. */
void orc_swiglu(const double* x, const uint16_t* Wg, const uint16_t* Wu, const uint16_t* Wd, int I, int h,
                double* out) {
    swiglu_w(x, Wg, NULL, NULL, Wu, NULL, NULL, Wd, NULL, NULL, I, h, out);
}

/* MoE FFN on one normalised (R1) input row xn [h]:
 * r = Wr xn; P = softmax(r); top-k; routed = sum_j w_j * SwiGLU_{e_j}(xn) in output order;
 * shared = sigmoid(g_s . xn) * SwiGLU_s(xn) (scale 1 without a gate vector);
 * out = routed + shared. idx/w receive the k routing decisions, gap their tie distance. */
void orc_moe_ffn(const orc_config* c, const orc_layer* L, const double* xn, double* out, int32_t* idx, double* w,
                 double* gap) {
    const int h = c->hidden, E = c->n_experts, kk = c->top_k, Ie = c->expert_inter;
    double* r = (double*)malloc(sizeof(double) * (size_t)E);
    double* t = (double*)malloc(sizeof(double) * (size_t)h);
    double* routed = (double*)calloc((size_t)h, sizeof(double));
    double* shared = (double*)calloc((size_t)h, sizeof(double));
    orc_matvec(L->w_router, E, h, xn, r);
    orc_route_topk(r, E, kk, c->norm_topk, idx, w, gap);
    for (int j = 0; j < kk; ++j) {
        int64_t e = idx[j];
        const int64_t msz = (int64_t)Ie * h;
        orc_swiglu(xn, L->e_gate + e * msz, L->e_up + e * msz, L->e_down + e * msz, Ie, h, t);
        for (int i = 0; i < h; ++i) routed[i] += w[j] * t[i];
    }
    if (c->shared_inter > 0) {
        orc_swiglu(xn, L->s_gate, L->s_up, L->s_down, c->shared_inter, h, t);
        double sc = 1.0;
        if (c->shared_gate && L->s_gate_vec) {
            double gdot = 0.0;
            for (int i = 0; i < h; ++i) gdot += (double)L->s_gate_vec[i] * xn[i];
            sc = sigmoid(gdot);
        }
        for (int i = 0; i < h; ++i) shared[i] = sc * t[i];
    }
    for (int i = 0; i < h; ++i) out[i] = routed[i] + shared[i];
    free(r);
    free(t);
    free(routed);
    free(shared);
}

/* ---------------------------------------------------------------- model */

struct orc_model {
    orc_config c;
    orc_weights w;
    orc_layer* layers;
    int n_seqs;
    uint16_t* kc; /* [n_seqs][L][max_ctx][kv] */
    uint16_t* vc;
    int32_t* route_idx; /* [L][k] of the last forward */
    double* route_w;    /* [L][k] */
    double* route_gap;  /* [L] */
    double* hidden;     /* [h] residual after the last layer of the last forward */
};

static int64_t kv_dim(const orc_config* c) { return (int64_t)c->nkv * c->d; }

static uint16_t* kslot(orc_model* m, uint16_t* base, int seq, int layer, int64_t pos) {
    const orc_config* c = &m->c;
    return base + (((int64_t)seq * c->layers + layer) * c->max_ctx + pos) * kv_dim(c);
}

orc_model* orc_create(const orc_config* c, const orc_weights* w, const orc_layer* layers, int n_seqs) {
    orc_model* m = (orc_model*)calloc(1, sizeof(orc_model));
    m->c = *c;
    m->w = *w;
    m->layers = (orc_layer*)malloc(sizeof(orc_layer) * (size_t)c->layers);
    memcpy(m->layers, layers, sizeof(orc_layer) * (size_t)c->layers);
    m->n_seqs = n_seqs;
    size_t cache = (size_t)n_seqs * c->layers * c->max_ctx * kv_dim(c);
    m->kc = (uint16_t*)calloc(cache, 2);
    m->vc = (uint16_t*)calloc(cache, 2);
    int k = c->top_k > 0 ? c->top_k : 1;
    m->route_idx = (int32_t*)calloc((size_t)c->layers * k, sizeof(int32_t));
    m->route_w = (double*)calloc((size_t)c->layers * k, sizeof(double));
    m->route_gap = (double*)calloc((size_t)c->layers, sizeof(double));
    m->hidden = (double*)calloc((size_t)c->hidden, sizeof(double));
    if (!m->kc || !m->vc) {
        orc_destroy(m);
        return NULL;
    }
    return m;
}

void orc_destroy(orc_model* m) {
    if (!m) return;
    free(m->layers);
    free(m->kc);
    free(m->vc);
    free(m->route_idx);
    free(m->route_w);
    free(m->route_gap);
    free(m->hidden);
    free(m);
}

/* One decoder layer for one token at `pos` of sequence `seq`; x is updated in place. */
static void layer_forward(orc_model* m, int li, int seq, int64_t pos, double* x) {
    const orc_config* c = &m->c;
    const orc_layer* L = &m->layers[li];
    const int h = c->hidden, d = c->d, nq = c->nq, nkv = c->nkv;
    const int64_t qd = (int64_t)nq * d, kvd = kv_dim(c), rows = qd + 2 * kvd;

    double* xn = (double*)malloc(sizeof(double) * (size_t)h);
    double* qkv = (double*)malloc(sizeof(double) * (size_t)rows);
    double* o = (double*)malloc(sizeof(double) * (size_t)qd);
    double* t = (double*)malloc(sizeof(double) * (size_t)h);

    /* 1. attention-input RMSNorm, R1 */
    orc_rmsnorm(x, L->attn_norm, h, c->eps, xn);
    for (int i = 0; i < h; ++i) xn[i] = orc_bf16(xn[i]);
    /* 2. fused QKV projection (+ bias before any norm or rotation) */
    matvec_w(L->wqkv, L->wqkv_q, L->wqkv_s, rows, h, xn, qkv);
    if (c->qkv_bias && L->bqkv)
        for (int64_t r = 0; r < rows; ++r) qkv[r] += (double)L->bqkv[r];
    double* q = qkv;
    double* k = qkv + qd;
    double* v = qkv + qd + kvd;
    /* 3. optional per-head QK-norm (applyHeadNorm): q heads with q_norm, k heads with k_norm */
    if (c->qk_norm) {
        orc_head_rmsnorm(q, nq, d, L->q_norm, c->eps);
        orc_head_rmsnorm(k, nkv, d, L->k_norm, c->eps);
    }
    /* 4. RoPE on q and k at pos */
    orc_rope(q, nq, d, pos, c->rope_base);
    orc_rope(k, nkv, d, pos, c->rope_base);
    /* 5. R2: q rounded; k, v rounded into the cache row `pos` (one write per position) */
    for (int64_t i = 0; i < qd; ++i) q[i] = orc_bf16(q[i]);
    uint16_t* krow = kslot(m, m->kc, seq, li, pos);
    uint16_t* vrow = kslot(m, m->vc, seq, li, pos);
    for (int64_t i = 0; i < kvd; ++i) {
        krow[i] = to_bits(orc_bf16(k[i]));
        vrow[i] = to_bits(orc_bf16(v[i]));
    }
    /* 6. causal GQA attention over rows 0..pos (the last `window` of them on a windowed
     *    layer), scale 1/sqrt(d), optional logit softcap; R3 */
    const int group = nq / nkv;
    const double scale = 1.0 / sqrt((double)d);
    const uint16_t* K0 = kslot(m, m->kc, seq, li, 0);
    const uint16_t* V0 = kslot(m, m->vc, seq, li, 0);
    const int64_t window = orc_layer_window(c, li);
    const int64_t first = window > 0 && pos + 1 > window ? pos + 1 - window : 0;
#pragma omp parallel for schedule(static) if (pos > 256)
    for (int hh = 0; hh < nq; ++hh) {
        int g = hh / group;
        orc_attend_window(q + (int64_t)hh * d, K0 + (int64_t)g * d, V0 + (int64_t)g * d, kvd, d, first, pos + 1,
                          scale, c->attn_softcap, o + (int64_t)hh * d);
    }
    for (int64_t i = 0; i < qd; ++i) o[i] = orc_bf16(o[i]);
    /* 7. o_proj (sandwich: RMS-normalised with post_attn_norm) and residual */
    matvec_w(L->wo, L->wo_q, L->wo_s, h, qd, o, t);
    if (c->sandwich) orc_rmsnorm(t, L->post_attn_norm, h, c->eps, t);
    for (int i = 0; i < h; ++i) x[i] += t[i];
    /* 8. FFN-input RMSNorm, R1 */
    orc_rmsnorm(x, L->ffn_norm, h, c->eps, xn);
    for (int i = 0; i < h; ++i) xn[i] = orc_bf16(xn[i]);
    if (c->n_experts <= 0) {
        /* 9. dense SwiGLU (sandwich: RMS-normalised with post_ffn_norm) */
        swiglu_w(xn, L->w_gate, L->w_gate_q, L->w_gate_s, L->w_up, L->w_up_q, L->w_up_s, L->w_down, L->w_down_q,
                 L->w_down_s, c->inter, h, t);
        if (c->sandwich) orc_rmsnorm(t, L->post_ffn_norm, h, c->eps, t);
        for (int i = 0; i < h; ++i) x[i] += t[i];
    } else {
        /* 10. MoE: router softmax, top-k, weighted routed experts, gated shared expert */
        const int kk = c->top_k;
        orc_moe_ffn(c, L, xn, t, m->route_idx + (int64_t)li * kk, m->route_w + (int64_t)li * kk,
                    &m->route_gap[li]);
        for (int i = 0; i < h; ++i) x[i] += t[i];
    }
    free(xn);
    free(qkv);
    free(o);
    free(t);
}

int orc_forward(orc_model* m, int seq, int32_t token, int64_t pos, double* logits) {
    const orc_config* c = &m->c;
    if (seq < 0 || seq >= m->n_seqs) return ORC_ERR_INVALID_ARG;
    if (token < 0 || token >= c->vocab) return ORC_ERR_INVALID_ARG;
    if (pos < 0 || pos >= c->max_ctx) return ORC_ERR_CONTEXT_OVERFLOW;
    const int h = c->hidden;
    double* x = (double*)malloc(sizeof(double) * (size_t)h);
    double* xn = (double*)malloc(sizeof(double) * (size_t)h);
    /* embedding row gather (embed scale 1) */
    for (int i = 0; i < h; ++i) x[i] = bf(m->w.embed[(int64_t)token * h + i]);
    for (int li = 0; li < c->layers; ++li) layer_forward(m, li, seq, pos, x);
    memcpy(m->hidden, x, sizeof(double) * (size_t)h);
    /* final RMSNorm (R1), LM head, optional final logit softcap */
    if (logits) {
        orc_rmsnorm(x, m->w.final_norm, h, c->eps, xn);
        for (int i = 0; i < h; ++i) xn[i] = orc_bf16(xn[i]);
        const uint16_t* head = c->tied ? m->w.embed : m->w.lm_head;
        matvec_w(head, c->tied ? NULL : m->w.lm_head_q, m->w.lm_head_s, c->vocab, h, xn, logits);
        if (c->final_softcap > 0.0)
            for (int64_t v = 0; v < c->vocab; ++v) logits[v] = c->final_softcap * tanh(logits[v] / c->final_softcap);
    }
    free(x);
    free(xn);
    return ORC_OK;
}

/* Prefill: the same per-token forward for pos0 .. pos0+T-1, logits of the last token. */
int orc_prefill(orc_model* m, int seq, const int32_t* tokens, int64_t T, int64_t pos0, double* logits) {
    if (T <= 0) return ORC_ERR_INVALID_ARG;
    if (pos0 < 0 || pos0 + T > m->c.max_ctx) return ORC_ERR_CONTEXT_OVERFLOW;
    for (int64_t t = 0; t < T; ++t) {
        int rc = orc_forward(m, seq, tokens[t], pos0 + t, t + 1 == T ? logits : NULL);
        if (rc != ORC_OK) return rc;
    }
    return ORC_OK;
}

int orc_argmax(const double* v, int64_t n) {
    int64_t best = 0;
    for (int64_t i = 1; i < n; ++i)
        if (v[i] > v[best]) best = i;
    return (int)best;
}

/* Test hooks: copy cache rows [pos0, pos0+n) of one layer of one sequence (bf16 [n][kv]). */
int orc_kv_write(orc_model* m, int seq, int layer, int64_t pos0, int64_t n, const uint16_t* k, const uint16_t* v) {
    const orc_config* c = &m->c;
    if (seq < 0 || seq >= m->n_seqs || layer < 0 || layer >= c->layers) return ORC_ERR_INVALID_ARG;
    if (pos0 < 0 || pos0 + n > c->max_ctx) return ORC_ERR_CONTEXT_OVERFLOW;
    memcpy(kslot(m, m->kc, seq, layer, pos0), k, (size_t)(n * kv_dim(c)) * 2);
    memcpy(kslot(m, m->vc, seq, layer, pos0), v, (size_t)(n * kv_dim(c)) * 2);
    return ORC_OK;
}

int orc_kv_read(orc_model* m, int seq, int layer, int64_t pos0, int64_t n, uint16_t* k, uint16_t* v) {
    const orc_config* c = &m->c;
    if (seq < 0 || seq >= m->n_seqs || layer < 0 || layer >= c->layers) return ORC_ERR_INVALID_ARG;
    if (pos0 < 0 || pos0 + n > c->max_ctx) return ORC_ERR_CONTEXT_OVERFLOW;
    memcpy(k, kslot(m, m->kc, seq, layer, pos0), (size_t)(n * kv_dim(c)) * 2);
    memcpy(v, kslot(m, m->vc, seq, layer, pos0), (size_t)(n * kv_dim(c)) * 2);
    return ORC_OK;
}

void orc_last_routes(const orc_model* m, int32_t* idx, double* w, double* gap) {
    int k = m->c.top_k > 0 ? m->c.top_k : 1;
    if (idx) memcpy(idx, m->route_idx, sizeof(int32_t) * (size_t)m->c.layers * k);
    if (w) memcpy(w, m->route_w, sizeof(double) * (size_t)m->c.layers * k);
    if (gap) memcpy(gap, m->route_gap, sizeof(double) * (size_t)m->c.layers);
}

void orc_last_hidden(const orc_model* m, double* out) { memcpy(out, m->hidden, sizeof(double) * (size_t)m->c.hidden); }

/* ---------------------------------------------------------------- standalone entry points */

/* Decode attention for B sequences, each with its own contiguous cache [ctx][nkv][d] (bf16).
 * For sequence b the query sits at position pos[b] and attends rows 0..pos[b].
 * If k_new/v_new are given, row pos[b] is overwritten with them first (after RoPE when
 * fused_rope). With fused_rope, q and k_new are rotated to pos[b] and rounded (R2).
 * out [B][nq][d], unrounded. The caches are modified in place (the append). */
void orc_gqa_decode(const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new, uint16_t* kcache,
                    uint16_t* vcache, int64_t ctx_stride, const int32_t* pos, int B, int nq, int nkv, int d,
                    double scale, int fused_rope, double rope_base, double* out) {
    const int64_t kvd = (int64_t)nkv * d;
    const int group = nq / nkv;
    for (int b = 0; b < B; ++b) {
        double* qb = (double*)malloc(sizeof(double) * (size_t)nq * d);
        for (int64_t i = 0; i < (int64_t)nq * d; ++i) qb[i] = bf(q[(int64_t)b * nq * d + i]);
        uint16_t* Kb = kcache + (int64_t)b * ctx_stride * kvd;
        uint16_t* Vb = vcache + (int64_t)b * ctx_stride * kvd;
        if (fused_rope) {
            orc_rope(qb, nq, d, pos[b], rope_base);
            for (int64_t i = 0; i < (int64_t)nq * d; ++i) qb[i] = orc_bf16(qb[i]);
        }
        if (k_new && v_new) {
            double* kb = (double*)malloc(sizeof(double) * (size_t)kvd);
            for (int64_t i = 0; i < kvd; ++i) kb[i] = bf(k_new[(int64_t)b * kvd + i]);
            if (fused_rope) orc_rope(kb, nkv, d, pos[b], rope_base);
            for (int64_t i = 0; i < kvd; ++i) {
                Kb[(int64_t)pos[b] * kvd + i] = to_bits(orc_bf16(kb[i]));
                Vb[(int64_t)pos[b] * kvd + i] = v_new[(int64_t)b * kvd + i];
            }
            free(kb);
        }
#pragma omp parallel for schedule(static)
        for (int hh = 0; hh < nq; ++hh) {
            int g = hh / group;
            orc_attend(qb + (int64_t)hh * d, Kb + (int64_t)g * d, Vb + (int64_t)g * d, kvd, d, (int64_t)pos[b] + 1,
                       scale, out + ((int64_t)b * nq + hh) * d);
        }
        free(qb);
    }
}

/* Routing of T rows of fp32 logits [T][E]. */
void orc_route_rows(const float* logits, int T, int E, int k, int renorm, int32_t* idx, double* w, double* gap) {
    double* r = (double*)malloc(sizeof(double) * (size_t)E);
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) r[e] = (double)logits[(int64_t)t * E + e];
        orc_route_topk(r, E, k, renorm, idx + (int64_t)t * k, w + (int64_t)t * k, gap ? gap + t : NULL);
    }
    free(r);
}

/* y[b][n] = sum_k W[n][k] x[b][k] for B bf16 input rows. */
void orc_gemv_rows(const uint16_t* W, const uint16_t* x, int B, int64_t N, int64_t K, double* y) {
    double* xv = (double*)malloc(sizeof(double) * (size_t)K);
    for (int b = 0; b < B; ++b) {
        for (int64_t k = 0; k < K; ++k) xv[k] = bf(x[(int64_t)b * K + k]);
        orc_matvec(W, N, K, xv, y + (int64_t)b * N);
    }
    free(xv);
}
