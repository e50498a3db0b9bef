/*
 * CPU oracle: plain fp64 definition of the decoder-only layer stack.
 * TEST INFRASTRUCTURE ONLY (tests/, the smoke check, the bench's CPU-baseline leg).
 * Shares no code with the CUDA library; see oracle.c for the precision contract.
 */
#ifndef ORACLE_H
#define ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_OK = 0, ORC_ERR_INVALID_ARG = 1, ORC_ERR_CONTEXT_OVERFLOW = 2 };

typedef struct orc_config {
    int32_t hidden, layers, nq, nkv, d, inter, vocab;
    int32_t tied, qkv_bias, qk_norm;
    int32_t n_experts, top_k, expert_inter, shared_inter, shared_gate, norm_topk;
    int32_t max_ctx;
    double eps, rope_base;
    /* sliding-window attention: layer l attends the last `sliding_window` positions when
     * (l + 1) % max(swa_pattern, 1) != 0 (0 = no window on any layer) */
    int32_t sliding_window, swa_pattern;
    int32_t sandwich; /* 1: post-attention and post-FFN RMSNorm before each residual add */
    int32_t q8;       /* 1: projections and LM head are int8 with one fp32 scale per row */
    double attn_softcap, final_softcap; /* 0 = off */
} orc_config;

typedef struct orc_weights {
    const uint16_t* embed;     /* bf16 [V][h] */
    const uint16_t* lm_head;   /* bf16 [V][h], unused when tied */
    const float* final_norm;   /* [h] */
    const int8_t* lm_head_q;   /* q8: int8 [V][h] (untied head only) */
    const float* lm_head_s;    /* q8: fp32 [V] row scales */
} orc_weights;

typedef struct orc_layer {
    const float* attn_norm;    /* [h] */
    const float* ffn_norm;     /* [h] */
    const uint16_t* wqkv;      /* bf16 [q+2kv][h], rows q | k | v */
    const float* bqkv;         /* [q+2kv] or NULL */
    const float* q_norm;       /* [d] or NULL */
    const float* k_norm;       /* [d] or NULL */
    const uint16_t* wo;        /* bf16 [h][q] */
    const uint16_t* w_gate;    /* dense: bf16 [I][h] */
    const uint16_t* w_up;      /* dense: bf16 [I][h] */
    const uint16_t* w_down;    /* dense: bf16 [h][I] */
    const uint16_t* w_router;  /* MoE: bf16 [E][h] */
    const uint16_t* e_gate;    /* MoE: bf16 [E][Ie][h] */
    const uint16_t* e_up;      /* MoE: bf16 [E][Ie][h] */
    const uint16_t* e_down;    /* MoE: bf16 [E][h][Ie] */
    const uint16_t* s_gate;    /* shared expert: bf16 [Is][h] */
    const uint16_t* s_up;      /* bf16 [Is][h] */
    const uint16_t* s_down;    /* bf16 [h][Is] */
    const float* s_gate_vec;   /* [h] or NULL */
    const float* post_attn_norm; /* sandwich: [h] */
    const float* post_ffn_norm;  /* sandwich: [h] */
    /* q8: the projections as int8 [rows][cols] with fp32 row scales [rows] */
    const int8_t* wqkv_q;
    const float* wqkv_s;
    const int8_t* wo_q;
    const float* wo_s;
    const int8_t* w_gate_q;
    const float* w_gate_s;
    const int8_t* w_up_q;
    const float* w_up_s;
    const int8_t* w_down_q;
    const float* w_down_s;
} orc_layer;

typedef struct orc_model orc_model;

double orc_bf16(double v);
void orc_matvec(const uint16_t* W, int64_t N, int64_t K, const double* x, double* y);
void orc_rmsnorm(const double* x, const float* g, int n, double eps, double* out);
void orc_head_rmsnorm(double* v, int heads, int d, const float* g, double eps);
void orc_rope(double* v, int heads, int d, int64_t pos, double base);
void orc_attend(const double* q, const uint16_t* K, const uint16_t* V, int64_t stride, int d, int64_t n,
                double scale, double* out);
void orc_attend_window(const double* q, const uint16_t* K, const uint16_t* V, int64_t stride, int d, int64_t first,
                       int64_t n, double scale, double softcap, double* out);
void orc_matvec_q8(const int8_t* Q, const float* S, int64_t N, int64_t K, const double* x, double* y);
int orc_layer_window(const orc_config* c, int layer);
void orc_route_topk(const double* logits, int E, int k, int renorm, int32_t* idx, double* w, double* gap);
void orc_swiglu(const double* x, const uint16_t* Wg, const uint16_t* Wu, const uint16_t* Wd, int I, int h,
                double* out);
void orc_swiglu_act(const double* x, const uint16_t* Wg, const uint16_t* Wu, int I, int h, double* act);

void orc_moe_ffn(const orc_config* c, const orc_layer* L, const double* xn, double* out, int32_t* idx, double* w,
                 double* gap);

orc_model* orc_create(const orc_config* c, const orc_weights* w, const orc_layer* layers, int n_seqs);
void orc_destroy(orc_model* m);
int orc_forward(orc_model* m, int seq, int32_t token, int64_t pos, double* logits);
int orc_prefill(orc_model* m, int seq, const int32_t* tokens, int64_t T, int64_t pos0, double* logits);
int orc_argmax(const double* v, int64_t n);
int orc_kv_write(orc_model* m, int seq, int layer, int64_t pos0, int64_t n, const uint16_t* k, const uint16_t* v);
int orc_kv_read(orc_model* m, int seq, int layer, int64_t pos0, int64_t n, uint16_t* k, uint16_t* v);
void orc_last_routes(const orc_model* m, int32_t* idx, double* w, double* gap);
void orc_last_hidden(const orc_model* m, double* out);

void orc_gqa_decode(const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new, uint16_t* kcache,
                    uint16_t* vcache, int64_t ctx_stride, const int32_t* pos, int B, int nq, int nkv, int d,
                    double scale, int fused_rope, double rope_base, double* out);
void orc_route_rows(const float* logits, int T, int E, int k, int renorm, int32_t* idx, double* w, double* gap);
void orc_gemv_rows(const uint16_t* W, const uint16_t* x, int B, int64_t N, int64_t K, double* y);

#ifdef __cplusplus
}
#endif
#endif
