// C ABI of the decoder-layer library: context, weights, paged KV cache, and the
// two orchestrated paths (chunked prefill, batched decode) plus the standalone
// hot-path entry points. Every step of the math runs in the kernels of this
// library; the host side only validates, allocates pages and launches.
//
// Interface follows ANEDVD src/engine.zig (Engine.init / forward / prefill /
// reset / deinit, ContextOverflow), frink_models decoder.rs (gqa_attention,
// MultiSeqKv) and cortiq_engine pipeline.rs (each token forwarded once and
// entered into the KV cache once; empty input refused).
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/dec_api.h"
#include "kernels.h"

using namespace dec;

namespace {

// Positions one dec_verify call may forward (the pages' multi-position verify checks up
// to a handful of draft tokens).
constexpr int kMaxVerify = 8;

thread_local std::string g_err;

dec_status fail(dec_status s, const std::string& msg) {
    g_err = msg;
    return s;
}

#define CUDA_TRY(expr)                                                                          \
    do {                                                                                        \
        cudaError_t e_ = (expr);                                                                \
        if (e_ != cudaSuccess)                                                                  \
            return fail(DEC_ERR_CUDA, std::string(#expr) + ": " + cudaGetErrorString(e_));      \
    } while (0)

// Test hook (dec_test_fail_alloc): the n-th device allocation from now on fails as if the
// device were out of memory; 0 = off.
std::atomic<long> g_fail_alloc_in{0};

template <typename T>
cudaError_t dmalloc(T** p, size_t count) {
    if (count == 0) count = 1;
    long n = g_fail_alloc_in.load();
    while (n > 0 && !g_fail_alloc_in.compare_exchange_weak(n, n - 1)) {
    }
    if (n == 1) {
        *p = nullptr;
        return cudaErrorMemoryAllocation;
    }
    return cudaMalloc(reinterpret_cast<void**>(p), count * sizeof(T));
}

bool is_host_ptr(const void* p) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return true;
    }
    return at.type == cudaMemoryTypeHost || at.type == cudaMemoryTypeUnregistered;
}

struct LayerDev {
    float *attn_norm = nullptr, *ffn_norm = nullptr, *bqkv = nullptr, *q_norm = nullptr, *k_norm = nullptr;
    uint16_t *wqkv = nullptr, *wo = nullptr, *wgu = nullptr, *wdown = nullptr;
    uint16_t *wrouter = nullptr, *egu = nullptr, *edown = nullptr, *sgu = nullptr, *sdown = nullptr;
    float* sgate_vec = nullptr;
    float *post_attn_norm = nullptr, *post_ffn_norm = nullptr;  // sandwich norms
    // q8_row models: the int8 projections (gate/up rows interleaved like wgu) and their row
    // scales; wqkv / wo / wgu / wdown then hold the same integers as bf16 (tensor-core path)
    int8_t *qkv_q = nullptr, *wo_q = nullptr, *gu_q = nullptr, *down_q = nullptr;
    float *qkv_s = nullptr, *wo_s = nullptr, *gu_s = nullptr, *down_s = nullptr;
    uint16_t *k_pool = nullptr, *v_pool = nullptr;
};

}  // namespace

struct dec_ctx {
    dec_config c{};
    int device = 0, num_sms = 148, smem_cap = 0;
    cudaStream_t stream = nullptr;  // stream all work is enqueued on
    cudaStream_t user = nullptr;    // the caller's stream
    bool bridge = false;            // caller gave the legacy default stream: own stream + events
    cudaEvent_t ev_in = nullptr, ev_out = nullptr;
    int qd = 0, kvd = 0, qkv_rows = 0, max_pages = 0, n_pages = 0;
    int max_tok = 0;  // rows of the per-step buffers: max(max_batch, prefill_chunk, kMaxVerify)
    std::vector<LayerDev> L;
    uint16_t *embed = nullptr, *head = nullptr;
    int8_t* head_q = nullptr;  // q8_row LM head and its row scales
    float* head_s = nullptr;
    float* final_norm = nullptr;
    // paging
    std::vector<int> free_pages;
    std::vector<std::vector<int>> seq_pages;
    std::vector<int> seq_len;
    std::vector<int32_t> h_bt;
    int32_t* d_bt = nullptr;
    // step buffers
    int32_t *d_tok = nullptr, *d_pos = nullptr;
    unsigned long long* d_amax = nullptr;  // packed greedy argmax, 32 words per row
    float2* rope_tab = nullptr;            // [max_context][d/2] (cos, sin): fp64 on the host, stored fp32
    float *x = nullptr, *qkv = nullptr, *logits = nullptr;
    float* ysub = nullptr;  // sandwich norms: a sublayer's output [max_tok][h] before its norm
    uint16_t *xn = nullptr, *qrot = nullptr, *attn = nullptr, *act = nullptr;
    float* gemm_ws = nullptr;  // tensor-core GEMM: pieces of tiles shared between CTAs
    int* gemm_cnt = nullptr;   // and their arrival counters (zero between launches)
    int gemm_cnt_n = 0;
    int* d_err = nullptr;        // set by a device wait that ran out (cleared by dec_check)
    // Host-to-device staging: two pinned slots used in turn, each fenced by an event
    // recorded after the copies that read it, so a call never waits for the device
    // unless the slot it needs is still being copied from (two calls back).
    int32_t* h_stage[2] = {nullptr, nullptr};
    cudaEvent_t ev_stage[2] = {nullptr, nullptr};
    int stage_next = 0;
    size_t stage_ints = 0;
    float** d_ldst = nullptr;    // device slot: where the head stores the logits (null: nowhere)
    int32_t* d_prompt = nullptr; // [max_context]
    int* h_err = nullptr;        // pinned copy of d_err for the synchronising paths
    int act_cols = 0;
    // MoE step buffers (rows: max_tok tokens, or max_tok * top_k (token, expert) slots)
    float *moe_logits = nullptr, *moe_w = nullptr, *moe_sgate = nullptr, *moe_y = nullptr, *moe_ys = nullptr;
    int32_t *moe_routes = nullptr, *moe_perm = nullptr, *moe_inv = nullptr, *moe_groups = nullptr, *moe_ngroups = nullptr;
    uint16_t* moe_act = nullptr;
    int head_rows = 0;  // rows of the logits / argmax buffers: max(max_batch, kMaxVerify)
    std::map<int, cudaGraphExec_t> graphs;
    int last_rows = 0;
    bool last_was_step = false;
};

namespace {

// ----------------------------------------------------------------- validation

dec_status check_config(const dec_config* c) {
    if (!c) return fail(DEC_ERR_INVALID_ARG, "config is NULL");
    if (c->hidden <= 0 || c->layers <= 0 || c->n_q_heads <= 0 || c->n_kv_heads <= 0 || c->vocab <= 0)
        return fail(DEC_ERR_INVALID_ARG, "hidden, layers, heads and vocab must be positive");
    if (c->n_q_heads % c->n_kv_heads != 0) return fail(DEC_ERR_INVALID_ARG, "n_q_heads % n_kv_heads != 0");
    if (c->n_q_heads / c->n_kv_heads > 16) return fail(DEC_ERR_UNSUPPORTED, "more than 16 q heads per kv head");
    if (c->head_dim != 64 && c->head_dim != 128) return fail(DEC_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
    if (c->hidden % 8 != 0) return fail(DEC_ERR_UNSUPPORTED, "hidden must be a multiple of 8");
    if (c->page_size != 16) return fail(DEC_ERR_UNSUPPORTED, "page_size must be 16");
    if (c->max_batch <= 0 || c->max_context <= 0 || c->prefill_chunk <= 0)
        return fail(DEC_ERR_INVALID_ARG, "max_batch, max_context and prefill_chunk must be positive");
    if (c->n_experts > 0) {
        if (c->n_experts > 256 || c->top_k <= 0 || c->top_k > 16 || c->top_k > c->n_experts)
            return fail(DEC_ERR_UNSUPPORTED, "MoE needs n_experts <= 256 and 0 < top_k <= min(16, n_experts)");
        if (c->expert_inter <= 0 || c->expert_inter % 8 != 0 || c->shared_inter < 0 || c->shared_inter % 8 != 0)
            return fail(DEC_ERR_UNSUPPORTED, "expert_inter / shared_inter must be multiples of 8");
    } else if (c->ffn_inter <= 0 || c->ffn_inter % 8 != 0) {
        return fail(DEC_ERR_UNSUPPORTED, "ffn_inter must be a positive multiple of 8");
    }
    if (!(c->rms_eps > 0.f)) return fail(DEC_ERR_INVALID_ARG, "rms_eps must be positive");
    if (c->sliding_window < 0 || c->swa_pattern < 0 || !(c->attn_softcap >= 0.f) || !(c->final_softcap >= 0.f))
        return fail(DEC_ERR_INVALID_ARG, "sliding_window, swa_pattern and the softcaps must be >= 0");
    if (c->sandwich_norms && c->n_experts > 0)
        return fail(DEC_ERR_UNSUPPORTED, "sandwich norms are built for the dense FFN only");
    if (c->weight_format != 0 && c->weight_format != 1) return fail(DEC_ERR_UNSUPPORTED, "weight_format must be 0 or 1");
    if (c->weight_format == 1 && (c->n_experts > 0 || c->tied_embeddings))
        return fail(DEC_ERR_UNSUPPORTED, "q8_row weights are built for dense models with an untied LM head");
    return DEC_OK;
}

// Attention window of layer li (0 = the whole context): every max(swa_pattern, 1)-th layer
// is global (cortiq layer_is_local).
int layer_window(const dec_config& k, int li) {
    if (k.sliding_window <= 0) return 0;
    const int pattern = k.swa_pattern > 1 ? k.swa_pattern : 1;
    return (li + 1) % pattern != 0 ? k.sliding_window : 0;
}

cudaError_t copy_in(void* dst, const void* src, size_t bytes, cudaStream_t st) {
    if (!src) return cudaErrorInvalidValue;
    return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDefault, st);
}

// Interleave rows of gate [rows][rb bytes] and up into dst [2*rows]: row 2j = gate j, 2j+1 = up j.
cudaError_t interleave_rows_in(void* dst, const void* gate, const void* up, size_t rows, size_t rb, cudaStream_t st) {
    if (!gate || !up) return cudaErrorInvalidValue;
    cudaError_t e = cudaMemcpy2DAsync(dst, 2 * rb, gate, rb, rb, rows, cudaMemcpyDefault, st);
    if (e != cudaSuccess) return e;
    return cudaMemcpy2DAsync(reinterpret_cast<uint8_t*>(dst) + rb, 2 * rb, up, rb, rb, rows, cudaMemcpyDefault, st);
}

cudaError_t interleave_in(uint16_t* dst, const void* gate, const void* up, size_t rows, int h, cudaStream_t st) {
    return interleave_rows_in(dst, gate, up, rows, (size_t)h * 2, st);
}

// ----------------------------------------------------------------- projections

// y = W x for `n` token rows: GEMV when n is small, tcgen05 GEMM otherwise. A q8_row
// projection also carries its int8 rows Q and row scales S (the GEMV streams Q; the GEMM
// multiplies W, the same integers in bf16, and scales each row in its epilogue).
struct Proj {
    const uint16_t* W;
    int M, K;
    const int8_t* Q = nullptr;
    const float* S = nullptr;
};

dec_status run_proj(dec_ctx* c, const Proj& p, int n, int epi, bool fused_norm, const float* xr, const float* g,
                    const uint16_t* xb, float* y, int ldy, const float* bias, uint16_t* act, int ldact,
                    cudaStream_t st, unsigned long long* amax = nullptr, float* const* y_ptr = nullptr,
                    float softcap = 0.f) {
    const int cap = c->smem_cap;
    if (n <= 8 && gemv_fits(n, p.K, cap, p.Q != nullptr)) {
        GemvArgs a{};
        a.W = p.W;
        a.Wq = p.Q;
        a.wscale = p.S;
        a.N = p.M;
        a.K = p.K;
        a.B = n;
        a.xb = fused_norm ? nullptr : xb;
        a.xr = fused_norm ? xr : nullptr;
        a.g = g;
        a.eps = c->c.rms_eps;
        a.ldx = p.K;
        a.y = y;
        a.y_ptr = y_ptr;
        a.ldy = ldy;
        a.bias = bias;
        a.act = act;
        a.ldact = ldact;
        a.amax = amax;
        a.softcap = softcap;
        a.err = c->d_err;
        a.smem_cap = cap;
        const int ge = epi == GEMM_STORE ? GEMV_STORE : epi == GEMM_RESID ? GEMV_RESID : GEMV_SWIGLU;
        CUDA_TRY(gemv_launch(a, ge, st, c->num_sms, true));
        return DEC_OK;
    }
    const uint16_t* in = xb;
    if (fused_norm) {
        CUDA_TRY(rmsnorm_launch(xr, g, n, p.K, c->c.rms_eps, c->xn, st, true));
        in = c->xn;
    }
    GemmPlan plan;
    CUDA_TRY(gemm_plan(&plan, p.W, p.M, p.K, in, n, c->num_sms, c->gemm_ws));
    GemmArgs a{};
    a.epi = epi;
    a.y = y;
    a.y_ptr = y_ptr;
    a.ldy = ldy;
    a.bias = bias;
    a.rscale = p.Q ? p.S : nullptr;
    a.act = act;
    a.ldact = ldact;
    a.amax = amax;
    a.softcap = softcap;
    a.cnt = c->gemm_cnt;
    a.err = c->d_err;
    if (gemm_cnt_needed(p.M, n) > c->gemm_cnt_n) return fail(DEC_ERR_UNSUPPORTED, "GEMM tile counters too small");
    CUDA_TRY(gemm_launch(plan, a, st, true));
    return DEC_OK;
}

// ----------------------------------------------------------------- MoE FFN of one layer

// xn = R1(rmsnorm(x)); router logits; top-k + shared gate; permutation by expert; grouped
// gate/up (SiLU*up) and down over the routed (token, expert) slots; shared expert; combine
// into the residual: x += sum_j w_j y_j + sigmoid(g . xn) y_shared.
dec_status moe_ffn(dec_ctx* c, int li, int n, cudaStream_t st) {
    const dec_config& k = c->c;
    LayerDev& L = c->L[li];
    const int h = k.hidden, E = k.n_experts, kk = k.top_k, Ie = k.expert_inter, Is = k.shared_inter;
    CUDA_TRY(rmsnorm_launch(c->x, L.ffn_norm, n, h, k.rms_eps, c->xn, st, true));
    dec_status s = run_proj(c, {L.wrouter, E, h}, n, GEMM_STORE, false, nullptr, nullptr, c->xn, c->moe_logits, E,
                            nullptr, nullptr, 0, st);
    if (s != DEC_OK) return s;
    int32_t* idx = c->moe_routes + (size_t)li * c->max_tok * kk;
    MoeRouteArgs r{};
    r.logits = c->moe_logits;
    r.E = E;
    r.k = kk;
    r.renorm = k.norm_topk_prob;
    r.idx = idx;
    r.w = c->moe_w;
    r.xn = c->xn;
    r.gvec = (Is > 0 && k.shared_gate) ? L.sgate_vec : nullptr;
    r.h = h;
    r.sgate = c->moe_sgate;
    CUDA_TRY(moe_route_launch(r, n, st, true));
    const int nb = grouped_nb_for(n);
    MoePermArgs p{};
    p.idx = idx;
    p.n = n;
    p.k = kk;
    p.E = E;
    p.nb = nb;
    p.perm_tok = c->moe_perm;
    p.inv = c->moe_inv;
    p.groups = c->moe_groups;
    p.n_groups = c->moe_ngroups;
    CUDA_TRY(moe_permute_launch(p, st, true));
    GroupedGemvArgs g{};
    g.W = L.egu;
    g.wstride = (size_t)2 * Ie * h;
    g.M = 2 * Ie;
    g.K = h;
    g.E = E;
    g.groups = c->moe_groups;
    g.n_groups = c->moe_ngroups;
    g.x = c->xn;
    g.x_map = c->moe_perm;
    g.ldx = h;
    g.act = c->moe_act;
    g.ldact = Ie;
    g.err = c->d_err;
    g.smem_cap = c->smem_cap;
    CUDA_TRY(grouped_gemv_launch(g, nb, true, st, c->num_sms, true));
    g.W = L.edown;
    g.wstride = (size_t)h * Ie;
    g.M = h;
    g.K = Ie;
    g.x = c->moe_act;
    g.x_map = nullptr;
    g.ldx = Ie;
    g.y = c->moe_y;
    g.ldy = h;
    g.act = nullptr;
    CUDA_TRY(grouped_gemv_launch(g, nb, false, st, c->num_sms, true));
    if (Is > 0) {
        s = run_proj(c, {L.sgu, 2 * Is, h}, n, GEMM_SWIGLU, false, nullptr, nullptr, c->xn, nullptr, 0, nullptr,
                     c->act, Is, st);
        if (s != DEC_OK) return s;
        s = run_proj(c, {L.sdown, h, Is}, n, GEMM_STORE, false, nullptr, nullptr, c->act, c->moe_ys, h, nullptr,
                     nullptr, 0, st);
        if (s != DEC_OK) return s;
    }
    MoeCombineArgs m{};
    m.x = c->x;
    m.y = c->moe_y;
    m.ys = Is > 0 ? c->moe_ys : nullptr;
    m.w = c->moe_w;
    m.inv = c->moe_inv;
    m.sgate = (Is > 0 && k.shared_gate && L.sgate_vec) ? c->moe_sgate : nullptr;
    m.k = kk;
    m.h = h;
    CUDA_TRY(moe_combine_launch(m, n, st, true));
    return DEC_OK;
}

// ----------------------------------------------------------------- one forward over n token rows

// Decode: n = B sequences, one token each, positions in d_pos; attention reads the
// per-sequence block table. Prefill: n tokens of one sequence at pos0..pos0+n-1.
dec_status forward_layers(dec_ctx* c, int n, bool decode, int seq, int pos0, cudaStream_t st) {
    const dec_config& k = c->c;
    const int h = k.hidden, d = k.head_dim;
    const float scale = 1.0f / sqrtf((float)d);
    for (int li = 0; li < k.layers; ++li) {
        LayerDev& L = c->L[li];
        // attention input norm + fused QKV (+bias)
        dec_status s = run_proj(c, {L.wqkv, c->qkv_rows, h, L.qkv_q, L.qkv_s}, n, GEMM_STORE, true, c->x,
                                L.attn_norm, nullptr, c->qkv, c->qkv_rows, L.bqkv, nullptr, 0, st);
        if (s != DEC_OK) return s;
        if (decode) {
            AttnDecodeArgs a{};
            a.qkv = c->qkv;
            a.ld_qkv = c->qkv_rows;
            a.q_norm = L.q_norm;
            a.k_norm = L.k_norm;
            a.eps = k.rms_eps;
            a.rope = 1;
            a.rope_base = k.rope_base;
            a.rope_tab = c->rope_tab;
            a.k_pool = L.k_pool;
            a.v_pool = L.v_pool;
            a.block_table = c->d_bt;
            a.max_pages = c->max_pages;
            a.pos = c->d_pos;
            a.B = n;
            a.nq = k.n_q_heads;
            a.nkv = k.n_kv_heads;
            a.d = d;
            a.scale = scale;
            a.window = layer_window(k, li);
            a.softcap = k.attn_softcap;
            // context splits merged inside a cluster: no scratch, chosen per batch size and span
            const int span = a.window > 0 ? std::min(a.window, k.max_context) : k.max_context;
            a.splits = attn_decode_splits(n, k.n_kv_heads, span, c->num_sms, true);
            a.part = nullptr;
            a.counters = nullptr;
            a.out = c->attn;
            a.err = c->d_err;
            CUDA_TRY(attn_decode_launch(a, st, true));
        } else {
            RopeAppendArgs r{};
            r.qkv = c->qkv;
            r.ld_qkv = c->qkv_rows;
            r.q_norm = L.q_norm;
            r.k_norm = L.k_norm;
            r.eps = k.rms_eps;
            r.rope_base = k.rope_base;
            r.rope_tab = c->rope_tab;
            r.T = n;
            r.pos0 = pos0;
            r.nq = k.n_q_heads;
            r.nkv = k.n_kv_heads;
            r.d = d;
            r.q_out = c->qrot;
            r.k_pool = L.k_pool;
            r.v_pool = L.v_pool;
            r.block_row = c->d_bt + (size_t)seq * c->max_pages;
            CUDA_TRY(rope_append_launch(r, st, true));
            AttnPrefillArgs a{};
            a.q = c->qrot;
            a.k_pool = L.k_pool;
            a.v_pool = L.v_pool;
            a.block_row = r.block_row;
            a.T = n;
            a.pos0 = pos0;
            a.nq = k.n_q_heads;
            a.nkv = k.n_kv_heads;
            a.d = d;
            a.scale = scale;
            a.window = layer_window(k, li);
            a.softcap = k.attn_softcap;
            a.splits = attn_prefill_splits(n, k.n_q_heads, k.n_kv_heads, attn_prefill_span(pos0, n, a.window),
                                           c->num_sms);
            a.out = c->attn;
            a.err = c->d_err;
            a.pool_rows = c->n_pages * k.n_kv_heads * 16;
            CUDA_TRY(attn_prefill_launch(a, st, true));
        }
        // o_proj + residual (sandwich: the output is RMS-normalised with its own gain first)
        if (k.sandwich_norms) {
            s = run_proj(c, {L.wo, h, c->qd, L.wo_q, L.wo_s}, n, GEMM_STORE, false, nullptr, nullptr, c->attn, c->ysub,
                         h, nullptr, nullptr, 0, st);
            if (s != DEC_OK) return s;
            CUDA_TRY(add_rmsnorm_launch(c->x, c->ysub, L.post_attn_norm, n, h, k.rms_eps, st, true));
        } else {
            s = run_proj(c, {L.wo, h, c->qd, L.wo_q, L.wo_s}, n, GEMM_RESID, false, nullptr, nullptr, c->attn, c->x, h,
                         nullptr, nullptr, 0, st);
            if (s != DEC_OK) return s;
        }
        if (k.n_experts > 0) {
            s = moe_ffn(c, li, n, st);
            if (s != DEC_OK) return s;
            continue;
        }
        // FFN: norm + fused gate/up + SiLU, then down + residual
        s = run_proj(c, {L.wgu, 2 * k.ffn_inter, h, L.gu_q, L.gu_s}, n, GEMM_SWIGLU, true, c->x, L.ffn_norm, nullptr,
                     nullptr, 0, nullptr, c->act, c->act_cols, st);
        if (s != DEC_OK) return s;
        if (k.sandwich_norms) {
            s = run_proj(c, {L.wdown, h, k.ffn_inter, L.down_q, L.down_s}, n, GEMM_STORE, false, nullptr, nullptr,
                         c->act, c->ysub, h, nullptr, nullptr, 0, st);
            if (s != DEC_OK) return s;
            CUDA_TRY(add_rmsnorm_launch(c->x, c->ysub, L.post_ffn_norm, n, h, k.rms_eps, st, true));
        } else {
            s = run_proj(c, {L.wdown, h, k.ffn_inter, L.down_q, L.down_s}, n, GEMM_RESID, false, nullptr, nullptr,
                         c->act, c->x, h, nullptr, nullptr, 0, st);
            if (s != DEC_OK) return s;
        }
    }
    return DEC_OK;
}

// Final norm + LM head for `n` rows starting at residual row `row0`. The logits [n][V] go
// to `y`, or, when y_ptr is given, to the device address it holds (read when the head
// runs, so one captured graph serves every destination); a null destination stores
// nothing. The greedy token of each row is folded into the head's epilogue (packed
// argmax words) either way.
dec_status head(dec_ctx* c, int row0, int n, cudaStream_t st, float* y, float* const* y_ptr) {
    const dec_config& k = c->c;
    CUDA_TRY(cudaMemsetAsync(c->d_amax, 0, sizeof(unsigned long long) * 32 * (size_t)n, st));
    return run_proj(c, {c->head, k.vocab, k.hidden, c->head_q, c->head_s}, n, GEMM_STORE, true,
                    c->x + (size_t)row0 * k.hidden,
                    c->final_norm, nullptr, y, k.vocab, nullptr, nullptr, 0, st, c->d_amax, y_ptr, k.final_softcap);
}

dec_status ensure_pages(dec_ctx* c, int seq, int upto) {
    // allocate pages so positions [0, upto) of seq are backed
    std::vector<int>& pg = c->seq_pages[seq];
    const int need = (upto + 15) / 16;
    while ((int)pg.size() < need) {
        if (c->free_pages.empty()) return fail(DEC_ERR_PAGES_EXHAUSTED, "KV page pool exhausted");
        const int p = c->free_pages.back();
        c->free_pages.pop_back();
        c->h_bt[(size_t)seq * c->max_pages + pg.size()] = p;
        pg.push_back(p);
    }
    return DEC_OK;
}

// One staging slot, in int32 words: tokens [max_tok] | positions [max_tok] | logits
// destination (one 8-byte pointer) | block-table rows [max_batch][max_pages] | prompt
// tokens [max_context].
struct StageLayout {
    size_t tok, pos, dst, bt, prompt, total;
};

StageLayout stage_layout(const dec_ctx* c) {
    StageLayout L;
    L.tok = 0;
    L.pos = L.tok + (size_t)c->max_tok;
    L.dst = (L.pos + (size_t)c->max_tok + 1) & ~(size_t)1;  // 8-byte aligned
    L.bt = L.dst + 2;
    L.prompt = L.bt + (size_t)c->c.max_batch * c->max_pages;
    L.total = L.prompt + (size_t)c->c.max_context;
    return L;
}

// The next staging slot. Its previous use was two calls ago; the event recorded after
// that use's copies has normally completed long since, so this rarely waits.
dec_status stage_acquire(dec_ctx* c, int32_t** slot, int* which) {
    const int i = c->stage_next;
    CUDA_TRY(cudaEventSynchronize(c->ev_stage[i]));
    c->stage_next ^= 1;
    *slot = c->h_stage[i];
    *which = i;
    return DEC_OK;
}

// Fence the slot: recorded on `st` right after the copies that read it.
dec_status stage_release(dec_ctx* c, int which, cudaStream_t st) {
    CUDA_TRY(cudaEventRecord(c->ev_stage[which], st));
    return DEC_OK;
}

// Copy the block-table rows of sequences [s0, s1) through the staging slot.
dec_status stage_bt_rows(dec_ctx* c, int32_t* slot, int s0, int s1, cudaStream_t st) {
    const StageLayout L = stage_layout(c);
    const size_t off = (size_t)s0 * c->max_pages, n = (size_t)(s1 - s0) * c->max_pages;
    memcpy(slot + L.bt + off, &c->h_bt[off], sizeof(int32_t) * n);
    CUDA_TRY(cudaMemcpyAsync(c->d_bt + off, slot + L.bt + off, sizeof(int32_t) * n, cudaMemcpyHostToDevice, st));
    return DEC_OK;
}

// After the stream has been synchronised: report a device wait that ran out (the error
// word a kernel sets when one of its bounded waits gives up) as DEC_ERR_TIMEOUT, and make
// the context usable again: clear the word and zero the GEMM tile counters that an
// abandoned reduction can leave behind.
dec_status take_device_error(dec_ctx* c, cudaStream_t st) {
    if (!*c->h_err) return DEC_OK;
    *c->h_err = 0;
    CUDA_TRY(cudaMemsetAsync(c->d_err, 0, sizeof(int), st));
    CUDA_TRY(cudaMemsetAsync(c->gemm_cnt, 0, sizeof(int) * (size_t)c->gemm_cnt_n, st));
    CUDA_TRY(cudaStreamSynchronize(st));
    return fail(DEC_ERR_TIMEOUT,
                "a bounded device wait ran out (this call or an earlier one on this context); the context "
                "has been reset for further calls");
}

// Synchronise and check the error word (the synchronising entry points).
dec_status sync_and_check(dec_ctx* c, cudaStream_t st) {
    CUDA_TRY(cudaMemcpyAsync(c->h_err, c->d_err, sizeof(int), cudaMemcpyDeviceToHost, st));
    CUDA_TRY(cudaStreamSynchronize(st));
    return take_device_error(c, st);
}

// Where the head should store the logits for a caller's logits_out: its own buffer for a
// device pointer, the context's buffer for a host pointer (copied out afterwards), nowhere
// for NULL.
float* logits_target(dec_ctx* c, float* out, bool* host) {
    *host = out && is_host_ptr(out);
    if (!out) return nullptr;
    return *host ? c->logits : out;
}

// Host logits: copy them out, synchronise and check the error word.
dec_status finish_host_logits(dec_ctx* c, float* out, int rows, cudaStream_t st) {
    const size_t bytes = (size_t)rows * c->c.vocab * sizeof(float);
    CUDA_TRY(cudaMemcpyAsync(out, c->logits, bytes, cudaMemcpyDeviceToHost, st));
    return sync_and_check(c, st);
}

// Order the context's stream after the caller's legacy-stream work, and back.
void enter(dec_ctx* c) {
    if (!c->bridge) return;
    cudaEventRecord(c->ev_in, nullptr);
    cudaStreamWaitEvent(c->stream, c->ev_in, 0);
}
void leave(dec_ctx* c) {
    if (!c->bridge) return;
    cudaEventRecord(c->ev_out, c->stream);
    cudaStreamWaitEvent(nullptr, c->ev_out, 0);
}

struct Scope {
    dec_ctx* c;
    explicit Scope(dec_ctx* c_) : c(c_) { enter(c); }
    ~Scope() { leave(c); }
};

// ----------------------------------------------------------------- standalone scratch (per device)

struct Scratch {
    float* attn_part = nullptr;
    size_t attn_part_n = 0;
    int* attn_cnt = nullptr;
    size_t attn_cnt_n = 0;
    float* ws = nullptr;
    size_t ws_n = 0;
    int* cnt = nullptr;
    size_t cnt_n = 0;
    int* err = nullptr;
    int32_t* moe_i = nullptr;  // perm [Tk] | inv [Tk] | groups [4 Tk] | n_groups [1]
    size_t moe_i_n = 0;
    uint16_t* moe_act = nullptr;
    size_t moe_act_n = 0;
    float* moe_y = nullptr;
    size_t moe_y_n = 0;
};
std::mutex g_scratch_mu;
std::map<int, Scratch> g_scratch;

template <typename T>
cudaError_t grow(T** p, size_t* have, size_t need, bool zero) {
    if (need <= *have) return cudaSuccess;
    if (*p) cudaFree(*p);
    *p = nullptr;
    *have = 0;
    cudaError_t e = cudaMalloc(reinterpret_cast<void**>(p), need * sizeof(T));
    if (e != cudaSuccess) return e;
    if (zero) {
        e = cudaMemset(*p, 0, need * sizeof(T));
        if (e != cudaSuccess) return e;
    }
    *have = need;
    return cudaSuccess;
}

int device_sms() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

int device_smem_cap() {
    int dev = 0, cap = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&cap, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    return cap - 1024;
}

}  // namespace

namespace dec {
// Message returned by dec_last_error() for entry points defined in other files.
void set_last_error(const std::string& msg) { g_err = msg; }
}  // namespace dec

// =================================================================== ABI

extern "C" {

const char* dec_last_error(void) { return g_err.c_str(); }

dec_status dec_init(const dec_config* cfg, const dec_weights* w, dec_stream_t stream, dec_ctx** out) {
    g_err.clear();
    if (!out) return fail(DEC_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    dec_status s = check_config(cfg);
    if (s != DEC_OK) return s;
    if (!w || !w->embed || !w->final_norm || !w->layers) return fail(DEC_ERR_INVALID_ARG, "weights missing");
    if (!cfg->tied_embeddings && !w->lm_head) return fail(DEC_ERR_INVALID_ARG, "lm_head missing (untied)");
    if (cfg->weight_format == 1) {
        bool ok = w->lm_head_scale != nullptr;
        for (int li = 0; li < cfg->layers && ok; ++li) {
            const dec_layer_weights& l = w->layers[li];
            ok = l.wqkv_scale && l.wo_scale && l.w_gate_scale && l.w_up_scale && l.w_down_scale;
        }
        if (!ok) return fail(DEC_ERR_INVALID_ARG, "q8_row weights need every row-scale array");
    }
    if (cfg->sandwich_norms) {
        for (int li = 0; li < cfg->layers; ++li)
            if (!w->layers[li].post_attn_norm || !w->layers[li].post_ffn_norm)
                return fail(DEC_ERR_INVALID_ARG, "sandwich norms need post_attn_norm and post_ffn_norm");
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    dec_ctx* c = new dec_ctx();
    c->c = *cfg;
    c->user = st;
    if (st == nullptr) {
        // CUDA graphs cannot be captured on the legacy default stream: work runs on an own
        // stream, ordered after and before the caller's default-stream work by events.
        c->bridge = true;
        if (cudaStreamCreateWithFlags(&c->stream, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&c->ev_in, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&c->ev_out, cudaEventDisableTiming) != cudaSuccess) {
            fail(DEC_ERR_CUDA, "stream/event creation failed");
            dec_free(c);
            return DEC_ERR_CUDA;
        }
        st = c->stream;
    } else {
        c->stream = st;
    }
    cudaGetDevice(&c->device);
    c->num_sms = device_sms();
    c->smem_cap = device_smem_cap();
    const dec_config& k = c->c;
    const int h = k.hidden, d = k.head_dim;
    c->qd = k.n_q_heads * d;
    c->kvd = k.n_kv_heads * d;
    c->qkv_rows = c->qd + 2 * c->kvd;
    c->max_pages = (k.max_context + 15) / 16;
    c->n_pages = k.n_pages > 0 ? k.n_pages : k.max_batch * c->max_pages;
    c->max_tok = std::max({k.max_batch, k.prefill_chunk, kMaxVerify});
    c->act_cols = std::max(k.ffn_inter, k.shared_inter);
    auto cleanup = [&](dec_status st_) {
        dec_free(c);
        return st_;
    };
    if (k.n_experts > 0) {  // the largest token group (8) must fit the grouped projections' shared memory
        const int nbmax = grouped_nb_for(c->max_tok);
        if (!grouped_fits(nbmax, h, c->smem_cap) || !grouped_fits(nbmax, k.expert_inter, c->smem_cap)) {
            fail(DEC_ERR_UNSUPPORTED, "hidden / expert_inter too long for the grouped expert projections");
            return cleanup(DEC_ERR_UNSUPPORTED);
        }
    }
    const bool q8 = k.weight_format == 1;
    // q8_row: int8 copy Q and row scales S of a [rows][cols] projection, plus the same
    // integers as bf16 in W for the tensor-core path (exact: every int8 is a bf16 value)
    auto load_q8 = [&](int8_t** Q, float** S, uint16_t** W, const void* src, const float* src_s, size_t rows,
                       size_t cols) -> cudaError_t {
        cudaError_t e = dmalloc(Q, rows * cols);
        if (e == cudaSuccess) e = copy_in(*Q, src, rows * cols, st);
        if (e == cudaSuccess) e = dmalloc(S, rows);
        if (e == cudaSuccess) e = copy_in(*S, src_s, rows * 4, st);
        if (e == cudaSuccess) e = dmalloc(W, rows * cols);
        if (e == cudaSuccess) e = widen_i8_launch(*Q, *W, rows * cols, st);
        return e;
    };
#define INIT_TRY(expr)                                                                         \
    do {                                                                                       \
        cudaError_t e_ = (expr);                                                               \
        if (e_ != cudaSuccess) {                                                               \
            dec_status code_ = e_ == cudaErrorMemoryAllocation ? DEC_ERR_OOM : DEC_ERR_CUDA;   \
            fail(code_, std::string(#expr) + ": " + cudaGetErrorString(e_));                   \
            cudaGetLastError();                                                                \
            return cleanup(code_);                                                             \
        }                                                                                      \
    } while (0)

    // ---- weights
    const size_t V = (size_t)k.vocab;
    INIT_TRY(dmalloc(&c->embed, V * h));
    INIT_TRY(copy_in(c->embed, w->embed, V * h * 2, st));
    if (k.tied_embeddings) {
        c->head = c->embed;
    } else if (q8) {
        INIT_TRY(load_q8(&c->head_q, &c->head_s, &c->head, w->lm_head, w->lm_head_scale, V, h));
    } else {
        INIT_TRY(dmalloc(&c->head, V * h));
        INIT_TRY(copy_in(c->head, w->lm_head, V * h * 2, st));
    }
    INIT_TRY(dmalloc(&c->final_norm, h));
    INIT_TRY(copy_in(c->final_norm, w->final_norm, (size_t)h * 4, st));
    c->L.resize(k.layers);
    const size_t page_elems = (size_t)c->n_pages * k.n_kv_heads * 16 * d;
    for (int li = 0; li < k.layers; ++li) {
        const dec_layer_weights& s_ = w->layers[li];
        LayerDev& L = c->L[li];
        INIT_TRY(dmalloc(&L.attn_norm, h));
        INIT_TRY(copy_in(L.attn_norm, s_.attn_norm, (size_t)h * 4, st));
        INIT_TRY(dmalloc(&L.ffn_norm, h));
        INIT_TRY(copy_in(L.ffn_norm, s_.ffn_norm, (size_t)h * 4, st));
        if (q8) {
            INIT_TRY(load_q8(&L.qkv_q, &L.qkv_s, &L.wqkv, s_.wqkv, s_.wqkv_scale, c->qkv_rows, h));
        } else {
            INIT_TRY(dmalloc(&L.wqkv, (size_t)c->qkv_rows * h));
            INIT_TRY(copy_in(L.wqkv, s_.wqkv, (size_t)c->qkv_rows * h * 2, st));
        }
        if (k.qkv_bias) {
            INIT_TRY(dmalloc(&L.bqkv, c->qkv_rows));
            INIT_TRY(copy_in(L.bqkv, s_.bqkv, (size_t)c->qkv_rows * 4, st));
        }
        if (k.qk_norm) {
            INIT_TRY(dmalloc(&L.q_norm, d));
            INIT_TRY(copy_in(L.q_norm, s_.q_norm, (size_t)d * 4, st));
            INIT_TRY(dmalloc(&L.k_norm, d));
            INIT_TRY(copy_in(L.k_norm, s_.k_norm, (size_t)d * 4, st));
        }
        if (k.sandwich_norms) {
            INIT_TRY(dmalloc(&L.post_attn_norm, h));
            INIT_TRY(copy_in(L.post_attn_norm, s_.post_attn_norm, (size_t)h * 4, st));
            INIT_TRY(dmalloc(&L.post_ffn_norm, h));
            INIT_TRY(copy_in(L.post_ffn_norm, s_.post_ffn_norm, (size_t)h * 4, st));
        }
        if (q8) {
            INIT_TRY(load_q8(&L.wo_q, &L.wo_s, &L.wo, s_.wo, s_.wo_scale, h, c->qd));
        } else {
            INIT_TRY(dmalloc(&L.wo, (size_t)h * c->qd));
            INIT_TRY(copy_in(L.wo, s_.wo, (size_t)h * c->qd * 2, st));
        }
        if (k.n_experts > 0) {
            const size_t E = k.n_experts, Ie = k.expert_inter, Is = k.shared_inter;
            INIT_TRY(dmalloc(&L.wrouter, E * h));
            INIT_TRY(copy_in(L.wrouter, s_.w_router, E * h * 2, st));
            INIT_TRY(dmalloc(&L.egu, E * 2 * Ie * h));  // per expert: gate/up rows interleaved
            INIT_TRY(interleave_in(L.egu, s_.e_gate, s_.e_up, E * Ie, h, st));
            INIT_TRY(dmalloc(&L.edown, E * h * Ie));
            INIT_TRY(copy_in(L.edown, s_.e_down, E * h * Ie * 2, st));
            if (Is > 0) {
                INIT_TRY(dmalloc(&L.sgu, 2 * Is * h));
                INIT_TRY(interleave_in(L.sgu, s_.s_gate, s_.s_up, Is, h, st));
                INIT_TRY(dmalloc(&L.sdown, (size_t)h * Is));
                INIT_TRY(copy_in(L.sdown, s_.s_down, (size_t)h * Is * 2, st));
                if (k.shared_gate && s_.s_gate_vec) {
                    INIT_TRY(dmalloc(&L.sgate_vec, h));
                    INIT_TRY(copy_in(L.sgate_vec, s_.s_gate_vec, (size_t)h * 4, st));
                }
            }
        } else if (q8) {
            const size_t I = k.ffn_inter;
            INIT_TRY(dmalloc(&L.gu_q, 2 * I * h));
            INIT_TRY(interleave_rows_in(L.gu_q, s_.w_gate, s_.w_up, I, (size_t)h, st));
            INIT_TRY(dmalloc(&L.gu_s, 2 * I));
            INIT_TRY(interleave_rows_in(L.gu_s, s_.w_gate_scale, s_.w_up_scale, I, 4, st));
            INIT_TRY(dmalloc(&L.wgu, 2 * I * h));
            INIT_TRY(widen_i8_launch(L.gu_q, L.wgu, 2 * I * h, st));
            INIT_TRY(load_q8(&L.down_q, &L.down_s, &L.wdown, s_.w_down, s_.w_down_scale, h, I));
        } else {
            INIT_TRY(dmalloc(&L.wgu, (size_t)2 * k.ffn_inter * h));
            INIT_TRY(interleave_in(L.wgu, s_.w_gate, s_.w_up, (size_t)k.ffn_inter, h, st));
            INIT_TRY(dmalloc(&L.wdown, (size_t)h * k.ffn_inter));
            INIT_TRY(copy_in(L.wdown, s_.w_down, (size_t)h * k.ffn_inter * 2, st));
        }
        INIT_TRY(dmalloc(&L.k_pool, page_elems));
        INIT_TRY(dmalloc(&L.v_pool, page_elems));
        INIT_TRY(cudaMemsetAsync(L.k_pool, 0, page_elems * 2, st));
        INIT_TRY(cudaMemsetAsync(L.v_pool, 0, page_elems * 2, st));
    }

    // ---- paging
    c->free_pages.resize(c->n_pages);
    for (int i = 0; i < c->n_pages; ++i) c->free_pages[i] = c->n_pages - 1 - i;  // pop_back gives 0, 1, ...
    c->seq_pages.assign(k.max_batch, {});
    c->seq_len.assign(k.max_batch, 0);
    c->h_bt.assign((size_t)k.max_batch * c->max_pages, 0);
    INIT_TRY(dmalloc(&c->d_bt, (size_t)k.max_batch * c->max_pages));
    INIT_TRY(cudaMemsetAsync(c->d_bt, 0, (size_t)k.max_batch * c->max_pages * 4, st));

    // ---- step buffers
    const int T = c->max_tok;
    INIT_TRY(dmalloc(&c->d_tok, T));
    INIT_TRY(dmalloc(&c->d_prompt, (size_t)k.max_context));
    INIT_TRY(dmalloc(&c->d_pos, T));
    c->head_rows = std::max(k.max_batch, kMaxVerify);  // decode rows, or the positions of one verify
    INIT_TRY(dmalloc(&c->d_amax, (size_t)32 * c->head_rows));
    {
        const int qkv_rows = k.n_q_heads * d + 2 * k.n_kv_heads * d;
        const int m_max = std::max({k.vocab, qkv_rows, k.hidden, 2 * k.ffn_inter, 2 * k.shared_inter, k.n_experts});
        c->gemm_cnt_n = gemm_cnt_needed(m_max, T);
        INIT_TRY(dmalloc(&c->gemm_ws, gemm_ws_floats(c->num_sms)));
        INIT_TRY(dmalloc(&c->gemm_cnt, c->gemm_cnt_n));
        INIT_TRY(cudaMemsetAsync(c->gemm_cnt, 0, (size_t)c->gemm_cnt_n * 4, st));
    }
    {
        // RoPE angles pos * base^(-2i/d), cos and sin evaluated in fp64, stored as fp32
        std::vector<float2> tab((size_t)k.max_context * (d / 2));
        for (int p = 0; p < k.max_context; ++p)
            for (int i = 0; i < d / 2; ++i) {
                const double theta = pow((double)k.rope_base, -2.0 * i / (double)d);
                const double ang = (double)p * theta;
                tab[(size_t)p * (d / 2) + i] = make_float2((float)cos(ang), (float)sin(ang));
            }
        INIT_TRY(dmalloc(&c->rope_tab, tab.size()));
        INIT_TRY(cudaMemcpy(c->rope_tab, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice));
    }
    INIT_TRY(dmalloc(&c->x, (size_t)T * h));
    if (k.sandwich_norms) INIT_TRY(dmalloc(&c->ysub, (size_t)T * h));
    INIT_TRY(dmalloc(&c->qkv, (size_t)T * c->qkv_rows));
    INIT_TRY(dmalloc(&c->logits, (size_t)c->head_rows * V));
    INIT_TRY(dmalloc(&c->xn, (size_t)T * std::max(h, c->qd)));
    INIT_TRY(dmalloc(&c->qrot, (size_t)T * c->qd));
    INIT_TRY(dmalloc(&c->attn, (size_t)T * c->qd));
    INIT_TRY(dmalloc(&c->act, (size_t)T * c->act_cols));
    if (k.n_experts > 0) {
        const size_t E = k.n_experts, kk = k.top_k, slots = (size_t)T * kk;
        INIT_TRY(dmalloc(&c->moe_logits, (size_t)T * E));
        INIT_TRY(dmalloc(&c->moe_w, slots));
        INIT_TRY(dmalloc(&c->moe_sgate, T));
        INIT_TRY(dmalloc(&c->moe_routes, (size_t)k.layers * slots));
        INIT_TRY(cudaMemsetAsync(c->moe_routes, 0, (size_t)k.layers * slots * 4, st));
        INIT_TRY(dmalloc(&c->moe_perm, slots));
        INIT_TRY(dmalloc(&c->moe_inv, slots));
        INIT_TRY(dmalloc(&c->moe_groups, 4 * (E + slots)));
        INIT_TRY(dmalloc(&c->moe_ngroups, 1));
        INIT_TRY(dmalloc(&c->moe_act, slots * k.expert_inter));
        INIT_TRY(dmalloc(&c->moe_y, slots * h));
        INIT_TRY(dmalloc(&c->moe_ys, (size_t)T * h));
    }
    INIT_TRY(dmalloc(&c->d_err, 1));
    INIT_TRY(cudaMemsetAsync(c->d_err, 0, 4, st));
    c->stage_ints = stage_layout(c).total;
    for (int i = 0; i < 2; ++i) {
        INIT_TRY(cudaMallocHost(reinterpret_cast<void**>(&c->h_stage[i]), sizeof(int32_t) * c->stage_ints));
        INIT_TRY(cudaEventCreateWithFlags(&c->ev_stage[i], cudaEventDisableTiming));
    }
    INIT_TRY(dmalloc(&c->d_ldst, 1));
    INIT_TRY(cudaMemsetAsync(c->d_ldst, 0, sizeof(float*), st));
    INIT_TRY(cudaMallocHost(reinterpret_cast<void**>(&c->h_err), sizeof(int)));
    *c->h_err = 0;

    INIT_TRY(cudaStreamSynchronize(st));
#undef INIT_TRY
    *out = c;
    return DEC_OK;
}

dec_status dec_free(dec_ctx* c) {
    if (!c) return DEC_OK;
    for (auto& kv : c->graphs) cudaGraphExecDestroy(kv.second);
    for (auto& L : c->L) {
        cudaFree(L.attn_norm);
        cudaFree(L.ffn_norm);
        cudaFree(L.bqkv);
        cudaFree(L.q_norm);
        cudaFree(L.k_norm);
        cudaFree(L.wqkv);
        cudaFree(L.wo);
        cudaFree(L.wgu);
        cudaFree(L.wdown);
        cudaFree(L.wrouter);
        cudaFree(L.egu);
        cudaFree(L.edown);
        cudaFree(L.sgu);
        cudaFree(L.sdown);
        cudaFree(L.sgate_vec);
        cudaFree(L.post_attn_norm);
        cudaFree(L.post_ffn_norm);
        cudaFree(L.qkv_q);
        cudaFree(L.qkv_s);
        cudaFree(L.wo_q);
        cudaFree(L.wo_s);
        cudaFree(L.gu_q);
        cudaFree(L.gu_s);
        cudaFree(L.down_q);
        cudaFree(L.down_s);
        cudaFree(L.k_pool);
        cudaFree(L.v_pool);
    }
    if (c->head != c->embed) cudaFree(c->head);
    cudaFree(c->head_q);
    cudaFree(c->head_s);
    cudaFree(c->embed);
    cudaFree(c->final_norm);
    cudaFree(c->d_bt);
    cudaFree(c->d_tok);
    cudaFree(c->d_prompt);
    cudaFree(c->d_pos);
    cudaFree(c->d_amax);
    cudaFree(c->rope_tab);
    cudaFree(c->x);
    cudaFree(c->ysub);
    cudaFree(c->qkv);
    cudaFree(c->logits);
    cudaFree(c->xn);
    cudaFree(c->qrot);
    cudaFree(c->attn);
    cudaFree(c->act);
    cudaFree(c->gemm_ws);
    cudaFree(c->gemm_cnt);
    cudaFree(c->moe_logits);
    cudaFree(c->moe_w);
    cudaFree(c->moe_sgate);
    cudaFree(c->moe_routes);
    cudaFree(c->moe_perm);
    cudaFree(c->moe_inv);
    cudaFree(c->moe_groups);
    cudaFree(c->moe_ngroups);
    cudaFree(c->moe_act);
    cudaFree(c->moe_y);
    cudaFree(c->moe_ys);
    cudaFree(c->d_err);
    cudaFree(c->d_ldst);
    for (int i = 0; i < 2; ++i) {
        if (c->ev_stage[i]) cudaEventSynchronize(c->ev_stage[i]);
        if (c->h_stage[i]) cudaFreeHost(c->h_stage[i]);
        if (c->ev_stage[i]) cudaEventDestroy(c->ev_stage[i]);
    }
    if (c->h_err) cudaFreeHost(c->h_err);
    if (c->bridge) {
        if (c->stream) cudaStreamDestroy(c->stream);
        if (c->ev_in) cudaEventDestroy(c->ev_in);
        if (c->ev_out) cudaEventDestroy(c->ev_out);
    }
    delete c;
    return DEC_OK;
}

dec_status dec_reset(dec_ctx* c, int32_t seq) {
    if (!c) return fail(DEC_ERR_INVALID_ARG, "ctx is NULL");
    if (seq < -1 || seq >= c->c.max_batch) return fail(DEC_ERR_INVALID_ARG, "seq out of range");
    for (int s = 0; s < c->c.max_batch; ++s) {
        if (seq != -1 && s != seq) continue;
        for (int p : c->seq_pages[s]) c->free_pages.push_back(p);
        c->seq_pages[s].clear();
        c->seq_len[s] = 0;
    }
    return DEC_OK;
}

dec_status dec_seq_len(dec_ctx* c, int32_t seq, int32_t* len_out) {
    if (!c || !len_out) return fail(DEC_ERR_INVALID_ARG, "NULL argument");
    if (seq < 0 || seq >= c->c.max_batch) return fail(DEC_ERR_INVALID_ARG, "seq out of range");
    *len_out = c->seq_len[seq];
    return DEC_OK;
}

dec_status dec_prefill(dec_ctx* c, int32_t seq, const int32_t* tokens, int32_t T, int32_t pos0, float* logits_out) {
    g_err.clear();
    if (!c) return fail(DEC_ERR_INVALID_ARG, "ctx is NULL");
    const dec_config& k = c->c;
    if (seq < 0 || seq >= k.max_batch) return fail(DEC_ERR_INVALID_ARG, "seq out of range");
    if (T <= 0 || !tokens) return fail(DEC_ERR_INVALID_ARG, "empty prompt");
    if (pos0 < 0 || (int64_t)pos0 + T > k.max_context) return fail(DEC_ERR_CONTEXT_OVERFLOW, "pos0 + T > max_context");
    if (pos0 != c->seq_len[seq]) return fail(DEC_ERR_INVALID_ARG, "pos0 must equal the sequence length");
    for (int i = 0; i < T; ++i)
        if (tokens[i] < 0 || tokens[i] >= k.vocab) return fail(DEC_ERR_INVALID_ARG, "token id out of range");
    dec_status s = ensure_pages(c, seq, pos0 + T);
    if (s != DEC_OK) return s;
    cudaStream_t st = c->stream;
    Scope scope(c);
    // the sequence's block-table row and all the prompt tokens in one staging slot, then the
    // chunks back to back with no host wait between them
    int32_t* slot = nullptr;
    int which = 0;
    s = stage_acquire(c, &slot, &which);
    if (s != DEC_OK) return s;
    const StageLayout SL = stage_layout(c);
    s = stage_bt_rows(c, slot, seq, seq + 1, st);
    if (s != DEC_OK) return s;
    memcpy(slot + SL.prompt, tokens, sizeof(int32_t) * T);
    CUDA_TRY(cudaMemcpyAsync(c->d_prompt, slot + SL.prompt, sizeof(int32_t) * T, cudaMemcpyHostToDevice, st));
    s = stage_release(c, which, st);
    if (s != DEC_OK) return s;
    const int C = k.prefill_chunk;
    int last_rows = 0;
    for (int done = 0; done < T; done += C) {
        const int n = std::min(C, T - done);
        CUDA_TRY(embed_launch(c->embed, c->d_prompt + done, n, k.hidden, c->x, st, false));
        s = forward_layers(c, n, false, seq, pos0 + done, st);
        if (s != DEC_OK) return s;
        last_rows = n;
    }
    bool host = false;
    float* dst = logits_target(c, logits_out, &host);
    s = head(c, last_rows - 1, 1, st, dst, nullptr);
    if (s != DEC_OK) return s;
    c->seq_len[seq] = pos0 + T;
    c->last_rows = 1;
    return host ? finish_host_logits(c, logits_out, 1, st) : DEC_OK;
}

dec_status dec_step(dec_ctx* c, const int32_t* tokens, const int32_t* pos, int32_t B, float* logits_out) {
    g_err.clear();
    if (!c) return fail(DEC_ERR_INVALID_ARG, "ctx is NULL");
    const dec_config& k = c->c;
    if (B <= 0 || B > k.max_batch) return fail(DEC_ERR_INVALID_ARG, "B out of range");
    if (!tokens || !pos) return fail(DEC_ERR_INVALID_ARG, "tokens/pos NULL");
    for (int b = 0; b < B; ++b) {
        if (tokens[b] < 0 || tokens[b] >= k.vocab) return fail(DEC_ERR_INVALID_ARG, "token id out of range");
        if (pos[b] < 0 || pos[b] >= k.max_context) return fail(DEC_ERR_CONTEXT_OVERFLOW, "pos >= max_context");
        if (pos[b] != c->seq_len[b]) return fail(DEC_ERR_INVALID_ARG, "pos must equal the sequence length");
    }
    cudaStream_t st = c->stream;
    Scope scope(c);
    int dirty_lo = B, dirty_hi = -1;
    for (int b = 0; b < B; ++b) {
        const size_t before = c->seq_pages[b].size();
        dec_status s = ensure_pages(c, b, pos[b] + 1);
        if (s != DEC_OK) return s;
        if (c->seq_pages[b].size() != before) {
            dirty_lo = std::min(dirty_lo, b);
            dirty_hi = std::max(dirty_hi, b);
        }
    }
    bool host = false;
    float* dst = logits_target(c, logits_out, &host);
    // tokens, positions, the logits destination and any block-table rows that gained a
    // page, through one staging slot (no host wait: the slot is fenced by its event)
    int32_t* slot = nullptr;
    int which = 0;
    dec_status s = stage_acquire(c, &slot, &which);
    if (s != DEC_OK) return s;
    const StageLayout SL = stage_layout(c);
    memcpy(slot + SL.tok, tokens, sizeof(int32_t) * B);
    memcpy(slot + SL.pos, pos, sizeof(int32_t) * B);
    memcpy(slot + SL.dst, &dst, sizeof(float*));
    CUDA_TRY(cudaMemcpyAsync(c->d_tok, slot + SL.tok, sizeof(int32_t) * B, cudaMemcpyHostToDevice, st));
    CUDA_TRY(cudaMemcpyAsync(c->d_pos, slot + SL.pos, sizeof(int32_t) * B, cudaMemcpyHostToDevice, st));
    CUDA_TRY(cudaMemcpyAsync(c->d_ldst, slot + SL.dst, sizeof(float*), cudaMemcpyHostToDevice, st));
    if (dirty_hi >= 0) {
        s = stage_bt_rows(c, slot, dirty_lo, dirty_hi + 1, st);
        if (s != DEC_OK) return s;
    }
    s = stage_release(c, which, st);
    if (s != DEC_OK) return s;

    auto it = c->graphs.find(B);
    if (it == c->graphs.end()) {
        cudaGraph_t g = nullptr;
        CUDA_TRY(cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal));
        s = DEC_OK;
        if (embed_launch(c->embed, c->d_tok, B, k.hidden, c->x, st, false) != cudaSuccess)
            s = fail(DEC_ERR_CUDA, "embed launch failed");
        if (s == DEC_OK) s = forward_layers(c, B, true, 0, 0, st);
        if (s == DEC_OK) s = head(c, 0, B, st, nullptr, c->d_ldst);
        cudaError_t e = cudaStreamEndCapture(st, &g);
        if (s != DEC_OK) {
            if (g) cudaGraphDestroy(g);
            return s;
        }
        if (e != cudaSuccess) return fail(DEC_ERR_CUDA, std::string("graph capture: ") + cudaGetErrorString(e));
        cudaGraphExec_t ex = nullptr;
        e = cudaGraphInstantiate(&ex, g, 0);
        cudaGraphDestroy(g);
        if (e != cudaSuccess) return fail(DEC_ERR_CUDA, std::string("graph instantiate: ") + cudaGetErrorString(e));
        it = c->graphs.emplace(B, ex).first;
    }
    CUDA_TRY(cudaGraphLaunch(it->second, st));
    for (int b = 0; b < B; ++b) c->seq_len[b] = pos[b] + 1;
    c->last_rows = B;
    return host ? finish_host_logits(c, logits_out, B, st) : DEC_OK;
}

dec_status dec_verify(dec_ctx* c, int32_t seq, const int32_t* tokens, int32_t N, int32_t pos0, float* logits_out) {
    g_err.clear();
    if (!c) return fail(DEC_ERR_INVALID_ARG, "ctx is NULL");
    const dec_config& k = c->c;
    if (seq < 0 || seq >= k.max_batch) return fail(DEC_ERR_INVALID_ARG, "seq out of range");
    if (N <= 0 || !tokens) return fail(DEC_ERR_INVALID_ARG, "no tokens");
    if (N > kMaxVerify) return fail(DEC_ERR_INVALID_ARG, "more than 8 positions");
    if (pos0 < 0 || (int64_t)pos0 + N > k.max_context) return fail(DEC_ERR_CONTEXT_OVERFLOW, "pos0 + N > max_context");
    if (pos0 != c->seq_len[seq]) return fail(DEC_ERR_INVALID_ARG, "pos0 must equal the sequence length");
    for (int i = 0; i < N; ++i)
        if (tokens[i] < 0 || tokens[i] >= k.vocab) return fail(DEC_ERR_INVALID_ARG, "token id out of range");
    dec_status s = ensure_pages(c, seq, pos0 + N);
    if (s != DEC_OK) return s;
    cudaStream_t st = c->stream;
    Scope scope(c);
    int32_t* slot = nullptr;
    int which = 0;
    s = stage_acquire(c, &slot, &which);
    if (s != DEC_OK) return s;
    const StageLayout SL = stage_layout(c);
    s = stage_bt_rows(c, slot, seq, seq + 1, st);
    if (s != DEC_OK) return s;
    memcpy(slot + SL.prompt, tokens, sizeof(int32_t) * N);
    CUDA_TRY(cudaMemcpyAsync(c->d_prompt, slot + SL.prompt, sizeof(int32_t) * N, cudaMemcpyHostToDevice, st));
    s = stage_release(c, which, st);
    if (s != DEC_OK) return s;
    // the N positions as one chunk: every projection streams its weights once for all of
    // them (the GEMV takes up to 8 columns); chunk-causal attention over the cache
    CUDA_TRY(embed_launch(c->embed, c->d_prompt, N, k.hidden, c->x, st, false));
    s = forward_layers(c, N, false, seq, pos0, st);
    if (s != DEC_OK) return s;
    bool host = false;
    float* dst = logits_target(c, logits_out, &host);
    s = head(c, 0, N, st, dst, nullptr);
    if (s != DEC_OK) return s;
    c->seq_len[seq] = pos0 + N;
    c->last_rows = N;
    return host ? finish_host_logits(c, logits_out, N, st) : DEC_OK;
}

dec_status dec_truncate(dec_ctx* c, int32_t seq, int32_t len) {
    g_err.clear();
    if (!c) return fail(DEC_ERR_INVALID_ARG, "ctx is NULL");
    if (seq < 0 || seq >= c->c.max_batch) return fail(DEC_ERR_INVALID_ARG, "seq out of range");
    if (len < 0 || len > c->seq_len[seq]) return fail(DEC_ERR_INVALID_ARG, "len must be in [0, sequence length]");
    // pages wholly past the new length go back to the pool; rows past it in the last kept
    // page are stale and are overwritten before anything reads them (a query at position p
    // reads rows 0..p only)
    std::vector<int>& pg = c->seq_pages[seq];
    const size_t keep = (size_t)(len + 15) / 16;
    while (pg.size() > keep) {
        c->free_pages.push_back(pg.back());
        pg.pop_back();
    }
    c->seq_len[seq] = len;
    return DEC_OK;
}

dec_status dec_check(dec_ctx* c) {
    if (!c) return fail(DEC_ERR_INVALID_ARG, "ctx is NULL");
    g_err.clear();
    Scope scope(c);
    return sync_and_check(c, c->stream);
}

dec_status dec_last_argmax(dec_ctx* c, int32_t* out, int32_t B) {
    if (!c || !out) return fail(DEC_ERR_INVALID_ARG, "NULL argument");
    if (B != c->last_rows) return fail(DEC_ERR_INVALID_ARG, "B differs from the last call's rows");
    std::vector<unsigned long long> w((size_t)32 * B);
    CUDA_TRY(cudaMemcpyAsync(w.data(), c->d_amax, sizeof(unsigned long long) * 32 * B, cudaMemcpyDeviceToHost,
                             c->stream));
    dec_status s = sync_and_check(c, c->stream);
    if (s != DEC_OK) return s;
    for (int b = 0; b < B; ++b) out[b] = argmax_unpack(w[(size_t)32 * b]);
    return DEC_OK;
}

dec_status dec_kv_write(dec_ctx* c, int32_t seq, int32_t layer, int32_t pos0, int32_t n, const void* k_,
                        const void* v_) {
    if (!c || !k_ || !v_) return fail(DEC_ERR_INVALID_ARG, "NULL argument");
    if (seq < 0 || seq >= c->c.max_batch || layer < 0 || layer >= c->c.layers || n <= 0 || pos0 < 0)
        return fail(DEC_ERR_INVALID_ARG, "bad seq/layer/range");
    if ((int64_t)pos0 + n > c->c.max_context) return fail(DEC_ERR_CONTEXT_OVERFLOW, "range beyond max_context");
    dec_status s = ensure_pages(c, seq, pos0 + n);
    if (s != DEC_OK) return s;
    cudaStream_t st = c->stream;
    int32_t* slot = nullptr;
    int which = 0;
    s = stage_acquire(c, &slot, &which);
    if (s != DEC_OK) return s;
    s = stage_bt_rows(c, slot, seq, seq + 1, st);
    if (s != DEC_OK) return s;
    s = stage_release(c, which, st);
    if (s != DEC_OK) return s;
    const size_t bytes = (size_t)n * c->kvd * 2;
    uint16_t *dk = nullptr, *dv = nullptr;
    CUDA_TRY(cudaMalloc(&dk, bytes));
    CUDA_TRY(cudaMalloc(&dv, bytes));
    cudaMemcpyAsync(dk, k_, bytes, cudaMemcpyDefault, st);
    cudaMemcpyAsync(dv, v_, bytes, cudaMemcpyDefault, st);
    cudaError_t e = kv_move_launch(c->L[layer].k_pool, c->L[layer].v_pool, c->d_bt + (size_t)seq * c->max_pages, pos0,
                                   n, c->c.n_kv_heads, c->c.head_dim, dk, dv, 1, st);
    cudaError_t e2 = cudaStreamSynchronize(st);
    cudaFree(dk);
    cudaFree(dv);
    if (e != cudaSuccess || e2 != cudaSuccess) return fail(DEC_ERR_CUDA, "kv write failed");
    c->seq_len[seq] = std::max(c->seq_len[seq], pos0 + n);
    return DEC_OK;
}

dec_status dec_kv_read(dec_ctx* c, int32_t seq, int32_t layer, int32_t pos0, int32_t n, void* k_, void* v_) {
    if (!c || !k_ || !v_) return fail(DEC_ERR_INVALID_ARG, "NULL argument");
    if (seq < 0 || seq >= c->c.max_batch || layer < 0 || layer >= c->c.layers || n <= 0 || pos0 < 0)
        return fail(DEC_ERR_INVALID_ARG, "bad seq/layer/range");
    if ((int64_t)pos0 + n > c->seq_len[seq]) return fail(DEC_ERR_INVALID_ARG, "range beyond the sequence length");
    cudaStream_t st = c->stream;
    const size_t bytes = (size_t)n * c->kvd * 2;
    uint16_t *dk = nullptr, *dv = nullptr;
    CUDA_TRY(cudaMalloc(&dk, bytes));
    CUDA_TRY(cudaMalloc(&dv, bytes));
    cudaError_t e = kv_move_launch(c->L[layer].k_pool, c->L[layer].v_pool, c->d_bt + (size_t)seq * c->max_pages, pos0,
                                   n, c->c.n_kv_heads, c->c.head_dim, dk, dv, 0, st);
    cudaMemcpyAsync(k_, dk, bytes, cudaMemcpyDefault, st);
    cudaMemcpyAsync(v_, dv, bytes, cudaMemcpyDefault, st);
    cudaError_t e2 = cudaStreamSynchronize(st);
    cudaFree(dk);
    cudaFree(dv);
    if (e != cudaSuccess || e2 != cudaSuccess) return fail(DEC_ERR_CUDA, "kv read failed");
    return DEC_OK;
}

dec_status dec_last_routes(dec_ctx* c, int32_t* idx, int32_t B) {
    if (!c || !idx) return fail(DEC_ERR_INVALID_ARG, "NULL argument");
    if (c->c.n_experts <= 0) return fail(DEC_ERR_UNSUPPORTED, "the model has no MoE layers");
    if (B <= 0 || B > c->max_tok) return fail(DEC_ERR_INVALID_ARG, "B out of range");
    const size_t kk = c->c.top_k;
    for (int l = 0; l < c->c.layers; ++l)
        CUDA_TRY(cudaMemcpyAsync(idx + (size_t)l * B * kk, c->moe_routes + (size_t)l * c->max_tok * kk,
                                 sizeof(int32_t) * B * kk, cudaMemcpyDeviceToHost, c->stream));
    CUDA_TRY(cudaStreamSynchronize(c->stream));
    return DEC_OK;
}

dec_status dec_last_hidden(dec_ctx* c, float* out, int32_t B) {
    if (!c || !out) return fail(DEC_ERR_INVALID_ARG, "NULL argument");
    if (B != c->last_rows && !(B == 1)) return fail(DEC_ERR_INVALID_ARG, "B differs from the last call's rows");
    CUDA_TRY(cudaMemcpyAsync(out, c->x, sizeof(float) * (size_t)B * c->c.hidden, cudaMemcpyDeviceToHost, c->stream));
    CUDA_TRY(cudaStreamSynchronize(c->stream));
    return DEC_OK;
}

// ------------------------------------------------------------------ standalone

dec_status gqa_decode_attn(const void* q, const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                           const int32_t* block_table, int32_t max_pages, const int32_t* pos, int32_t B, int32_t nq,
                           int32_t nkv, int32_t d, int32_t page_size, float scale, int32_t fused_rope,
                           float rope_base, void* out, dec_stream_t stream) {
    g_err.clear();
    if (!q || !k_pool || !v_pool || !block_table || !pos || !out) return fail(DEC_ERR_INVALID_ARG, "NULL pointer");
    if ((k_new == nullptr) != (v_new == nullptr)) return fail(DEC_ERR_INVALID_ARG, "k_new and v_new: both or neither");
    if (B <= 0 || nq <= 0 || nkv <= 0 || nq % nkv != 0 || max_pages <= 0)
        return fail(DEC_ERR_INVALID_ARG, "bad B / heads / max_pages");
    if (nq / nkv > 16) return fail(DEC_ERR_UNSUPPORTED, "more than 16 q heads per kv head");
    if (d != 64 && d != 128) return fail(DEC_ERR_UNSUPPORTED, "d must be 64 or 128");
    if (page_size != 16) return fail(DEC_ERR_UNSUPPORTED, "page_size must be 16");
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    int dev = 0;
    cudaGetDevice(&dev);
    Scratch& S = g_scratch[dev];
    const int sms = device_sms();
    const int splits = attn_decode_splits(B, nkv, max_pages * 16, sms, false);
    CUDA_TRY(grow(&S.attn_part, &S.attn_part_n, (size_t)B * nq * splits * (d + 2), false));
    CUDA_TRY(grow(&S.attn_cnt, &S.attn_cnt_n, (size_t)B * nkv, true));
    size_t one = 0;
    if (!S.err) CUDA_TRY(grow(&S.err, &one, 1, true));
    AttnDecodeArgs a{};
    a.q_bf = static_cast<const uint16_t*>(q);
    a.k_new = static_cast<const uint16_t*>(k_new);
    a.v_new = static_cast<const uint16_t*>(v_new);
    a.eps = 1e-6f;
    a.rope = fused_rope;
    a.rope_base = rope_base;
    a.k_pool = static_cast<uint16_t*>(k_pool);
    a.v_pool = static_cast<uint16_t*>(v_pool);
    a.block_table = block_table;
    a.max_pages = max_pages;
    a.pos = pos;
    a.B = B;
    a.nq = nq;
    a.nkv = nkv;
    a.d = d;
    a.scale = scale;
    a.splits = splits;
    a.part = S.attn_part;
    a.counters = S.attn_cnt;
    a.out = static_cast<uint16_t*>(out);
    a.err = S.err;
    CUDA_TRY(attn_decode_launch(a, reinterpret_cast<cudaStream_t>(stream), false));
    return DEC_OK;
}

dec_status moe_route_topk(const float* logits, int32_t T, int32_t E, int32_t k, int32_t renorm, int32_t* idx_out,
                          float* w_out, dec_stream_t stream) {
    g_err.clear();
    if (!logits || !idx_out || !w_out) return fail(DEC_ERR_INVALID_ARG, "NULL pointer");
    if (T <= 0 || E <= 0 || k <= 0 || k > E) return fail(DEC_ERR_INVALID_ARG, "bad T / E / k");
    if (E > 256 || k > 16) return fail(DEC_ERR_UNSUPPORTED, "E <= 256 and k <= 16");
    // the same routing kernel as the MoE layer, without the shared-expert gate
    MoeRouteArgs r{};
    r.logits = logits;
    r.E = E;
    r.k = k;
    r.renorm = renorm;
    r.idx = idx_out;
    r.w = w_out;
    CUDA_TRY(moe_route_launch(r, T, reinterpret_cast<cudaStream_t>(stream), false));
    return DEC_OK;
}

dec_status moe_experts(const void* x, const int32_t* idx, const float* w, int32_t T, int32_t h, int32_t E,
                       int32_t k, int32_t I, const void* Wgu, const void* Wd, float* out, dec_stream_t stream) {
    g_err.clear();
    if (!x || !idx || !w || !Wgu || !Wd || !out) return fail(DEC_ERR_INVALID_ARG, "NULL pointer");
    if (T <= 0 || h <= 0 || E <= 0 || k <= 0 || k > E || I <= 0) return fail(DEC_ERR_INVALID_ARG, "bad T / h / E / k / I");
    if (E > 256 || k > 16) return fail(DEC_ERR_UNSUPPORTED, "E <= 256 and k <= 16");
    if (h % 8 != 0 || I % 8 != 0) return fail(DEC_ERR_UNSUPPORTED, "h and I must be multiples of 8");
    const int nb = grouped_nb_for(T);
    const int cap = device_smem_cap();
    if (!grouped_fits(nb, h, cap) || !grouped_fits(nb, I, cap))
        return fail(DEC_ERR_UNSUPPORTED, "rows too long for shared memory");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    int dev = 0;
    cudaGetDevice(&dev);
    Scratch& S = g_scratch[dev];
    size_t one = 0;
    if (!S.err) CUDA_TRY(grow(&S.err, &one, 1, true));
    const size_t tk = (size_t)T * k;
    CUDA_TRY(grow(&S.moe_i, &S.moe_i_n, 6 * tk + 1, false));
    CUDA_TRY(grow(&S.moe_act, &S.moe_act_n, tk * I, false));
    CUDA_TRY(grow(&S.moe_y, &S.moe_y_n, tk * h, false));
    int32_t* perm = S.moe_i;
    int32_t* inv = perm + tk;
    int32_t* groups = inv + tk;
    int32_t* n_groups = groups + 4 * tk;
    MoePermArgs p{};
    p.idx = idx;
    p.n = T;
    p.k = k;
    p.E = E;
    p.nb = nb;
    p.perm_tok = perm;
    p.inv = inv;
    p.groups = groups;
    p.n_groups = n_groups;
    CUDA_TRY(moe_permute_launch(p, st, false));
    GroupedGemvArgs g{};
    g.W = static_cast<const uint16_t*>(Wgu);
    g.wstride = (size_t)2 * I * h;
    g.M = 2 * I;
    g.K = h;
    g.E = E;
    g.groups = groups;
    g.n_groups = n_groups;
    g.x = static_cast<const uint16_t*>(x);
    g.x_map = perm;
    g.ldx = h;
    g.act = S.moe_act;
    g.ldact = I;
    g.err = S.err;
    g.smem_cap = cap;
    const int sms = device_sms();
    CUDA_TRY(grouped_gemv_launch(g, nb, true, st, sms, false));
    g.W = static_cast<const uint16_t*>(Wd);
    g.wstride = (size_t)h * I;
    g.M = h;
    g.K = I;
    g.x = S.moe_act;
    g.x_map = nullptr;
    g.ldx = I;
    g.act = nullptr;
    g.y = S.moe_y;
    g.ldy = h;
    CUDA_TRY(grouped_gemv_launch(g, nb, false, st, sms, false));
    CUDA_TRY(cudaMemsetAsync(out, 0, (size_t)T * h * sizeof(float), st));
    MoeCombineArgs m{};
    m.x = out;
    m.y = S.moe_y;
    m.w = w;
    m.inv = inv;
    m.k = k;
    m.h = h;
    CUDA_TRY(moe_combine_launch(m, T, st, false));
    return DEC_OK;
}

dec_status weight_gemv(const void* W, const void* x, int32_t B, int32_t N, int32_t K, float* y, dec_stream_t stream) {
    g_err.clear();
    if (!W || !x || !y) return fail(DEC_ERR_INVALID_ARG, "NULL pointer");
    if (B <= 0 || N <= 0 || K <= 0) return fail(DEC_ERR_INVALID_ARG, "B, N, K must be positive");
    if (K % 8 != 0) return fail(DEC_ERR_UNSUPPORTED, "K must be a multiple of 8");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    int dev = 0;
    cudaGetDevice(&dev);
    Scratch& S = g_scratch[dev];
    size_t one = 0;
    if (!S.err) CUDA_TRY(grow(&S.err, &one, 1, true));
    const int sms = device_sms();
    const int cap = device_smem_cap();
    if (B <= 8 && gemv_fits(B, K, cap)) {
        GemvArgs a{};
        a.W = static_cast<const uint16_t*>(W);
        a.N = N;
        a.K = K;
        a.B = B;
        a.xb = static_cast<const uint16_t*>(x);
        a.ldx = K;
        a.y = y;
        a.ldy = N;
        a.err = S.err;
        a.smem_cap = cap;
        CUDA_TRY(gemv_launch(a, GEMV_STORE, st, sms, false));
        return DEC_OK;
    }
    CUDA_TRY(grow(&S.ws, &S.ws_n, gemm_ws_floats(sms), false));
    CUDA_TRY(grow(&S.cnt, &S.cnt_n, (size_t)gemm_cnt_needed(N, B), true));
    GemmPlan plan;
    CUDA_TRY(gemm_plan(&plan, static_cast<const uint16_t*>(W), N, K, static_cast<const uint16_t*>(x), B, sms, S.ws));
    GemmArgs a{};
    a.epi = GEMM_STORE;
    a.y = y;
    a.ldy = N;
    a.cnt = S.cnt;
    a.err = S.err;
    CUDA_TRY(gemm_launch(plan, a, st, false));
    return DEC_OK;
}

dec_status ffn_gate_up(const void* Wgu, const float* x, const float* gain, float eps, int32_t B, int32_t I, int32_t K,
                       void* act, dec_stream_t stream) {
    g_err.clear();
    if (!Wgu || !x || !gain || !act) return fail(DEC_ERR_INVALID_ARG, "NULL pointer");
    if (B <= 0 || I <= 0 || K <= 0 || !(eps > 0.f)) return fail(DEC_ERR_INVALID_ARG, "B, I, K, eps must be positive");
    if (K % 8 != 0 || I % 2 != 0) return fail(DEC_ERR_UNSUPPORTED, "K must be a multiple of 8 and I even");
    const int cap = device_smem_cap();
    if (B > 8 || !gemv_fits(B, K, cap)) return fail(DEC_ERR_UNSUPPORTED, "B * K too large for the GEMV");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    int dev = 0;
    cudaGetDevice(&dev);
    Scratch& S = g_scratch[dev];
    size_t one = 0;
    if (!S.err) CUDA_TRY(grow(&S.err, &one, 1, true));
    // the decode step's launch: RMSNorm prologue, interleaved gate/up rows, SiLU(g) * u epilogue
    GemvArgs a{};
    a.W = static_cast<const uint16_t*>(Wgu);
    a.N = 2 * I;
    a.K = K;
    a.B = B;
    a.xr = x;
    a.g = gain;
    a.eps = eps;
    a.ldx = K;
    a.act = static_cast<uint16_t*>(act);
    a.ldact = I;
    a.err = S.err;
    a.smem_cap = cap;
    CUDA_TRY(gemv_launch(a, GEMV_SWIGLU, st, device_sms(), false));
    return DEC_OK;
}

dec_status weight_gemv_q8(const void* Wq, const float* scale, const void* x, int32_t B, int32_t N, int32_t K, float* y,
                          dec_stream_t stream) {
    g_err.clear();
    if (!Wq || !scale || !x || !y) return fail(DEC_ERR_INVALID_ARG, "NULL pointer");
    if (B <= 0 || N <= 0 || K <= 0) return fail(DEC_ERR_INVALID_ARG, "B, N, K must be positive");
    if (K % 16 != 0) return fail(DEC_ERR_UNSUPPORTED, "K must be a multiple of 16");
    const int cap = device_smem_cap();
    if (B > 8 || !gemv_fits(B, K, cap, true)) return fail(DEC_ERR_UNSUPPORTED, "B * K too large for the q8 GEMV");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    int dev = 0;
    cudaGetDevice(&dev);
    Scratch& S = g_scratch[dev];
    size_t one = 0;
    if (!S.err) CUDA_TRY(grow(&S.err, &one, 1, true));
    GemvArgs a{};
    a.Wq = static_cast<const int8_t*>(Wq);
    a.wscale = scale;
    a.N = N;
    a.K = K;
    a.B = B;
    a.xb = static_cast<const uint16_t*>(x);
    a.ldx = K;
    a.y = y;
    a.ldy = N;
    a.err = S.err;
    a.smem_cap = cap;
    CUDA_TRY(gemv_launch(a, GEMV_STORE, st, device_sms(), false));
    return DEC_OK;
}

dec_status dec_check_standalone(dec_stream_t stream) {
    g_err.clear();
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    CUDA_TRY(cudaStreamSynchronize(st));
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    int dev = 0;
    cudaGetDevice(&dev);
    auto it = g_scratch.find(dev);
    if (it == g_scratch.end() || !it->second.err) return DEC_OK;
    Scratch& S = it->second;
    int e = 0;
    CUDA_TRY(cudaMemcpy(&e, S.err, sizeof(int), cudaMemcpyDeviceToHost));
    if (!e) return DEC_OK;
    // clear the word and the GEMM tile counters an abandoned reduction can leave behind
    CUDA_TRY(cudaMemset(S.err, 0, sizeof(int)));
    if (S.cnt) CUDA_TRY(cudaMemset(S.cnt, 0, sizeof(int) * S.cnt_n));
    CUDA_TRY(cudaDeviceSynchronize());
    return fail(DEC_ERR_TIMEOUT, "a bounded device wait of a standalone call ran out; its output is not valid");
}

dec_status dec_test_fail_alloc(int32_t n) {
    g_fail_alloc_in.store(n > 0 ? n : 0);
    return DEC_OK;
}

dec_status dec_test_gemm_wait(int32_t extra_pieces, int64_t limit_cycles) {
    if (extra_pieces < 0 || limit_cycles < 0) return fail(DEC_ERR_INVALID_ARG, "negative argument");
    gemm_set_test_wait(extra_pieces, limit_cycles);
    return DEC_OK;
}

int32_t dec_test_streamk_check(int32_t M, int32_t N, int32_t K, int32_t ctas) {
    return gemm_streamk_check(M, N, K, ctas);
}

}  // extern "C"
