/*
 * dec_api.h — C ABI of the B200 decoder-layer library (libdec.so).
 *
 * The library runs the per-token forward of a decoder-only transformer layer
 * stack over a paged bf16 KV cache, as chunked prefill and as batched
 * single-token decode, entirely in CUDA kernels written for sm_100a.
 *
 * Sources (the pages this interface follows):
 *   ANEDVD src/engine.zig — Engine.init / forward / prefill / reset / deinit,
 *     the ContextOverflow error and its test "an over-long prompt is refused".
 *   frink_models decoder.rs — gqa_attention (CUDA gqa_decode), MultiSeqKv
 *     (per-sequence caches for batched decode), route_top_k.
 *   cortiq_engine pipeline.rs — the prefill/decode contract (every token is
 *     forwarded once and enters the KV cache once; logits come from the last
 *     forwarded token), empty input refused.
 *
 * Conventions for every entry point:
 *   - Matrices are row-major [out][in] bf16 (passed as void*, 2 bytes per
 *     element, IEEE bfloat16 bits). 1-D parameters (norm gains, biases, the
 *     shared-expert gate vector) are fp32 arrays.
 *   - Every call returns a dec_status. On failure nothing has been launched
 *     unless the status is DEC_ERR_CUDA; dec_last_error() gives a message
 *     (thread-local, valid until the next call on the same thread).
 *   - Work is enqueued on the caller's stream and is not synchronised unless
 *     a host output buffer is given (documented per call). Host inputs are copied
 *     through pinned staging memory before the call returns, so the caller may reuse
 *     its buffers at once.
 *   - A stream argument of 0 means the legacy default stream.
 *   - Device waits are bounded. A kernel whose wait runs out sets an error word and
 *     returns (nothing traps). The word is reported as DEC_ERR_TIMEOUT by the next call
 *     that synchronises (a host logits buffer, dec_last_argmax, dec_check; for the
 *     standalone calls dec_check_standalone), which also clears it; the output of the
 *     failed call is not valid.
 */
#ifndef DEC_API_H
#define DEC_API_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* dec_stream_t; /* same type as cudaStream_t */

typedef enum dec_status {
    DEC_OK = 0,
    DEC_ERR_INVALID_ARG = 1,      /* bad pointer, shape, token id or position */
    DEC_ERR_CONTEXT_OVERFLOW = 2, /* pos0 + T > max_context (ANEDVD ContextOverflow) */
    DEC_ERR_PAGES_EXHAUSTED = 3,  /* the KV page pool has no free page */
    DEC_ERR_OOM = 4,              /* device allocation failed */
    DEC_ERR_CUDA = 5,             /* a CUDA call failed; see dec_last_error() */
    DEC_ERR_TIMEOUT = 6,          /* a bounded wait ran out */
    DEC_ERR_UNSUPPORTED = 7       /* shape outside what the kernels handle */
} dec_status;

/* Model shape. Zero disables an optional feature. */
typedef struct dec_config {
    int32_t hidden;          /* h */
    int32_t layers;          /* L */
    int32_t n_q_heads;       /* nq */
    int32_t n_kv_heads;      /* nkv; nq % nkv == 0; q head i reads kv head i / (nq / nkv) */
    int32_t head_dim;        /* d: 64 or 128 */
    int32_t ffn_inter;       /* I of the dense SwiGLU FFN (0 for MoE models) */
    int32_t vocab;           /* V */
    int32_t tied_embeddings; /* 1: the LM head is the embedding matrix */
    int32_t qkv_bias;        /* 1: an fp32 bias is added to q, k, v before QK-norm and RoPE */
    int32_t qk_norm;         /* 1: per-head RMSNorm of q and k (weights [d]) before RoPE */
    int32_t n_experts;       /* E routed experts (0 = dense FFN) */
    int32_t top_k;           /* experts per token */
    int32_t expert_inter;    /* routed expert inter size */
    int32_t shared_inter;    /* shared expert inter size (0 = none) */
    int32_t shared_gate;     /* 1: the shared expert is scaled by sigmoid(gate_vec . xn) */
    int32_t norm_topk_prob;  /* 1: the k routing weights are renormalised to sum to 1 */
    float rms_eps;           /* RMSNorm epsilon */
    float rope_base;         /* RoPE base (theta) */
    int32_t max_batch;       /* sequences decoded together (dec_step's B <= max_batch) */
    int32_t max_context;     /* positions per sequence */
    int32_t page_size;       /* KV page size in tokens: 16 */
    int32_t prefill_chunk;   /* tokens per prefill chunk (layer-major within a chunk) */
    int32_t n_pages;         /* KV pages in the pool; 0 = max_batch * ceil(max_context / page_size) */
    /* Sliding-window attention (ANEDVD attentionDecode .window; cortiq layer_window): layer l
     * is windowed when sliding_window > 0 and (l + 1) % max(swa_pattern, 1) != 0, and its
     * query at position p then attends positions p - sliding_window + 1 .. p only. */
    int32_t sliding_window;
    int32_t swa_pattern;
    float attn_softcap;      /* > 0: each scaled attention score s becomes c * tanh(s / c) */
    float final_softcap;     /* > 0: each logit v becomes c * tanh(v / c) (ANEDVD runHead) */
    int32_t sandwich_norms;  /* 1: the o_proj and the dense FFN outputs are RMS-normalised with
                                post_attn_norm / post_ffn_norm before each residual add */
    int32_t weight_format;   /* 0: bf16 projections; 1: q8_row: the QKV, o, gate, up and down
                                projections and the untied LM head are int8 [rows][cols] with one
                                fp32 scale per row, W[n][k] = scale[n] * q[n][k] (dense models) */
} dec_config;

/* One layer's weights. Pointers may be host or device memory; they are read
 * during dec_init only (the library keeps its own repacked copies). */
typedef struct dec_layer_weights {
    const float* attn_norm;  /* [h] */
    const float* ffn_norm;   /* [h] */
    const void* wqkv;        /* bf16 [nq*d + 2*nkv*d][h]: rows q, then k, then v */
    const float* bqkv;       /* [nq*d + 2*nkv*d] or NULL */
    const float* q_norm;     /* [d] or NULL */
    const float* k_norm;     /* [d] or NULL */
    const void* wo;          /* bf16 [h][nq*d] */
    const void* w_gate;      /* dense: bf16 [I][h] */
    const void* w_up;        /* dense: bf16 [I][h] */
    const void* w_down;      /* dense: bf16 [h][I] */
    const void* w_router;    /* MoE: bf16 [E][h] */
    const void* e_gate;      /* MoE: bf16 [E][Ie][h] */
    const void* e_up;        /* MoE: bf16 [E][Ie][h] */
    const void* e_down;      /* MoE: bf16 [E][h][Ie] */
    const void* s_gate;      /* shared expert: bf16 [Is][h] or NULL */
    const void* s_up;        /* bf16 [Is][h] */
    const void* s_down;      /* bf16 [h][Is] */
    const float* s_gate_vec; /* [h] or NULL */
    const float* post_attn_norm; /* sandwich_norms: [h] */
    const float* post_ffn_norm;  /* sandwich_norms: [h] */
    /* weight_format 1: the row scales of wqkv, wo, w_gate, w_up, w_down (whose pointers then
     * hold int8 values, same shapes) */
    const float* wqkv_scale;     /* [nq*d + 2*nkv*d] */
    const float* wo_scale;       /* [h] */
    const float* w_gate_scale;   /* [I] */
    const float* w_up_scale;     /* [I] */
    const float* w_down_scale;   /* [h] */
} dec_layer_weights;

typedef struct dec_weights {
    const void* embed;                /* bf16 [V][h] */
    const void* lm_head;              /* bf16 [V][h]; ignored when tied_embeddings */
    const float* final_norm;          /* [h] */
    const dec_layer_weights* layers;  /* host array of L entries */
    const float* lm_head_scale;       /* weight_format 1: [V] row scales of the int8 lm_head */
} dec_weights;

typedef struct dec_ctx dec_ctx;

/* Build a context on the current device: validate the shape, copy and repack the
 * weights into library-owned device memory (fused gate/up), allocate the paged
 * KV pool, the block table and the workspace. Like ANEDVD Engine.init, but the
 * caller's weight buffers may be freed as soon as this returns (the copies are
 * complete: the call synchronises `stream`).
 * Errors: NULL cfg / w / out, or a non-positive size -> INVALID_ARG; a shape the kernels
 * do not handle (more than 16 query heads per kv head, head_dim other than 64 / 128,
 * hidden or an FFN width not a multiple of
 * 8, page_size other than 16, more than 256 experts or top_k above 16, MoE rows too long
 * for the grouped projections' shared memory, sandwich norms or q8_row weights with MoE,
 * q8_row with tied embeddings) -> UNSUPPORTED; device memory -> OOM. */
dec_status dec_init(const dec_config* cfg, const dec_weights* w, dec_stream_t stream, dec_ctx** out);

/* Release everything dec_init allocated (ANEDVD Engine.deinit). NULL is a no-op. */
dec_status dec_free(dec_ctx* ctx);

/* Forget sequence `seq` (or all sequences when seq == -1): its pages return to the
 * pool and its length becomes 0 (ANEDVD Engine.reset; cortiq kv_cache.clear). */
dec_status dec_reset(dec_ctx* ctx, int32_t seq);

/* Prefill T prompt tokens of sequence `seq` at positions pos0 .. pos0+T-1
 * (ANEDVD Engine.prefill; cortiq prefill_batch). Runs layer-major over chunks of
 * cfg.prefill_chunk tokens; every token's k and v enter the cache once.
 *   tokens     host int32 [T], each in [0, V)
 *   pos0       must equal the sequence's current length (each token enters once)
 *   logits_out fp32 [V]: logits of the last token. A device pointer is written by the
 *              LM head directly (stream-ordered, no synchronisation); a host pointer
 *              makes the call synchronise before returning; NULL stores no logits (the
 *              greedy token is still kept for dec_last_argmax).
 * Stream-ordered: with a device or NULL logits_out the call returns without waiting for
 * the device.
 * Errors: T <= 0 or a bad token -> INVALID_ARG; pos0 + T > max_context ->
 * CONTEXT_OVERFLOW (exact fit allowed); no free page -> PAGES_EXHAUSTED. */
dec_status dec_prefill(dec_ctx* ctx, int32_t seq, const int32_t* tokens, int32_t T, int32_t pos0,
                       float* logits_out);

/* One decode step for sequences 0..B-1 (ANEDVD Engine.forward, batched as frink
 * MultiSeqKv): token tokens[b] at position pos[b] of sequence b.
 *   tokens, pos host int32 [B]; pos[b] must equal sequence b's current length and be
 *               < max_context (else CONTEXT_OVERFLOW).
 *   logits_out  fp32 [B][V], device or host pointer as in dec_prefill. NULL is the
 *               greedy-only step: the LM head stores no logits at all and keeps only
 *               each row's argmax (read with dec_last_argmax), as the pages' folded
 *               head downloads the argmax instead of the full-vocabulary logits
 *               (frink_models decoder.rs FoldedLmHead).
 * The whole step is replayed from a CUDA graph captured on the first call for each B;
 * the logits destination is read by the head on the device, so the same graph serves
 * device, host and NULL outputs. With a device or NULL logits_out the call returns
 * without waiting for the device. */
dec_status dec_step(dec_ctx* ctx, const int32_t* tokens, const int32_t* pos, int32_t B, float* logits_out);

/* Multi-position verify (cortiq_engine pipeline.rs forward_pair: several positions of one
 * sequence share one pass over the weights, as speculative decoding's check of draft
 * tokens needs): forward tokens[0..N-1] of sequence `seq` at positions pos0 .. pos0+N-1
 * and return the logits of every position. Equal to N dec_step calls on that sequence,
 * but each projection streams its weights once for all N positions.
 *   tokens     host int32 [N], 1 <= N <= 8, each in [0, V)
 *   pos0       must equal the sequence's current length; the N rows enter the cache
 *   logits_out fp32 [N][V] (row i = position pos0 + i), device, host or NULL as in dec_prefill
 * dec_last_argmax(ctx, out, N) then gives the greedy token of every position. Reject
 * draft tokens with dec_truncate.
 * Errors: N outside [1, 8], a bad token or pos0 -> INVALID_ARG; pos0 + N > max_context ->
 * CONTEXT_OVERFLOW; no free page -> PAGES_EXHAUSTED. */
dec_status dec_verify(dec_ctx* ctx, int32_t seq, const int32_t* tokens, int32_t N, int32_t pos0,
                      float* logits_out);

/* Roll sequence `seq` back to its first `len` positions (cortiq_engine pipeline.rs
 * truncate_last: the KV rows of rejected draft tokens are dropped). Pages past the new
 * length return to the pool. Host-side only: nothing is launched and nothing waits.
 * Errors: len < 0 or len > the current length -> INVALID_ARG. */
dec_status dec_truncate(dec_ctx* ctx, int32_t seq, int32_t len);

/* Greedy tokens of the last dec_step / dec_prefill / dec_verify: argmax over each logits row,
 * lowest index on ties. out: host int32 [B] (B = rows of the last call). Synchronises;
 * returns DEC_ERR_TIMEOUT if a device wait of an earlier call ran out. */
dec_status dec_last_argmax(dec_ctx* ctx, int32_t* out, int32_t B);

/* Synchronise the context's stream and report whether a bounded device wait of any
 * earlier call on this context ran out (DEC_ERR_TIMEOUT; the outputs of the failing call
 * are not valid). Clears the error word and the tile counters an abandoned GEMM
 * reduction leaves behind, so later calls run normally. */
dec_status dec_check(dec_ctx* ctx);

/* ---------------------------------------------------------------- standalone hot-path calls */

/* Causal GQA decode attention over a paged bf16 KV cache (frink gqa_attention /
 * launch_gqa_decode; ANEDVD cpu.attentionDecode). For each sequence b the query
 * sits at position p = pos[b] and attends cache rows 0..p:
 *   out[b][h] = sum_j softmax_j(q[b][h] . K[b][j] * scale) V[b][j],  kv head h / (nq/nkv).
 *   q          device bf16 [B][nq][d]
 *   k_new/v_new device bf16 [B][nkv][d], or both NULL: the row p already holds them
 *   k_pool/v_pool device bf16 [n_pages][nkv][page_size][d]; row j of sequence b is slot
 *              j % page_size of page block_table[b][j / page_size]
 *   block_table device int32 [B][max_pages]
 *   pos        device int32 [B], 0 <= pos[b] < max_pages * page_size
 *   fused_rope 1: q and k_new are rotated to position p (half-split pairs, angle
 *              p * rope_base^(-2i/d)) and rounded to bf16 before use; k_new/v_new are
 *              written to row p first (the cache append). 0: used as given.
 *   out        device bf16 [B][nq][d]
 * Scratch for the split-context partial results is allocated by the library on
 * first use and kept for later calls on the same device. d must be 64 or 128,
 * page_size 16. */
dec_status gqa_decode_attn(const void* q, const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                           const int32_t* block_table, int32_t max_pages, const int32_t* pos, int32_t B,
                           int32_t nq, int32_t nkv, int32_t d, int32_t page_size, float scale,
                           int32_t fused_rope, float rope_base, void* out, dec_stream_t stream);

/* gqa_decode_attn without any device allocation. The source pages have no
 * counterpart to this call; it exists for callers that must not let a library
 * allocate device memory: programs whose device memory is reserved up front by their
 * own pool allocator, latency-bound loops that cannot absorb the synchronisation a
 * cudaMalloc/cudaFree may cause, and plugin hosts that forbid allocation after
 * start-up. Arguments, layout and results are those of gqa_decode_attn.
 *   - Scratch lives in one fixed array inside the library image, present on every
 *     device that loads the library until the process exits: room for 16384
 *     (sequence, kv head) pairs and 1048576 floats of split partials. Shapes that need
 *     more are refused with DEC_ERR_UNSUPPORTED before anything is launched.
 *   - The first call on a device looks up the array's device address (a one-time
 *     set-up per device); make that first call before any stream capture begins.
 *   - Every call uses the same array. The call clears the merge counters it needs
 *     (an asynchronous memset on `stream`) before its kernel; calls whose work can
 *     overlap on the GPU (different streams, or several threads) race on the array
 *     and must be serialised by the caller.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine. */
dec_status gqa_decode_attn_noalloc(const void* q, const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                                   const int32_t* block_table, int32_t max_pages, const int32_t* pos, int32_t B,
                                   int32_t nq, int32_t nkv, int32_t d, int32_t page_size, float scale,
                                   int32_t fused_rope, float rope_base, void* out, dec_stream_t stream);

/* MoE routing (ANEDVD cpu.moeRoute; frink route_top_k; cortiq MoeFfn): for each of
 * T rows of router logits, P = softmax over all E, then the k most probable experts
 * in descending order (lower index first on equal probability); weights P, or P /
 * sum_topk P when renorm. logits device fp32 [T][E]; idx_out device int32 [T][k];
 * w_out device fp32 [T][k]. E <= 256, k <= E. */
dec_status moe_route_topk(const float* logits, int32_t T, int32_t E, int32_t k, int32_t renorm, int32_t* idx_out,
                          float* w_out, dec_stream_t stream);

/* Routed experts of the MoE FFN for T token rows whose routing is given (ANEDVD
 * moeExpertAccum; frink decoder.rs expert loop; cortiq MoeFfn):
 *   out[t] = sum_j w[t][j] * SwiGLU_{idx[t][j]}(x[t]),
 *   SwiGLU_e(x) = Wd_e . bf16(SiLU(Wg_e . x) * (Wu_e . x)),
 * summed in top-k order. The tokens are permuted by expert and each expert's weights
 * stream once per group of at most 8 of its tokens (the same kernels as the MoE layer).
 *   x     device bf16 [T][h]
 *   idx   device int32 [T][k]; an entry outside [0, E) contributes nothing
 *   w     device fp32 [T][k]
 *   Wgu   device bf16 [E][2I][h]: gate row i of expert e at row 2i, up row i at 2i+1
 *   Wd    device bf16 [E][h][I]
 *   out   device fp32 [T][h], overwritten; stream-ordered, the call does not synchronise.
 * Errors: NULL pointer, T/h/E/k/I <= 0 or k > E -> INVALID_ARG; E > 256, k > 16, h or I
 * not a multiple of 8, or rows too long for shared memory -> UNSUPPORTED. Scratch
 * buffers are kept per device and grow on demand; calls must be serialised. */
dec_status moe_experts(const void* x, const int32_t* idx, const float* w, int32_t T, int32_t h, int32_t E,
                       int32_t k, int32_t I, const void* Wgu, const void* Wd, float* out, dec_stream_t stream);

/* Weight-streaming projection y[b][n] = sum_k W[n][k] x[b][k] (ANEDVD 1x1 conv
 * kernels; every projection of the layer). W device bf16 [N][K]; x device bf16
 * [B][K]; y device fp32 [B][N]. K % 8 == 0. B <= 8 streams W once through the
 * CUDA-core GEMV; larger B runs the tcgen05 tensor-core GEMM. */
dec_status weight_gemv(const void* W, const void* x, int32_t B, int32_t N, int32_t K, float* y,
                       dec_stream_t stream);

/* Synchronise `stream` and report whether a bounded device wait of a standalone call
 * (weight_gemv, weight_gemv_q8, moe_experts) on the current device ran out since the last check:
 * DEC_ERR_TIMEOUT, and the word and the GEMM tile counters are cleared. */
dec_status dec_check_standalone(dec_stream_t stream);

/* The front half of the dense SwiGLU FFN in one weight-streaming pass, as the decode step runs
 * it (ANEDVD engine.zig: rmsnormColumn, then the fused gate/up/SiLU program of
 * makeFusedFfnKernel): for each of B rows,
 *   xn = bf16(x * (1 / sqrt(mean(x^2) + eps)) * gain),
 *   act[i] = bf16(SiLU(Wgu[2i] . xn) * (Wgu[2i+1] . xn)),  SiLU(z) = z / (1 + e^-z).
 *   Wgu  device bf16 [2I][K]: gate row i at 2i, up row i at 2i+1
 *   x    device fp32 [B][K] (the residual stream); gain device fp32 [K]
 *   act  device bf16 [B][I]
 * B <= 8. Errors: NULL pointer or a non-positive size -> INVALID_ARG; K not a multiple of 8,
 * I odd, B > 8 or B * K beyond shared memory -> UNSUPPORTED. Stream-ordered. */
dec_status ffn_gate_up(const void* Wgu, const float* x, const float* gain, float eps, int32_t B, int32_t I, int32_t K,
                       void* act, dec_stream_t stream);

/* q8_row weight-streaming projection (cortiq_engine pipeline.rs q8_row_parts: int8 rows with
 * one fp32 scale per row): y[b][n] = scale[n] * sum_k Wq[n][k] x[b][k], the row's exactly
 * dequantised dot product, accumulated in fp32. Each weight byte is read once.
 *   Wq device int8 [N][K]; scale device fp32 [N]; x device bf16 [B][K]; y device fp32 [B][N]
 * Errors: NULL pointer or a non-positive size -> INVALID_ARG; K not a multiple of 16, B > 8
 * or B * K beyond the kernel's shared memory -> UNSUPPORTED. Stream-ordered; a device wait
 * that runs out is reported by dec_check_standalone. */
dec_status weight_gemv_q8(const void* Wq, const float* scale, const void* x, int32_t B, int32_t N, int32_t K,
                          float* y, dec_stream_t stream);

/* ---------------------------------------------------------------- test hooks */

/* The n-th device allocation made by the library from now on fails as if the device
 * were out of memory (n = 0 turns this off). Process-wide; for testing the OOM paths. */
dec_status dec_test_fail_alloc(int32_t n);

/* The stream-K reduction wait of tensor-core GEMM launches made after this call waits
 * for `extra_pieces` more partial tiles than exist, giving up after `limit_cycles` SM
 * clock cycles (0 = the normal limit of about 1 s). (0, 0) restores normal operation.
 * Process-wide; a dec_step graph keeps the setting it was captured with. For testing the
 * DEC_ERR_TIMEOUT path: a CTA whose wait runs out skips its remaining outputs but still
 * drains its accumulators, so it leaves with all its loads and MMAs complete. */
dec_status dec_test_gemm_wait(int32_t extra_pieces, int64_t limit_cycles);

/* Host-side check (no GPU needed) of the work split the persistent tensor-core GEMM uses
 * for an M x N x K product over `ctas` CTAs (it launches min(SMs, units / 8) of them, a
 * unit being one 128-row tile x one 64-wide k block): every unit is covered once, every
 * partial tile another CTA finishes is the first segment its CTA processes, and every tile
 * split between CTAs has exactly one finisher, the CTA holding its last k blocks, whose
 * expected pieces all exist. Returns the number of violations (0 = sound), or -1 for a
 * non-positive argument. */
int32_t dec_test_streamk_check(int32_t M, int32_t N, int32_t K, int32_t ctas);

/* Copy cache rows [pos0, pos0+n) of layer `layer` of sequence `seq` to / from host
 * buffers bf16 [n][nkv*d] (k and v). dec_kv_write also extends the sequence's length
 * to pos0+n when that is longer (allocating pages). Both synchronise. */
dec_status dec_kv_read(dec_ctx* ctx, int32_t seq, int32_t layer, int32_t pos0, int32_t n, void* k, void* v);
dec_status dec_kv_write(dec_ctx* ctx, int32_t seq, int32_t layer, int32_t pos0, int32_t n, const void* k,
                        const void* v);

/* Routing decisions of the last dec_step: host int32 [L][B][top_k]. Synchronises. */
dec_status dec_last_routes(dec_ctx* ctx, int32_t* idx, int32_t B);

/* Residual stream after the last layer of the last dec_step: host fp32 [B][h]. Synchronises. */
dec_status dec_last_hidden(dec_ctx* ctx, float* out, int32_t B);

/* Current length of sequence `seq`. */
dec_status dec_seq_len(dec_ctx* ctx, int32_t seq, int32_t* len_out);

/* Message for the last failure on this thread ("" if none). */
const char* dec_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* DEC_API_H */
