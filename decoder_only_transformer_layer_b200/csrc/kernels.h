// Internal launcher interface between the C ABI (dec_api.cu) and the kernels.
// All pointers are device pointers; bf16 tensors are uint16_t bit patterns.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

namespace dec {

// ----------------------------------------------------------------- GEMV (decode projections)

enum GemvEpi { GEMV_STORE = 0, GEMV_RESID = 1, GEMV_SWIGLU = 2 };

struct GemvArgs {
    const uint16_t* W;  // [N][K]
    const int8_t* Wq;   // q8_row weights [N][K] (used instead of W when set), with
    const float* wscale;  // one fp32 scale per row: W[n][k] = wscale[n] * Wq[n][k]
    int N, K;
    int B, nb;          // active columns; nb = compiled column count (set by the launcher)
    const uint16_t* xb; // bf16 input [B][ldx], or
    const float* xr;    // fp32 residual [B][ldx] normalised in the prologue with gain g
    const float* g;
    float eps;
    int ldx;
    float* y;           // STORE: y[b*ldy+n] = acc (+bias); RESID: y[b*ldy+n] += acc
    float* const* y_ptr;  // STORE: when set, the destination is *y_ptr, read on the device
                          // (a null *y_ptr stores nothing: only the greedy argmax is kept)
    int ldy;
    const float* bias;
    uint16_t* act;      // SWIGLU: act[b*ldact + n/2] = bf16(silu(acc[even]) * acc[odd])
    int ldact;
    unsigned long long* amax;  // STORE: per column, packed greedy argmax of y (null = off)
    float softcap;      // STORE: > 0 stores (and takes the argmax of) softcap * tanh(v / softcap)
    int* err;
    int smem_cap;
};

int gemv_nb_for(int B);
bool gemv_fits(int B, int K, int smem_cap, bool q8 = false);
cudaError_t gemv_launch(GemvArgs a, int epi, cudaStream_t st, int num_sms, bool pdl);

// ----------------------------------------------------------------- tcgen05 GEMM (prefill, large batch)

enum GemmEpi { GEMM_STORE = 0, GEMM_RESID = 1, GEMM_SWIGLU = 2 };

struct GemmPlan {
    CUtensorMap tmA;  // weights [M][K], box 64 x 128
    CUtensorMap tmB;  // activations [N][K], box 64 x BN
    const float* ws;
    int M, N, K, bn, nc;  // nc: persistent CTAs (stream-K ranges)
    int splitk;           // >= 2: cluster split-K with this many CTAs per tile (N <= 128, few tiles)
};

struct GemmArgs {
    int M, N, K;      // D[M][N] = A[M][K] . B[N][K]^T, stored transposed: y[n][m]
    int epi;
    float* y;
    float* const* y_ptr;  // STORE: as GemvArgs::y_ptr
    int ldy;
    const float* bias;
    const float* rscale;  // per weight row: the product is scaled by rscale[m] first (null = 1);
                          // q8_row weights run as their exact bf16 integer values times it
    uint16_t* act;
    int ldact;
    unsigned long long* amax;  // STORE: per token, packed greedy argmax of y (null = off)
    float softcap;    // STORE: as GemvArgs::softcap
    float* ws;        // set from the plan: fp32 pieces of tiles shared between CTAs
    int* cnt;         // gemm_cnt_needed(M, N) zeroed tile counters (left zeroed)
    int* err;
    int wait_extra;   // set by the launcher from gemm_set_test_wait (0 in normal use)
    long long wait_limit;
};

// Test hook: the stream-K reduction wait of later GEMM launches waits for `extra_pieces`
// more pieces than a tile has (so it cannot be satisfied) and gives up after `limit_cycles`
// (0 = the normal limit). A CTA leaves that wait with every operand load and MMA of its
// own completed and no reduction load issued, so it exits cleanly; the tile counters it
// leaves behind must be zeroed by the host before the next launch.
void gemm_set_test_wait(int extra_pieces, long long limit_cycles);
// Host-side check of the persistent GEMM's work split (see gemm_tc.cu); violations or -1.
int gemm_streamk_check(int M, int N, int K, int nc);

// Build the tensor maps for one GEMM shape (host; encodes the A, B and workspace
// addresses). ws holds gemm_ws_floats(num_sms) floats.
cudaError_t gemm_plan(GemmPlan* p, const uint16_t* A, int M, int K, const uint16_t* B, int N, int num_sms,
                      const float* ws);
size_t gemm_ws_floats(int num_sms);
int gemm_cnt_needed(int M, int N);
cudaError_t gemm_launch(const GemmPlan& p, GemmArgs a, cudaStream_t st, bool pdl);
// Tensor map over a row-major bf16 [rows][K] matrix, read in 128B-swizzled boxes of 64
// columns x box_rows rows (host; fails on a base or stride the TMA unit cannot take).
cudaError_t tmap_bf16_rows(CUtensorMap* tm, const uint16_t* base, int rows, int K, int box_rows);

// ----------------------------------------------------------------- attention

struct AttnDecodeArgs {
    // query and new row: fp32 qkv rows (model path) or bf16 tensors (standalone call)
    const float* qkv;
    int ld_qkv;
    const uint16_t* q_bf;   // [B][nq][d]
    const uint16_t* k_new;  // [B][nkv][d] or null
    const uint16_t* v_new;
    const float* q_norm;    // [d] or null (model path only)
    const float* k_norm;
    float eps;
    int rope;               // rotate q and the new k to pos
    float rope_base;
    const float2* rope_tab; // [max_ctx][d/2] (cos, sin), or null: evaluated in the kernel
    uint16_t* k_pool;       // [n_pages][nkv][16][d]
    uint16_t* v_pool;
    const int32_t* block_table;
    int max_pages;
    const int32_t* pos;     // [B]
    int B, nq, nkv, d;
    float scale;
    int window;             // > 0: the query at p attends keys p-window+1 .. p only
    float softcap;          // > 0: each scaled score s becomes softcap * tanh(s / softcap)
    int splits;
    float* part;            // [B][nq][splits][d+2], or null: the splits merge inside a cluster (<= 16)
    int* counters;          // [B][nkv] (with part)
    uint16_t* out;          // [B][nq*d]
    int* err;
};
cudaError_t attn_decode_launch(const AttnDecodeArgs& a, cudaStream_t st, bool pdl);
int attn_decode_splits(int B, int nkv, int max_ctx, int num_sms, bool cluster);

struct RopeAppendArgs {
    const float* qkv;  // [T][ld]
    int ld_qkv;
    const float* q_norm;
    const float* k_norm;
    float eps;
    float rope_base;
    const float2* rope_tab;  // [max_ctx][d/2] (cos, sin), or null
    int T, pos0, nq, nkv, d;
    uint16_t* q_out;   // [T][nq][d]
    uint16_t* k_pool;
    uint16_t* v_pool;
    const int32_t* block_row;  // block table row of the sequence
};
cudaError_t rope_append_launch(const RopeAppendArgs& a, cudaStream_t st, bool pdl);

struct AttnPrefillArgs {
    const uint16_t* q;  // [T][nq][d] (rotated, bf16)
    const uint16_t* k_pool;
    const uint16_t* v_pool;
    const int32_t* block_row;
    int T, pos0, nq, nkv, d;
    float scale;
    int window;         // as AttnDecodeArgs
    float softcap;
    int splits;         // key splits (1..8): the split CTAs of a row block form one cluster
    uint16_t* out;      // [T][nq*d]
    int* err;
    int pool_rows;      // rows of the pools viewed as [pages * nkv * 16][d] (tensor-core path)
};
cudaError_t attn_prefill_launch(const AttnPrefillArgs& a, cudaStream_t st, bool pdl);
// The tensor-core prefill attention (tcgen05, TMEM): head dim 128, power-of-two groups.
bool attn_prefill_tc_ok(const AttnPrefillArgs& a);
cudaError_t attn_prefill_tc_launch(const AttnPrefillArgs& a, cudaStream_t st, bool pdl);
// A bf16 tensor map with 128-byte swizzle: dims[0] contiguous; strides[i] (bytes) of dims[i + 1].
cudaError_t tmap_bf16_sw128(CUtensorMap* tm, const void* base, int rank, const uint64_t* dims,
                            const uint64_t* strides, const uint32_t* box);
int attn_prefill_splits(int T, int nq, int nkv, int ctx, int num_sms);
// Keys a prefill chunk's rows may see: the whole causal prefix, or with a window the last
// window + T - 1 positions (sizes the key splits).
inline int attn_prefill_span(int pos0, int T, int window) {
    const int n = pos0 + T;
    return window > 0 && window + T - 1 < n ? window + T - 1 : n;
}

// Greedy argmax as one 64-bit word per row: high half an order-preserving key of the
// fp32 value, low half ~index (so on equal values the lowest index is the largest word).
// The zero word is below every real value. atomicMax of these words is order-free.
__host__ __device__ inline unsigned long long argmax_pack(float v, int idx) {
    unsigned int b;
    memcpy(&b, &v, 4);
    const unsigned int key = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return ((unsigned long long)key << 32) | (unsigned long long)(0xFFFFFFFFu - (unsigned int)idx);
}
__host__ __device__ inline int argmax_unpack(unsigned long long w) { return (int)(0xFFFFFFFFu - (unsigned int)w); }

// ----------------------------------------------------------------- elementwise / small

cudaError_t embed_launch(const uint16_t* E, const int32_t* tok, int B, int h, float* x, cudaStream_t st, bool pdl);
cudaError_t rmsnorm_launch(const float* x, const float* g, int T, int h, float eps, uint16_t* out, cudaStream_t st,
                           bool pdl);
// out[i] = bf16(q[i]) for n int8 values (exact: every int8 is a bf16 value).
cudaError_t widen_i8_launch(const int8_t* q, uint16_t* out, size_t n, cudaStream_t st);
// Sandwich norm: x[t] += y[t] * rsqrt(mean(y[t]^2) + eps) * g for T rows of h (fp32).
cudaError_t add_rmsnorm_launch(float* x, const float* y, const float* g, int T, int h, float eps, cudaStream_t st,
                               bool pdl);

}  // namespace dec

#include <map>
#include <mutex>
#include <string>
#include <utility>
namespace dec {
void set_last_error(const std::string& msg);

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) only when a kernel needs more dynamic
// shared memory on this device than already granted (the call costs host time on every
// launch otherwise).
inline cudaError_t ensure_smem(const void* fn, int bytes) {
    static std::mutex mu;
    static std::map<std::pair<const void*, int>, int> granted;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    int& g = granted[std::make_pair(fn, dev)];
    if (g >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) g = bytes;
    return e;
}

// ----------------------------------------------------------------- MoE

struct MoeRouteArgs {
    const float* logits;  // [n][E]
    int E, k, renorm;
    int32_t* idx;         // [n][k]
    float* w;             // [n][k]
    const uint16_t* xn;   // [n][h] normalised rows (shared-expert gate input)
    const float* gvec;    // [h] shared-expert gate vector, or null (gate = 1)
    int h;
    float* sgate;         // [n] sigmoid(gvec . xn), or null
};
cudaError_t moe_route_launch(const MoeRouteArgs& a, int n, cudaStream_t st, bool pdl);

struct MoePermArgs {
    const int32_t* idx;   // [n][k]
    int n, k, E, nb;
    int32_t* perm_tok;    // [n*k] token of each permuted slot
    int32_t* inv;         // [n*k] permuted slot of (token, j)
    int32_t* groups;      // [max_groups][4]: expert, first slot, count, 0
    int32_t* n_groups;    // [1]
};
cudaError_t moe_permute_launch(const MoePermArgs& a, cudaStream_t st, bool pdl);

struct GroupedGemvArgs {
    const uint16_t* W;    // expert 0 weights [M][K]; expert e at W + e * wstride
    size_t wstride;
    int M, K;
    int E;                // experts in W (the tensor-core path reads W as [E*M][K])
    const int32_t* groups;
    const int32_t* n_groups;
    const uint16_t* x;    // token rows (bf16), row of slot p = x_map ? x_map[p] : p
    const int32_t* x_map;
    int ldx;
    float* y;             // STORE: y[p][row]
    int ldy;
    uint16_t* act;        // SWIGLU: act[p][row/2]
    int ldact;
    int* err;
    int smem_cap;
};
int grouped_nb_for(int n);
bool grouped_uses_mma(int nb, int M, int K, size_t wstride, int smem_cap);
bool grouped_fits(int nb, int K, int smem_cap);
cudaError_t grouped_gemv_launch(const GroupedGemvArgs& a, int nb, bool swiglu, cudaStream_t st, int num_sms,
                                bool pdl);

struct MoeCombineArgs {
    float* x;             // [n][h] residual
    const float* y;       // [n*k][h] routed slot outputs
    const float* ys;      // [n][h] shared expert output, or null
    const float* w;       // [n][k]
    const int32_t* inv;   // [n][k]
    const float* sgate;   // [n] or null
    int k, h;
};
cudaError_t moe_combine_launch(const MoeCombineArgs& a, int n, cudaStream_t st, bool pdl);
cudaError_t kv_move_launch(uint16_t* pool_k, uint16_t* pool_v, const int32_t* block_row, int pos0, int n, int nkv,
                           int d, uint16_t* dense_k, uint16_t* dense_v, int to_pool, cudaStream_t st);
}  // namespace dec
