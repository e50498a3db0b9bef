// Small memory-bound steps of the layer stack:
//  * embedding row gather (ANEDVD Engine.forward embed; cortiq embed_single),
//    embed scale 1;
//  * RMSNorm of fp32 residual rows to bf16 (ANEDVD rmsnormColumn / rmsnormChunk:
//    x * (1/sqrt(mean(x^2) + eps)) * w, written in the device input precision);
//  * greedy argmax over logits, lowest index on ties;
//  * MoE routing: softmax over all experts, top-k, optional renormalisation
//    (ANEDVD cpu.moeRoute; frink route_top_k; cortiq MoeFfn).
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace dec {

namespace {

template <typename K, typename Args>
cudaError_t launch_ex(K kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl, const Args& args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, args);
}

struct EmbedArgs {
    const uint16_t* E;
    const int32_t* tok;
    int h;
    float* x;
};

__global__ void embed_kernel(EmbedArgs a) {
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x;
    const uint16_t* row = a.E + (size_t)a.tok[b] * a.h;
    float* dst = a.x + (size_t)b * a.h;
    for (int i = threadIdx.x * 8; i < a.h; i += blockDim.x * 8) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + i);
        float4 lo = make_float4(bf_lo(v.x), bf_hi(v.x), bf_lo(v.y), bf_hi(v.y));
        float4 hi = make_float4(bf_lo(v.z), bf_hi(v.z), bf_lo(v.w), bf_hi(v.w));
        *reinterpret_cast<float4*>(dst + i) = lo;
        *reinterpret_cast<float4*>(dst + i + 4) = hi;
    }
}

struct NormArgs {
    const float* x;
    const float* g;
    int h;
    float eps;
    uint16_t* out;
};

__global__ void __launch_bounds__(256) rmsnorm_kernel(NormArgs a) {
    __shared__ float red[8];
    pdl_trigger();
    pdl_wait();
    const int t = blockIdx.x;
    const float* x = a.x + (size_t)t * a.h;
    float ss = 0.f;
    for (int i = threadIdx.x * 4; i < a.h; i += 256 * 4) {
        const float4 v = *reinterpret_cast<const float4*>(x + i);
        ss = fmaf(v.x, v.x, ss);
        ss = fmaf(v.y, v.y, ss);
        ss = fmaf(v.z, v.z, ss);
        ss = fmaf(v.w, v.w, ss);
    }
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) tot += red[w];
    const float inv = 1.0f / sqrtf(tot / (float)a.h + a.eps);
    uint16_t* o = a.out + (size_t)t * a.h;
    for (int i = threadIdx.x * 4; i < a.h; i += 256 * 4) {
        const float4 v = *reinterpret_cast<const float4*>(x + i);
        const float4 g = *reinterpret_cast<const float4*>(a.g + i);
        uint2 r;
        r.x = pack_bf2(v.x * inv * g.x, v.y * inv * g.y);
        r.y = pack_bf2(v.z * inv * g.z, v.w * inv * g.w);
        *reinterpret_cast<uint2*>(o + i) = r;
    }
}

struct ArgmaxArgs {
    const float* logits;
    int V;
    int32_t* out;
};

__global__ void __launch_bounds__(1024) argmax_kernel(ArgmaxArgs a) {
    __shared__ float bv[32];
    __shared__ int bi[32];
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x;
    const float* l = a.logits + (size_t)b * a.V;
    float best = -INFINITY;
    int idx = 0x7fffffff;
    for (int i = threadIdx.x; i < a.V; i += blockDim.x) {
        const float v = l[i];
        if (v > best || (v == best && i < idx)) {
            best = v;
            idx = i;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, idx, o);
        if (ov > best || (ov == best && oi < idx)) {
            best = ov;
            idx = oi;
        }
    }
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
        bv[w] = best;
        bi[w] = idx;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const int nw = blockDim.x >> 5;
        for (int k = 1; k < nw; ++k)
            if (bv[k] > best || (bv[k] == best && bi[k] < idx)) {
                best = bv[k];
                idx = bi[k];
            }
        a.out[b] = idx;
    }
}

struct TopkArgs {
    const float* logits;
    int E, k, renorm;
    int32_t* idx;
    float* w;
};

// One warp per row: E <= 256 logits held 8 per lane.
__global__ void __launch_bounds__(32) topk_kernel(TopkArgs a) {
    pdl_trigger();
    pdl_wait();
    const int t = blockIdx.x, lane = threadIdx.x;
    const float* r = a.logits + (size_t)t * a.E;
    float v[8];
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int e = lane + 32 * j;
        v[j] = e < a.E ? r[e] : -INFINITY;
        mx = fmaxf(mx, v[j]);
    }
    mx = warp_max(mx);
    float p[8], sum = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int e = lane + 32 * j;
        p[j] = e < a.E ? expf(v[j] - mx) : 0.f;
        sum += p[j];
    }
    sum = warp_sum(sum);
    const float inv = 1.0f / sum;
#pragma unroll
    for (int j = 0; j < 8; ++j) p[j] *= inv;
    bool taken[8] = {false, false, false, false, false, false, false, false};
    float sel_p[16];
    int sel_i[16];
    float tot = 0.f;
    for (int q = 0; q < a.k; ++q) {
        float bp = -1.f;
        int be = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = lane + 32 * j;
            if (e < a.E && !taken[j] && (p[j] > bp || (p[j] == bp && e < be))) {
                bp = p[j];
                be = e;

            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float op = __shfl_xor_sync(0xffffffffu, bp, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (op > bp || (op == bp && oe < be)) {
                bp = op;
                be = oe;
            }
        }
        if ((be & 31) == lane) taken[be >> 5] = true;

        if (q < 16) {
            sel_p[q] = bp;
            sel_i[q] = be;
        }
        tot += bp;
    }
    if (lane == 0) {
        for (int q = 0; q < a.k && q < 16; ++q) {
            a.idx[(size_t)t * a.k + q] = sel_i[q];
            a.w[(size_t)t * a.k + q] = a.renorm ? sel_p[q] / tot : sel_p[q];
        }
    }
}

}  // namespace

cudaError_t embed_launch(const uint16_t* E, const int32_t* tok, int B, int h, float* x, cudaStream_t st, bool pdl) {
    EmbedArgs a{E, tok, h, x};
    return launch_ex(embed_kernel, dim3(B), dim3(128), 0, st, pdl, a);
}

cudaError_t rmsnorm_launch(const float* x, const float* g, int T, int h, float eps, uint16_t* out, cudaStream_t st,
                           bool pdl) {
    NormArgs a{x, g, h, eps, out};
    return launch_ex(rmsnorm_kernel, dim3(T), dim3(256), 0, st, pdl, a);
}

cudaError_t argmax_launch(const float* logits, int B, int V, int32_t* out, cudaStream_t st, bool pdl) {
    ArgmaxArgs a{logits, V, out};
    return launch_ex(argmax_kernel, dim3(B), dim3(1024), 0, st, pdl, a);
}

cudaError_t topk_launch(const float* logits, int T, int E, int k, int renorm, int32_t* idx, float* w,
                        cudaStream_t st, bool pdl) {
    if (E > 256 || k > 16 || k > E || k <= 0) return cudaErrorInvalidValue;
    TopkArgs a{logits, E, k, renorm, idx, w};
    return launch_ex(topk_kernel, dim3(T), dim3(32), 0, st, pdl, a);
}

}  // namespace dec

// ----------------------------------------------------------------- KV test hooks (scatter / gather)

namespace dec {

namespace {

struct KvMoveArgs {
    uint16_t* pool_k;
    uint16_t* pool_v;
    const int32_t* block_row;
    int pos0, n, nkv, d;
    uint16_t* dense_k;  // [n][nkv*d]
    uint16_t* dense_v;
    int to_pool;
};

__global__ void kv_move_kernel(KvMoveArgs a) {
    const int i = blockIdx.x;  // position index
    const int p = a.pos0 + i;
    const int phys = a.block_row[p / 16], slot = p % 16;
    const int kvd = a.nkv * a.d;
    for (int e = threadIdx.x; e < kvd; e += blockDim.x) {
        const int g = e / a.d, c = e % a.d;
        const size_t po = (((size_t)phys * a.nkv + g) * 16 + slot) * a.d + c;
        const size_t dn = (size_t)i * kvd + e;
        if (a.to_pool) {
            a.pool_k[po] = a.dense_k[dn];
            a.pool_v[po] = a.dense_v[dn];
        } else {
            a.dense_k[dn] = a.pool_k[po];
            a.dense_v[dn] = a.pool_v[po];
        }
    }
}

}  // namespace

cudaError_t kv_move_launch(uint16_t* pool_k, uint16_t* pool_v, const int32_t* block_row, int pos0, int n, int nkv,
                           int d, uint16_t* dense_k, uint16_t* dense_v, int to_pool, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    KvMoveArgs a{pool_k, pool_v, block_row, pos0, n, nkv, d, dense_k, dense_v, to_pool};
    kv_move_kernel<<<n, 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace dec
