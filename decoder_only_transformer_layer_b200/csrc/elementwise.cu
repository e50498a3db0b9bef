// Small memory-bound steps of the layer stack:
//  * embedding row gather (ANEDVD Engine.forward embed; cortiq embed_single),
//    embed scale 1;
//  * RMSNorm of fp32 residual rows to bf16 (ANEDVD rmsnormColumn / rmsnormChunk:
//    x * (1/sqrt(mean(x^2) + eps)) * w, written in the device input precision);
//  * the sandwich norm's residual add (ANEDVD Engine.forward: the o_proj and FFN outputs
//    pass through rmsnormFlat with their own gains before joining the residual), fp32;
//  * moving cache rows between the paged pool and dense arrays (test hooks).
// The greedy argmax is folded into the LM-head epilogues (gemv.cu, gemm_tc.cu) and the
// MoE routing lives in moe.cu.
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

// Rows up to 256 threads x 4 floats x kNormU are held in registers: every load of a row is
// issued before the first use (one memory round trip per row instead of one per piece), and
// the gains, which do not depend on the previous kernel, are loaded before waiting on it.
// Thread tid sums the squares of pieces tid, tid + 256, ... in that order on either path.
constexpr int kNormU = 8;

__global__ void __launch_bounds__(256) rmsnorm_kernel(NormArgs a) {
    __shared__ float red[8];
    const int t = blockIdx.x, tid = threadIdx.x;
    const bool held = a.h <= 256 * 4 * kNormU;
    float4 gv[kNormU], xv[kNormU];
    if (held) {
#pragma unroll
        for (int u = 0; u < kNormU; ++u)
            if ((u * 256 + tid) * 4 < a.h) gv[u] = *reinterpret_cast<const float4*>(a.g + (u * 256 + tid) * 4);
    }
    pdl_trigger();
    pdl_wait();
    const float* x = a.x + (size_t)t * a.h;
    float ss = 0.f;
    if (held) {
#pragma unroll
        for (int u = 0; u < kNormU; ++u)
            if ((u * 256 + tid) * 4 < a.h) xv[u] = *reinterpret_cast<const float4*>(x + (u * 256 + tid) * 4);
#pragma unroll
        for (int u = 0; u < kNormU; ++u) {
            if ((u * 256 + tid) * 4 < a.h) {
                ss = fmaf(xv[u].x, xv[u].x, ss);
                ss = fmaf(xv[u].y, xv[u].y, ss);
                ss = fmaf(xv[u].z, xv[u].z, ss);
                ss = fmaf(xv[u].w, xv[u].w, ss);
            }
        }
    } else {
        for (int i = tid * 4; i < a.h; i += 256 * 4) {
            const float4 v = *reinterpret_cast<const float4*>(x + i);
            ss = fmaf(v.x, v.x, ss);
            ss = fmaf(v.y, v.y, ss);
            ss = fmaf(v.z, v.z, ss);
            ss = fmaf(v.w, v.w, ss);
        }
    }
    ss = warp_sum(ss);
    if ((tid & 31) == 0) red[tid >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) tot += red[w];
    const float inv = 1.0f / sqrtf(tot / (float)a.h + a.eps);
    uint16_t* o = a.out + (size_t)t * a.h;
    if (held) {
#pragma unroll
        for (int u = 0; u < kNormU; ++u) {
            const int i = (u * 256 + tid) * 4;
            if (i < a.h) {
                uint2 r;
                r.x = pack_bf2(xv[u].x * inv * gv[u].x, xv[u].y * inv * gv[u].y);
                r.y = pack_bf2(xv[u].z * inv * gv[u].z, xv[u].w * inv * gv[u].w);
                *reinterpret_cast<uint2*>(o + i) = r;
            }
        }
    } else {
        for (int i = tid * 4; i < a.h; i += 256 * 4) {
            const float4 v = *reinterpret_cast<const float4*>(x + i);
            const float4 g = *reinterpret_cast<const float4*>(a.g + i);
            uint2 r;
            r.x = pack_bf2(v.x * inv * g.x, v.y * inv * g.y);
            r.y = pack_bf2(v.z * inv * g.z, v.w * inv * g.w);
            *reinterpret_cast<uint2*>(o + i) = r;
        }
    }
}

struct AddNormArgs {
    float* x;        // [T][h] residual, updated
    const float* y;  // [T][h] sublayer output
    const float* g;
    int h;
    float eps;
};

// x[t] += y[t] * (1 / sqrt(mean(y[t]^2) + eps)) * g, one CTA per row, all in fp32 (rows held
// in registers as in rmsnorm_kernel).
__global__ void __launch_bounds__(256) add_rmsnorm_kernel(AddNormArgs a) {
    __shared__ float red[8];
    const int t = blockIdx.x, tid = threadIdx.x;
    const bool held = a.h <= 256 * 4 * kNormU;
    float4 gv[kNormU], yv[kNormU], xv[kNormU];
    if (held) {
#pragma unroll
        for (int u = 0; u < kNormU; ++u)
            if ((u * 256 + tid) * 4 < a.h) gv[u] = *reinterpret_cast<const float4*>(a.g + (u * 256 + tid) * 4);
    }
    pdl_trigger();
    pdl_wait();
    const float* y = a.y + (size_t)t * a.h;
    float* x = a.x + (size_t)t * a.h;
    float ss = 0.f;
    if (held) {
#pragma unroll
        for (int u = 0; u < kNormU; ++u) {
            if ((u * 256 + tid) * 4 < a.h) {
                yv[u] = *reinterpret_cast<const float4*>(y + (u * 256 + tid) * 4);
                xv[u] = *reinterpret_cast<const float4*>(x + (u * 256 + tid) * 4);
            }
        }
#pragma unroll
        for (int u = 0; u < kNormU; ++u) {
            if ((u * 256 + tid) * 4 < a.h) {
                ss = fmaf(yv[u].x, yv[u].x, ss);
                ss = fmaf(yv[u].y, yv[u].y, ss);
                ss = fmaf(yv[u].z, yv[u].z, ss);
                ss = fmaf(yv[u].w, yv[u].w, ss);
            }
        }
    } else {
        for (int i = tid * 4; i < a.h; i += 256 * 4) {
            const float4 v = *reinterpret_cast<const float4*>(y + i);
            ss = fmaf(v.x, v.x, ss);
            ss = fmaf(v.y, v.y, ss);
            ss = fmaf(v.z, v.z, ss);
            ss = fmaf(v.w, v.w, ss);
        }
    }
    ss = warp_sum(ss);
    if ((tid & 31) == 0) red[tid >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) tot += red[w];
    const float inv = 1.0f / sqrtf(tot / (float)a.h + a.eps);
    if (held) {
#pragma unroll
        for (int u = 0; u < kNormU; ++u) {
            const int i = (u * 256 + tid) * 4;
            if (i < a.h) {
                float4 r = xv[u];
                r.x += yv[u].x * inv * gv[u].x;
                r.y += yv[u].y * inv * gv[u].y;
                r.z += yv[u].z * inv * gv[u].z;
                r.w += yv[u].w * inv * gv[u].w;
                *reinterpret_cast<float4*>(x + i) = r;
            }
        }
    } else {
        for (int i = tid * 4; i < a.h; i += 256 * 4) {
            const float4 v = *reinterpret_cast<const float4*>(y + i);
            const float4 g = *reinterpret_cast<const float4*>(a.g + i);
            float4 r = *reinterpret_cast<const float4*>(x + i);
            r.x += v.x * inv * g.x;
            r.y += v.y * inv * g.y;
            r.z += v.z * inv * g.z;
            r.w += v.w * inv * g.w;
            *reinterpret_cast<float4*>(x + i) = r;
        }
    }
}

// out[i] = bf16(q[i]): every int8 value is exactly a bf16 value (at most 8 significant bits).
__global__ void widen_i8_kernel(const int8_t* q, uint16_t* out, size_t n) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        out[i] = f2bf((float)q[i]);
}

}  // namespace

cudaError_t widen_i8_launch(const int8_t* q, uint16_t* out, size_t n, cudaStream_t st) {
    widen_i8_kernel<<<1184, 256, 0, st>>>(q, out, n);
    return cudaGetLastError();
}

cudaError_t add_rmsnorm_launch(float* x, const float* y, const float* g, int T, int h, float eps, cudaStream_t st,
                               bool pdl) {
    AddNormArgs a{x, y, g, h, eps};
    return launch_ex(add_rmsnorm_kernel, dim3(T), dim3(256), 0, st, pdl, a);
}

cudaError_t embed_launch(const uint16_t* E, const int32_t* tok, int B, int h, float* x, cudaStream_t st, bool pdl) {
    EmbedArgs a{E, tok, h, x};
    return launch_ex(embed_kernel, dim3(B), dim3(128), 0, st, pdl, a);
}

cudaError_t rmsnorm_launch(const float* x, const float* g, int T, int h, float eps, uint16_t* out, cudaStream_t st,
                           bool pdl) {
    NormArgs a{x, g, h, eps, out};
    return launch_ex(rmsnorm_kernel, dim3(T), dim3(256), 0, st, pdl, a);
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
