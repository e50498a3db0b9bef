// Weight-streaming skinny projection for decode: y[b][n] = sum_k W[n][k] x[b][k]
// for up to NB columns, W bf16 [N][K] read from HBM exactly once.
//
// These are the projections of the layer (ANEDVD src/engine.zig: the qkv, o,
// fused gate/up/SiLU/down and LM-head 1x1 conv kernels; the decode-time
// "dominant matvec" of runHead). At small batch they are HBM-bound: every
// weight byte is used NB times, so the kernel is built to keep HBM busy, not
// the tensor cores.
//
// Design (B200):
//  * one CTA per SM (persistent over a contiguous range of 4-row blocks), 8
//    consumer warps + 1 producer warp;
//  * the producer streams 4-row x KC-column weight stages (KC <= 4096) into a
//    shared-memory ring with cp.async.bulk (TMA engine, L2 evict-first), up to 8
//    stages in flight per SM. Large copies matter: 2 KB copies held the kernel near
//    60% of HBM bandwidth and 8 KB copies near 6.6 TB/s on a pure read, while 32 KB
//    copies reach 7.2-7.4 TB/s; when a stage holds whole rows (K <= 4096) its 4 rows
//    are one contiguous block and move in one copy, else one copy per row. The producer starts BEFORE
//    griddepcontrol.wait: weights do not depend on the previous kernel, so their
//    stream overlaps its tail;
//  * the input columns sit in shared memory as bf16; with a fused RMSNorm they
//    are normalised from the fp32 residual in the prologue (R1 rounding point);
//  * warps 2r and 2r+1 own the two column halves of row r of each stage:
//    16-byte shared loads, fp32 FMA, a warp reduction per row and a fixed-order
//    sum of the two halves (deterministic, no atomics on data);
//  * epilogues: store (+bias, optional greedy argmax), residual add, or SwiGLU on
//    interleaved gate/up rows (row 2j = gate j, row 2j+1 = up j) writing bf16
//    silu(g)*u (R4).
#include "common.cuh"
#include "kernels.h"

namespace dec {

namespace {

constexpr int kRows = 4;               // rows per stage
constexpr int kKC = 4096;              // max columns per stage (8 KB per row copy)
constexpr int kWarps = 8;              // consumer warps: 2 per row
constexpr int kConsumers = kWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kMaxStages = 16;         // short rows (small K) keep more stages in flight

struct Layout {
    int kc, stages;
    uint32_t stage_bytes, ring_off, x_off, red_off, total;
};

__host__ __device__ inline Layout make_layout(int nb, int K, int smem_cap) {
    Layout L;
    L.kc = K < kKC ? K : kKC;
    L.stage_bytes = (uint32_t)kRows * L.kc * 2;
    const uint32_t bars = 2 * kMaxStages * 8;
    L.red_off = bars;                                  // [kWarps][16] floats + 64 floats scratch
    const uint32_t red = (uint32_t)(kWarps * 16 + 64) * 4;
    L.x_off = (L.red_off + red + 127) & ~127u;
    const uint32_t xbytes = ((uint32_t)nb * K * 2 + 127) & ~127u;
    L.ring_off = L.x_off + xbytes;
    int st = (int)((smem_cap - (int)L.ring_off) / (int)L.stage_bytes);
    L.stages = st > kMaxStages ? kMaxStages : st;
    L.total = L.ring_off + (uint32_t)(L.stages > 0 ? L.stages : 0) * L.stage_bytes;
    return L;
}

DEC_DEVINL float dot8(uint4 w, uint4 x, float acc) {
    acc = fmaf(bf_lo(w.x), bf_lo(x.x), acc);
    acc = fmaf(bf_hi(w.x), bf_hi(x.x), acc);
    acc = fmaf(bf_lo(w.y), bf_lo(x.y), acc);
    acc = fmaf(bf_hi(w.y), bf_hi(x.y), acc);
    acc = fmaf(bf_lo(w.z), bf_lo(x.z), acc);
    acc = fmaf(bf_hi(w.z), bf_hi(x.z), acc);
    acc = fmaf(bf_lo(w.w), bf_lo(x.w), acc);
    acc = fmaf(bf_hi(w.w), bf_hi(x.w), acc);
    return acc;
}

DEC_DEVINL void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory"); }

template <int NB, int EPI>
__global__ void __launch_bounds__(kThreads, 1) gemv_kernel(GemvArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Layout L = make_layout(NB, a.K, a.smem_cap);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    float* red = reinterpret_cast<float*>(smem + L.red_off);
    uint16_t* xs = reinterpret_cast<uint16_t*>(smem + L.x_off);
    uint8_t* ring = smem + L.ring_off;

    const int nrb = (a.N + kRows - 1) / kRows;
    const int nkc = (a.K + L.kc - 1) / L.kc;
    // contiguous range of row blocks for this CTA
    const int rb0 = (int)((int64_t)blockIdx.x * nrb / gridDim.x);
    const int rb1 = (int)((int64_t)(blockIdx.x + 1) * nrb / gridDim.x);

    if (threadIdx.x == 0) {
        for (int s = 0; s < L.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();
    pdl_trigger();

    if (warp == kWarps) {
        // ------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            int s = 0;
            uint32_t ph = 0;
            for (int rb = rb0; rb < rb1; ++rb) {
                const int r0 = rb * kRows;
                const int nrows = min(kRows, a.N - r0);
                for (int kc = 0; kc < nkc; ++kc) {
                    const int k0 = kc * L.kc;
                    const int kcols = min(L.kc, a.K - k0);
                    if (!mbar_wait_bounded(&empty[s], ph ^ 1, a.err)) goto producer_done;
                    mbar_arrive_expect_tx(&full[s], (uint32_t)(nrows * kcols * 2));
                    uint8_t* dst = ring + (size_t)s * L.stage_bytes;
                    if (kcols == a.K) {  // whole rows: the stage is one contiguous block
                        bulk_g2s_stream(dst, a.W + (size_t)r0 * a.K, (uint32_t)(nrows * kcols * 2), &full[s], pol);
                    } else {
                        for (int r = 0; r < nrows; ++r)
                            bulk_g2s_stream(dst + (size_t)r * L.kc * 2, a.W + (size_t)(r0 + r) * a.K + k0,
                                            (uint32_t)kcols * 2, &full[s], pol);
                    }
                    if (++s == L.stages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
            }
        }
    producer_done:
        pdl_wait();
        return;
    }

    // ---------------------------------------------------- consumers: input columns
    pdl_wait();
    const int tid = threadIdx.x;
    for (int b = 0; b < NB; ++b) {
        uint16_t* xrow = xs + (size_t)b * a.K;
        if (b >= a.B) {
            for (int k = tid * 8; k < a.K; k += kConsumers * 8) *reinterpret_cast<uint4*>(xrow + k) = make_uint4(0, 0, 0, 0);
            continue;
        }
        if (a.xr) {
            // fused RMSNorm of the fp32 residual row: R1 rounding to bf16
            const float* xr = a.xr + (size_t)b * a.ldx;
            float ss = 0.f;
            for (int k = tid * 4; k < a.K; k += kConsumers * 4) {
                const float4 v = *reinterpret_cast<const float4*>(xr + k);
                ss = fmaf(v.x, v.x, ss);
                ss = fmaf(v.y, v.y, ss);
                ss = fmaf(v.z, v.z, ss);
                ss = fmaf(v.w, v.w, ss);
            }
            ss = warp_sum(ss);
            if (lane == 0) red[kWarps * 16 + warp] = ss;
            consumer_sync();
            float tot = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) tot += red[kWarps * 16 + w];
            const float inv = 1.0f / sqrtf(tot / (float)a.K + a.eps);
            for (int k = tid * 4; k < a.K; k += kConsumers * 4) {
                const float4 v = *reinterpret_cast<const float4*>(xr + k);
                const float4 g = *reinterpret_cast<const float4*>(a.g + k);
                uint2 o;
                o.x = pack_bf2(v.x * inv * g.x, v.y * inv * g.y);
                o.y = pack_bf2(v.z * inv * g.z, v.w * inv * g.w);
                *reinterpret_cast<uint2*>(xrow + k) = o;
            }
            consumer_sync();  // red[] reused by the next column
        } else {
            const uint16_t* xb = a.xb + (size_t)b * a.ldx;
            for (int k = tid * 8; k < a.K; k += kConsumers * 8)
                *reinterpret_cast<uint4*>(xrow + k) = *reinterpret_cast<const uint4*>(xb + k);
        }
    }
    consumer_sync();

    // ---------------------------------------------------- consumers: stream
    // A timed-out wait marks the call failed (a.err) and skips the remaining work, but
    // every warp still passes the same named barriers so none of them can hang.
    const int r_in = warp >> 1, half = warp & 1;
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    unsigned long long best = 0;  // lane b of an even warp: packed argmax of column b over its rows
    for (int rb = rb0; rb < rb1; ++rb) {
        const int row = rb * kRows + r_in;
        const bool valid = row < a.N;
        float acc[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[b] = 0.f;
        for (int kc = 0; kc < nkc; ++kc) {
            const int k0 = kc * L.kc;
            const int npc = min(L.kc, a.K - k0) >> 3;  // 16-byte pieces of this chunk
            const int hp = (npc + 1) >> 1;
            const int p0 = half * hp, p1 = min(npc, p0 + hp);
            if (ok && !mbar_wait_bounded(&full[s], ph, a.err)) ok = false;
            if (valid && ok) {
                const uint4* wrow =
                    reinterpret_cast<const uint4*>(ring + (size_t)s * L.stage_bytes + (size_t)r_in * L.kc * 2);
                for (int p = p0 + lane; p < p1; p += 32) {
                    const uint4 w8 = wrow[p];
#pragma unroll
                    for (int b = 0; b < NB; ++b) {
                        const uint4 x8 = *reinterpret_cast<const uint4*>(xs + (size_t)b * a.K + k0 + p * 8);
                        acc[b] = dot8(w8, x8, acc[b]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (++s == L.stages) {
                s = 0;
                ph ^= 1;
            }
        }
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[b] = warp_sum(acc[b]);
        if (lane == 0) {
#pragma unroll
            for (int b = 0; b < NB; ++b) red[warp * 16 + b] = acc[b];
        }
        consumer_sync();
        // row sum = first column half + second column half, in that order
        if constexpr (EPI != GEMV_SWIGLU) {
            if (half == 0 && lane < a.B && valid && ok) {
                const float v = red[warp * 16 + lane] + red[(warp + 1) * 16 + lane];
                if constexpr (EPI == GEMV_STORE) {
                    const float o = v + (a.bias ? a.bias[row] : 0.f);
                    a.y[(size_t)lane * a.ldy + row] = o;
                    if (a.amax) {
                        const unsigned long long w = argmax_pack(o, row);
                        if (w > best) best = w;
                    }
                } else {
                    a.y[(size_t)lane * a.ldy + row] += v;
                }
            }
        } else {
            if ((r_in & 1) == 0 && half == 0 && valid && ok && lane < a.B) {
                const float g = red[warp * 16 + lane] + red[(warp + 1) * 16 + lane];
                const float u = red[(warp + 2) * 16 + lane] + red[(warp + 3) * 16 + lane];
                const float sg = g * (1.0f / (1.0f + expf(-g)));
                a.act[(size_t)lane * a.ldact + (row >> 1)] = f2bf(sg * u);
            }
        }
        consumer_sync();
    }
    if constexpr (EPI == GEMV_STORE) {
        if (a.amax) {  // greedy argmax: CTA reduction, then one atomic per column
            unsigned long long* wb = reinterpret_cast<unsigned long long*>(red);  // [8 warps][8 columns]
            if (lane < NB) wb[warp * 8 + lane] = best;
            consumer_sync();
            if (warp == 0 && lane < a.B) {
                unsigned long long m = 0;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) m = wb[w * 8 + lane] > m ? wb[w * 8 + lane] : m;
                if (m) atomicMax(&a.amax[(size_t)lane * 32], m);
            }
        }
    }
}

template <int NB, int EPI>
cudaError_t launch_nb(const GemvArgs& a0, cudaStream_t st, int num_sms, bool pdl) {
    GemvArgs a = a0;
    const Layout L = make_layout(NB, a.K, a.smem_cap);
    if (L.stages < 3) return cudaErrorInvalidValue;
    auto kern = gemv_kernel<NB, EPI>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), (int)L.total);
    if (e != cudaSuccess) return e;
    const int nrb = (a.N + kRows - 1) / kRows;
    const int grid = nrb < num_sms ? nrb : num_sms;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int EPI>
cudaError_t launch_epi(const GemvArgs& a, cudaStream_t st, int num_sms, bool pdl) {
    switch (a.nb) {
        case 1: return launch_nb<1, EPI>(a, st, num_sms, pdl);
        case 2: return launch_nb<2, EPI>(a, st, num_sms, pdl);
        case 4: return launch_nb<4, EPI>(a, st, num_sms, pdl);
        case 8: return launch_nb<8, EPI>(a, st, num_sms, pdl);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

int gemv_nb_for(int B) { return B <= 1 ? 1 : B <= 2 ? 2 : B <= 4 ? 4 : B <= 8 ? 8 : 0; }

bool gemv_fits(int B, int K, int smem_cap) {
    const int nb = gemv_nb_for(B);
    if (nb == 0 || K % 8 != 0 || K <= 0) return false;
    const Layout L = make_layout(nb, K, smem_cap);
    return L.stages >= 3;
}

cudaError_t gemv_launch(GemvArgs a, int epi, cudaStream_t st, int num_sms, bool pdl) {
    a.nb = gemv_nb_for(a.B);
    if (epi == GEMV_SWIGLU && (a.N % kRows) != 0) return cudaErrorInvalidValue;
    switch (epi) {
        case GEMV_STORE: return launch_epi<GEMV_STORE>(a, st, num_sms, pdl);
        case GEMV_RESID: return launch_epi<GEMV_RESID>(a, st, num_sms, pdl);
        case GEMV_SWIGLU: return launch_epi<GEMV_SWIGLU>(a, st, num_sms, pdl);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace dec
