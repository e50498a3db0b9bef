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
//  * q8_row weights (int8 rows, one fp32 scale per row; cortiq's q8_row_parts): the
//    same stream at half the bytes. Each 16-byte piece holds 16 weights; a weight is
//    widened exactly by permuting its offset-binary byte into the mantissa of 2^23 and
//    subtracting 2^23 + 128 (the magic-number int-to-float conversion, Kim et al.,
//    "Who Says Elephants Can't Run", 2022), then packed fp32x2 FMAs (sm_100) accumulate
//    q * x against the fp32 input columns; the row scale is applied once, in the
//    epilogue, so y = scale * sum_k q x exactly as the row's dequantised dot product;
//  * epilogues: store (+bias, optional greedy argmax; the destination may be read
//    from device memory, and a null one stores nothing), residual add, or SwiGLU on
//    interleaved gate/up rows (row 2j = gate j, row 2j+1 = up j) writing bf16
//    silu(g)*u (R4).
#include "common.cuh"
#include "kernels.h"

namespace dec {

namespace {

constexpr int kRows = 4;               // rows per stage (bf16)
constexpr int kKC = 4096;              // max bf16 columns per stage (8 KB per row copy)
constexpr int kKCq = 4096;             // max int8 columns per stage (4 KB per row copy)
constexpr int kWarps = 8;              // consumer warps: 2 per row
constexpr int kConsumers = kWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kMaxStages = 16;         // short rows (small K) keep more stages in flight
constexpr int kXU = 4;                 // fp32 input pieces (16 bytes) per thread held for the fused norm
constexpr int kXC = 8;                 // bf16 input pieces (16 bytes) per thread in flight when copied

// Rows per stage. q8_row with one or two input columns takes 8 rows: the same bytes per stage
// as bf16, and twice the rows between two reductions.
__host__ __device__ constexpr int rows_per_stage(int nb, bool q8) { return q8 && nb <= 2 ? 8 : kRows; }

struct Layout {
    int kc, stages;
    uint32_t stage_bytes, ring_off, x_off, red_off, total;
};

// bf16 weights: 2-byte elements; q8_row weights: 1-byte elements. The input columns sit in
// shared memory as bf16 either way.
__host__ __device__ inline Layout make_layout(int nb, int K, int smem_cap, bool q8 = false) {
    Layout L;
    const int kcmax = q8 ? kKCq : kKC;
    L.kc = K < kcmax ? K : kcmax;
    L.stage_bytes = (uint32_t)rows_per_stage(nb, q8) * L.kc * (q8 ? 1 : 2);
    // shorter stages when fewer than 4 of them would fit (long rows, several input columns)
    const uint32_t fixed = (((uint32_t)(2 * kMaxStages * 8) + (uint32_t)(2 * kWarps * 64 + 64) * 4 + 127) & ~127u) +
                           (((uint32_t)nb * K * 2 + 127) & ~127u);
    while (L.kc > 1024 && L.kc % 16 == 0 && (int)fixed + 4 * (int)L.stage_bytes > smem_cap) {
        L.kc /= 2;
        L.stage_bytes /= 2;
    }
    const uint32_t bars = 2 * kMaxStages * 8;
    L.red_off = bars;  // two [kWarps][64] float areas (q8 alternates them) + 64 floats scratch
    const uint32_t red = (uint32_t)(2 * kWarps * 64 + 64) * 4;
    L.x_off = (L.red_off + red + 127) & ~127u;
    const uint32_t xbytes = ((uint32_t)nb * K * 2 + 127) & ~127u;  // bf16 input columns
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

// The final logit softcap c tanh(o / c), out of line: a call is taken only when the cap is
// set, so the uncapped epilogue never evaluates the tanh speculatively.
__device__ __noinline__ float softcap_apply(float o, float c) { return c * tanhf(o / c); }

DEC_DEVINL void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory"); }

// The four int8 values of w as exact fp32 values: byte i of w ^ 0x80808080 (q + 128) goes
// into the mantissa of 2^23, and 2^23 + 128 is subtracted.
DEC_DEVINL void widen4(uint32_t w, float2& q01, float2& q23) {
    const uint32_t u = w ^ 0x80808080u;
    const float2 m = make_float2(-8388736.f, -8388736.f);
    q01 = fadd2(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540)),
                            __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7541))),
                m);
    q23 = fadd2(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7542)),
                            __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7543))),
                m);
}

// Warp sums of V values per lane (V a power of two, at most 32) by a butterfly that halves
// the values at each exchange: V - 1 + 5 - log2(V) shuffles instead of 5 V. On return lane l
// holds the sum of value index vidx<V>(l) over all 32 lanes in v[0].
template <int V>
DEC_DEVINL void warp_sum_scatter(float (&v)[V], int lane) {
#pragma unroll
    for (int n = V, m = 16; n > 1; n >>= 1, m >>= 1) {
        const bool hi = lane & m;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float send = hi ? v[i] : v[i + n / 2];
            const float keep = hi ? v[i + n / 2] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
#pragma unroll
    for (int m = 16 / V; m >= 1; m >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
}
// the value index lane l holds after warp_sum_scatter<V>; lanes with (l & (32 / V - 1)) == 0 own it
template <int V>
DEC_DEVINL int vidx(int lane) {
    int idx = 0;
#pragma unroll
    for (int n = V, m = 16; n > 1; n >>= 1, m >>= 1) idx += (lane & m) ? n / 2 : 0;
    return idx;
}

// 16 int8 weights as exact fp32 pairs
DEC_DEVINL void widen16(uint4 w, float2 (&q)[8]) {
    widen4(w.x, q[0], q[1]);
    widen4(w.y, q[2], q[3]);
    widen4(w.z, q[4], q[5]);
    widen4(w.w, q[6], q[7]);
}
// 16 bf16 input columns as fp32 pairs
DEC_DEVINL void load_x16(const uint16_t* x, float2 (&xv)[8]) {
    const uint4 a = reinterpret_cast<const uint4*>(x)[0], c = reinterpret_cast<const uint4*>(x)[1];
    const uint32_t u[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) xv[j] = make_float2(bf_lo(u[j]), bf_hi(u[j]));
}

template <int NB, int EPI, bool Q8>
__global__ void __launch_bounds__(kThreads, 1) gemv_kernel(GemvArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int ES = Q8 ? 1 : 2;  // bytes per weight
    const Layout L = make_layout(NB, a.K, a.smem_cap, Q8);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    float* red = reinterpret_cast<float*>(smem + L.red_off);
    uint16_t* xs = reinterpret_cast<uint16_t*>(smem + L.x_off);  // bf16 input columns [NB][K]
    const uint8_t* Wb = Q8 ? reinterpret_cast<const uint8_t*>(a.Wq) : reinterpret_cast<const uint8_t*>(a.W);
    uint8_t* ring = smem + L.ring_off;

    constexpr int RW = rows_per_stage(NB, Q8);
    const int nrb = (a.N + RW - 1) / RW;
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
                const int r0 = rb * RW;
                const int nrows = min(RW, a.N - r0);
                for (int kc = 0; kc < nkc; ++kc) {
                    const int k0 = kc * L.kc;
                    const int kcols = min(L.kc, a.K - k0);
                    if (!mbar_wait_bounded(&empty[s], ph ^ 1, a.err)) goto producer_done;
                    mbar_arrive_expect_tx(&full[s], (uint32_t)(nrows * kcols * ES));
                    uint8_t* dst = ring + (size_t)s * L.stage_bytes;
                    if (kcols == a.K) {  // whole rows: the stage is one contiguous block
                        bulk_g2s_stream(dst, Wb + (size_t)r0 * a.K * ES, (uint32_t)(nrows * kcols * ES), &full[s],
                                        pol);
                    } else {
                        for (int r = 0; r < nrows; ++r)
                            bulk_g2s_stream(dst + (size_t)r * L.kc * ES, Wb + ((size_t)(r0 + r) * a.K + k0) * ES,
                                            (uint32_t)kcols * ES, &full[s], pol);
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
    // Each thread holds several 16-byte pieces of a column in registers: all its loads are
    // issued before the first use, so a column costs one memory round trip, not one per piece.
    // The norm gains are weights: they are loaded before the wait on the previous kernel.
    const int tid = threadIdx.x;
    const bool held = a.xr != nullptr && a.K <= kConsumers * 4 * kXU;
    float4 gv[kXU];
    if (held) {
#pragma unroll
        for (int u = 0; u < kXU; ++u) {
            const int k = (u * kConsumers + tid) * 4;
            if (k < a.K) gv[u] = *reinterpret_cast<const float4*>(a.g + k);
        }
    }
    pdl_wait();
    for (int b = 0; b < NB; ++b) {
        uint16_t* xrow = xs + (size_t)b * a.K;
        if (b >= a.B) {
            for (int k = tid * 8; k < a.K; k += kConsumers * 8) *reinterpret_cast<uint4*>(xrow + k) = make_uint4(0, 0, 0, 0);
            continue;
        }
        if (a.xr) {
            // fused RMSNorm of the fp32 residual row: R1 rounding to bf16. Thread tid sums the
            // squares of pieces tid, tid + 256, ... in that order on either path.
            const float* xr = a.xr + (size_t)b * a.ldx;
            float ss = 0.f;
            float4 xv[kXU];
            if (held) {
#pragma unroll
                for (int u = 0; u < kXU; ++u) {
                    const int k = (u * kConsumers + tid) * 4;
                    if (k < a.K) xv[u] = *reinterpret_cast<const float4*>(xr + k);
                }
#pragma unroll
                for (int u = 0; u < kXU; ++u) {
                    if ((u * kConsumers + tid) * 4 < a.K) {
                        ss = fmaf(xv[u].x, xv[u].x, ss);
                        ss = fmaf(xv[u].y, xv[u].y, ss);
                        ss = fmaf(xv[u].z, xv[u].z, ss);
                        ss = fmaf(xv[u].w, xv[u].w, ss);
                    }
                }
            } else {
                for (int k = tid * 4; k < a.K; k += kConsumers * 4) {
                    const float4 v = *reinterpret_cast<const float4*>(xr + k);
                    ss = fmaf(v.x, v.x, ss);
                    ss = fmaf(v.y, v.y, ss);
                    ss = fmaf(v.z, v.z, ss);
                    ss = fmaf(v.w, v.w, ss);
                }
            }
            ss = warp_sum(ss);
            if (lane == 0) red[2 * kWarps * 64 + warp] = ss;
            consumer_sync();
            float tot = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) tot += red[2 * kWarps * 64 + w];
            const float inv = 1.0f / sqrtf(tot / (float)a.K + a.eps);
            if (held) {
#pragma unroll
                for (int u = 0; u < kXU; ++u) {
                    const int k = (u * kConsumers + tid) * 4;
                    if (k < a.K) {
                        uint2 o;
                        o.x = pack_bf2(xv[u].x * inv * gv[u].x, xv[u].y * inv * gv[u].y);
                        o.y = pack_bf2(xv[u].z * inv * gv[u].z, xv[u].w * inv * gv[u].w);
                        *reinterpret_cast<uint2*>(xrow + k) = o;
                    }
                }
            } else {
                for (int k = tid * 4; k < a.K; k += kConsumers * 4) {
                    const float4 v = *reinterpret_cast<const float4*>(xr + k);
                    const float4 g = *reinterpret_cast<const float4*>(a.g + k);
                    uint2 o;
                    o.x = pack_bf2(v.x * inv * g.x, v.y * inv * g.y);
                    o.y = pack_bf2(v.z * inv * g.z, v.w * inv * g.w);
                    *reinterpret_cast<uint2*>(xrow + k) = o;
                }
            }
            consumer_sync();  // red[] reused by the next column
        } else {
            const uint16_t* xb = a.xb + (size_t)b * a.ldx;
            for (int k0 = tid * 8; k0 < a.K; k0 += kConsumers * 8 * kXC) {
                uint4 v[kXC];
#pragma unroll
                for (int u = 0; u < kXC; ++u) {
                    const int k = k0 + u * kConsumers * 8;
                    if (k < a.K) v[u] = *reinterpret_cast<const uint4*>(xb + k);
                }
#pragma unroll
                for (int u = 0; u < kXC; ++u) {
                    const int k = k0 + u * kConsumers * 8;
                    if (k < a.K) *reinterpret_cast<uint4*>(xrow + k) = v[u];
                }
            }
        }
    }
    consumer_sync();

    // ---------------------------------------------------- consumers: stream
    // A timed-out wait marks the call failed (a.err) and skips the remaining work, but
    // every warp still passes the same named barriers so none of them can hang.
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    float* const y = (EPI == GEMV_STORE && a.y_ptr) ? *a.y_ptr : a.y;  // null: argmax only
    if constexpr (Q8) {
        // q8_row: consumer thread t owns the 16-column pieces t, t + 256, ... of ALL rows of
        // a stage, so each input column is read from shared memory once per stage (bf16,
        // half the weight bytes) and reused for the stage's rows; the rows' partial sums
        // are reduced over the warps after the stage.
        unsigned long long best = 0;  // thread t < RW * NB: argmax of column t % NB
        int par = 0;                  // the reduction area of this stage (they alternate)
        for (int rb = rb0; rb < rb1; ++rb) {
            float2 acc[RW][NB];
#pragma unroll
            for (int r = 0; r < RW; ++r)
#pragma unroll
                for (int b = 0; b < NB; ++b) acc[r][b] = make_float2(0.f, 0.f);
            for (int kc = 0; kc < nkc; ++kc) {
                const int k0 = kc * L.kc;
                const int npc = min(L.kc, a.K - k0) >> 4;  // 16-column pieces of this chunk
                if (ok && !mbar_wait_bounded(&full[s], ph, a.err)) ok = false;
                if (ok) {
                    const uint8_t* st8 = ring + (size_t)s * L.stage_bytes;
                    for (int p = tid; p < npc; p += kConsumers) {
                        // rows past N hold stale bytes: their sums are never stored
                        if constexpr (NB <= 2) {  // input columns held, one weight row at a time
                            float2 xv[NB][8];
#pragma unroll
                            for (int b = 0; b < NB; ++b) load_x16(xs + (size_t)b * a.K + k0 + p * 16, xv[b]);
#pragma unroll
                            for (int r = 0; r < RW; ++r) {
                                float2 q[8];
                                widen16(*reinterpret_cast<const uint4*>(st8 + (size_t)r * L.kc + p * 16), q);
#pragma unroll
                                for (int b = 0; b < NB; ++b)
#pragma unroll
                                    for (int j = 0; j < 8; ++j) acc[r][b] = ffma2(q[j], xv[b][j], acc[r][b]);
                            }
                        } else {  // weight rows held, one input column at a time
                            float2 q[RW][8];
#pragma unroll
                            for (int r = 0; r < RW; ++r)
                                widen16(*reinterpret_cast<const uint4*>(st8 + (size_t)r * L.kc + p * 16), q[r]);
#pragma unroll
                            for (int b = 0; b < NB; ++b) {
                                float2 xv[8];
                                load_x16(xs + (size_t)b * a.K + k0 + p * 16, xv);
#pragma unroll
                                for (int r = 0; r < RW; ++r)
#pragma unroll
                                    for (int j = 0; j < 8; ++j) acc[r][b] = ffma2(q[r][j], xv[j], acc[r][b]);
                            }
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
            // per (row, column): warp partial sums, then the 8 warps summed in warp order. The
            // two reduction areas alternate, so one barrier per stage suffices: the area written
            // here was last read two stages ago, before this stage's barrier of those readers.
            float* rd = red + par * kWarps * 64;
            par ^= 1;
            {
                constexpr int V = RW * NB;  // 8, 16 or 32 sums, index r * NB + b
                float v[V];
#pragma unroll
                for (int r = 0; r < RW; ++r)
#pragma unroll
                    for (int b = 0; b < NB; ++b) v[r * NB + b] = acc[r][b].x + acc[r][b].y;
                warp_sum_scatter<V>(v, lane);
                if ((lane & (32 / V - 1)) == 0) rd[warp * 64 + vidx<V>(lane)] = v[0];
            }
            consumer_sync();
            if (tid < RW * NB) {
                const int r = tid / NB, b = tid % NB, row = rb * RW + r;
                float v = 0.f;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) v += rd[w * 64 + tid];
                if (row < a.N && b < a.B && ok) {
                    v *= a.wscale[row];  // the row's scale, once, on its exact integer-weight dot product
                    if constexpr (EPI == GEMV_STORE) {
                        float o = v + (a.bias ? a.bias[row] : 0.f);
                        if (a.softcap > 0.f) o = softcap_apply(o, a.softcap);  // final logit softcap
                        if (y) y[(size_t)b * a.ldy + row] = o;
                        if (a.amax) {
                            const unsigned long long pw = argmax_pack(o, row);
                            if (pw > best) best = pw;
                        }
                    } else if constexpr (EPI == GEMV_RESID) {
                        y[(size_t)b * a.ldy + row] += v;
                    } else if ((r & 1) == 0) {  // SwiGLU: gate row r, up row r + 1
                        float u = 0.f;
#pragma unroll
                        for (int w = 0; w < kWarps; ++w) u += rd[w * 64 + tid + NB];
                        u *= a.wscale[row + 1];
                        const float sg = silu_f(v);
                        a.act[(size_t)b * a.ldact + (row >> 1)] = f2bf(sg * u);
                    }
                }
            }
        }
        if constexpr (EPI == GEMV_STORE) {
            if (a.amax) {  // greedy argmax: CTA reduction, then one atomic per column
                consumer_sync();  // the last stage's readers are done with the reduction areas
                unsigned long long* wb = reinterpret_cast<unsigned long long*>(red);  // [RW][NB]
                if (tid < RW * NB) wb[tid] = best;
                consumer_sync();
                if (tid < NB && tid < a.B) {
                    unsigned long long m = 0;
#pragma unroll
                    for (int r = 0; r < RW; ++r) m = wb[r * NB + tid] > m ? wb[r * NB + tid] : m;
                    if (m) atomicMax(&a.amax[(size_t)tid * 32], m);
                }
            }
        }
        return;
    } else {
        const int r_in = warp >> 1, half = warp & 1;
        unsigned long long best = 0;  // lane b of an even warp: packed argmax of column b over its rows
        int par = 0;                  // the reduction area of this stage (they alternate, as above)
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
            float* rd = red + par * kWarps * 64;
            par ^= 1;
#pragma unroll
            for (int b = 0; b < NB; ++b) acc[b] = warp_sum(acc[b]);
            if (lane == 0) {
#pragma unroll
                for (int b = 0; b < NB; ++b) rd[warp * 16 + b] = acc[b];
            }
            consumer_sync();
            // row sum = first column half + second column half, in that order
            if constexpr (EPI != GEMV_SWIGLU) {
                if (half == 0 && lane < a.B && valid && ok) {
                    const float v = rd[warp * 16 + lane] + rd[(warp + 1) * 16 + lane];
                    if constexpr (EPI == GEMV_STORE) {
                        float o = v + (a.bias ? a.bias[row] : 0.f);
                        if (a.softcap > 0.f) o = softcap_apply(o, a.softcap);  // final logit softcap
                        if (y) y[(size_t)lane * a.ldy + row] = o;
                        if (a.amax) {
                            const unsigned long long w = argmax_pack(o, row);
                            if (w > best) best = w;
                        }
                    } else {
                        y[(size_t)lane * a.ldy + row] += v;
                    }
                }
            } else {
                if ((r_in & 1) == 0 && half == 0 && valid && ok && lane < a.B) {
                    const float g = rd[warp * 16 + lane] + rd[(warp + 1) * 16 + lane];
                    const float u = rd[(warp + 2) * 16 + lane] + rd[(warp + 3) * 16 + lane];
                    const float sg = silu_f(g);
                    a.act[(size_t)lane * a.ldact + (row >> 1)] = f2bf(sg * u);
                }
            }
        }
        if constexpr (EPI == GEMV_STORE) {
            if (a.amax) {  // greedy argmax: CTA reduction, then one atomic per column
                consumer_sync();  // the last stage's readers are done with the reduction areas
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
}

template <int NB, int EPI, bool Q8>
cudaError_t launch_nb(const GemvArgs& a0, cudaStream_t st, int num_sms, bool pdl) {
    GemvArgs a = a0;
    const Layout L = make_layout(NB, a.K, a.smem_cap, Q8);
    if (L.stages < 3) return cudaErrorInvalidValue;
    auto kern = gemv_kernel<NB, EPI, Q8>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), (int)L.total);
    if (e != cudaSuccess) return e;
    constexpr int RW = rows_per_stage(NB, Q8);
    const int nrb = (a.N + RW - 1) / RW;
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

template <int EPI, bool Q8>
cudaError_t launch_epi(const GemvArgs& a, cudaStream_t st, int num_sms, bool pdl) {
    switch (a.nb) {
        case 1: return launch_nb<1, EPI, Q8>(a, st, num_sms, pdl);
        case 2: return launch_nb<2, EPI, Q8>(a, st, num_sms, pdl);
        case 4: return launch_nb<4, EPI, Q8>(a, st, num_sms, pdl);
        case 8: return launch_nb<8, EPI, Q8>(a, st, num_sms, pdl);
        default: return cudaErrorInvalidValue;
    }
}

template <int EPI>
cudaError_t launch_fmt(const GemvArgs& a, cudaStream_t st, int num_sms, bool pdl) {
    return a.Wq ? launch_epi<EPI, true>(a, st, num_sms, pdl) : launch_epi<EPI, false>(a, st, num_sms, pdl);
}

}  // namespace

int gemv_nb_for(int B) { return B <= 1 ? 1 : B <= 2 ? 2 : B <= 4 ? 4 : B <= 8 ? 8 : 0; }

bool gemv_fits(int B, int K, int smem_cap, bool q8) {
    const int nb = gemv_nb_for(B);
    if (nb == 0 || K % (q8 ? 16 : 8) != 0 || K <= 0) return false;
    const Layout L = make_layout(nb, K, smem_cap, q8);
    return L.stages >= 3;
}

cudaError_t gemv_launch(GemvArgs a, int epi, cudaStream_t st, int num_sms, bool pdl) {
    a.nb = gemv_nb_for(a.B);
    if (epi == GEMV_SWIGLU && (a.N % rows_per_stage(a.nb, a.Wq != nullptr)) != 0) return cudaErrorInvalidValue;
    if (a.Wq && (!a.wscale || a.K % 16 != 0)) return cudaErrorInvalidValue;
    switch (epi) {
        case GEMV_STORE: return launch_fmt<GEMV_STORE>(a, st, num_sms, pdl);
        case GEMV_RESID: return launch_fmt<GEMV_RESID>(a, st, num_sms, pdl);
        case GEMV_SWIGLU: return launch_fmt<GEMV_SWIGLU>(a, st, num_sms, pdl);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace dec
