// Mixture-of-experts FFN of the layer (ANEDVD src/engine.zig: cpu.moeRoute, the routed
// expert loop moeExpertAccum and the sigmoid-scaled shared expert; frink_models decoder.rs:
// route_top_k, shared-expert gate; cortiq_engine pipeline.rs: MoeFfn):
//   P = softmax(router . xn) over all E experts; the k most probable experts (lower index
//   first on ties), weights P or P / sum_topk P; out = sum_j w_j SwiGLU_{e_j}(xn) +
//   sigmoid(g . xn) SwiGLU_shared(xn); x += out.
//
// B200 design: the tokens of a step or prefill chunk are permuted by expert (counts,
// offsets, a deterministic token list per expert), split into groups of at most NB tokens,
// and each expert's weights stream once per group. Where an expert's weight rows tile into
// 128-row blocks, every group runs on the tensor pipe (work item = group x 128-row block,
// TMA boxes, mma.sync with the group's tokens as the n dimension of 8); otherwise a grouped
// weight-streaming GEMV on the CUDA cores (work item = group x 4-row weight block, the same
// bulk-copy ring as the dense GEMV). Either way
// the group's token rows sit in shared memory and the epilogue writes SiLU(gate)*up (bf16)
// or the projection (fp32) per (token, expert) slot.
// A combine kernel adds the weighted slots and the gated shared expert to the residual in
// a fixed order (routed experts in top-k order, then the shared expert).
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

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

// ------------------------------------------------------------------ routing + shared gate

// One warp per token: softmax over E <= 256 logits (8 per lane), k picks by probability with
// the lower index first on ties, optional renormalisation; the shared-expert gate
// sigmoid(gvec . xn) from the same normalised row.
__global__ void __launch_bounds__(32) moe_route_kernel(MoeRouteArgs a) {
    pdl_trigger();
    pdl_wait();
    const int t = blockIdx.x, lane = threadIdx.x;
    const float* r = a.logits + (size_t)t * a.E;
    float v[8], mx = -INFINITY;
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
    float tot = 0.f;
    float sel_p[16];
    int sel_i[16];
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
        sel_p[q & 15] = bp;
        sel_i[q & 15] = be;
        tot += bp;
    }
    float gate = 1.f;
    if (a.gvec) {
        const uint16_t* xr = a.xn + (size_t)t * a.h;
        float d = 0.f;
        for (int i = lane; i < a.h; i += 32) d = fmaf(a.gvec[i], bf2f(xr[i]), d);
        d = warp_sum(d);
        gate = 1.0f / (1.0f + expf(-d));
    }
    if (lane == 0) {
        for (int q = 0; q < a.k; ++q) {
            a.idx[(size_t)t * a.k + q] = sel_i[q];
            a.w[(size_t)t * a.k + q] = a.renorm ? sel_p[q] / tot : sel_p[q];
        }
        if (a.sgate) a.sgate[t] = gate;
    }
}

// ------------------------------------------------------------------ permutation by expert

// One CTA: counts per expert, offsets, per-expert token lists in (token, slot) order, the
// inverse map, and the groups of at most nb tokens (expert order) for the grouped
// projections. Warp w owns a contiguous range of routing slots: it counts them into its
// own histogram, the histograms are scanned over warps (per expert) and over experts
// (warp shuffles), and each warp then places its slots 32 at a time, ranking lanes that
// share an expert by lane order, so every expert's list keeps slot order.
constexpr int kPermWarps = 8;

__global__ void __launch_bounds__(kPermWarps * 32) moe_permute_kernel(MoePermArgs a) {
    __shared__ int hist[kPermWarps][256];  // counts, then each warp's next position per expert
    __shared__ int cnt[256], off[256], goff[256];
    pdl_trigger();
    pdl_wait();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int total = a.n * a.k, E = a.E;
    int* hflat = &hist[0][0];
    for (int i = tid; i < kPermWarps * 256; i += kPermWarps * 32) hflat[i] = 0;
    __syncthreads();
    const int r0 = (int)((int64_t)total * warp / kPermWarps);
    const int r1 = (int)((int64_t)total * (warp + 1) / kPermWarps);
    for (int i = r0 + lane; i < r1; i += 32) {
        const int e = a.idx[i];
        if (e >= 0 && e < E)
            atomicAdd(&hist[warp][e], 1);
        else
            a.inv[i] = -1;  // dropped: the combine skips it
    }
    __syncthreads();
    {  // thread e: count of expert e and the exclusive prefix of its histogram over warps
        int c = 0;
        if (tid < E)
            for (int w = 0; w < kPermWarps; ++w) {
                const int h = hist[w][tid];
                hist[w][tid] = c;
                c += h;
            }
        cnt[tid] = tid < E ? c : 0;
    }
    __syncthreads();
    if (warp == 0) {  // exclusive scans over the 256 experts, 8 per lane: slot and group offsets
        int lc[8], lg[8], s = 0, gs = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            lc[j] = cnt[lane * 8 + j];
            lg[j] = (lc[j] + a.nb - 1) / a.nb;
            s += lc[j];
            gs += lg[j];
        }
        int si = s, gi = gs;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int t1 = __shfl_up_sync(0xffffffffu, si, d);
            const int t2 = __shfl_up_sync(0xffffffffu, gi, d);
            if (lane >= d) {
                si += t1;
                gi += t2;
            }
        }
        int o = si - s, g = gi - gs;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            off[lane * 8 + j] = o;
            goff[lane * 8 + j] = g;
            o += lc[j];
            g += lg[j];
        }
        if (lane == 31) *a.n_groups = gi;
    }
    __syncthreads();
    for (int i = tid; i < kPermWarps * 256; i += kPermWarps * 32) hflat[i] += off[i & 255];
    __syncthreads();
    for (int b0 = r0; b0 < r1; b0 += 32) {
        const int i = b0 + lane;
        const int e = i < r1 ? a.idx[i] : -1;
        const bool valid = e >= 0 && e < E;
        const unsigned m = __match_any_sync(0xffffffffu, valid ? e : 1024 + lane);
        if (valid) {
            const int p = hist[warp][e] + __popc(m & ((1u << lane) - 1u));
            a.perm_tok[p] = i / a.k;
            a.inv[i] = p;
        }
        __syncwarp();
        if (valid && lane == 31 - __clz(m)) hist[warp][e] += __popc(m);
        __syncwarp();
    }
    if (tid < E) {
        const int e = tid, o = off[e], c = cnt[e];
        int g = goff[e];
        for (int s = 0; s < c; s += a.nb, ++g) {
            a.groups[g * 4 + 0] = e;
            a.groups[g * 4 + 1] = o + s;
            a.groups[g * 4 + 2] = min(a.nb, c - s);
            a.groups[g * 4 + 3] = 0;
        }
    }
}

// ------------------------------------------------------------------ grouped weight-streaming GEMV

constexpr int kRows = 4;
constexpr int kKC = 4096;
constexpr int kWarps = 8;
constexpr int kConsumers = kWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kMaxStages = 16;

struct Layout {
    int kc, stages;
    uint32_t stage_bytes, ring_off, x_off, red_off, total;
};

__host__ __device__ inline Layout make_layout(int nb, int K, int smem_cap) {
    Layout L;
    L.kc = K < kKC ? K : kKC;
    L.stage_bytes = (uint32_t)kRows * L.kc * 2;
    L.red_off = 2 * kMaxStages * 8;
    const uint32_t red = (uint32_t)(kWarps * 16) * 4;
    L.x_off = (L.red_off + red + 127) & ~127u;
    L.ring_off = L.x_off + (((uint32_t)nb * K * 2 + 127) & ~127u);
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

// Work item i = (group i / nrb, 4-row block i % nrb); group = (expert e, first permuted slot
// p0, token count c <= NB). Weights of expert e: W + e * wstride, rows [M][K].
template <int NB, int SWIGLU>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemv_kernel(GroupedGemvArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Layout L = make_layout(NB, a.K, a.smem_cap);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    float* red = reinterpret_cast<float*>(smem + L.red_off);
    uint16_t* xs = reinterpret_cast<uint16_t*>(smem + L.x_off);
    uint8_t* ring = smem + L.ring_off;

    if (threadIdx.x == 0) {
        for (int s = 0; s < L.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();
    pdl_trigger();
    pdl_wait();  // the groups come from the previous kernel

    const int nrb = (a.M + kRows - 1) / kRows;
    const int nkc = (a.K + L.kc - 1) / L.kc;
    const int items = *a.n_groups * nrb;
    const int i0 = (int)((int64_t)blockIdx.x * items / gridDim.x);
    const int i1 = (int)((int64_t)(blockIdx.x + 1) * items / gridDim.x);

    if (warp == kWarps) {
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            int s = 0;
            uint32_t ph = 0;
            for (int it = i0; it < i1; ++it) {
                const int g = it / nrb, rb = it % nrb;
                const uint16_t* W = a.W + (size_t)a.groups[g * 4] * a.wstride;
                const int r0 = rb * kRows;
                const int nrows = min(kRows, a.M - r0);
                for (int kc = 0; kc < nkc; ++kc) {
                    const int k0 = kc * L.kc;
                    const int kcols = min(L.kc, a.K - k0);
                    if (!mbar_wait_bounded(&empty[s], ph ^ 1, a.err)) return;
                    mbar_arrive_expect_tx(&full[s], (uint32_t)(nrows * kcols * 2));
                    uint8_t* dst = ring + (size_t)s * L.stage_bytes;
                    if (kcols == a.K) {  // whole rows: one contiguous block
                        bulk_g2s_stream(dst, W + (size_t)r0 * a.K, (uint32_t)(nrows * kcols * 2), &full[s], pol);
                    } else {
                        for (int r = 0; r < nrows; ++r)
                            bulk_g2s_stream(dst + (size_t)r * L.kc * 2, W + (size_t)(r0 + r) * a.K + k0,
                                            (uint32_t)kcols * 2, &full[s], pol);
                    }
                    if (++s == L.stages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
            }
        }
        return;
    }

    const int tid = threadIdx.x;
    const int r_in = warp >> 1, half = warp & 1;
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    int cur_g = -1, c = 0, p0 = 0;
    for (int it = i0; it < i1; ++it) {
        const int g = it / nrb, rb = it % nrb;
        if (g != cur_g) {  // load the group's token rows
            cur_g = g;
            p0 = a.groups[g * 4 + 1];
            c = a.groups[g * 4 + 2];
            consumer_sync();
            for (int b = 0; b < NB; ++b) {
                uint16_t* xrow = xs + (size_t)b * a.K;
                if (b < c) {
                    const int src = a.x_map ? a.x_map[p0 + b] : p0 + b;
                    const uint16_t* xr = a.x + (size_t)src * a.ldx;
                    for (int k = tid * 8; k < a.K; k += kConsumers * 8)
                        *reinterpret_cast<uint4*>(xrow + k) = *reinterpret_cast<const uint4*>(xr + k);
                } else {
                    for (int k = tid * 8; k < a.K; k += kConsumers * 8)
                        *reinterpret_cast<uint4*>(xrow + k) = make_uint4(0, 0, 0, 0);
                }
            }
            consumer_sync();
        }
        const int row = rb * kRows + r_in;
        const bool valid = row < a.M;
        float acc[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[b] = 0.f;
        for (int kc = 0; kc < nkc; ++kc) {
            const int k0 = kc * L.kc;
            const int npc = min(L.kc, a.K - k0) >> 3;
            const int hp = (npc + 1) >> 1;
            const int q0 = half * hp, q1 = min(npc, q0 + hp);
            if (ok && !mbar_wait_bounded(&full[s], ph, a.err)) ok = false;
            if (valid && ok) {
                const uint4* wrow =
                    reinterpret_cast<const uint4*>(ring + (size_t)s * L.stage_bytes + (size_t)r_in * L.kc * 2);
                for (int p = q0 + lane; p < q1; p += 32) {
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
        if (!SWIGLU) {
            if (half == 0 && lane < c && valid && ok)
                a.y[(size_t)(p0 + lane) * a.ldy + row] = red[warp * 16 + lane] + red[(warp + 1) * 16 + lane];
        } else if ((r_in & 1) == 0 && half == 0 && valid && ok && lane < c) {
            const float gv = red[warp * 16 + lane] + red[(warp + 1) * 16 + lane];
            const float uv = red[(warp + 2) * 16 + lane] + red[(warp + 3) * 16 + lane];
            const float sg = silu_f(gv);
            a.act[(size_t)(p0 + lane) * a.ldact + (row >> 1)] = f2bf(sg * uv);
        }
        consumer_sync();
    }
}

// ------------------------------------------------------------------ grouped GEMM on the tensor pipe

// Groups of up to 8 tokens: the CUDA-core GEMV above converts every token element once per
// weight row and becomes ALU-bound with 8 tokens (and streams small 4-row items with 1), so
// here each group's token rows are the n = 8 operand of mma.sync m16n8k16 (bf16 in, fp32
// accumulate; token rows past the group's count are zero). A work item is (group, 128-row weight
// block); the TMA unit streams the block in 128B-swizzled boxes of 64 columns x 128 rows,
// and consumer warp w owns rows 16w .. 16w+15 of the block over the whole K, so no partial
// sums cross warps. Token rows sit in shared memory with a 16-byte pad per row, which
// makes the ldmatrix reads of both operands free of bank conflicts.
constexpr int kTcRows = 128;
constexpr int kTcK = 64;
constexpr uint32_t kTcBox = kTcRows * kTcK * 2;  // 16 KB
constexpr int kTcMaxStages = 8;
constexpr int kTcTok = 8;

struct TcLayout {
    int kp, stages;  // padded token row (elements); operand ring depth
    uint32_t xs_off, ring_off, total;
};

__host__ __device__ inline TcLayout make_tc_layout(int K, int smem_cap) {
    TcLayout L;
    L.kp = ((K + kTcK - 1) / kTcK) * kTcK + 8;
    L.xs_off = 2 * kTcMaxStages * 8;
    L.ring_off = (L.xs_off + (uint32_t)kTcTok * L.kp * 2 + 1023) & ~1023u;
    int st = (int)(((long long)smem_cap - 1024 - (long long)L.ring_off) / (long long)kTcBox);
    L.stages = st > kTcMaxStages ? kTcMaxStages : st;
    L.total = L.ring_off + (uint32_t)(L.stages > 0 ? L.stages : 0) * kTcBox + 1024;  // + base alignment
    return L;
}

template <int SWIGLU>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_mma_kernel(const __grid_constant__ CUtensorMap tmW, GroupedGemvArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);  // swizzle atoms: 1 KB
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const TcLayout L = make_tc_layout(a.K, a.smem_cap);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kTcMaxStages;
    uint16_t* xs = reinterpret_cast<uint16_t*>(smem + L.xs_off);
    uint8_t* ring = smem + L.ring_off;
    if (threadIdx.x == 0) prefetch_tmap(&tmW);

    if (threadIdx.x == 0) {
        for (int s = 0; s < L.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();
    pdl_trigger();
    pdl_wait();  // the groups come from the previous kernel

    const int nrb = a.M / kTcRows;
    const int nkb = (a.K + kTcK - 1) / kTcK;
    const int items = *a.n_groups * nrb;
    const int i0 = (int)((int64_t)blockIdx.x * items / gridDim.x);
    const int i1 = (int)((int64_t)(blockIdx.x + 1) * items / gridDim.x);

    if (warp == kWarps) {
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            int s = 0;
            uint32_t ph = 0;
            for (int it = i0; it < i1; ++it) {
                const int g = it / nrb, rb = it % nrb;
                const int row = a.groups[g * 4] * a.M + rb * kTcRows;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait_bounded(&empty[s], ph ^ 1, a.err)) return;
                    mbar_arrive_expect_tx(&full[s], kTcBox);  // columns past K arrive zero-filled
                    tma_load_2d_hint(ring + (size_t)s * kTcBox, &tmW, kb * kTcK, row, &full[s], pol);
                    if (++s == L.stages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
            }
        }
        return;
    }

    // ldmatrix lane roles. A (x4): matrices (rows 0-7 | 8-15) x (k 0-7 | 8-15) of the warp's
    // 16 rows; B (x4): token rows 0-7 at k offsets 0, 8, 16, 24 (two k16 steps).
    const int mi = lane >> 3, ri = lane & 7;
    const int a_row = warp * 16 + ri + ((mi & 1) << 3);
    const uint32_t a_row_off = (uint32_t)a_row * 128;
    const int a_sw = a_row & 7;
    const int a_chunk = mi >> 1;
    const uint16_t* b_base = xs + (size_t)ri * L.kp + mi * 8;
    const int g4 = lane >> 2, t4 = lane & 3;

    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    int cur_g = -1, c = 0, p0 = 0;
    for (int it = i0; it < i1; ++it) {
        const int g = it / nrb, rb = it % nrb;
        if (g != cur_g) {  // the group's token rows, zero past the c tokens and past K
            cur_g = g;
            p0 = a.groups[g * 4 + 1];
            c = a.groups[g * 4 + 2];
            consumer_sync();
            const int kw = L.kp - 8;
            for (int b = 0; b < kTcTok; ++b) {
                uint16_t* xrow = xs + (size_t)b * L.kp;
                const uint16_t* xr = nullptr;
                if (b < c) xr = a.x + (size_t)(a.x_map ? a.x_map[p0 + b] : p0 + b) * a.ldx;
                for (int k = threadIdx.x * 8; k < kw; k += kConsumers * 8)
                    *reinterpret_cast<uint4*>(xrow + k) =
                        (xr && k < a.K) ? *reinterpret_cast<const uint4*>(xr + k) : make_uint4(0, 0, 0, 0);
            }
            consumer_sync();
        }
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int kb = 0; kb < nkb; ++kb) {
            if (ok && !mbar_wait_bounded(&full[s], ph, a.err)) ok = false;
            if (ok) {
                const uint8_t* stage = ring + (size_t)s * kTcBox + a_row_off;
                const uint16_t* bk = b_base + kb * kTcK;
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t bf[4];
                    ldsm_x4(bf, bk + h2 * 32);
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int chunk = (h2 * 2 + j) * 2 + a_chunk;
                        uint32_t af[4];
                        ldsm_x4(af, stage + ((chunk ^ a_sw) << 4));
                        mma_bf16_16816(acc, af, bf + 2 * j);
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
        // acc: rows r0 = 16w + g4 and r0 + 8 of the block, tokens 2*t4 and 2*t4 + 1.
        const int r0 = rb * kTcRows + warp * 16 + g4;
        const int tok = 2 * t4;
        if (!SWIGLU) {
            if (ok) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int tq = tok + (q & 1), rq = r0 + ((q >> 1) << 3);
                    if (tq < c) a.y[(size_t)(p0 + tq) * a.ldy + rq] = acc[q];
                }
            }
        } else {
            // gate rows are even, up rows odd: the up partner of lane l sits in lane l + 4
            float up[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) up[q] = __shfl_down_sync(0xffffffffu, acc[q], 4);
            if (ok && (g4 & 1) == 0) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int tq = tok + (q & 1), rq = r0 + ((q >> 1) << 3);
                    if (tq < c) {
                        const float gv = acc[q];
                        const float sg = silu_f(gv);
                        a.act[(size_t)(p0 + tq) * a.ldact + (rq >> 1)] = f2bf(sg * up[q]);
                    }
                }
            }
        }
    }
}

// ------------------------------------------------------------------ combine

// x[t][i] += (sum_j w[t][j] * y[inv[t*k+j]][i]) + sgate[t] * ys[t][i]
__global__ void __launch_bounds__(256) moe_combine_kernel(MoeCombineArgs a) {
    pdl_trigger();
    pdl_wait();
    const int t = blockIdx.x;
    int slot[16];
    float wt[16];
    for (int j = 0; j < a.k && j < 16; ++j) {
        slot[j] = a.inv[(size_t)t * a.k + j];
        wt[j] = a.w[(size_t)t * a.k + j];
    }
    const float sg = a.sgate ? a.sgate[t] : 1.f;
    for (int i = blockIdx.y * 256 + threadIdx.x; i < a.h; i += 256 * gridDim.y) {
        float routed = 0.f;
        for (int j = 0; j < a.k && j < 16; ++j)
            if (slot[j] >= 0) routed += wt[j] * a.y[(size_t)slot[j] * a.h + i];
        const float shared = a.ys ? sg * a.ys[(size_t)t * a.h + i] : 0.f;
        a.x[(size_t)t * a.h + i] += routed + shared;
    }
}

template <int NB, int SW>
cudaError_t launch_grouped_nb(const GroupedGemvArgs& a, cudaStream_t st, int num_sms, bool pdl) {
    const Layout L = make_layout(NB, a.K, a.smem_cap);
    if (L.stages < 3) return cudaErrorInvalidValue;
    auto kern = grouped_gemv_kernel<NB, SW>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), (int)L.total);
    if (e != cudaSuccess) return e;
    return launch_ex(kern, dim3(num_sms), dim3(kThreads), L.total, st, pdl, a);
}

template <int SW>
cudaError_t launch_grouped_mma(const GroupedGemvArgs& a, cudaStream_t st, int num_sms, bool pdl) {
    const TcLayout L = make_tc_layout(a.K, a.smem_cap);
    CUtensorMap tm;
    cudaError_t e = tmap_bf16_rows(&tm, a.W, a.E * a.M, a.K, kTcRows);
    if (e != cudaSuccess) return e;
    auto kern = grouped_mma_kernel<SW>;
    e = ensure_smem(reinterpret_cast<const void*>(kern), (int)L.total);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_sms);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, tm, a);
}

}  // namespace

cudaError_t moe_route_launch(const MoeRouteArgs& a, int n, cudaStream_t st, bool pdl) {
    if (a.E > 256 || a.k > 16 || a.k > a.E || a.k <= 0) return cudaErrorInvalidValue;
    return launch_ex(moe_route_kernel, dim3(n), dim3(32), 0, st, pdl, a);
}

cudaError_t moe_permute_launch(const MoePermArgs& a, cudaStream_t st, bool pdl) {
    if (a.E > 256) return cudaErrorInvalidValue;
    return launch_ex(moe_permute_kernel, dim3(1), dim3(256), 0, st, pdl, a);
}

int grouped_nb_for(int n) { return n <= 1 ? 1 : n <= 2 ? 2 : n <= 4 ? 4 : 8; }

bool grouped_fits(int nb, int K, int smem_cap) {
    if (K % 8 != 0) return false;
    return make_layout(nb, K, smem_cap).stages >= 3;
}

// Groups (of any size up to 8 tokens) go to the tensor pipe when the weights tile into
// 128-row blocks that stay inside one expert and the TMA unit can read them as one
// [E*M][K] matrix.
bool grouped_uses_mma(int nb, int M, int K, size_t wstride, int smem_cap) {
    return nb >= 1 && nb <= kTcTok && M % kTcRows == 0 && K % 8 == 0 && wstride == (size_t)M * K &&
           make_tc_layout(K, smem_cap).stages >= 3;
}

cudaError_t grouped_gemv_launch(const GroupedGemvArgs& a, int nb, bool swiglu, cudaStream_t st, int num_sms,
                                bool pdl) {
    if (swiglu && a.M % kRows != 0) return cudaErrorInvalidValue;
    if (grouped_uses_mma(nb, a.M, a.K, a.wstride, a.smem_cap) && a.E > 0 &&
        (reinterpret_cast<uintptr_t>(a.W) & 15) == 0)
        return swiglu ? launch_grouped_mma<1>(a, st, num_sms, pdl) : launch_grouped_mma<0>(a, st, num_sms, pdl);
#define DEC_G(NB_)                                                                                   \
    case NB_:                                                                                        \
        return swiglu ? launch_grouped_nb<NB_, 1>(a, st, num_sms, pdl) : launch_grouped_nb<NB_, 0>(a, st, num_sms, pdl);
    switch (nb) {
        DEC_G(1)
        DEC_G(2)
        DEC_G(4)
        DEC_G(8)
        default: return cudaErrorInvalidValue;
    }
#undef DEC_G
}

cudaError_t moe_combine_launch(const MoeCombineArgs& a, int n, cudaStream_t st, bool pdl) {
    if (a.k > 16) return cudaErrorInvalidValue;
    // few tokens: split each row over CTAs, so the combine is not one CTA's serial walk of h
    const int cols = (a.h + 255) / 256;
    const int gy = std::min(cols, std::max(1, 1024 / std::max(n, 1)));
    return launch_ex(moe_combine_kernel, dim3(n, gy), dim3(256), 0, st, pdl, a);
}

}  // namespace dec
