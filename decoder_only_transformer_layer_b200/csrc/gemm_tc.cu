// Tensor-core projection for prefill chunks and large decode batches:
//   D[m][n] = sum_k A[m][k] * B[n][k],  A = weights bf16 [M][K], B = activations
//   bf16 [N][K] (N = tokens), both K-major; stored transposed as y[n][m].
//
// These are the same projections as the decode GEMV (ANEDVD src/engine.zig:
// the chunk-wide 1x1 convs of Engine.prefill; cortiq_engine pipeline.rs: the
// chunk GEMMs of prefill_batch), used where the token count makes them a real
// dense contraction.
//
// B200 design (sm_100a, tcgen05):
//  * persistent: one CTA per SM; the (128 x BN tile, 64-wide k block) units of the
//    product (BN = 32/64/128 tokens) are cut into equal contiguous ranges, one per
//    CTA (stream-K), so every SM streams the same share of the weights whatever the
//    tile count; a tile shared by several CTAs is finished by the CTA holding its
//    last k blocks: the others publish their fp32 pieces first thing, and the
//    finisher adds them, in k order, to its own accumulator (deterministic, no
//    atomics on data, and no CTA waits for another's wait);
//  * warp 4 / lane 0 drives TMA: 128B-swizzled 64-wide K slices of A and B into a
//    6-8 stage shared-memory ring (mbarrier complete_tx); the weight slices of
//    the first stages are issued before griddepcontrol.wait (they do not depend
//    on the previous kernel), the activation slices after it;
//  * warp 5 / lane 0 issues tcgen05.mma.cta_group::1.kind::f16 (M=128, N=BN,
//    K=16 per instruction, fp32 accumulator in TMEM) and frees each stage with
//    tcgen05.commit; the accumulator is double-buffered in TMEM (2 x BN columns),
//    so one tile's epilogue overlaps the next tile's main loop;
//  * warps 0-3 and 6-9 read the accumulator with tcgen05.ld (warp w owns TMEM lanes
//    32 (w % 4).. = weight rows; warps 0-3 one half of the columns, 6-9 the other;
//    the cluster split-K kernel likewise) and apply the epilogue: store (+bias, + greedy
//    argmax; the destination may be read from device memory, and a null one stores
//    nothing), residual add, or SwiGLU on interleaved gate/up rows (bf16 silu(g)*u).
#include <cuda.h>

#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace dec {

namespace {

constexpr int BM = 128, BK = 64;


template <int BN>
struct Cfg {
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int STAGES = BN <= 64 ? 8 : BN <= 128 ? 6 : 4;
    static constexpr int TMEM_COLS = 2 * BN;  // two accumulator buffers (64/128/256/512 columns)
    static constexpr int SMEM = STAGES * STAGE + 1024 + 256;
};

template <int BN>
__host__ __device__ constexpr uint32_t idesc_bf16() {
    return idesc_bf16_mn<BM, BN>();
}

// The STORE value: the optional final logit softcap c tanh(v / c).
DEC_DEVINL float store_value(const GemmArgs& a, float v) {
    return a.softcap > 0.f ? a.softcap * tanhf(v / a.softcap) : v;
}

// Apply the epilogue EPI to the 16 values v[j] of (row, t0 + j). All lanes of the warp call
// it together (the SwiGLU pairing uses a shuffle). Every global load of a chunk is issued
// before any store, so the 16 accesses overlap instead of waiting on one another.
template <int EPI>
DEC_DEVINL void epilogue16_t(const GemmArgs& a, int row, int t0, const float (&v_in)[16]) {
    const bool row_ok = row < a.M;
    float v[16];
    const float rs = (a.rscale && row_ok) ? a.rscale[row] : 1.f;  // q8_row: the row's scale
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = v_in[j] * rs;
    if constexpr (EPI == GEMM_SWIGLU) {
        // rows 2i (gate) and 2i+1 (up) sit in adjacent lanes; the even lane finishes the
        // even tokens and the odd lane the odd ones, so every lane evaluates 8 SiLUs
        const bool odd = (threadIdx.x & 1) != 0;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
            const float own = odd ? v[2 * jj + 1] : v[2 * jj];
            const float other = __shfl_xor_sync(0xffffffffu, odd ? v[2 * jj] : v[2 * jj + 1], 1);
            const float g = odd ? other : own, u = odd ? own : other;
            const int t = t0 + 2 * jj + (odd ? 1 : 0);
            if (row_ok && t < a.N) {
                const float sg = silu_f(g);
                a.act[(size_t)t * a.ldact + (row >> 1)] = f2bf(sg * u);
            }
        }
    } else if constexpr (EPI == GEMM_RESID) {
        if (!row_ok) return;
        float* yr = a.y + (size_t)t0 * a.ldy + row;
        const size_t ld = a.ldy;
        float old[16];
        if (t0 + 16 <= a.N) {  // a whole chunk: no per-token test
#pragma unroll
            for (int j = 0; j < 16; ++j) old[j] = yr[j * ld];
#pragma unroll
            for (int j = 0; j < 16; ++j) yr[j * ld] = old[j] + v[j];
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) old[j] = t0 + j < a.N ? yr[j * ld] : 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (t0 + j < a.N) yr[j * ld] = old[j] + v[j];
        }
    } else {
        if (!row_ok) return;
        float* const y = a.y_ptr ? *a.y_ptr : a.y;  // null: only the greedy argmax is kept
        if (!y) return;
        const float bias = a.bias ? a.bias[row] : 0.f;
        float* yr = y + (size_t)t0 * a.ldy + row;
        const size_t ld = a.ldy;
        // the softcap test stays outside the loop: the plain path carries no tanh at all
        if (a.softcap > 0.f) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (t0 + j < a.N) yr[j * ld] = store_value(a, v[j] + bias);
        } else if (t0 + 16 <= a.N) {  // a whole chunk: no per-token test
#pragma unroll
            for (int j = 0; j < 16; ++j) yr[j * ld] = v[j] + bias;
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (t0 + j < a.N) yr[j * ld] = v[j] + bias;
        }
    }
}

// The same with the epilogue chosen at run time (the persistent stream-K kernel).
DEC_DEVINL void epilogue16(const GemmArgs& a, int row, int t0, const float (&v_in)[16]) {
    if (a.epi == GEMM_SWIGLU)
        epilogue16_t<GEMM_SWIGLU>(a, row, t0, v_in);
    else if (a.epi == GEMM_RESID)
        epilogue16_t<GEMM_RESID>(a, row, t0, v_in);
    else
        epilogue16_t<GEMM_STORE>(a, row, t0, v_in);
}

// Greedy argmax of the STORE epilogue: warp maximum of the packed (value, row) words of
// each token, one atomicMax per warp and token (token words 256 bytes apart).
DEC_DEVINL void argmax16(const GemmArgs& a, int row, int t0, const float (&v)[16]) {
    const int lane = threadIdx.x & 31;
    const float bias = (a.bias && row < a.M) ? a.bias[row] : 0.f;
    const float rs = (a.rscale && row < a.M) ? a.rscale[row] : 1.f;
    float o[16];
    if (a.softcap > 0.f) {
#pragma unroll
        for (int j = 0; j < 16; ++j) o[j] = store_value(a, v[j] * rs + bias);
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) o[j] = v[j] * rs + bias;
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        unsigned long long w = (row < a.M && t0 + j < a.N) ? argmax_pack(o[j], row) : 0ull;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const unsigned long long u = __shfl_xor_sync(0xffffffffu, w, o);
            w = u > w ? u : w;
        }
        if (lane == 0 && w) atomicMax(&a.amax[(size_t)(t0 + j) * 32], w);
    }
}

// ----------------------------------------------------------------- stream-K work split
//
// The (tile, 64-wide k block) units of the whole product, tile-major, are cut into
// gridDim.x equal contiguous ranges, one per persistent CTA. A CTA's range is a run of
// segments, one per tile it touches: whole tiles in the middle, and at its two ends
// pieces of tiles it shares with the neighbouring CTAs.
struct Work {
    long long U;  // stream-K units (the first tsk tiles x nkb)
    int nkb, tiles_n, bn, nc;
    int tsk;      // tiles split by stream-K (tiles [0, tsk))
    int dp;       // whole tiles per CTA after them, round-robin: CTA c takes tsk + c + j nc
};

// With several column tiles (N > BN) and at least two tiles per CTA, all but about one
// round of tiles go round-robin, so the CTAs working at the same time share weight blocks
// in L2; the rest (at least one tile per CTA, so no piece is shorter than a tile's worth of
// k blocks on average) is split by stream-K and processed first. With one column tile
// every tile is split by stream-K.
__host__ __device__ inline Work make_work(const GemmArgs& a, int bn, int nc) {
    Work w;
    w.nkb = (a.K + BK - 1) / BK;
    w.tiles_n = (a.N + bn - 1) / bn;
    w.bn = bn;
    w.nc = nc;
    const int T = ((a.M + BM - 1) / BM) * w.tiles_n;
    w.dp = (w.tiles_n > 1 && T >= 2 * w.nc) ? T / w.nc - 1 : 0;
    w.tsk = T - w.dp * w.nc;
    w.U = (long long)w.tsk * w.nkb;
    return w;
}

__host__ __device__ inline long long unit0(const Work& w, int c) { return w.U * c / w.nc; }
// CTA whose range holds stream-K unit u (w.U > 0).
__host__ __device__ inline int cta_of(const Work& w, long long u) { return (int)(((u + 1) * w.nc - 1) / w.U); }

struct Range {
    long long u0, u1;
    int c, tf, nsk, nseg, iters;  // nsk: stream-K segments, then w.dp whole tiles
};

__host__ __device__ inline Range cta_range(const Work& w, int c) {
    Range r;
    r.c = c;
    r.u0 = unit0(w, c);
    r.u1 = unit0(w, c + 1);
    r.tf = (int)(r.u0 / w.nkb);
    r.nsk = r.u1 > r.u0 ? (int)((r.u1 - 1) / w.nkb) - r.tf + 1 : 0;
    r.nseg = r.nsk + w.dp;
    r.iters = (int)(r.u1 - r.u0) + w.dp * w.nkb;
    return r;
}

struct Seg {
    int tile, kb0, kb1, slot;  // slot: 0 = first tile of the range, 1 = any later one
};

// The j-th segment in processing order: the head piece of the range's last tile first (a
// piece some later CTA finishes, so it is published as early as possible), then the
// first tile (this CTA holds its last k blocks and finishes it), then the middle tiles,
// then the round-robin whole tiles.
__host__ __device__ inline Seg segment(const Work& w, const Range& r, int j) {
    Seg s;
    if (j >= r.nsk) {
        s.tile = w.tsk + r.c + (j - r.nsk) * w.nc;
        s.kb0 = 0;
        s.kb1 = w.nkb;
        s.slot = 1;
        return s;
    }
    int i = j;
    if (r.nsk >= 2) i = j == 0 ? r.nsk - 1 : j - 1;
    s.tile = r.tf + i;
    const long long t0 = (long long)s.tile * w.nkb;
    s.kb0 = (int)((r.u0 > t0 ? r.u0 : t0) - t0);
    s.kb1 = (int)((r.u1 < t0 + w.nkb ? r.u1 : t0 + w.nkb) - t0);
    s.slot = i == 0 ? 0 : 1;
    return s;
}

// Workspace slot of CTA cc's piece of (stream-K) `tile`.
__host__ __device__ inline int piece_slot(const Work& w, int cc, int tile) { return (int)(unit0(w, cc) / w.nkb) == tile ? 0 : 1; }

// Walks the k blocks of a range in processing order (the producer's view).
struct SegIter {
    Work w;
    Range r;
    Seg s;
    int j, kb, m0, n0;
    DEC_DEVINL SegIter(const Work& w_, const Range& r_) : w(w_), r(r_), j(0) { load(); }
    DEC_DEVINL void load() {
        if (j >= r.nseg) return;
        s = segment(w, r, j);
        kb = s.kb0;
        m0 = s.tile / w.tiles_n * BM;
        n0 = s.tile % w.tiles_n * w.bn;
    }
    DEC_DEVINL void next() {
        if (++kb >= s.kb1) {
            ++j;
            load();
        }
    }
};

// Barrier of the eight epilogue warps only.
DEC_DEVINL void epi_bar8() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

DEC_DEVINL int ld_acquire_gpu(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Whether P pieces of a shared tile have been published (tile counter >= P), waiting for
// them (bounded: on time-out sets the error flag and returns false). Only the CTA that
// finishes the tile calls it, after its own piece's MMAs have completed.
DEC_DEVINL bool tile_ready(const GemmArgs& a, int tile, int P, volatile int* flag_s) {
    if (threadIdx.x == 0) {
        int r = 1;
        const long long st = clock64();
        const long long limit = a.wait_limit > 0 ? a.wait_limit : (1ll << 31);
        while (ld_acquire_gpu(&a.cnt[tile]) < P + a.wait_extra) {
            if (clock64() - st > limit) {
                atomicExch(a.err, 1);
                r = 0;
                break;
            }
        }
        *flag_s = r;
    }
    epi_bar8();
    const int r = *flag_s;
    epi_bar8();
    return r != 0;
}

template <int BN>
__global__ void __launch_bounds__(320, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   GemmArgs a) {
    using C = Cfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE);
    uint64_t* empty = full + C::STAGES;
    uint64_t* accf = empty + C::STAGES;  // [2] accumulator buffer ready for the epilogue
    uint64_t* acce = accf + 2;           // [2] accumulator buffer drained by the epilogue
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + 2);
    int* flag_s = reinterpret_cast<int*>(tmem_slot + 1);  // a wait for a tile's pieces timed out

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 4 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    const Work w = make_work(a, BN, gridDim.x);
    const int c = blockIdx.x;
    const Range rg = cta_range(w, c);

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accf[b], 1);
            mbar_init(&acce[b], 256);
        }
        fence_mbar_init();
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(C::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_trigger();

    if (warp == 4) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            // A weight block read by one column tile only streams through L2 (evict-first);
            // with several column tiles it is read again, so it keeps the normal policy.
            const uint64_t pol = policy_evict_first();
            const bool once = w.tiles_n == 1;
            auto load_a = [&](void* dst, int kb, int m0, uint64_t* bar) {
                if (once)
                    tma_load_2d_hint(dst, &tmA, kb * BK, m0, bar, pol);
                else
                    tma_load_2d(dst, &tmA, kb * BK, m0, bar);
            };
            const int total = rg.iters;
            const int pre = total < C::STAGES ? total : C::STAGES;
            // the weight slices of the first stages do not depend on the previous kernel
            SegIter it(w, rg);
            for (int i = 0; i < pre; ++i, it.next()) {
                mbar_arrive_expect_tx(&full[i], C::STAGE);
                load_a(smem + i * C::STAGE, it.kb, it.m0, &full[i]);
            }
            pdl_wait();
            SegIter jt(w, rg);
            for (int i = 0; i < pre; ++i, jt.next())
                tma_load_2d(smem + i * C::STAGE + C::A_BYTES, &tmB, jt.kb * BK, jt.n0, &full[i]);
            for (int i = pre; i < total; ++i, it.next()) {
                const int s = i % C::STAGES;
                const uint32_t u = (uint32_t)(i / C::STAGES);
                if (!mbar_wait_bounded(&empty[s], (u & 1u) ^ 1u, a.err)) break;
                mbar_arrive_expect_tx(&full[s], C::STAGE);
                load_a(smem + s * C::STAGE, it.kb, it.m0, &full[s]);
                tma_load_2d(smem + s * C::STAGE + C::A_BYTES, &tmB, it.kb * BK, it.n0, &full[s]);
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        pdl_wait();
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            constexpr uint32_t idesc = idesc_bf16<BN>();
            const uint32_t sbase = smem_u32(smem);
            int i = 0;
            bool ok = true;
            for (int j = 0; j < rg.nseg && ok; ++j) {
                const Seg sg = segment(w, rg, j);
                const int buf = j & 1;
                if (j >= 2 && !mbar_wait_bounded(&acce[buf], (uint32_t)(((j >> 1) - 1) & 1), a.err)) break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(buf * BN);
                for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++i) {
                    const int s = i % C::STAGES;
                    const uint32_t u = (uint32_t)(i / C::STAGES);
                    if (!mbar_wait_bounded(&full[s], u & 1u, a.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t abase = sbase + s * C::STAGE, bbase = abase + C::A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        tc_mma(d, sdesc_sw128(abase + kk * 32), sdesc_sw128(bbase + kk * 32), idesc,
                               (kb > sg.kb0 || kk > 0) ? 1u : 0u);
                    tc_commit(&empty[s]);
                }
                tc_commit(&accf[buf]);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------ epilogue (warps 0-3 and 6-9): warp w reads
        // TMEM lanes 32 (w % 4) .. (rows), warps 0-3 the first half of the columns, 6-9 the
        // second (one warp a scheduler left the last tile's SwiGLU epilogue latency-bound)
        pdl_wait();
        const int q4 = warp & 3;
        constexpr int HC = BN / 2;  // columns of each half
        const int cb = warp >= 6 ? HC : 0;
        const int rloc = q4 * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        // ok turns false when a wait for a shared tile's pieces runs out: the remaining
        // accumulators are still drained (every MMA completes and every TMA load is consumed
        // before TMEM is freed), only their outputs are skipped
        bool ok = true;
        for (int j = 0; j < rg.nseg; ++j) {
            const Seg sg = segment(w, rg, j);
            const int buf = j & 1;
            if (!mbar_wait_bounded(&accf[buf], (uint32_t)((j >> 1) & 1), a.err)) break;
            tc_fence_after();
            const uint32_t acc = tmem + lane_off + (uint32_t)(buf * BN);
            const bool whole = sg.kb0 == 0 && sg.kb1 == w.nkb;
            // A shared tile is finished by the CTA holding its last k blocks. The other pieces
            // are the first segment their CTAs process (segment() order), so they are
            // published early and nobody waits for the finisher.
            const bool fin = !whole && sg.kb1 == w.nkb;
            if (fin && ok) ok = tile_ready(a, sg.tile, c - cta_of(w, (long long)sg.tile * w.nkb), flag_s);
            if ((whole || fin) && ok) {
                int c_lo = c, slot_lo = 0;
                if (fin) {
                    c_lo = cta_of(w, (long long)sg.tile * w.nkb);
                    slot_lo = piece_slot(w, c_lo, sg.tile);
                }
                const int row = sg.tile / w.tiles_n * BM + rloc, n0 = sg.tile % w.tiles_n * BN;
                for (int c0 = cb; c0 < cb + HC; c0 += 16) {
                    uint32_t r[16];
                    tmem_ld16_issue(acc + (uint32_t)c0, r);
                    // the published pieces ([column][row] fp32) in k order, then this CTA's
                    float v[16];
#pragma unroll
                    for (int q = 0; q < 16; ++q) v[q] = 0.f;
                    for (int cc = c_lo; cc < c; ++cc) {
                        const float* pc =
                            a.ws + ((size_t)cc * 2 + (cc == c_lo ? slot_lo : 0)) * (BM * BN) + (size_t)c0 * BM + rloc;
#pragma unroll
                        for (int q = 0; q < 16; ++q) v[q] += __ldcg(pc + (size_t)q * BM);
                    }
                    tmem_ld_wait16(r);
                    if (fin) {
#pragma unroll
                        for (int q = 0; q < 16; ++q) v[q] += __uint_as_float(r[q]);
                    } else {
#pragma unroll
                        for (int q = 0; q < 16; ++q) v[q] = __uint_as_float(r[q]);
                    }
                    epilogue16(a, row, n0 + c0, v);
                    if (a.amax && a.epi == GEMM_STORE) argmax16(a, row, n0 + c0, v);
                }
            } else if (!whole && !fin) {
                // publish this piece ([column][row] fp32, coalesced) and free the accumulator
                float* mine = a.ws + ((size_t)c * 2 + sg.slot) * (BM * BN);
                for (int c0 = cb; c0 < cb + HC; c0 += 16) {
                    uint32_t r[16];
                    tmem_ld16_issue(acc + (uint32_t)c0, r);
                    tmem_ld_wait16(r);
#pragma unroll
                    for (int q = 0; q < 16; ++q) __stcg(mine + (size_t)(c0 + q) * BM + rloc, __uint_as_float(r[q]));
                }
                __threadfence();
            }
            tc_fence_before();
            mbar_arrive(&acce[buf]);
            if (!whole) {
                epi_bar8();
                if (threadIdx.x == 0) {
                    if (!fin)
                        atomicAdd(&a.cnt[sg.tile], 1);
                    else if (ok)
                        atomicExch(&a.cnt[sg.tile], 0);  // every piece is read: ready for the next launch
                    // (after a wait that ran out the host zeroes the counters)
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS)
                     : "memory");
    }
}

// ----------------------------------------------------------------- cluster split-K
//
// Products with one column tile (N <= 128: prefill chunks, decode batches) and few 128-row
// tiles (the QKV, o_proj and down projections) split each tile's k blocks over the S <= 8
// CTAs of one thread-block cluster. Every CTA streams 1/S of the tile's weights into its
// own TMEM accumulator. The partial tiles are then summed inside the cluster: once every CTA
// of the cluster is past its MMAs (one cluster barrier: every operand ring is drained), each
// CTA reads its accumulator rows and sends every 32-row-aligned slice to the CTA that owns
// it, straight from registers (st.async, completing as transaction bytes on the owner's
// mbarrier; its own slice it keeps). The owner sums the S partials of its rows in rank
// order (deterministic) and applies the epilogue. There is no global round trip, no wait
// on CTAs outside the cluster, and no second cluster barrier: no CTA reads another's
// shared memory. (Staging every partial and copying slices with the DMA engine, which
// reads the sender's shared memory and so needs a last barrier before anyone leaves, took
// 0.2-0.4 us longer a launch.)
//
// Shared memory after the main loop (it overlays the drained operand ring):
// [recv: S slots x rows per owner x LDR floats], LDR = BN + 4.

constexpr int kMaxSplitK = 8;

// Rows of the tile each owner CTA finishes: a multiple of 32 (one warp's lanes).
__host__ __device__ constexpr int splitk_rows(int S) { return 32 * ((4 + S - 1) / S); }

template <int BN>
__host__ __device__ constexpr size_t splitk_recv_bytes(int S) {
    return (size_t)S * splitk_rows(S) * (BN + 4) * 4;
}

// The largest receive area over every S <= kMaxSplitK (every split's partial of the rows a
// CTA finishes, its own included).
template <int BN>
__host__ __device__ constexpr size_t splitk_exchange_bytes() {
    size_t m = 0;
    for (int S = 2; S <= kMaxSplitK; ++S) m = splitk_recv_bytes<BN>(S) > m ? splitk_recv_bytes<BN>(S) : m;
    return m;
}

template <int BN>
__host__ __device__ constexpr size_t splitk_body_bytes() {
    return (size_t)Cfg<BN>::STAGES * Cfg<BN>::STAGE > splitk_exchange_bytes<BN>()
               ? (size_t)Cfg<BN>::STAGES * Cfg<BN>::STAGE
               : splitk_exchange_bytes<BN>();
}

template <int BN>
__host__ __device__ constexpr int splitk_smem() {
    return (int)splitk_body_bytes<BN>() + 1024 + 256;
}

template <int BN, int EPI>
__global__ void __launch_bounds__(320, 1)
    gemm_splitk_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmArgs a,
                       int S) {
    using C = Cfg<BN>;
    constexpr int LDR = BN + 4;  // receive rows padded by 16 bytes: conflict-free 16-byte stores
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + splitk_body_bytes<BN>());
    uint64_t* empty = full + C::STAGES;
    uint64_t* accf = empty + C::STAGES;  // the accumulator is complete
    uint64_t* recvb = accf + 1;          // the other CTAs' slices of this CTA's rows have landed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(recvb + 1);
    float* recv = reinterpret_cast<float*>(smem);  // [S][rows per owner][LDR], over the drained ring

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (int)cluster_rank();
    const int tile = blockIdx.x / S;
    const int m0 = tile * BM;
    const int nkb = (a.K + BK - 1) / BK;
    const int kb0 = (int)((long long)nkb * rank / S), kb1 = (int)((long long)nkb * (rank + 1) / S);
    const int iters = kb1 - kb0;
    if (warp == 4 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }

    const int RS = splitk_rows(S);
    const int my0 = rank * RS, my1 = min(BM, my0 + RS);  // the rows this CTA finishes
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        mbar_init(recvb, 1);
        // the S - 1 other CTAs each send (my1 - my0) rows of BN floats; armed before the
        // cluster barrier, so no byte can arrive before the count
        if (my1 > my0) mbar_arrive_expect_tx(recvb, (uint32_t)(S - 1) * (my1 - my0) * BN * 4);
        fence_mbar_init();
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(BN)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_trigger();

    if (warp == 4) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer (each weight block
            // is read once: evict-first)
            const uint64_t pol = policy_evict_first();
            const int pre = iters < C::STAGES ? iters : C::STAGES;
            for (int i = 0; i < pre; ++i) {  // weights do not depend on the previous kernel
                mbar_arrive_expect_tx(&full[i], C::STAGE);
                tma_load_2d_hint(smem + i * C::STAGE, &tmA, (kb0 + i) * BK, m0, &full[i], pol);
            }
            pdl_wait();
            for (int i = 0; i < pre; ++i) tma_load_2d(smem + i * C::STAGE + C::A_BYTES, &tmB, (kb0 + i) * BK, 0, &full[i]);
            for (int i = pre; i < iters; ++i) {
                const int s = i % C::STAGES;
                const uint32_t u = (uint32_t)(i / C::STAGES);
                if (!mbar_wait_bounded(&empty[s], (u & 1u) ^ 1u, a.err)) break;
                mbar_arrive_expect_tx(&full[s], C::STAGE);
                tma_load_2d_hint(smem + s * C::STAGE, &tmA, (kb0 + i) * BK, m0, &full[s], pol);
                tma_load_2d(smem + s * C::STAGE + C::A_BYTES, &tmB, (kb0 + i) * BK, 0, &full[s]);
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        pdl_wait();
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            constexpr uint32_t idesc = idesc_bf16<BN>();
            const uint32_t sbase = smem_u32(smem);
            for (int i = 0; i < iters; ++i) {
                const int s = i % C::STAGES;
                const uint32_t u = (uint32_t)(i / C::STAGES);
                if (!mbar_wait_bounded(&full[s], u & 1u, a.err)) break;
                tc_fence_after();
                const uint32_t abase = sbase + s * C::STAGE, bbase = abase + C::A_BYTES;
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)
                    tc_mma(tmem, sdesc_sw128(abase + kk * 32), sdesc_sw128(bbase + kk * 32), idesc,
                           (i > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&empty[s]);
            }
            tc_commit(accf);
        }
        __syncwarp();
    } else {
        pdl_wait();
        mbar_wait_bounded(accf, 0, a.err);  // on a time-out the partial is garbage, the flag is set
        tc_fence_after();
    }
    // every CTA of the cluster is past its MMAs: every ring is drained, free to receive
    cluster_sync();
    // epilogue warps 0-3 and 6-9: warp w reads TMEM lanes 32 (w % 4).. (rows), warps 0-3
    // one half of the columns, 6-9 the other
    const bool epi = warp < 4 || warp >= 6;
    const int ew = warp < 4 ? warp : warp - 2;  // 0..7
    if (epi) {
        // my partial of each row into slot [rank] of the row's owner: kept here for my own
        // rows, st.async from registers (transaction bytes on the owner's recvb) for the
        // others, so no copy reads this CTA's shared memory once it moves on
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;  // = TMEM lane
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        const int cb = warp >= 6 ? BN / 2 : 0;
        const int o = row / RS, lr = row - o * RS;  // owner and row within its slice
        float* slot = recv + ((size_t)rank * RS + lr) * LDR;
        const uint32_t rdst = o == rank ? 0u : dsmem_map(smem_u32(slot), o);
        const uint32_t rbar = o == rank ? 0u : dsmem_map(smem_u32(recvb), o);
        for (int c0 = cb; c0 < cb + BN / 2; c0 += 16) {
            uint32_t r[16];
            if (iters > 0) {
                tmem_ld16_issue(tmem + lane_off + (uint32_t)c0, r);
                tmem_ld_wait16(r);
            } else {
#pragma unroll
                for (int q = 0; q < 16; ++q) r[q] = 0u;
            }
            if (o == rank) {
#pragma unroll
                for (int q = 0; q < 16; q += 4)
                    *reinterpret_cast<uint4*>(slot + c0 + q) = make_uint4(r[q], r[q + 1], r[q + 2], r[q + 3]);
            } else {
#pragma unroll
                for (int q = 0; q < 16; q += 4)
                    st_async_4f(rdst + (uint32_t)(c0 + q) * 4, __uint_as_float(r[q]), __uint_as_float(r[q + 1]),
                                __uint_as_float(r[q + 2]), __uint_as_float(r[q + 3]), rbar);
            }
        }
        epi_bar8();  // my own slot is written
    }

    if (epi && my1 > my0) {
        // the owner sums its rows' partials in rank order and applies the epilogue:
        // units of (32 rows, 16 columns), lane = row
        const bool got = mbar_wait_cluster_bounded(recvb, 0, a.err);
        const int groups = (my1 - my0) / 32;
        for (int u = ew; got && u < groups * (BN / 16); u += 8) {
            const int gi = u / (BN / 16), c0 = (u % (BN / 16)) * 16;
            const int lr = gi * 32 + lane;
            float acc[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) acc[q] = 0.f;
            for (int z = 0; z < S; ++z) {
                const float4* src = reinterpret_cast<const float4*>(recv + ((size_t)z * RS + lr) * LDR + c0);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 v = src[q];
                    acc[4 * q] += v.x;
                    acc[4 * q + 1] += v.y;
                    acc[4 * q + 2] += v.z;
                    acc[4 * q + 3] += v.w;
                }
            }
            const int row = m0 + my0 + lr;
            epilogue16_t<EPI>(a, row, c0, acc);
            if constexpr (EPI == GEMM_STORE) {
                if (a.amax) argmax16(a, row, c0, acc);
            }
        }
    }
    // nothing reads another CTA's shared memory, and every CTA's incoming bytes completed
    // before it got here: no cluster barrier before leaving
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(BN) : "memory");
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

cudaError_t encode_2d(CUtensorMap* tm, const uint16_t* base, int rows, int K, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int BN>
cudaError_t launch_bn(const GemmPlan& p, const GemmArgs& a, cudaStream_t st, bool pdl) {
    using C = Cfg<BN>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(gemm_tc_kernel<BN>), C::SMEM);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.nc);
    cfg.blockDim = dim3(320);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BN>, p.tmA, p.tmB, a);
}

template <int BN, int EPI>
cudaError_t launch_splitk(const GemmPlan& p, const GemmArgs& a, cudaStream_t st, bool pdl) {
    const int smem = splitk_smem<BN>();
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(gemm_splitk_kernel<BN, EPI>), smem);
    if (e != cudaSuccess) return e;
    const int tiles = (p.M + BM - 1) / BM;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(tiles * p.splitk);
    cfg.blockDim = dim3(320);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    attr[na].id = cudaLaunchAttributeClusterDimension;  // the S splits of a tile: one cluster
    attr[na].val.clusterDim.x = p.splitk;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, gemm_splitk_kernel<BN, EPI>, p.tmA, p.tmB, a, p.splitk);
}

template <int EPI>
cudaError_t launch_splitk_bn(const GemmPlan& p, const GemmArgs& a, cudaStream_t st, bool pdl) {
    switch (p.bn) {
        case 32: return launch_splitk<32, EPI>(p, a, st, pdl);
        case 64: return launch_splitk<64, EPI>(p, a, st, pdl);
        case 128: return launch_splitk<128, EPI>(p, a, st, pdl);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t tmap_bf16_sw128(CUtensorMap* tm, const void* base, int rank, const uint64_t* dims,
                            const uint64_t* strides, const uint32_t* box) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || rank < 1 || rank > 5) return cudaErrorNotSupported;
    cuuint64_t d[5], st[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        bx[i] = box[i];
        es[i] = 1;
        if (i + 1 < rank) st[i] = strides[i];
    }
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), d, st, bx, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Row-major bf16 [rows][K] read in 128B-swizzled boxes of 64 columns x box_rows rows.
cudaError_t tmap_bf16_rows(CUtensorMap* tm, const uint16_t* base, int rows, int K, int box_rows) {
    return encode_2d(tm, base, rows, K, box_rows);
}

// Column tile: the whole batch up to 128 tokens; 256 beyond (more work per operand byte
// once the product is compute-bound).
int gemm_bn(int N) { return N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : 256; }

namespace {
// How many clusters of S CTAs of gemm_splitk_kernel<BN> the device holds at once (GPCs hold
// whole clusters, so this can be below SMs / S). Cached per device, column tile and S.
template <int BN>
int splitk_resident(int S) {
    static std::mutex mu;
    static std::map<std::pair<int, int>, int> known;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    auto it = known.find(std::make_pair(dev, S));
    if (it != known.end()) return it->second;
    int n = 0;
    if (ensure_smem(reinterpret_cast<const void*>(gemm_splitk_kernel<BN, GEMM_STORE>), splitk_smem<BN>()) ==
        cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(S * 8);
        cfg.blockDim = dim3(320);
        cfg.dynamicSmemBytes = splitk_smem<BN>();
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = S;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, gemm_splitk_kernel<BN, GEMM_STORE>, &cfg) != cudaSuccess) {
            n = 0;               // the stream-K kernel runs instead
            cudaGetLastError();  // and the refused query leaves no error behind
        }
    }
    known[std::make_pair(dev, S)] = n;
    return n;
}

template <int BN>
int splitk_pick(int tiles, int nkb, int num_sms) {
    int S = num_sms / tiles;
    if (S > kMaxSplitK) S = kMaxSplitK;
    if (S > nkb / 4) S = nkb / 4;
    for (; S >= 2; --S) {
        if (tiles * S * 2 < num_sms) return 0;  // the clusters would leave most SMs idle
        if (splitk_resident<BN>(S) >= tiles) return S;  // one wave: every cluster resident at once
    }
    return 0;
}
}  // namespace

// Cluster split-K for one column tile (N <= 128) when the 128-row tiles are too few to
// fill the SMs: the largest S <= min(8, SMs / tiles, k blocks / 4) CTAs per tile whose
// clusters are all resident at once and still cover at least half of the SMs; 0 = use the
// persistent stream-K kernel.
int gemm_splitk(int M, int N, int K, int num_sms) {
    if (N > 128) return 0;
    const int tiles = (M + BM - 1) / BM;
    const int nkb = (K + BK - 1) / BK;
    switch (gemm_bn(N)) {
        case 32: return splitk_pick<32>(tiles, nkb, num_sms);
        case 64: return splitk_pick<64>(tiles, nkb, num_sms);
        default: return splitk_pick<128>(tiles, nkb, num_sms);
    }
}

// One persistent CTA per SM, each with at least 8 k blocks of work.
int gemm_ctas(int M, int N, int K, int num_sms) {
    const int bn = gemm_bn(N);
    const long long units = (long long)((M + BM - 1) / BM) * ((N + bn - 1) / bn) * ((K + BK - 1) / BK);
    long long nc = units / 8;
    if (nc > num_sms) nc = num_sms;
    if (nc < 1) nc = 1;
    return (int)nc;
}

// Host-side check of the persistent kernel's work split for an M x N x K product over
// `nc` CTAs (the plan the kernel derives from its grid): every (tile, k block) unit is
// covered exactly once; every piece that another CTA finishes is the first segment its
// CTA processes (so it is published before that CTA waits on anything, which is what
// keeps the finishers' waits free of cycles); every tile split between CTAs has exactly
// one finisher, the CTA holding its last k blocks, whose expected pieces are the other
// CTAs' segments of the tile in the slots it reads. Returns the number of violations.
int gemm_streamk_check(int M, int N, int K, int nc) {
    if (M <= 0 || N <= 0 || K <= 0 || nc <= 0) return -1;
    GemmArgs a{};
    a.M = M;
    a.N = N;
    a.K = K;
    const Work w = make_work(a, gemm_bn(N), nc);
    const int T = ((M + BM - 1) / BM) * w.tiles_n;
    std::vector<int> cover((size_t)T * w.nkb, 0), fins(T, 0), pieces(T, 0);
    int bad = 0;
    for (int c = 0; c < nc; ++c) {
        const Range r = cta_range(w, c);
        for (int j = 0; j < r.nseg; ++j) {
            const Seg sg = segment(w, r, j);
            if (sg.tile < 0 || sg.tile >= T || sg.kb0 < 0 || sg.kb1 > w.nkb || sg.kb0 >= sg.kb1) {
                ++bad;
                continue;
            }
            for (int kb = sg.kb0; kb < sg.kb1; ++kb) ++cover[(size_t)sg.tile * w.nkb + kb];
            const bool whole = sg.kb0 == 0 && sg.kb1 == w.nkb, fin = !whole && sg.kb1 == w.nkb;
            if (!whole && !fin) {
                ++pieces[sg.tile];
                if (j != 0) ++bad;                                // published late
                if (sg.slot != piece_slot(w, c, sg.tile)) ++bad;  // not where the finisher reads
            }
            if (fin) {
                ++fins[sg.tile];
                if (c - cta_of(w, (long long)sg.tile * w.nkb) < 1) ++bad;  // nothing to wait for
            }
        }
    }
    for (size_t u = 0; u < cover.size(); ++u) bad += cover[u] != 1;
    for (int t = 0; t < T; ++t) {
        if (t >= w.tsk) {  // round-robin whole tiles
            bad += fins[t] != 0 || pieces[t] != 0;
            continue;
        }
        const long long t0 = (long long)t * w.nkb;
        const int P = cta_of(w, t0 + w.nkb - 1) - cta_of(w, t0) + 1;
        if (P == 1)
            bad += fins[t] != 0 || pieces[t] != 0;
        else
            bad += fins[t] != 1 || pieces[t] != P - 1;
    }
    return bad;
}

size_t gemm_ws_floats(int num_sms) { return (size_t)2 * num_sms * BM * 256; }

int gemm_cnt_needed(int M, int N) { return ((M + BM - 1) / BM) * ((N + 31) / 32); }

cudaError_t gemm_plan(GemmPlan* p, const uint16_t* A, int M, int K, const uint16_t* B, int N, int num_sms,
                      const float* ws) {
    if (M <= 0 || N <= 0 || K <= 0 || K % 8 != 0 || !ws) return cudaErrorInvalidValue;
    p->M = M;
    p->N = N;
    p->K = K;
    p->bn = gemm_bn(N);
    p->nc = gemm_ctas(M, N, K, num_sms);
    p->splitk = gemm_splitk(M, N, K, num_sms);
    p->ws = ws;
    cudaError_t e = encode_2d(&p->tmA, A, M, K, BM);
    if (e != cudaSuccess) return e;
    return encode_2d(&p->tmB, B, N, K, p->bn);
}

namespace {
int g_test_extra = 0;
long long g_test_limit = 0;
}  // namespace

void gemm_set_test_wait(int extra_pieces, long long limit_cycles) {
    g_test_extra = extra_pieces > 0 ? extra_pieces : 0;
    g_test_limit = limit_cycles > 0 ? limit_cycles : 0;
}

cudaError_t gemm_launch(const GemmPlan& p, GemmArgs a, cudaStream_t st, bool pdl) {
    a.wait_extra = g_test_extra;
    a.wait_limit = g_test_limit;
    a.M = p.M;
    a.N = p.N;
    a.K = p.K;
    a.ws = const_cast<float*>(p.ws);
    if (p.splitk >= 2) {
        switch (a.epi) {
            case GEMM_STORE: return launch_splitk_bn<GEMM_STORE>(p, a, st, pdl);
            case GEMM_RESID: return launch_splitk_bn<GEMM_RESID>(p, a, st, pdl);
            case GEMM_SWIGLU: return launch_splitk_bn<GEMM_SWIGLU>(p, a, st, pdl);
            default: return cudaErrorInvalidValue;
        }
    }
    if (!a.cnt) return cudaErrorInvalidValue;
    switch (p.bn) {
        case 32: return launch_bn<32>(p, a, st, pdl);
        case 64: return launch_bn<64>(p, a, st, pdl);
        case 128: return launch_bn<128>(p, a, st, pdl);
        case 256: return launch_bn<256>(p, a, st, pdl);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace dec
