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
//  * one 128 x BN output tile per CTA (BN = 32/64/128 tokens), split over K when
//    the tile count would leave SMs idle; split partials are summed in split order
//    by the last CTA of the tile (deterministic, no atomics on data);
//  * warp 0 / lane 0 drives TMA: 128B-swizzled 64-wide K slices of A and B into a
//    6-8 stage shared-memory ring (mbarrier complete_tx); the weight slices of
//    the first stages are issued before griddepcontrol.wait (they do not depend
//    on the previous kernel), the activation slices after it;
//  * warp 1 / lane 0 issues tcgen05.mma.cta_group::1.kind::f16 (M=128, N=BN,
//    K=16 per instruction, fp32 accumulator in TMEM) and frees each stage with
//    tcgen05.commit;
//  * all 4 warps read the accumulator with tcgen05.ld (warp w owns TMEM lanes
//    32w..32w+31 = weight rows) and apply the epilogue: store (+bias), residual
//    add, or SwiGLU on interleaved gate/up rows (bf16 silu(g)*u).
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"

namespace dec {

namespace {

constexpr int BM = 128, BK = 64;

template <int BN>
struct Cfg {
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int STAGES = BN <= 64 ? 8 : 6;
    static constexpr int TMEM_COLS = BN < 32 ? 32 : BN;
    static constexpr int SMEM = STAGES * STAGE + 1024 + 256;
};

DEC_DEVINL uint64_t sdesc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);  // start address
    d |= (uint64_t)1 << 16;                    // leading byte offset (16 B; unused for swizzled K-major)
    d |= (uint64_t)(1024 >> 4) << 32;          // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1 << 46;                    // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;                    // 128-byte swizzle
    return d;
}

template <int BN>
__host__ __device__ constexpr uint32_t idesc_bf16() {
    return (1u << 4)                      // accumulator F32
           | (1u << 7)                    // A BF16
           | (1u << 10)                   // B BF16
           | ((uint32_t)(BN >> 3) << 17)  // N
           | ((uint32_t)(BM >> 4) << 24); // M
}

DEC_DEVINL void tma_load_2d(void* dst, const CUtensorMap* tm, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

DEC_DEVINL void tma_load_2d_hint(void* dst, const CUtensorMap* tm, int x, int y, uint64_t* bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, "
        "{%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}

DEC_DEVINL void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
DEC_DEVINL void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

DEC_DEVINL void tc_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accum) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
}

DEC_DEVINL void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

DEC_DEVINL void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// tcgen05.ld of 16 columns without waiting; the values are valid after tmem_ld_wait32.
DEC_DEVINL void tmem_ld16_issue(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// Wait for outstanding tcgen05.ld; the registers are in-out operands so no use of them can
// be scheduled before the wait.
DEC_DEVINL void tmem_ld_wait32(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                   "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                   "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}


// Apply the epilogue to the 16 values v[j] of (row, t0 + j). All lanes of the warp call
// it together (the SwiGLU pairing uses a shuffle). Every global load of a chunk is issued
// before any store, so the 16 accesses overlap instead of waiting on one another.
DEC_DEVINL void epilogue16(const GemmArgs& a, int row, int t0, const float (&v)[16]) {
    const bool row_ok = row < a.M;
    if (a.epi == GEMM_SWIGLU) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float partner = __shfl_xor_sync(0xffffffffu, v[j], 1);
            if (row_ok && (row & 1) == 0 && t0 + j < a.N) {
                const float sg = v[j] * (1.0f / (1.0f + expf(-v[j])));
                a.act[(size_t)(t0 + j) * a.ldact + (row >> 1)] = f2bf(sg * partner);
            }
        }
        return;
    }
    if (!row_ok) return;
    if (a.epi == GEMM_RESID) {
        float old[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) old[j] = t0 + j < a.N ? a.y[(size_t)(t0 + j) * a.ldy + row] : 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (t0 + j < a.N) a.y[(size_t)(t0 + j) * a.ldy + row] = old[j] + v[j];
    } else {
        const float bias = a.bias ? a.bias[row] : 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (t0 + j < a.N) a.y[(size_t)(t0 + j) * a.ldy + row] = v[j] + bias;
    }
}

// Greedy argmax of the STORE epilogue: warp maximum of the packed (value, row) words of
// each token, one atomicMax per warp and token (token words 256 bytes apart).
DEC_DEVINL void argmax16(const GemmArgs& a, int row, int t0, const float (&v)[16]) {
    const int lane = threadIdx.x & 31;
    const float bias = (a.bias && row < a.M) ? a.bias[row] : 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        unsigned long long w = (row < a.M && t0 + j < a.N) ? argmax_pack(v[j] + bias, row) : 0ull;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const unsigned long long u = __shfl_xor_sync(0xffffffffu, w, o);
            w = u > w ? u : w;
        }
        if (lane == 0 && w) atomicMax(&a.amax[(size_t)(t0 + j) * 32], w);
    }
}

template <int BN>
__global__ void __launch_bounds__(128, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmArgs a) {
    using C = Cfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE);
    uint64_t* empty = full + C::STAGES;
    uint64_t* accb = empty + C::STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accb + 1);
    int* ticket = reinterpret_cast<int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN, z = blockIdx.z;
    const int nkb = (a.K + BK - 1) / BK;
    const int kb0 = (int)((int64_t)z * nkb / a.splits), kb1 = (int)((int64_t)(z + 1) * nkb / a.splits);
    const int nk = kb1 - kb0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accb, 1);
        fence_mbar_init();
    }
    if (warp == 2) {
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

    bool ok = true;
    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer
        const uint64_t pol = policy_evict_first();
        const int pre = nk < C::STAGES ? nk : C::STAGES;
        for (int i = 0; i < pre; ++i) {
            mbar_arrive_expect_tx(&full[i], C::STAGE);
            tma_load_2d_hint(smem + i * C::STAGE, &tmA, (kb0 + i) * BK, m0, &full[i], pol);
        }
        pdl_wait();
        for (int i = 0; i < pre; ++i) tma_load_2d(smem + i * C::STAGE + C::A_BYTES, &tmB, (kb0 + i) * BK, n0, &full[i]);
        for (int i = pre; i < nk; ++i) {
            const int s = i % C::STAGES;
            const uint32_t u = (uint32_t)(i / C::STAGES);
            if (!mbar_wait_bounded(&empty[s], (u & 1u) ^ 1u, a.err)) break;
            mbar_arrive_expect_tx(&full[s], C::STAGE);
            tma_load_2d_hint(smem + s * C::STAGE, &tmA, (kb0 + i) * BK, m0, &full[s], pol);
            tma_load_2d(smem + s * C::STAGE + C::A_BYTES, &tmB, (kb0 + i) * BK, n0, &full[s]);
        }
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = idesc_bf16<BN>();
        const uint32_t sbase = smem_u32(smem);
        for (int i = 0; i < nk; ++i) {
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
                tc_mma(tmem, sdesc_sw128(abase + kk * 32), sdesc_sw128(bbase + kk * 32), idesc,
                       (i > 0 || kk > 0) ? 1u : 0u);
            tc_commit(&empty[s]);
        }
        tc_commit(accb);
    }
    if (warp != 0) pdl_wait();  // every thread passes the grid dependency before finishing

    // ---------------------------------------------------- epilogue
    __syncwarp();
    const bool acc_ready = mbar_wait_bounded(accb, 0, a.err);
    tc_fence_after();
    const int rloc = warp * 32 + lane;
    const int row = m0 + rloc;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    // Split-K: the a.splits CTAs of this tile form one cluster. CTA r owns rows
    // [r*rp, r*rp + rp) of the tile; every CTA pushes its partial of those rows into the
    // owner's receive buffer (drained stage ring, [split][row][BN + 4] fp32, vector stores
    // to distributed shared memory, no waiting), then after one cluster barrier each owner
    // sums its rows over the splits in split order from local shared memory (deterministic).
    const int S = a.splits;
    const int rp = (((BM + S - 1) / S) + 1) & ~1;  // even, so SwiGLU pairs stay in one slice
    constexpr int LDR = BN + 4;                    // padded row: conflict-free vector access
    const uint32_t recv = smem_u32(smem);
    const int owner = rloc / rp, lr = rloc - owner * rp;
    if (S > 1) cluster_sync();  // every CTA's stage ring is drained before any partial lands in it
    for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld16_issue(lane_base + (uint32_t)c0, r);
        tmem_ld16_issue(lane_base + (uint32_t)c0 + 16, r + 16);
        tmem_ld_wait32(r);
        if (!acc_ready) continue;
        if (S == 1) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float v[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[16 * h + j]);
                epilogue16(a, row, n0 + c0 + 16 * h, v);
                if (a.amax && a.epi == GEMM_STORE) argmax16(a, row, n0 + c0 + 16 * h, v);
            }
        } else {
            const uint32_t dst = recv + (uint32_t)(((z * rp + lr) * LDR + c0) * 4);
#pragma unroll
            for (int q = 0; q < 8; ++q) dsmem_st4(dst + q * 16, owner, r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS)
                     : "memory");
    }
    (void)ok;
    (void)ticket;
    if (S == 1) return;

    cluster_sync();  // all partials have arrived; from here on only local shared memory is read
    const int r_lo = min(BM, z * rp), nr = min(BM, r_lo + rp) - r_lo;
    const float* rb = reinterpret_cast<const float*>(smem);
    if (!acc_ready || nr <= 0) return;
    if (a.epi == GEMM_SWIGLU) {
        const int np = nr / 2;
        for (int i = threadIdx.x; i < np * (BN / 4); i += 128) {
            const int lp = 2 * (i % np), c4 = 4 * (i / np);
            float4 g = make_float4(0.f, 0.f, 0.f, 0.f), u = g;
            for (int s2 = 0; s2 < S; ++s2) {
                const float4 pg = *reinterpret_cast<const float4*>(rb + (s2 * rp + lp) * LDR + c4);
                const float4 pu = *reinterpret_cast<const float4*>(rb + (s2 * rp + lp + 1) * LDR + c4);
                g.x += pg.x, g.y += pg.y, g.z += pg.z, g.w += pg.w;
                u.x += pu.x, u.y += pu.y, u.z += pu.z, u.w += pu.w;
            }
            const int grow = m0 + r_lo + lp;
            if (grow >= a.M) continue;
            const float gv[4] = {g.x, g.y, g.z, g.w}, uv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int t = n0 + c4 + q;
                if (t >= a.N) continue;
                const float sg = gv[q] * (1.0f / (1.0f + expf(-gv[q])));
                a.act[(size_t)t * a.ldact + (grow >> 1)] = f2bf(sg * uv[q]);
            }
        }
    } else {
        for (int i = threadIdx.x; i < nr * (BN / 4); i += 128) {
            const int l = i % nr, c4 = 4 * (i / nr);
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int s2 = 0; s2 < S; ++s2) {
                const float4 p = *reinterpret_cast<const float4*>(rb + (s2 * rp + l) * LDR + c4);
                v.x += p.x, v.y += p.y, v.z += p.z, v.w += p.w;
            }
            const int grow = m0 + r_lo + l;
            if (grow >= a.M) continue;
            const float vv[4] = {v.x, v.y, v.z, v.w};
            const float bias = (a.epi == GEMM_STORE && a.bias) ? a.bias[grow] : 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int t = n0 + c4 + q;
                if (t >= a.N) continue;
                float* dst = a.y + (size_t)t * a.ldy + grow;
                if (a.epi == GEMM_RESID) {
                    *dst += vv[q];
                } else {
                    *dst = vv[q] + bias;
                    if (a.amax) atomicMax(&a.amax[(size_t)t * 32], argmax_pack(vv[q] + bias, grow));
                }
            }
        }
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
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((p.M + BM - 1) / BM, (p.N + BN - 1) / BN, p.splits);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (p.splits > 1) {  // the split CTAs of a tile form one cluster (reduction through DSMEM)
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = 1;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = p.splits;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BN>, p.tmA, p.tmB, a);
}

}  // namespace

int gemm_tiles(const GemmPlan& p) { return ((p.M + BM - 1) / BM) * ((p.N + p.bn - 1) / p.bn); }

int gemm_choose_splits(int M, int N, int K, int num_sms, int* bn_out) {
    const int bn = N <= 32 ? 32 : N <= 64 ? 64 : 128;
    if (bn_out) *bn_out = bn;
    const int tiles = ((M + BM - 1) / BM) * ((N + bn - 1) / bn);
    const int nkb = (K + BK - 1) / BK;
    int best = 1;
    double best_eff = 0.0;
    for (int s = 1; s <= 8 && s <= nkb / 4 + 1; ++s) {
        const int ctas = tiles * s;
        const int waves = (ctas + num_sms - 1) / num_sms;
        const double eff = (double)ctas / ((double)waves * num_sms);
        if (eff > best_eff + 0.05) {
            best_eff = eff;
            best = s;
        }
        if (eff >= 0.85) break;
    }
    if (best > nkb) best = nkb;
    return best;
}

cudaError_t gemm_plan(GemmPlan* p, const uint16_t* A, int M, int K, const uint16_t* B, int N, int num_sms) {
    if (M <= 0 || N <= 0 || K <= 0 || K % 8 != 0) return cudaErrorInvalidValue;
    p->M = M;
    p->N = N;
    p->K = K;
    p->splits = gemm_choose_splits(M, N, K, num_sms, &p->bn);
    cudaError_t e = encode_2d(&p->tmA, A, M, K, BM);
    if (e != cudaSuccess) return e;
    return encode_2d(&p->tmB, B, N, K, p->bn);
}

cudaError_t gemm_launch(const GemmPlan& p, GemmArgs a, cudaStream_t st, bool pdl) {
    a.M = p.M;
    a.N = p.N;
    a.K = p.K;
    a.splits = p.splits;
    switch (p.bn) {
        case 32: return launch_bn<32>(p, a, st, pdl);
        case 64: return launch_bn<64>(p, a, st, pdl);
        case 128: return launch_bn<128>(p, a, st, pdl);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace dec
