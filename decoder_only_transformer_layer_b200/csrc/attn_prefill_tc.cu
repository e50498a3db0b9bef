// Causal GQA attention of a prefill chunk on the tensor cores (tcgen05, TMEM accumulators).
//
// The chunk's rows are (token, head) pairs of one kv head's group: a CTA owns 128 of them
// (128 / G tokens x the G query heads that share the kv head), so every key and value it
// loads serves all G heads. Per 128-key block of the paged cache:
//   S = Q K^T          tcgen05.mma M=128 N=128 K=16 (x 8 over d = 128), fp32 in TMEM
//   P = exp2(S' - m)   8 softmax warps, two per row quarter (TMEM lanes), each taking one
//                      half of the keys and exchanging the row maximum through shared
//                      memory; S' is the scaled (or softcapped) score in log2 units; P
//                      written back over S in TMEM as
//                      two bf16 terms P_hi + P_lo (P_hi the top 16 bits of the fp32 P, P_lo
//                      those of the exact rest: 15 significant bits; a single bf16 P moved
//                      the Llama-3-8B-shape logits by ~0.6%, past the parity bar)
//   O += P V           tcgen05.mma M=128 N=128 K=16, A (P) from TMEM, B (V) from shared
//                      memory (x 8 over keys, x 2 terms)
// with S double-buffered in TMEM, so the scores of block j + 1 are computed while the
// softmax warps work on block j. K and V stream through separate 3-stage rings, each with
// its own producer warp: a K stage is released as soon as its scores are computed, a V
// stage when its PV product is, so the loads of later blocks overlap the softmax. The running maximum m is moved, and O and l rescaled,
// only when a row's maximum grows by more than 2^8 (P <= 2^8 never overflows, and O / l
// is unchanged by the choice of m), so O stays in TMEM untouched almost always.
// Keys past a row's position (or before its window) are masked per element; blocks before
// every row's window are skipped.
// With S > 1 key splits (short chunks would otherwise fill few SMs) the S CTAs of a row
// block form a cluster, each taking a contiguous run of key blocks. After one cluster
// barrier (every ring drained) each sends its rows' unnormalised O with their m and l
// straight from TMEM-loaded registers to the owner of the rows (128 / S of them), with
// st.async completing on the owner's mbarrier, and the owner merges the S partials in
// split order (deterministic). No CTA reads another's shared memory, so there is no
// second barrier before leaving.
//
// Operand layouts in shared memory (all 128-byte swizzled, 1024-byte aligned):
//   Q  [2 d-halves][128 rows][64 d]   A of S, K-major      (TMA 3-D box {64, G, 128/G})
//   K  [2 d-halves][128 keys][64 d]   B of S, K-major      (TMA box {64, 16} per page)
//   V  [2 d-halves][128 keys][64 d]   B of O, MN-major (d contiguous)
// TMEM (512 columns): S/P of even blocks at 0, of odd blocks at 128 (P_hi in the first 64
// columns, P_lo in the next 64, two keys per column), O at 256.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace dec {

namespace {

constexpr int kTcRows = 128;  // (token, head) rows per CTA: the MMA's M
constexpr int kTcKeys = 128;  // keys per block: N of S, K of O
constexpr int kTcPage = 16;
constexpr float kTcLog2e = 1.4426950408889634f;
constexpr float kTcRescale = 8.0f;  // log2 units

constexpr int kTcStages = 3;
constexpr uint32_t kStage = 32768;  // one 128-key block of K or of V
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = 32768;
constexpr uint32_t kOffV = kOffK + kTcStages * kStage;
constexpr uint32_t kOffBar = kOffV + kTcStages * kStage;
// after the last block: [recv: S][128 / S][LDR] every split's partial of this CTA's rows
constexpr int kLdr = 132;  // O[128], m, l, 2 pad: 16-byte rows, conflict-free
constexpr uint32_t kOffRecv = kOffK;
static_assert(kOffRecv + kTcRows * kLdr * 4 <= kOffBar, "the merge area fits in the drained rings");
constexpr uint32_t kOffXch = kOffBar + 256;  // softmax warp pairs' row maxima and sums
constexpr uint32_t kTcSmem = kOffXch + 2 * kTcRows * 4 + 1024;  // + alignment slack
static_assert(kTcSmem <= 232448, "fits the 227 KB a CTA may use");

// Shared-memory descriptor of a 128-byte-swizzled MN-major operand: each 128-byte row holds
// 64 consecutive MN elements of one k, 8 rows (8 k) form a 1024-byte swizzle atom. The
// leading byte offset is the stride between 64-element atoms along MN (the two d-halves of
// V, 16 KB apart), the stride byte offset the stride between 8-row groups along K (1 KB).
DEC_DEVINL uint64_t sdesc_sw128_mn(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)(16384 >> 4) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// kind::f16 instruction descriptor: bf16 A (K-major) and B (MN-major when b_mn), fp32 D.
template <int M, int N, bool B_MN>
__host__ __device__ constexpr uint32_t idesc_tc() {
    return (1u << 4) | (1u << 7) | (1u << 10) | (B_MN ? (1u << 16) : 0u) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

DEC_DEVINL void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
// D (+)= A B with A read from TMEM (lanes = rows, two 16-bit elements per column, the lower
// k in the low half) and B from shared memory.
DEC_DEVINL void tc_mma_tmem_a(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc, uint32_t accum) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
}

// Two fp32 values' top halves as the two bf16 of one word (a's in the low half): the
// values truncated to bf16.
DEC_DEVINL uint32_t hi_halves(float a, float b) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(d) : "r"(__float_as_uint(a)), "r"(__float_as_uint(b)));
    return d;
}
DEC_DEVINL float trunc_bf(float x) { return __uint_as_float(__float_as_uint(x) & 0xFFFF0000u); }

// Barrier `id` (1..15) over `n` threads of the CTA (a multiple of 32).
DEC_DEVINL void named_bar_sync(uint32_t id, uint32_t n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

DEC_DEVINL void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// No instruction: tells the compiler the 32 registers change here, so no use of values
// loaded before a tcgen05.wait::ld on another array can move above that wait.
DEC_DEVINL void reg_fence32(uint32_t (&r)[32]) {
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                   "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                   "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}

DEC_DEVINL void tma_load_3d(void* dst, const CUtensorMap* tm, int x, int y, int z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

// The softcapped score c tanh(raw scale / c) in log2 units, out of line so the uncapped
// path never evaluates the tanh.
__device__ __noinline__ float capped_score(float raw, float scale, float c) {
    return c * tanhf(raw * scale / c) * kTcLog2e;
}

// 2^x by the hardware's approximate exponential (a few fp32 ulp; 2^-inf = 0). The P it
// gives is rounded to bf16 terms.
DEC_DEVINL float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Pass 1 over NC x 32 raw scores of a row (keys key0 ..), in place: keys outside [lo, pos]
// become -inf; with CAP the others become the softcapped score in log2 units (`sc` the
// attention scale, `c` the cap), without it they stay raw (the scale, positive, is applied
// in pass 2). Returns their maximum (four independent partial maxima).
template <bool CAP, int NC>
DEC_DEVINL float scores_log2(uint32_t (&v)[NC][32], float sc, float c, bool whole, int key0, int lo, int pos) {
    float bm4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    if (whole) {
#pragma unroll
        for (int k = 0; k < NC; ++k)
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                const float x = CAP ? capped_score(__uint_as_float(v[k][q]), sc, c) : __uint_as_float(v[k][q]);
                if (CAP) v[k][q] = __float_as_uint(x);
                bm4[q & 3] = fmaxf(bm4[q & 3], x);
            }
    } else {
#pragma unroll
        for (int k = 0; k < NC; ++k)
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                const int key = key0 + 32 * k + q;
                float x = CAP ? capped_score(__uint_as_float(v[k][q]), sc, c) : __uint_as_float(v[k][q]);
                x = key > pos || key < lo ? -INFINITY : x;
                v[k][q] = __float_as_uint(x);
                bm4[q & 3] = fmaxf(bm4[q & 3], x);
            }
    }
    return fmaxf(fmaxf(bm4[0], bm4[1]), fmaxf(bm4[2], bm4[3]));
}

struct TcPrefArgs {
    AttnPrefillArgs a;
    int G, tok_per_cta;
};

__global__ void __launch_bounds__(352, 1)
    attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, TcPrefArgs args) {
    const AttnPrefillArgs& a = args.a;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t* q_full = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* k_full = q_full + 1;               // [kTcStages]
    uint64_t* k_empty = k_full + kTcStages;      // [kTcStages]
    uint64_t* v_full = k_empty + kTcStages;      // [kTcStages]
    uint64_t* v_empty = v_full + kTcStages;      // [kTcStages]
    uint64_t* s_full = v_empty + kTcStages;      // [2]
    uint64_t* p_full = s_full + 2;    // the softmax warps read S[j & 1] and wrote P over it
    uint64_t* pv_done = p_full + 1;   // [2] O += P V of block j completed: pv_done[j & 1]
    uint64_t* recvb = pv_done + 2;    // the other splits' rows of this CTA have landed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(recvb + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = args.G, TPC = args.tok_per_cta;
    const int g = blockIdx.y;
    const int t0 = blockIdx.x * TPC;                  // first token of this CTA
    const int t_last = min(a.T - 1, t0 + TPC - 1);    // last valid token
    const int hi_key = a.pos0 + t_last;               // the largest key any row sees
    const int lo_key = a.window > 0 ? max(0, a.pos0 + t0 + 1 - a.window) : 0;  // the smallest
    const int S = gridDim.z, z = blockIdx.z;           // key splits (a cluster), this split
    const int RS = kTcRows / S;                        // rows each split finishes
    const int kb_lo = lo_key / kTcKeys, nb_all = hi_key / kTcKeys - kb_lo + 1;
    const int kb0 = kb_lo + (int)((long long)nb_all * z / S);  // this split's key blocks
    const int nb = kb_lo + (int)((long long)nb_all * (z + 1) / S) - kb0;
    const int np = (a.pos0 + a.T + kTcPage - 1) / kTcPage;  // pages holding keys of this chunk

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < kTcStages; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) mbar_init(&s_full[i], 1);
        mbar_init(p_full, 8);
        mbar_init(&pv_done[0], 1);
        mbar_init(&pv_done[1], 1);
        mbar_init(recvb, 1);
        // armed before the first cluster barrier, so no byte can arrive before the count
        if (S > 1) mbar_arrive_expect_tx(recvb, (uint32_t)(S - 1) * RS * kLdr * 4);
        fence_mbar_init();
    }
    if (warp == 8 && lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(512)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tO = tmem + 2 * kTcKeys;  // S[0], S[1]: columns 0..255; O: 256..383
    pdl_trigger();

    if (warp == 8 || warp == 10) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producers: K (warp 8, with
            // q first) and V (warp 10)
            const bool isv = warp == 10;
            uint64_t* full = isv ? v_full : k_full;
            uint64_t* empty = isv ? v_empty : k_empty;
            const CUtensorMap* tm = isv ? &tmV : &tmK;
            uint8_t* ring = smem + (isv ? kOffV : kOffK);
            pdl_wait();  // q and the chunk's own keys come from the previous kernels
            if (!isv) {
                mbar_arrive_expect_tx(q_full, 32768);
                for (int h2 = 0; h2 < 2; ++h2)
                    tma_load_3d(smem + kOffQ + h2 * 16384, &tmQ, h2 * 64, g * G, t0, q_full);
            }
            for (int j = 0; j < nb; ++j) {
                const int s = j % kTcStages;
                if (j >= kTcStages && !mbar_wait_bounded(&empty[s], (j / kTcStages - 1) & 1, a.err)) break;
                mbar_arrive_expect_tx(&full[s], kStage);
                uint8_t* d = ring + s * kStage;
                for (int pi = 0; pi < kTcKeys / kTcPage; ++pi) {
                    // pages past the chunk's last one hold only masked keys: any finite page
                    // will do, so they reload the last page
                    const int page = min((kb0 + j) * (kTcKeys / kTcPage) + pi, np - 1);
                    const int row = (a.block_row[page] * a.nkv + g) * kTcPage;
                    for (int h2 = 0; h2 < 2; ++h2) tma_load_2d(d + h2 * 16384 + pi * 2048, tm, h2 * 64, row, &full[s]);
                }
            }
        }
        __syncwarp();
    } else if (warp == 9) {
        pdl_wait();
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            constexpr uint32_t id_s = idesc_tc<128, 128, false>();
            constexpr uint32_t id_o = idesc_tc<128, 128, true>();
            const uint32_t sb = smem_u32(smem);
            bool ok = mbar_wait_bounded(q_full, 0, a.err);
            // S(j) into TMEM columns (j & 1) * 128; the K stage is free once these complete
            auto issue_s = [&](int j) {
                const int s = j % kTcStages;
                const uint32_t kb = sb + kOffK + s * kStage;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc_mma(tS + (j & 1) * kTcKeys, sdesc_sw128(sb + kOffQ + (kk >> 2) * 16384 + (kk & 3) * 32),
                           sdesc_sw128(kb + (kk >> 2) * 16384 + (kk & 3) * 32), id_s, kk > 0 ? 1u : 0u);
                tc_commit(&s_full[j & 1]);
                tc_commit(&k_empty[s]);
            };
            if (ok && nb > 0) {
                ok = mbar_wait_bounded(&k_full[0], 0, a.err);
                tc_fence_after();
                if (ok) issue_s(0);
            }
            for (int j = 0; j < nb && ok; ++j) {
                if (j + 1 < nb) {
                    // TMEM columns ((j + 1) & 1) * 128 held P(j - 1), whose PV product was
                    // issued before this (tcgen05 MMAs of one thread run in order)
                    const int s1 = (j + 1) % kTcStages;
                    if (!mbar_wait_bounded(&k_full[s1], ((j + 1) / kTcStages) & 1, a.err)) break;
                    tc_fence_after();
                    issue_s(j + 1);
                }
                const int sv = j % kTcStages;
                if (!mbar_wait_bounded(p_full, j & 1, a.err)) break;
                if (!mbar_wait_bounded(&v_full[sv], (j / kTcStages) & 1, a.err)) break;
                tc_fence_after();
                const uint32_t vb = sb + kOffV + sv * kStage;
                const uint32_t tp = tS + (j & 1) * kTcKeys;  // P_hi at tp, P_lo at tp + 64
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t vdesc = sdesc_sw128_mn(vb + kk * 2048);
                    tc_mma_tmem_a(tO, tp + kk * 8, vdesc, id_o, (j > 0 || kk > 0) ? 1u : 0u);
                    tc_mma_tmem_a(tO, tp + 64 + kk * 8, vdesc, id_o, 1u);
                }
                tc_commit(&pv_done[j & 1]);
                tc_commit(&v_empty[sv]);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------ softmax + epilogue (warps 0-7): warps w and w + 4
        // share the 32 rows (TMEM lanes) 32 (w % 4) ..; warp w takes keys 0-63 of each block,
        // warp w + 4 keys 64-127
        const int quad = warp & 3, half = warp >> 2;
        const int r = quad * 32 + lane;  // row = TMEM lane
        const int tl = r / G;             // token within the CTA
        const int t = t0 + tl;
        const bool valid = tl < TPC && t < a.T;
        const int pos = a.pos0 + t;       // the row's last visible key
        const int lo = a.window > 0 ? pos + 1 - a.window : 0;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const float sl2 = a.scale * kTcLog2e;
        const bool cap = a.softcap > 0.f;
        float* xch = reinterpret_cast<float*>(smem + kOffXch);  // [2 halves][128 rows]
        const uint32_t pair_bar = 1 + quad;                     // named barrier of warps w, w + 4
        float m = -INFINITY, l = 0.f;  // l: this half's keys only
        pdl_wait();
        bool ok = true;
        for (int j = 0; j < nb; ++j) {
            const int key0 = (kb0 + j) * kTcKeys;
            if (ok && !mbar_wait_bounded(&s_full[j & 1], (j >> 1) & 1, a.err)) ok = false;
            tc_fence_after();
            const uint32_t sa = tS + (j & 1) * kTcKeys + lane_off;
            // The row sees keys [lo, pos]: a block wholly inside needs no per-key test, one
            // wholly outside contributes nothing.
            const bool none = !valid || key0 > pos || key0 + kTcKeys - 1 < lo;
            const bool whole = !none && key0 + kTcKeys - 1 <= pos && key0 >= lo;
            // this half's 64 scores of the row, in one TMEM round trip
            uint32_t v[2][32];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                tmem_ld16_issue(sa + 64 * half + 32 * c, v[c]);
                tmem_ld16_issue(sa + 64 * half + 32 * c + 16, v[c] + 16);
            }
            tmem_ld_wait32(v[1]);
            reg_fence32(v[0]);
            // pass 1: the scores in log2 units, masked, and their maximum
            // (the cap and mask tests sit outside the loops: a test, let alone a possible
            // call, per element made this pass cost more than the rest of the block)
            float bm = -INFINITY;
            if (!none) {
                if (cap)
                    bm = scores_log2<true>(v, a.scale, a.softcap, whole, key0 + 64 * half, lo, pos);
                else
                    bm = scores_log2<false>(v, 0.f, 0.f, whole, key0 + 64 * half, lo, pos) * sl2;
            }
            // the row maximum over both halves (the first barrier: the partner has read the
            // last value; the second also orders both halves' score loads before either
            // writes P over the scores)
            if (j > 0) named_bar_sync(pair_bar, 64);
            xch[half * 128 + r] = bm;
            tc_fence_before();
            named_bar_sync(pair_bar, 64);
            tc_fence_after();
            bm = fmaxf(bm, xch[(half ^ 1) * 128 + r]);
            const float mn = fmaxf(m, bm);
            const bool grow = m != -INFINITY && mn > m + kTcRescale;
            if (__any_sync(0xffffffffu, grow)) {
                // move the reference maximum: O and l of the rows that grew scale by 2^(m - mn)
                // (each half rescales its 64 columns of O) once O += P V of block j - 1 is in.
                // Nothing else waits for it: P of block j goes where P of block j - 2 was,
                // whose product completed before the scores of block j did.
                if (j > 0 && ok && !mbar_wait_bounded(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, a.err)) ok = false;
                tc_fence_after();
                const float corr = grow ? ex2f(m - mn) : 1.f;
                for (int c0 = 64 * half; c0 < 64 * half + 64; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld16_issue(tO + lane_off + c0, o);
                    tmem_ld16_issue(tO + lane_off + c0 + 16, o + 16);
                    tmem_ld_wait32(o);
#pragma unroll
                    for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * corr);
                    tmem_st16(tO + lane_off + c0, o);
                    tmem_st16(tO + lane_off + c0 + 16, o + 16);
                }
                tmem_st_wait();
                l *= corr;
            }
            if (grow || m == -INFINITY) m = mn;
            // pass 2: P = 2^(S' - m) as bf16 hi + lo, written over the row's scores in TMEM
            // (keys 2i, 2i + 1 in column i of each term), and the row sum (four independent
            // partial sums); masked scores are -inf and give 0. P_hi is P truncated to bf16,
            // P_lo the exact rest P - P_hi truncated: |P - P_hi - P_lo| < 2^-14 P.
            // Pairs of keys go through the packed fp32x2 pipe: x = s mul - m, the sums, and
            // P - P_hi.
            const bool zero = none || m == -INFINITY;
            const float2 mul2 = cap ? make_float2(1.f, 1.f) : make_float2(sl2, sl2);
            const float2 nm2 = make_float2(-m, -m), neg1 = make_float2(-1.f, -1.f);
            float2 sum2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t ph[16], pl[16];
                if (zero) {
#pragma unroll
                    for (int q = 0; q < 16; ++q) ph[q] = pl[q] = 0u;
                } else {
#pragma unroll
                    for (int q = 0; q < 32; q += 2) {
                        const float2 x =
                            ffma2(make_float2(__uint_as_float(v[c][q]), __uint_as_float(v[c][q + 1])), mul2, nm2);
                        const float2 p = make_float2(ex2f(x.x), ex2f(x.y));
                        sum2[(q >> 1) & 1] = fadd2(sum2[(q >> 1) & 1], p);
                        ph[q / 2] = hi_halves(p.x, p.y);
                        const float2 rest = ffma2(make_float2(trunc_bf(p.x), trunc_bf(p.y)), neg1, p);
                        pl[q / 2] = hi_halves(rest.x, rest.y);
                    }
                }
                const int cg = 2 * half + c;  // keys 32 cg .. 32 cg + 31 of the block
                tmem_st16(sa + 16 * cg, ph);
                tmem_st16(sa + 64 + 16 * cg, pl);
            }
            l += (sum2[0].x + sum2[1].x) + (sum2[0].y + sum2[1].y);
            tmem_st_wait();  // the MMA reads P from TMEM
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        // ---- epilogue: the row sum over both halves
        named_bar_sync(pair_bar, 64);
        xch[half * 128 + r] = l;
        named_bar_sync(pair_bar, 64);
        l += xch[(half ^ 1) * 128 + r];
        if (nb > 0 && ok && !mbar_wait_bounded(&pv_done[(nb - 1) & 1], ((nb - 1) >> 1) & 1, a.err)) ok = false;
        tc_fence_after();
        if (S == 1) {
            // O / l, bf16, to out[t][g G + (r % G)][:] (each half its 64 columns)
            const float inv = l > 0.f ? 1.0f / l : 0.f;
            uint16_t* dst = a.out + ((size_t)t * a.nq + (size_t)g * G + (r % G)) * 128;
            for (int c0 = 64 * half; c0 < 64 * half + 64; c0 += 32) {
                uint32_t v[32];
                tmem_ld16_issue(tO + lane_off + c0, v);
                tmem_ld16_issue(tO + lane_off + c0 + 16, v + 16);
                tmem_ld_wait32(v);
                if (valid && ok) {
#pragma unroll
                    for (int q = 0; q < 32; q += 8) {
                        uint4 o;
                        o.x = pack_bf2(__uint_as_float(v[q]) * inv, __uint_as_float(v[q + 1]) * inv);
                        o.y = pack_bf2(__uint_as_float(v[q + 2]) * inv, __uint_as_float(v[q + 3]) * inv);
                        o.z = pack_bf2(__uint_as_float(v[q + 4]) * inv, __uint_as_float(v[q + 5]) * inv);
                        o.w = pack_bf2(__uint_as_float(v[q + 6]) * inv, __uint_as_float(v[q + 7]) * inv);
                        *reinterpret_cast<uint4*>(dst + c0 + q) = o;
                    }
                }
            }
        } else {
            // every split of the cluster is past its MMAs: every ring is drained, free to
            // receive (the producer and MMA warps arrive below)
            cluster_sync();
            // this split's partial of row r (unnormalised O, m, l) into slot [z] of the row's
            // owner: kept here for own rows, st.async from registers (transaction bytes on the
            // owner's recvb) for the others, so no copy reads this CTA's shared memory
            const int own = r / RS, lr = r - own * RS;
            float* slot = reinterpret_cast<float*>(smem + kOffRecv) + ((size_t)z * RS + lr) * kLdr;
            const uint32_t rdst = own == z ? 0u : dsmem_map(smem_u32(slot), own);
            const uint32_t rbar = own == z ? 0u : dsmem_map(smem_u32(recvb), own);
            auto put4 = [&](int c, uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3) {
                if (own == z)
                    *reinterpret_cast<uint4*>(slot + c) = make_uint4(x0, x1, x2, x3);
                else
                    st_async_4f(rdst + (uint32_t)c * 4, __uint_as_float(x0), __uint_as_float(x1), __uint_as_float(x2),
                                __uint_as_float(x3), rbar);
            };
            for (int c0 = 64 * half; c0 < 64 * half + 64; c0 += 32) {
                uint32_t v[32];
                if (nb > 0) {
                    tmem_ld16_issue(tO + lane_off + c0, v);
                    tmem_ld16_issue(tO + lane_off + c0 + 16, v + 16);
                    tmem_ld_wait32(v);
                } else {
#pragma unroll
                    for (int q = 0; q < 32; ++q) v[q] = 0u;  // no key blocks: O = 0, m = -inf, l = 0
                }
#pragma unroll
                for (int q = 0; q < 32; q += 4) put4(c0 + q, v[q], v[q + 1], v[q + 2], v[q + 3]);
            }
            if (half == 0) put4(128, __float_as_uint(m), __float_as_uint(l), 0u, 0u);
            named_bar_sync(5, 256);  // every own row is in place before the merge reads it
        }
    }
    if (S > 1) {
        if (warp >= 8) cluster_sync();  // the producer and MMA warps' arrivals
        if (warp < 4) {
            // rows [z RS, z RS + RS): 128 / RS threads a row, 128 / (128 / RS) columns each
            const int tpr = kTcRows / RS;
            const int lr = threadIdx.x / tpr, part = threadIdx.x % tpr, cols = 128 / tpr;
            const int rr = z * RS + lr;  // the row in the CTA's 128
            const bool got = mbar_wait_cluster_bounded(recvb, 0, a.err);
            const int tt = t0 + rr / G;
            auto part_row = [&](int zz) {
                return reinterpret_cast<const float*>(smem + kOffRecv) + ((size_t)zz * RS + lr) * kLdr;
            };
            float M = -INFINITY;
            for (int zz = 0; zz < S; ++zz) M = fmaxf(M, part_row(zz)[128]);
            float L = 0.f;
            float acc[128 / 2];  // at most 64 columns per thread (RS <= 64)
#pragma unroll
            for (int c = 0; c < 64; ++c) acc[c] = 0.f;
            for (int zz = 0; zz < S; ++zz) {
                const float* pr = part_row(zz);
                const float mz = pr[128];
                if (mz == -INFINITY) continue;
                const float wz = ex2f(mz - M);
                L += wz * pr[129];
#pragma unroll
                for (int c = 0; c < 64; c += 4) {
                    if (c < cols) {
                        const float4 v = *reinterpret_cast<const float4*>(pr + part * cols + c);
                        acc[c] += wz * v.x;
                        acc[c + 1] += wz * v.y;
                        acc[c + 2] += wz * v.z;
                        acc[c + 3] += wz * v.w;
                    }
                }
            }
            if (got && tt < a.T && (rr / G) < TPC) {
                const float inv = L > 0.f ? 1.0f / L : 0.f;
                uint16_t* dst = a.out + ((size_t)tt * a.nq + (size_t)g * G + (rr % G)) * 128 + part * cols;
#pragma unroll
                for (int c = 0; c < 64; c += 8) {
                    if (c < cols) {
                        uint4 o;
                        o.x = pack_bf2(acc[c] * inv, acc[c + 1] * inv);
                        o.y = pack_bf2(acc[c + 2] * inv, acc[c + 3] * inv);
                        o.z = pack_bf2(acc[c + 4] * inv, acc[c + 5] * inv);
                        o.w = pack_bf2(acc[c + 6] * inv, acc[c + 7] * inv);
                        *reinterpret_cast<uint4*>(dst + c) = o;
                    }
                }
            }
        }
        // nothing reads another CTA's shared memory, and this CTA's incoming bytes completed
        // before its merge: no cluster barrier before leaving
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
    }
}

}  // namespace

// The tensor-core kernel takes head dim 128, groups of 1, 2, 4, ..., 128 query heads, and
// chunks of at least one CTA's tokens (the q box never exceeds the chunk).
bool attn_prefill_tc_ok(const AttnPrefillArgs& a) {
    const int G = a.nkv > 0 ? a.nq / a.nkv : 0;
    return a.d == 128 && G >= 1 && G <= kTcRows && (G & (G - 1)) == 0 && a.nq % a.nkv == 0 && a.pool_rows > 0 &&
           a.T >= kTcRows / G;
}

cudaError_t attn_prefill_tc_launch(const AttnPrefillArgs& a, cudaStream_t st, bool pdl) {
    if (a.T <= 0) return cudaSuccess;
    if (!attn_prefill_tc_ok(a)) return cudaErrorInvalidValue;
    const int G = a.nq / a.nkv;
    TcPrefArgs args;
    args.a = a;
    args.G = G;
    args.tok_per_cta = kTcRows / G;
    // key splits: a power of two (rows split evenly between the owners), enough CTAs to
    // cover the SMs, at most one per key block of the longest row, at most 8 (a portable
    // cluster)
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    const int ctas = ((a.T + args.tok_per_cta - 1) / args.tok_per_cta) * a.nkv;
    const int span_blocks = (attn_prefill_span(a.pos0, a.T, a.window) + kTcKeys - 1) / kTcKeys + 1;
    int S = 1;
    while (S < 8 && ctas * S * 2 <= sms && S * 2 <= span_blocks) S *= 2;
    CUtensorMap tmQ, tmK, tmV;
    {
        const uint64_t dims[3] = {128, (uint64_t)a.nq, (uint64_t)a.T};
        const uint64_t strides[2] = {128 * 2, (uint64_t)a.nq * 128 * 2};
        const uint32_t box[3] = {64, (uint32_t)G, (uint32_t)(kTcRows / G)};
        cudaError_t e = tmap_bf16_sw128(&tmQ, a.q, 3, dims, strides, box);
        if (e != cudaSuccess) return e;
    }
    {
        const uint64_t dims[2] = {128, (uint64_t)a.pool_rows};
        const uint64_t strides[1] = {128 * 2};
        const uint32_t box[2] = {64, kTcPage};
        cudaError_t e = tmap_bf16_sw128(&tmK, a.k_pool, 2, dims, strides, box);
        if (e != cudaSuccess) return e;
        e = tmap_bf16_sw128(&tmV, a.v_pool, 2, dims, strides, box);
        if (e != cudaSuccess) return e;
    }
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(attn_prefill_tc_kernel), (int)kTcSmem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((a.T + args.tok_per_cta - 1) / args.tok_per_cta, a.nkv, S);
    cfg.blockDim = dim3(352);
    cfg.dynamicSmemBytes = kTcSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (S > 1) {  // the key splits of a row block: one cluster
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = 1;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = S;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, attn_prefill_tc_kernel, tmQ, tmK, tmV, args);
}

}  // namespace dec
