// Causal GQA attention over a paged bf16 KV cache, decode and chunked prefill.
//
// What it computes (ANEDVD src/engine.zig: ropeAndCache, cpu.attentionDecode,
// cpu.attentionPrefill; frink_models decoder.rs: gqa_attention / the CUDA
// gqa_decode kernel; cortiq_engine pipeline.rs: attn_scale = 1/sqrt(head_dim)):
//   q head h reads kv head g = h / (nq / nkv); the query at position p attends
//   cache rows 0..p; o = sum_j softmax_j(q . k_j * scale) v_j. Optionally (ANEDVD's
//   attentionDecode options .window and .logit_softcap; cortiq's per-layer window)
//   only rows p-W+1..p are attended, and each scaled score s becomes c tanh(s / c).
// Before attention q and the new k get an optional per-head RMSNorm (QK-norm)
// and RoPE (half-split pairs (i, i + d/2), angle p * base^(-2i/d), evaluated in
// fp64), and are rounded to bf16; k and v enter the cache once, at row p.
//
// B200 design:
//  * decode: one CTA per (sequence, kv head, context split); the G = nq/nkv
//    query heads of the group share one pass over the K/V pages (GQA packing
//    into the 16 rows of an m16n8k16 tensor-core tile); 4 warps take pages in
//    turn, each with a double-buffered cp.async page ring; online softmax in
//    fp32 with quad shuffles; splits merged deterministically by the last CTA
//    of each (sequence, kv head);
//  * the softmax weights P enter the PV product as two bf16 terms (P_hi + P_lo)
//    so that the weighted sum keeps fp32-level accuracy; Q.K is exact in fp32
//    (both operands are the rounded bf16 values);
//  * QK-norm, RoPE and the cache append of the new token are fused into the
//    decode kernel: the CTA whose split holds row p writes it before reading.
//  * prefill: the chunk's q/k/v are rotated and appended by rope_append_kernel;
//    the attention kernel then gives each warp 16 (token, head) rows, shares
//    64-key blocks of the cache among its 4 warps and skips fully masked pages.
#include <math.h>

#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"
#include "kernels.h"

namespace dec {

namespace {

constexpr int kPage = 16;
constexpr int kDecodeMaxSplits = 16;  // context splits of one (sequence, kv head): one cluster
constexpr float kLog2e = 1.4426950408889634f;

// A raw q.k product -> the softmax argument in log2 units: times scale, then the logit
// softcap c tanh(s / c) when c > 0.
DEC_DEVINL float score_log2(float raw, float scale, float softcap) {
    const float s = raw * scale;
    return (softcap > 0.f ? softcap * tanhf(s / softcap) : s) * kLog2e;
}

// A warp transforms one head vector of D fp32 values: optional RMSNorm with weight
// nw, optional RoPE at position pos, rounding to bf16. Lane l holds elements
// l + 32 m; element l + 32 m (m < D/64) pairs with element l + 32 (m + D/64).
// With `tab` (the row of a host-built table for this position: (cos, sin) per pair,
// evaluated in fp64 and rounded to fp32) the angles are read; without it they are
// evaluated here in fp64.
template <int D>
DEC_DEVINL void head_transform(const float* vals_in, bool in_bf16, const uint16_t* in_b, const float* nw,
                               float eps, bool rope, int pos, float base, uint16_t* dst,
                               const float2* tab = nullptr) {
    constexpr int E = D / 32;
    const int lane = threadIdx.x & 31;
    float v[E];
#pragma unroll
    for (int m = 0; m < E; ++m) v[m] = in_bf16 ? bf2f(in_b[lane + 32 * m]) : vals_in[lane + 32 * m];
    if (nw) {
        float ss = 0.f;
#pragma unroll
        for (int m = 0; m < E; ++m) ss = fmaf(v[m], v[m], ss);
        ss = warp_sum(ss);
        const float inv = 1.0f / sqrtf(ss / (float)D + eps);
#pragma unroll
        for (int m = 0; m < E; ++m) v[m] = v[m] * inv * nw[lane + 32 * m];
    }
    if (rope) {
#pragma unroll
        for (int m = 0; m < E / 2; ++m) {
            float c, s;
            if (tab) {
                const float2 cs = tab[lane + 32 * m];
                c = cs.x;
                s = cs.y;
            } else {
                rope_cs(pos, lane + 32 * m, D, base, &c, &s);
            }
            const float x0 = v[m], x1 = v[m + E / 2];
            v[m] = x0 * c - x1 * s;
            v[m + E / 2] = x0 * s + x1 * c;
        }
    }
#pragma unroll
    for (int m = 0; m < E; ++m) dst[lane + 32 * m] = f2bf(v[m]);
}

// Per-position constants of head_transform, read before the grid-dependency wait (they do
// not depend on the previous kernel): this lane's (cos, sin) pairs and norm gains.
template <int D>
struct HeadRegs {
    float2 cs[D / 64];
    float qn[D / 32], kn[D / 32];
};

template <int D>
DEC_DEVINL void load_head_regs(HeadRegs<D>& r, const float2* tab, const float* qn, const float* kn) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int m = 0; m < D / 64; ++m) r.cs[m] = tab ? tab[lane + 32 * m] : make_float2(1.f, 0.f);
#pragma unroll
    for (int m = 0; m < D / 32; ++m) {
        r.qn[m] = qn ? qn[lane + 32 * m] : 1.f;
        r.kn[m] = kn ? kn[lane + 32 * m] : 1.f;
    }
}

// head_transform with the norm gains (nw, or null for none) and the angles held in
// registers: the same arithmetic in the same order.
template <int D>
DEC_DEVINL void head_transform_regs(const float* vals_in, const float* nw, bool norm, float eps, bool rope,
                                    const float2* cs, uint16_t* dst) {
    constexpr int E = D / 32;
    const int lane = threadIdx.x & 31;
    float v[E];
#pragma unroll
    for (int m = 0; m < E; ++m) v[m] = vals_in[lane + 32 * m];
    if (norm) {
        float ss = 0.f;
#pragma unroll
        for (int m = 0; m < E; ++m) ss = fmaf(v[m], v[m], ss);
        ss = warp_sum(ss);
        const float inv = 1.0f / sqrtf(ss / (float)D + eps);
#pragma unroll
        for (int m = 0; m < E; ++m) v[m] = v[m] * inv * nw[m];
    }
    if (rope) {
#pragma unroll
        for (int m = 0; m < E / 2; ++m) {
            const float c = cs[m].x, s = cs[m].y;
            const float x0 = v[m], x1 = v[m + E / 2];
            v[m] = x0 * c - x1 * s;
            v[m + E / 2] = x0 * s + x1 * c;
        }
    }
#pragma unroll
    for (int m = 0; m < E; ++m) dst[lane + 32 * m] = f2bf(v[m]);
}

// Online-softmax state update for one 16-key page held as two m16n8 score tiles.
// sc[nt][0..1]: row g, keys nt*8 + 2t + {0,1}; sc[nt][2..3]: row g + 8.
// Scores are already in log2 units; masked entries are -inf. Returns P in sc.
DEC_DEVINL void softmax_page(float (&sc)[2][4], float (&m)[2], float (&l)[2], float (&corr)[2]) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        float mx = fmaxf(fmaxf(sc[0][2 * r], sc[0][2 * r + 1]), fmaxf(sc[1][2 * r], sc[1][2 * r + 1]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float mn = fmaxf(m[r], mx);
        if (mn == -INFINITY) {  // every key so far masked for this row
            corr[r] = 1.f;
            sc[0][2 * r] = sc[0][2 * r + 1] = sc[1][2 * r] = sc[1][2 * r + 1] = 0.f;
            continue;
        }
        corr[r] = exp2f(m[r] - mn);
        m[r] = mn;
        float sum = 0.f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const float p = exp2f(sc[nt][2 * r + c] - mn);
                sc[nt][2 * r + c] = p;
                sum += p;
            }
        l[r] = l[r] * corr[r] + sum;
    }
}

// O += P V for one 16-key page: P (rows g, g+8) from sc, V page rows in shared memory
// with row stride LD, chunks swizzled as load_page_warp stores them. P enters as bf16 hi + lo parts. PACK (at most 8 query rows): row
// g + 8 of the A tile carries P_lo of row g, so one MMA per tile takes both terms; the
// accumulator's rows g and g + 8 then hold the two terms' products of row g.
template <int D, int LD, bool PACK>
DEC_DEVINL void pv_page(const float (&sc)[2][4], const uint16_t* vd, float (&o)[D / 8][4]) {
    const int lane = threadIdx.x & 31;
    uint32_t ph[4], pl[4];
    const float* p0 = sc[0];
    const float* p1 = sc[1];
    float v[8] = {p0[0], p0[1], p0[2], p0[3], p1[0], p1[1], p1[2], p1[3]};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float a = v[2 * i], b = v[2 * i + 1];
        const float ah = round_bf(a), bh = round_bf(b);
        ph[i] = pack_bf2(ah, bh);
        pl[i] = pack_bf2(a - ah, b - bh);
    }
    const int key = (lane & 7) + ((lane >> 3) & 1) * 8;
    // A fragment: [0] row g keys 2t.., [1] row g + 8 keys 2t.., [2] row g keys 8 + 2t..,
    // [3] row g + 8 keys 8 + 2t..
    const uint32_t pk[4] = {ph[0], pl[0], ph[2], pl[2]};
#pragma unroll
    for (int dt2 = 0; dt2 < D / 16; ++dt2) {
        uint32_t vb[4];
        ldsm_x4_trans(vb, vd + key * LD + (((dt2 * 2 + (lane >> 4)) ^ (key & 7)) << 3));
        const uint32_t b0[2] = {vb[0], vb[1]}, b1[2] = {vb[2], vb[3]};
        if constexpr (PACK) {
            mma_bf16_16816(o[2 * dt2], pk, b0);
            mma_bf16_16816(o[2 * dt2 + 1], pk, b1);
        } else {
            mma_bf16_16816(o[2 * dt2], ph, b0);
            mma_bf16_16816(o[2 * dt2], pl, b0);
            mma_bf16_16816(o[2 * dt2 + 1], ph, b1);
            mma_bf16_16816(o[2 * dt2 + 1], pl, b1);
        }
    }
}

// S = Q K^T for one 16-key page: Q fragments qf (rows 0..15), K page rows in shared memory
// (swizzled as load_page_warp stores them).
template <int D, int LD>
DEC_DEVINL void qk_page(const uint32_t (&qf)[D / 16][4], const uint16_t* kd, float (&sc)[2][4]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) sc[nt][c] = 0.f;
    const int key = (lane & 7) + (lane >> 4) * 8;
    // even and odd k steps accumulate separately: two dependent chains of D / 32 MMAs per
    // tile instead of one of D / 16
    float s2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t kb[4];
        ldsm_x4(kb, kd + key * LD + (((ks * 2 + ((lane >> 3) & 1)) ^ (key & 7)) << 3));
        const uint32_t b0[2] = {kb[0], kb[1]}, b1[2] = {kb[2], kb[3]};
        mma_bf16_16816((ks & 1) ? s2[0] : sc[0], qf[ks], b0);
        mma_bf16_16816((ks & 1) ? s2[1] : sc[1], qf[ks], b1);
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) sc[nt][c] += s2[nt][c];
}

template <int D, int LD>
DEC_DEVINL void load_q_frags(const uint16_t* qs, uint32_t (&qf)[D / 16][4]) {
    const int lane = threadIdx.x & 31;
    const int row = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) ldsm_x4(qf[ks], qs + row * LD + ks * 16 + (lane >> 4) * 8);
}

// Copy one page (16 rows x D) of K and V of kv head g into shared rows of stride LD (one
// warp). Decode pages are unpadded (LD = D) with the 16-byte chunks of row r stored at
// chunk ^ (r % 8): the 8 rows an ldmatrix phase reads then fall in distinct banks.
template <int D, int LD>
DEC_DEVINL void load_page_warp(const uint16_t* kpool, const uint16_t* vpool, int phys, int nkv, int g,
                               uint16_t* kd, uint16_t* vd) {
    const int lane = threadIdx.x & 31;
    const size_t base = ((size_t)phys * nkv + g) * kPage * D;
    constexpr int CH = kPage * D / 8;  // 16-byte chunks per page
#pragma unroll
    for (int c = lane; c < CH; c += 32) {
        const int row = c / (D / 8), col = (c % (D / 8)) * 8;
        const int sw = (((col >> 3) ^ (row & 7)) << 3);
        cp_async16(kd + row * LD + sw, kpool + base + row * D + col);
        cp_async16(vd + row * LD + sw, vpool + base + row * D + col);
    }
    cp_async_commit();
}

// ================================================================== decode

// Page ring depth per warp: 8-warp CTAs (split contexts, few pages each) keep 2 pages in
// flight per warp, 4-warp CTAs (one CTA per sequence and kv head, many pages) keep 3.
// Shared memory of the decode kernel: the page rings (the warps' partials reuse them after
// the page loop) and, for a cluster merge, the receive area of the rows a CTA finishes. At
// ~110 KB two CTAs fit on an SM, so a 16-CTA cluster can be placed on 8 SMs of a GPC (at
// 1 CTA per SM some 16-CTA clusters waited for a second wave).
template <int D, int NW, int RING>
__host__ __device__ constexpr size_t dec_rings_bytes() {
    const size_t ring = (size_t)NW * RING * 2 * kPage * D * 2;
    const size_t wo = (size_t)NW * 16 * D * 4;
    return ring > wo ? ring : wo;
}

template <int D, int NW, int RING>
__global__ void __launch_bounds__(NW * 32) attn_decode_kernel(AttnDecodeArgs a) {
    constexpr int LD = D + 8;      // q tile rows
    constexpr int PLD = D;         // page rows (chunk-swizzled)
    constexpr int PAGE = kPage * PLD;
    constexpr int LDR = D + 4;  // receive rows: o[D], m, l, 2 pad (16-byte aligned)
    constexpr int NT = NW * 32;
    __shared__ __align__(16) uint16_t qs[16 * LD];
    __shared__ __align__(16) uint16_t newkv[2][D];  // the appended k and v rows (bf16)
    __shared__ float wm[NW][16], wl[NW][16];
    __shared__ __align__(8) uint64_t recv_bar;  // the partials of this CTA's rows have landed
    extern __shared__ __align__(16) uint8_t dyn[];
    uint16_t* kvbuf = reinterpret_cast<uint16_t*>(dyn);  // [NW warps][RING][K,V][16][D]
    float* wo = reinterpret_cast<float*>(dyn);           // [NW][16][D] after the page loop
    // [rows owned][splits][LDR]: every split's partial of the rows this CTA finishes
    float* recv = reinterpret_cast<float*>(dyn + dec_rings_bytes<D, NW, RING>());

    const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z, S = gridDim.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int G = a.nq / a.nkv;
    // Without a scratch buffer the splits of one (sequence, kv head) form a cluster and
    // merge in distributed shared memory. The partials land in a receive area that overlaps
    // the page rings, so a CTA arrives on the cluster barrier only once its page loop is
    // done, and nobody writes into another CTA's shared memory before every CTA has arrived.
    const bool cl = S > 1 && a.part == nullptr;
    __shared__ int ticket_s;
    // At most 8 query heads per group: P_lo rides in the tile's spare rows 8-15 (pv_page).
    const bool pack = G <= 8;
    if (cl) {
        // Each CTA will send its partial rows straight to the CTA finishing them (st.async,
        // completing as transaction bytes on that CTA's recv_bar). The barrier is initialised
        // before this CTA arrives on the cluster barrier; senders wait on it before sending.
        if (tid == 0) {
            mbar_init(&recv_bar, 1);
            fence_mbar_init();
        }
        asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    }

    // ---- independent of the previous kernel: positions, block table and the cache pages
    // (the row being appended is patched in after it is written, below)
    const int p = a.pos[b];
    const int n = p + 1;
    const int kf = a.window > 0 && n > a.window ? n - a.window : 0;  // first attended key
    const int np = (n + kPage - 1) / kPage;
    const int pf = kf / kPage;  // first page with an attended key
    const int pps = (np - pf + S - 1) / S;
    const int pg0 = pf + s * pps, pg1 = min(np, pg0 + pps);
    const int32_t* bt = a.block_table + (size_t)b * a.max_pages;
    const bool has_last = pg0 < pg1 && pg1 == np;
    const float sl2 = a.scale * kLog2e;
    // this warp's pages: pg0 + warp + NW i, i < cnt; the first RING are fetched now. Lane j
    // holds the block-table entry of page i = base + j and of page i = base + 32 + j, so a
    // refill never waits on a block-table load (the next 32 are fetched 32 pages ahead).
    uint16_t* wbuf = kvbuf + (size_t)warp * RING * 2 * PAGE;
    const int cnt = pg0 + warp < pg1 ? (pg1 - pg0 - warp + NW - 1) / NW : 0;
    int bt_base = 0;
    int bt_cur = lane < cnt ? bt[pg0 + warp + NW * lane] : 0;
    int bt_next = lane + 32 < cnt ? bt[pg0 + warp + NW * (lane + 32)] : 0;
    auto page_entry = [&](int i) {  // warp-collective; i grows by one per call
        if (i >= bt_base + 32) {
            bt_base += 32;
            bt_cur = bt_next;
            bt_next = lane + bt_base + 32 < cnt ? bt[pg0 + warp + NW * (lane + bt_base + 32)] : 0;
        }
        return __shfl_sync(0xffffffffu, bt_cur, i - bt_base);
    };
    int issued = 0;
    for (; issued < cnt && issued < RING; ++issued) {
        uint16_t* slot = wbuf + (size_t)issued * 2 * PAGE;
        load_page_warp<D, PLD>(a.k_pool, a.v_pool, page_entry(issued), a.nkv, g, slot, slot + PAGE);
    }
    // the model path's angles and QK-norm gains do not depend on the previous kernel either
    const float2* tab = a.rope_tab ? a.rope_tab + (size_t)p * (D / 2) : nullptr;
    HeadRegs<D> hr;
    const bool regs = a.qkv != nullptr && (tab != nullptr || !a.rope);
    if (regs) load_head_regs<D>(hr, a.rope ? tab : nullptr, a.q_norm, a.k_norm);

    pdl_trigger();
    pdl_wait();
    const bool have_new = a.qkv != nullptr || a.k_new != nullptr;
    const size_t off_p = has_last ? (((size_t)bt[p / kPage] * a.nkv + g) * kPage + (p % kPage)) * D : 0;

    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    const int t4 = lane & 3, gr = lane >> 2;

    if (pg0 < pg1) {
        // ---- q tile of the group (rows >= G are zero); the split holding row p appends it
        for (int r = warp; r < 16; r += NW) {
            uint16_t* dst = qs + r * LD;
            if (r < G) {
                const int h = g * G + r;
                if (regs)
                    head_transform_regs<D>(a.qkv + (size_t)b * a.ld_qkv + (size_t)h * D, hr.qn, a.q_norm != nullptr,
                                           a.eps, a.rope, hr.cs, dst);
                else if (a.qkv)
                    head_transform<D>(a.qkv + (size_t)b * a.ld_qkv + (size_t)h * D, false, nullptr, a.q_norm, a.eps,
                                      a.rope, p, a.rope_base, dst, tab);
                else
                    head_transform<D>(nullptr, true, a.q_bf + ((size_t)b * a.nq + h) * D, nullptr, a.eps, a.rope, p,
                                      a.rope_base, dst);
            } else {
                for (int i = lane; i < D; i += 32) dst[i] = 0;
            }
        }
        if (has_last && have_new && warp < 2) {
            // the new row: k gets QK-norm and RoPE, v is only rounded; staged in shared
            // memory (patched into the page fetched before it existed) and appended to the cache
            if (warp == 0) {
                if (regs)
                    head_transform_regs<D>(a.qkv + (size_t)b * a.ld_qkv + (size_t)(a.nq + g) * D, hr.kn,
                                           a.k_norm != nullptr, a.eps, a.rope, hr.cs, newkv[0]);
                else if (a.qkv)
                    head_transform<D>(a.qkv + (size_t)b * a.ld_qkv + (size_t)(a.nq + g) * D, false, nullptr, a.k_norm,
                                      a.eps, a.rope, p, a.rope_base, newkv[0], tab);
                else
                    head_transform<D>(nullptr, true, a.k_new + ((size_t)b * a.nkv + g) * D, nullptr, a.eps, a.rope, p,
                                      a.rope_base, newkv[0]);
            } else {
                if (a.qkv)
                    head_transform<D>(a.qkv + (size_t)b * a.ld_qkv + (size_t)(a.nq + a.nkv + g) * D, false, nullptr,
                                      nullptr, a.eps, false, p, a.rope_base, newkv[1], tab);
                else
                    head_transform<D>(nullptr, true, a.v_new + ((size_t)b * a.nkv + g) * D, nullptr, a.eps, false, p,
                                      a.rope_base, newkv[1]);
            }
            __syncwarp();
            uint16_t* dst = (warp == 0 ? a.k_pool : a.v_pool) + off_p;
            for (int c = lane * 8; c < D; c += 256)
                *reinterpret_cast<uint4*>(dst + c) = *reinterpret_cast<const uint4*>(&newkv[warp][c]);
        }
        __syncthreads();  // q tile and the staged row are ready

        uint32_t qf[D / 16][4];
        load_q_frags<D, LD>(qs, qf);

        // each warp streams its pages through a RING-page cp.async ring; a slot is refilled
        // as soon as its page has been used
        for (int i = 0; i < cnt; ++i) {
            const int pg = pg0 + warp + NW * i;
            switch (issued - i - 1) {  // groups that may stay in flight
                case 0: cp_async_wait<0>(); break;
                case 1: cp_async_wait<1>(); break;
                case 2: cp_async_wait<2>(); break;
                default: cp_async_wait<3>(); break;
            }
            __syncwarp();
            uint16_t* kd = wbuf + (size_t)(i % RING) * 2 * PAGE;
            if (pg == np - 1 && has_last && have_new) {
                // the page was fetched before row p existed: copy the staged row in
                const int pr = p % kPage;
                uint16_t* row = kd + (lane < 16 ? 0 : PAGE) + pr * PLD;
                for (int c = (lane & 15) * 8; c < D; c += 128)
                    *reinterpret_cast<uint4*>(row + ((((c >> 3) ^ (pr & 7))) << 3)) =
                        *reinterpret_cast<const uint4*>(&newkv[lane >> 4][c]);
                __syncwarp();
            }
            float sc[2][4];
            qk_page<D, PLD>(qf, kd, sc);
            // the softcap test stays outside the loops: the plain path carries no tanh at all
            if (a.softcap > 0.f) {
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int c = 0; c < 4; ++c) sc[nt][c] = score_log2(sc[nt][c], a.scale, a.softcap);
            } else {
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int c = 0; c < 4; ++c) sc[nt][c] *= sl2;
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int key = pg * kPage + nt * 8 + 2 * t4 + (c & 1);
                    if (!(key < n && key >= kf)) sc[nt][c] = -INFINITY;
                }
            float corr[2];
            softmax_page(sc, m, l, corr);
            if (pack) corr[1] = corr[0];  // rows g + 8 hold row g's P_lo products
#pragma unroll
            for (int q = 0; q < D / 8; ++q) {
                o[q][0] *= corr[0];
                o[q][1] *= corr[0];
                o[q][2] *= corr[1];
                o[q][3] *= corr[1];
            }
            if (pack)
                pv_page<D, PLD, true>(sc, kd + PAGE, o);
            else
                pv_page<D, PLD, false>(sc, kd + PAGE, o);
            __syncwarp();
            if (issued < cnt) {
                load_page_warp<D, PLD>(a.k_pool, a.v_pool, page_entry(issued), a.nkv, g, kd, kd + PAGE);
                ++issued;
            }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
            l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
        }
    }
    if (pack) {
        // row g's two terms; rows 8-15 are past the group
#pragma unroll
        for (int q = 0; q < D / 8; ++q) {
            o[q][0] += o[q][2];
            o[q][1] += o[q][3];
        }
    }

    // ---- merge the 4 warps of the CTA through shared memory (a CTA without pages
    // contributes m = -inf, l = 0, o = 0)
    __syncthreads();  // page buffers are free
    if (t4 == 0) {
        wm[warp][gr] = m[0];
        wm[warp][gr + 8] = m[1];
        wl[warp][gr] = l[0];
        wl[warp][gr + 8] = l[1];
    }
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
        float* r0 = wo + ((size_t)warp * 16 + gr) * D + i * 8 + 2 * t4;
        float* r1 = wo + ((size_t)warp * 16 + gr + 8) * D + i * 8 + 2 * t4;
        r0[0] = o[i][0];
        r0[1] = o[i][1];
        r1[0] = o[i][2];
        r1[1] = o[i][3];
    }
    __syncthreads();
    // Split partial of row r: o (relative to M) and M, L. In a cluster row r is finished by
    // CTA r % S, which receives every split's partial of it in slot [r / S][s]; otherwise the
    // partials go to the scratch and the last CTA of (b, g) merges them.
    uint32_t rbar = 0;
    if (cl) {
        asm volatile("barrier.cluster.wait.aligned;" ::: "memory");  // every recv_bar is initialised
    }
    for (int idx = tid; idx < G * (D / 4); idx += NT) {
        const int r = idx / (D / 4), c = (idx % (D / 4)) * 4;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, wm[w][r]);
        float L = 0.f;
        float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            if (wm[w][r] == -INFINITY) continue;
            const float f = exp2f(wm[w][r] - M);
            L += f * wl[w][r];
            const float4 v = *reinterpret_cast<const float4*>(wo + ((size_t)w * 16 + r) * D + c);
            O.x += f * v.x;
            O.y += f * v.y;
            O.z += f * v.z;
            O.w += f * v.w;
        }
        if (S == 1) {
            const float inv = 1.0f / L;
            uint2 pk;
            pk.x = pack_bf2(O.x * inv, O.y * inv);
            pk.y = pack_bf2(O.z * inv, O.w * inv);
            *reinterpret_cast<uint2*>(a.out + (size_t)b * a.nq * D + (size_t)(g * G + r) * D + c) = pk;
        } else if (cl) {
            const int own = r % S;
            const uint32_t dst = dsmem_map(smem_u32(recv + ((size_t)(r / S) * S + s) * LDR), own);
            rbar = dsmem_map(smem_u32(&recv_bar), own);
            st_async_4f(dst + c * 4, O.x, O.y, O.z, O.w, rbar);
            if (c == 0) st_async_2f(dst + D * 4, M, L, rbar);
        } else {
            float* pp = a.part + (((size_t)b * a.nq + g * G + r) * S + s) * (D + 2);
            pp[c] = O.x;
            pp[c + 1] = O.y;
            pp[c + 2] = O.z;
            pp[c + 3] = O.w;
            if (c == 0) {
                pp[D] = M;
                pp[D + 1] = L;
            }
        }
    }
    if (S == 1) return;

    if (cl) {
        // ---- rows r = s, s + S, ...: weighted sum over the splits in split order
        const int owned = s < G ? (G - 1 - s) / S + 1 : 0;
        if (owned == 0) return;  // nothing reads this CTA's shared memory
        if (tid == 0) mbar_arrive_expect_tx(&recv_bar, (uint32_t)(owned * S * (D * 4 + 8)));
        const bool got = mbar_wait_cluster_bounded(&recv_bar, 0, a.err);
        for (int j = 0; j < owned; ++j) {
            const int r = s + j * S;
            const float* rv = recv + (size_t)j * S * LDR;
            // (unrolled to the cluster bound: the split weights are computed once per row,
            // and the loads of every split are in flight together)
            float mz[kDecodeMaxSplits], wz[kDecodeMaxSplits];
            float M = -INFINITY;
#pragma unroll
            for (int z = 0; z < kDecodeMaxSplits; ++z) {
                mz[z] = z < S ? rv[(size_t)z * LDR + D] : -INFINITY;
                M = fmaxf(M, mz[z]);
            }
            float L = 0.f;
#pragma unroll
            for (int z = 0; z < kDecodeMaxSplits; ++z) {
                wz[z] = mz[z] != -INFINITY ? exp2f(mz[z] - M) : 0.f;
                if (mz[z] != -INFINITY) L += wz[z] * rv[(size_t)z * LDR + D + 1];
            }
            const float invL = 1.0f / L;
            for (int c = tid; c < D; c += NT) {
                float O = 0.f;
#pragma unroll
                for (int z = 0; z < kDecodeMaxSplits; ++z)
                    if (mz[z] != -INFINITY) O += wz[z] * rv[(size_t)z * LDR + c];
                if (got) a.out[(size_t)b * a.nq * D + (size_t)(g * G + r) * D + c] = f2bf(O * invL);
            }
        }
        return;
    }

    // ---- the last CTA of (b, g) merges the splits in split order
    __threadfence();
    __syncthreads();
    if (tid == 0) ticket_s = atomicAdd(&a.counters[b * a.nkv + g], 1);
    __syncthreads();
    if (ticket_s != S - 1) return;
    __threadfence();
    // weights of each split: f_z = exp2(m_z - M) / sum_z exp2(m_z - M) l_z (one warp per head)
    float* fz = reinterpret_cast<float*>(kvbuf);  // [G][splits]
    for (int r = warp; r < G; r += NW) {
        const float* pp = a.part + ((size_t)b * a.nq + g * G + r) * S * (D + 2);
        float M = -INFINITY;
        for (int z = lane; z < S; z += 32) M = fmaxf(M, __ldcg(pp + (size_t)z * (D + 2) + D));
        M = warp_max(M);
        float L = 0.f;
        for (int z = lane; z < S; z += 32) {
            const float mz = __ldcg(pp + (size_t)z * (D + 2) + D);
            const float f = mz == -INFINITY ? 0.f : exp2f(mz - M);
            fz[r * S + z] = f;
            L += f * __ldcg(pp + (size_t)z * (D + 2) + D + 1);
        }
        L = warp_sum(L);
        __syncwarp();
        for (int z = lane; z < S; z += 32) fz[r * S + z] /= L;
    }
    __syncthreads();
    // weighted sum over splits in split order; loads of one split are coalesced across threads
    for (int idx = tid; idx < G * D; idx += NT) {
        const int r = idx / D, c = idx % D;
        const int h = g * G + r;
        const float* pp = a.part + ((size_t)b * a.nq + h) * S * (D + 2) + c;
        const float* f = fz + r * S;
        float O = 0.f;
        int z = 0;
        for (; z + 4 <= S; z += 4) {
            const float p0 = __ldcg(pp + (size_t)z * (D + 2)), p1 = __ldcg(pp + (size_t)(z + 1) * (D + 2));
            const float p2 = __ldcg(pp + (size_t)(z + 2) * (D + 2)), p3 = __ldcg(pp + (size_t)(z + 3) * (D + 2));
            O += f[z] * p0;
            O += f[z + 1] * p1;
            O += f[z + 2] * p2;
            O += f[z + 3] * p3;
        }
        for (; z < S; ++z) O += f[z] * __ldcg(pp + (size_t)z * (D + 2));
        a.out[(size_t)b * a.nq * D + (size_t)h * D + c] = f2bf(O);
    }
    if (tid == 0) a.counters[b * a.nkv + g] = 0;
}

// ================================================================== prefill: rotate + append

template <int D>
__global__ void __launch_bounds__(128) rope_append_kernel(RopeAppendArgs a) {
    const int t = blockIdx.x;
    const int warp = threadIdx.x >> 5;
    pdl_trigger();
    pdl_wait();
    const int p = a.pos0 + t;
    const float* row = a.qkv + (size_t)t * a.ld_qkv;
    const int phys = a.block_row[p / kPage];
    const int slot = p % kPage;
    const int nh = a.nq + 2 * a.nkv;
    const float2* tab = a.rope_tab ? a.rope_tab + (size_t)p * (D / 2) : nullptr;
    for (int hh = blockIdx.y * 4 + warp; hh < nh; hh += 4 * gridDim.y) {
        if (hh < a.nq) {
            head_transform<D>(row + (size_t)hh * D, false, nullptr, a.q_norm, a.eps, true, p, a.rope_base,
                              a.q_out + ((size_t)t * a.nq + hh) * D, tab);
        } else if (hh < a.nq + a.nkv) {
            const int j = hh - a.nq;
            head_transform<D>(row + (size_t)hh * D, false, nullptr, a.k_norm, a.eps, true, p, a.rope_base,
                              a.k_pool + (((size_t)phys * a.nkv + j) * kPage + slot) * D, tab);
        } else {
            const int j = hh - a.nq - a.nkv;
            head_transform<D>(row + (size_t)hh * D, false, nullptr, nullptr, a.eps, false, p, a.rope_base,
                              a.v_pool + (((size_t)phys * a.nkv + j) * kPage + slot) * D);
        }
    }
}

// ================================================================== prefill attention

constexpr int kPrefRows = 64;      // (token, head) rows per CTA: 4 warps x 16
constexpr int kPrefKeys = 64;      // keys per shared block (4 pages)
constexpr int kPrefMaxSplits = 8;  // key splits of one row block: the CTAs of one cluster

// K and V blocks, double-buffered, rows padded to D + 8 (conflict-free ldmatrix).
template <int D>
constexpr size_t prefill_smem() {
    return (size_t)2 * 2 * kPrefKeys * (D + 8) * 2;
}

// S = Q K^T for one 64-key block: sc[nt] holds keys 8 nt .. 8 nt + 7 of the block.
template <int D, int LD>
DEC_DEVINL void qk_block(const uint32_t (&qf)[D / 16][4], const uint16_t* kd, float (&sc)[8][4]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
    const int key = (lane & 7) + (lane >> 4) * 8;
    const int col = ((lane >> 3) & 1) * 8;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
        for (int kp = 0; kp < 4; ++kp) {
            uint32_t kb[4];
            ldsm_x4(kb, kd + (kp * 16 + key) * LD + ks * 16 + col);
            const uint32_t b0[2] = {kb[0], kb[1]}, b1[2] = {kb[2], kb[3]};
            mma_bf16_16816(sc[2 * kp], qf[ks], b0);
            mma_bf16_16816(sc[2 * kp + 1], qf[ks], b1);
        }
    }
}

// Online-softmax update over one 64-key block (log2 units; masked entries -inf).
// Rows g (r = 0) and g + 8 (r = 1) of the warp's 16; the quad's four threads hold
// the block's 64 columns of a row. Returns P in sc and the rescale factor of o.
DEC_DEVINL void softmax_block(float (&sc)[8][4], float (&m)[2], float (&l)[2], float (&corr)[2]) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        float mx = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) mx = fmaxf(mx, fmaxf(sc[nt][2 * r], sc[nt][2 * r + 1]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float mn = fmaxf(m[r], mx);
        if (mn == -INFINITY) {  // every key so far masked for this row
            corr[r] = 1.f;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) sc[nt][2 * r] = sc[nt][2 * r + 1] = 0.f;
            continue;
        }
        corr[r] = exp2f(m[r] - mn);
        m[r] = mn;
        float sum = 0.f;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const float p = exp2f(sc[nt][2 * r + c] - mn);
                sc[nt][2 * r + c] = p;
                sum += p;
            }
        l[r] = l[r] * corr[r] + sum;
    }
}

// O += P V for one 64-key block; P enters as bf16 hi + lo parts.
template <int D, int LD>
DEC_DEVINL void pv_block(const float (&sc)[8][4], const uint16_t* vd, float (&o)[D / 8][4]) {
    const int lane = threadIdx.x & 31;
    const int key = (lane & 7) + ((lane >> 3) & 1) * 8;
    const int col = (lane >> 4) * 8;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float v[8] = {sc[2 * j][0],     sc[2 * j][1],     sc[2 * j][2],     sc[2 * j][3],
                            sc[2 * j + 1][0], sc[2 * j + 1][1], sc[2 * j + 1][2], sc[2 * j + 1][3]};
        uint32_t ph[4], pl[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float x = v[2 * i], y = v[2 * i + 1];
            const float xh = round_bf(x), yh = round_bf(y);
            ph[i] = pack_bf2(xh, yh);
            pl[i] = pack_bf2(x - xh, y - yh);
        }
#pragma unroll
        for (int dt2 = 0; dt2 < D / 16; ++dt2) {
            uint32_t vb[4];
            ldsm_x4_trans(vb, vd + (j * 16 + key) * LD + dt2 * 16 + col);
            const uint32_t b0[2] = {vb[0], vb[1]}, b1[2] = {vb[2], vb[3]};
            mma_bf16_16816(o[2 * dt2], ph, b0);
            mma_bf16_16816(o[2 * dt2 + 1], ph, b1);
            mma_bf16_16816(o[2 * dt2], pl, b0);
            mma_bf16_16816(o[2 * dt2 + 1], pl, b1);
        }
    }
}

// One CTA: 64 (token, head) rows of kv head g -- row r is token r / G, head g G + r % G --
// against key split blockIdx.z of the keys those rows may see. With several splits the
// split CTAs form one cluster: after the key loop each pushes its unnormalised rows
// (o, running max m, sum l) into the shared memory of the CTA that owns the row, and
// the owners merge the splits in rank order.
template <int D>
__global__ void __launch_bounds__(128, 3) attn_prefill_kernel(AttnPrefillArgs a) {
    constexpr int LD = D + 8;
    extern __shared__ __align__(16) uint8_t dyn[];
    uint16_t* kb = reinterpret_cast<uint16_t*>(dyn);  // [2][64][LD]
    uint16_t* vb = kb + 2 * kPrefKeys * LD;           // [2][64][LD]

    // row blocks in reverse: under the causal mask the last rows see the most keys, so the
    // longest CTAs are dispatched first and the shortest fill the tail
    const int qb = gridDim.x - 1 - blockIdx.x, g = blockIdx.y, s = blockIdx.z, S = gridDim.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int G = a.nq / a.nkv;
    const int R = a.T * G;
    pdl_trigger();
    pdl_wait();

    const int rbase = qb * kPrefRows;
    const int t_last = min(a.T - 1, (rbase + kPrefRows - 1) / G);
    const int n_cta = a.pos0 + t_last + 1;  // keys any row of this CTA may see
    const int W = a.window;
    // with a window, the first key any row of this CTA may see (its first row's window start)
    const int kf_cta = W > 0 ? max(0, a.pos0 + rbase / G - W + 1) : 0;
    const int nblk = (n_cta + kPrefKeys - 1) / kPrefKeys;
    const int bf = kf_cta / kPrefKeys;
    const int bps = (nblk - bf + S - 1) / S;
    const int blk0 = bf + s * bps, blk1 = min(nblk, blk0 + bps);

    // this thread's rows (g and g + 8 of the warp's 16) and their last visible key
    const int r0 = rbase + warp * 16;
    const int gr = lane >> 2, t4 = lane & 3;
    const int ra = r0 + gr, rb = r0 + gr + 8;
    const int lim_a = ra < R ? a.pos0 + ra / G : -1;
    const int lim_b = rb < R ? a.pos0 + rb / G : -1;
    const int warp_hi = r0 < R ? a.pos0 + min(R - 1, r0 + 15) / G : -1;  // largest limit of the warp
    const int warp_lo = r0 + 15 < R ? a.pos0 + r0 / G : -1;              // smallest (-1: padding rows)
    // with a window: keys below wlo_min are outside every row's window, keys from wlo_max on
    // inside every row's window
    const int wlo_min = W > 0 && r0 < R ? a.pos0 + r0 / G - W + 1 : 0;
    const int wlo_max = W > 0 ? warp_hi - W + 1 : 0;

    // Q fragments straight from global memory (A layout of m16n8k16)
    uint32_t qf[D / 16][4];
    {
        const uint32_t* qa = ra < R ? reinterpret_cast<const uint32_t*>(
                                          a.q + ((size_t)(ra / G) * a.nq + g * G + ra % G) * D)
                                    : nullptr;
        const uint32_t* qbp = rb < R ? reinterpret_cast<const uint32_t*>(
                                           a.q + ((size_t)(rb / G) * a.nq + g * G + rb % G) * D)
                                     : nullptr;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            qf[ks][0] = qa ? __ldg(qa + ks * 8 + t4) : 0u;
            qf[ks][1] = qbp ? __ldg(qbp + ks * 8 + t4) : 0u;
            qf[ks][2] = qa ? __ldg(qa + ks * 8 + 4 + t4) : 0u;
            qf[ks][3] = qbp ? __ldg(qbp + ks * 8 + 4 + t4) : 0u;
        }
    }

    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    const float sl2 = a.scale * kLog2e;

    // keys at or past n_cta are not read: their rows are zero-filled (weight 0, finite)
    auto load_block = [&](int blk, int buf) {
        uint16_t* kd = kb + buf * kPrefKeys * LD;
        uint16_t* vd = vb + buf * kPrefKeys * LD;
        constexpr int CH = kPrefKeys * D / 8;
        for (int c = tid; c < CH; c += 128) {
            const int key = c / (D / 8), col = (c % (D / 8)) * 8;
            const int kg = blk * kPrefKeys + key;
            if (kg < n_cta) {
                const int phys = a.block_row[kg / kPage];
                const size_t off = (((size_t)phys * a.nkv + g) * kPage + kg % kPage) * D + col;
                cp_async16(kd + key * LD + col, a.k_pool + off);
                cp_async16(vd + key * LD + col, a.v_pool + off);
            } else {
                *reinterpret_cast<uint4*>(kd + key * LD + col) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4*>(vd + key * LD + col) = make_uint4(0, 0, 0, 0);
            }
        }
        cp_async_commit();
    };

    int buf = 0;
    if (blk0 < blk1) load_block(blk0, 0);
    for (int blk = blk0; blk < blk1; ++blk) {
        if (blk + 1 < blk1) {
            load_block(blk + 1, buf ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const int k0 = blk * kPrefKeys;
        // else every key of the block is masked for this warp's rows (past the causal edge,
        // or before every row's window)
        if (k0 <= warp_hi && k0 + kPrefKeys - 1 >= wlo_min) {
            float sc[8][4];
            qk_block<D, LD>(qf, kb + buf * kPrefKeys * LD, sc);
            if (a.softcap > 0.f) {
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int c = 0; c < 4; ++c) sc[nt][c] = score_log2(sc[nt][c], a.scale, a.softcap);
            } else {
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int c = 0; c < 4; ++c) sc[nt][c] *= sl2;
            }
            // the causal edge (or padding rows), or a window start, crosses the block
            if (k0 + kPrefKeys - 1 > warp_lo || (W > 0 && k0 < wlo_max)) {
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int key = k0 + nt * 8 + 2 * t4 + (c & 1);
                        const int lim = c < 2 ? lim_a : lim_b;
                        if (key > lim || (W > 0 && key <= lim - W)) sc[nt][c] = -INFINITY;
                    }
            }
            float corr[2];
            softmax_block(sc, m, l, corr);
#pragma unroll
            for (int i = 0; i < D / 8; ++i) {
                o[i][0] *= corr[0];
                o[i][1] *= corr[0];
                o[i][2] *= corr[1];
                o[i][3] *= corr[1];
            }
            pv_block<D, LD>(sc, vb + buf * kPrefKeys * LD, o);
        }
        __syncthreads();  // buffer reuse
        buf ^= 1;
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
        l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
    }

    if (S == 1) {
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int r = hr == 0 ? ra : rb;
            if (r >= R) continue;
            const int t = r / G, h = g * G + r % G;
            const float inv = 1.0f / l[hr];
            uint32_t* dst = reinterpret_cast<uint32_t*>(a.out + (size_t)t * a.nq * D + (size_t)h * D);
#pragma unroll
            for (int i = 0; i < D / 8; ++i) dst[i * 4 + t4] = pack_bf2(o[i][2 * hr] * inv, o[i][2 * hr + 1] * inv);
        }
        return;
    }

    // ---- split merge inside the cluster; the K/V buffers become the receive area
    constexpr int LDR = D + 4;  // o[D], m, l, 2 pad: 16-byte aligned rows
    const int rp = (kPrefRows + S - 1) / S;  // rows owned by each CTA of the cluster
    const int rank = (int)cluster_rank();
    float* recv = reinterpret_cast<float*>(dyn);  // [S][rp][LDR]
    cluster_sync();  // every CTA's key loop is done before partials land in its buffers
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        const int lr = warp * 16 + gr + 8 * hr;
        const int owner = lr / rp, orow = lr - owner * rp;
        const uint32_t dst = smem_u32(recv + ((size_t)rank * rp + orow) * LDR);
#pragma unroll
        for (int i = 0; i < D / 8; ++i) dsmem_st2f(dst + (i * 8 + 2 * t4) * 4, owner, o[i][2 * hr], o[i][2 * hr + 1]);
        if (t4 == 0) dsmem_st2f(dst + D * 4, owner, m[hr], l[hr]);
    }
    cluster_sync();  // all partials have arrived; only local shared memory is read below
    const int lr0 = rank * rp, nr = min(kPrefRows, lr0 + rp) - lr0;
    for (int idx = tid; idx < nr * (D / 4); idx += 128) {
        const int orow = idx / (D / 4), c4 = (idx % (D / 4)) * 4;
        const int r = rbase + lr0 + orow;
        if (r >= R) continue;
        float M = -INFINITY;
        for (int z = 0; z < S; ++z) M = fmaxf(M, recv[((size_t)z * rp + orow) * LDR + D]);
        float L = 0.f;
        float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int z = 0; z < S; ++z) {
            const float* pz = recv + ((size_t)z * rp + orow) * LDR;
            const float mz = pz[D];
            if (mz == -INFINITY) continue;
            const float f = exp2f(mz - M);
            L += f * pz[D + 1];
            const float4 v = *reinterpret_cast<const float4*>(pz + c4);
            O.x += f * v.x;
            O.y += f * v.y;
            O.z += f * v.z;
            O.w += f * v.w;
        }
        const float inv = 1.0f / L;
        const int t = r / G, h = g * G + r % G;
        uint2 pk;
        pk.x = pack_bf2(O.x * inv, O.y * inv);
        pk.y = pack_bf2(O.z * inv, O.w * inv);
        *reinterpret_cast<uint2*>(a.out + (size_t)t * a.nq * D + (size_t)h * D + c4) = pk;
    }
}

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

}  // namespace

// One wave of (sequence, kv head, split) CTAs, each split at least 8 pages long; merged
// in a cluster, at most kDecodeMaxSplits (the CTAs of one cluster).
int attn_decode_splits(int B, int nkv, int max_ctx, int num_sms, bool cluster) {
    const int ctas = B * nkv;
    int s = (num_sms + ctas - 1) / ctas;
    const int pages = (max_ctx + kPage - 1) / kPage;
    const int max_s = (pages + 7) / 8;
    if (s > max_s) s = max_s;
    if (cluster && s > kDecodeMaxSplits) s = kDecodeMaxSplits;
    if (s < 1) s = 1;
    return s;
}

template <int D, int NW, int RING>
size_t decode_smem(int G, int splits, bool cl) {
    size_t sm = dec_rings_bytes<D, NW, RING>();
    if (cl) sm += (size_t)((G + splits - 1) / splits) * splits * (D + 4) * 4;  // receive area
    return sm;
}

template <int D, int NW, int RING>
cudaError_t decode_launch_dw(const AttnDecodeArgs& a, cudaStream_t st, bool pdl) {
    const int G = a.nq / a.nkv;
    const bool cl = a.splits > 1 && a.part == nullptr;
    const size_t smem = decode_smem<D, NW, RING>(G, a.splits, cl);
    auto kern = attn_decode_kernel<D, NW, RING>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), (int)smem);
    if (e != cudaSuccess) return e;
    if (cl && a.splits > 8) {
        static std::once_flag once;
        static cudaError_t ce = cudaSuccess;
        std::call_once(once, [] {
            ce = cudaFuncSetAttribute(attn_decode_kernel<D, NW, RING>, cudaFuncAttributeNonPortableClusterSizeAllowed,
                                      1);
        });
        if (ce != cudaSuccess) return ce;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.splits, a.nkv, a.B);
    cfg.blockDim = dim3(NW * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (cl) {  // the splits of a (sequence, kv head) merge inside one cluster
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = a.splits;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

// How many clusters of S CTAs of attn_decode_kernel<D, 4, 4> the device holds at once (GPCs
// hold whole clusters, so at one CTA per SM this can be below SMs / S). Cached per device,
// group size and S.
template <int D>
int decode_resident(int G, int S) {
    static std::mutex mu;
    static std::map<std::tuple<int, int, int>, int> known;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_tuple(dev, G, S);
    auto it = known.find(key);
    if (it != known.end()) return it->second;
    int n = 0;
    auto kern = attn_decode_kernel<D, 4, 4>;
    const size_t smem = decode_smem<D, 4, 4>(G, S, true);
    bool ok = ensure_smem(reinterpret_cast<const void*>(kern), (int)smem) == cudaSuccess;
    if (ok && S > 8) ok = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
    if (ok) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(S, 8, 1);
        cfg.blockDim = dim3(128);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = S;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();  // a refused query leaves no error behind
    known[key] = n;
    return n;
}

// 4 warps. Split contexts merged in a cluster get 4-page rings at one CTA per SM (every
// page of a split of up to 16 pages is in flight before the wait on the previous kernel,
// and no warp shares its scheduler with another CTA's), with the largest split count whose
// clusters are all resident at once; otherwise 3-page rings, two CTAs per SM. (8 warps
// with 2-page rings measured slower at batch 1: 20.8 against 11-13 us per launch of the
// Llama-3-8B shape. 16-CTA clusters at one CTA per SM: one of the 8 waited for a second
// wave.)
template <int D>
cudaError_t decode_launch_d(const AttnDecodeArgs& a, cudaStream_t st, bool pdl) {
    if (a.splits > 1 && a.part == nullptr) {
        const int G = a.nq / a.nkv, clusters = a.B * a.nkv;
        for (int S = a.splits; S >= 2; --S) {
            if (decode_resident<D>(G, S) >= clusters) {
                AttnDecodeArgs b = a;
                b.splits = S;
                return decode_launch_dw<D, 4, 4>(b, st, pdl);
            }
        }
    }
    return decode_launch_dw<D, 4, 3>(a, st, pdl);
}

cudaError_t attn_decode_launch(const AttnDecodeArgs& a, cudaStream_t st, bool pdl) {
    if (a.splits < 1 || a.nkv <= 0 || a.nq % a.nkv != 0 || a.nq / a.nkv > 16) return cudaErrorInvalidValue;
    if (a.splits > 1 && a.part == nullptr && a.splits > kDecodeMaxSplits) return cudaErrorInvalidValue;
    // the scratch merge keeps [G][splits] weights in the page rings
    if ((size_t)(a.nq / a.nkv) * a.splits * 4 > dec_rings_bytes<64, 4, 3>()) return cudaErrorInvalidValue;
    if (a.d == 128) return decode_launch_d<128>(a, st, pdl);
    if (a.d == 64) return decode_launch_d<64>(a, st, pdl);
    return cudaErrorInvalidValue;
}

cudaError_t rope_append_launch(const RopeAppendArgs& a, cudaStream_t st, bool pdl) {
    if (a.T <= 0) return cudaSuccess;
    // one (token, 4 heads) per CTA: each warp transforms one head, so a head costs one memory
    // round trip instead of a warp walking a dozen heads one after another
    const dim3 grid(a.T, (a.nq + 2 * a.nkv + 3) / 4);
    if (a.d == 128) return launch_ex(rope_append_kernel<128>, grid, dim3(128), 0, st, pdl, a);
    if (a.d == 64) return launch_ex(rope_append_kernel<64>, grid, dim3(128), 0, st, pdl, a);
    return cudaErrorInvalidValue;
}

// Key splits per 64-row block so that the grid fills about one wave at three CTAs per SM;
// at most one split per 64-key block and at most a portable cluster (8).
int attn_prefill_splits(int T, int nq, int nkv, int ctx, int num_sms) {
    const int G = nq / nkv;
    const int qblocks = (T * G + kPrefRows - 1) / kPrefRows;
    const int ctas = qblocks * nkv;
    int s = (3 * num_sms) / ctas;
    const int blocks = (ctx + kPrefKeys - 1) / kPrefKeys;
    if (s > blocks) s = blocks;
    if (s > kPrefMaxSplits) s = kPrefMaxSplits;
    if (s < 1) s = 1;
    return s;
}

template <int D>
cudaError_t prefill_launch_d(const AttnPrefillArgs& a, cudaStream_t st, bool pdl) {
    const int G = a.nq / a.nkv;
    const int qblocks = (a.T * G + kPrefRows - 1) / kPrefRows;
    const size_t smem = prefill_smem<D>();
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(attn_prefill_kernel<D>), (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(qblocks, a.nkv, a.splits);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (a.splits > 1) {  // the key splits of a row block form one cluster (merge through DSMEM)
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = 1;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = a.splits;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, attn_prefill_kernel<D>, a);
}

cudaError_t attn_prefill_launch(const AttnPrefillArgs& a, cudaStream_t st, bool pdl) {
    if (a.T <= 0) return cudaSuccess;
    if (attn_prefill_tc_ok(a)) return attn_prefill_tc_launch(a, st, pdl);
    if (a.splits < 1 || a.splits > kPrefMaxSplits) return cudaErrorInvalidValue;
    if (a.d == 128) return prefill_launch_d<128>(a, st, pdl);
    if (a.d == 64) return prefill_launch_d<64>(a, st, pdl);
    return cudaErrorInvalidValue;
}

}  // namespace dec
