"""Parity of the standalone hot-path entry points (weight_gemv, gqa_decode_attn,
moe_route_topk) with the CPU oracle, through the C ABI, on seeded inputs."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
import decoder_only_transformer_layer_b200 as dec
from _util import assert_parity, bits_to_f64, build_paged, from_dev_bf16, gather_paged, max_err, to_dev_bf16

pytestmark = pytest.mark.gpu

# fp32 accumulation of exact bf16 products: relative error far below this bar
KERNEL_REL = 2e-5

GEMV_CASES = [(1, 6152, 4096), (1, 1000, 688), (1, 4100, 576), (2, 517, 1408), (3, 999, 2048), (4, 300, 14336),
              (8, 256, 576), (8, 129, 4096), (1, 9, 64)]
GEMM_CASES = [(9, 300, 704), (16, 1024, 4096), (32, 777, 2048), (64, 1500, 1408), (100, 640, 576),
              (128, 6144, 4096), (160, 2100, 448), (256, 512, 1024), (33, 129, 14336), (300, 1000, 2048),
              (512, 768, 4096)]
# one column tile and few row tiles: the cluster split-K path (S = 3, 4, 4, 8 CTAs per tile;
# a ragged last row tile; column tiles of 32, 64 and 128 tokens)
SPLITK_CASES = [(128, 4096, 4096), (128, 4096, 14336), (32, 6144, 4096), (64, 4100, 4096), (16, 2048, 4096),
                (128, 2048, 2048)]


@pytest.mark.parametrize("B,N,K", GEMV_CASES + GEMM_CASES + SPLITK_CASES)
def test_weight_gemv_matches_oracle(B, N, K):
    W = synth.bf16_normal((N, K), 1, N * 7 + K, 0.0, 0.02)
    x = synth.bf16_normal((B, K), 2, B * 13 + K, 0.0, 1.0)
    ref = oracle.gemv_rows(W, x)
    y = torch.full((B, N), float("nan"), device="cuda")
    dec.weight_gemv(to_dev_bf16(W, torch), to_dev_bf16(x, torch), y)
    torch.cuda.synchronize()
    got = y.cpu().numpy()
    d, r = assert_parity(got, ref, what=f"gemv B={B} N={N} K={K}")
    assert r <= KERNEL_REL, f"kernel-level bar: rel={r:.2e}"


def test_weight_gemv_repeatable_bitwise():
    W = synth.bf16_normal((2000, 4096), 3, 1, 0.0, 0.02)
    for B in (1, 64):
        x = synth.bf16_normal((B, 4096), 4, B, 0.0, 1.0)
        Wd, xd = to_dev_bf16(W, torch), to_dev_bf16(x, torch)
        outs = []
        for _ in range(3):
            y = torch.zeros((B, 2000), device="cuda")
            dec.weight_gemv(Wd, xd, y)
            outs.append(y.cpu().numpy())
        assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[1], outs[2])


def _attn_case(B, nq, nkv, d, pos, rope, new, seed, base=10000.0):
    ctx = int(max(pos)) + 1
    q = synth.bf16_normal((B, nq, d), seed, 1, 0.0, 1.0)
    kc = synth.bf16_normal((B, ctx, nkv, d), seed, 2, 0.0, 1.0)
    vc = synth.bf16_normal((B, ctx, nkv, d), seed, 3, 0.0, 1.0)
    kn = synth.bf16_normal((B, nkv, d), seed, 4, 0.0, 1.0) if new else None
    vn = synth.bf16_normal((B, nkv, d), seed, 5, 0.0, 1.0) if new else None
    kpool, vpool, bt = build_paged(kc, vc, 16, seed)
    scale = 1.0 / math.sqrt(d)
    posa = np.asarray(pos, np.int32)
    ko, vo = kc.copy(), vc.copy()
    ref = oracle.gqa_decode(q, kn, vn, ko, vo, posa, nq, nkv, d, scale, rope, base)
    kp, vp = to_dev_bf16(kpool, torch), to_dev_bf16(vpool, torch)
    out = torch.zeros((B, nq, d), dtype=torch.bfloat16, device="cuda")
    dec.gqa_decode_attn(to_dev_bf16(q, torch), None if kn is None else to_dev_bf16(kn, torch),
                        None if vn is None else to_dev_bf16(vn, torch), kp, vp,
                        torch.from_numpy(bt).cuda(), torch.from_numpy(posa).cuda(), nq, nkv, d, scale, rope, base, out)
    torch.cuda.synchronize()
    got = bits_to_f64(from_dev_bf16(out))
    return got, ref, (from_dev_bf16(kp), from_dev_bf16(vp), bt, ko, vo, ctx)


def _check_attn(got, ref, what, rope=False):
    assert_parity(got, ref, what=what)
    # output is bf16: every element within one bf16 quantum of the exact value
    q = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    if rope:
        # Fused RoPE rotates q and the new key in fp32 here and in fp64 in the oracle; a
        # rotated element rounded to bf16 can land one ulp (2^-8 relative) apart, which moves
        # every score of that head by up to about 2^-8 of one product term, and the output by
        # a small fraction of its scale: allow 2^-6 of the largest output on top.
        q = q + 2.0 ** -6 * np.max(np.abs(ref))
    assert np.all(np.abs(got - ref) <= q + 1e-6), f"{what}: beyond one bf16 quantum"


@pytest.mark.parametrize("rope,new", [(0, 0), (1, 1), (0, 1), (1, 0)])
def test_gqa_decode_small_ragged(rope, new):
    got, ref, (kp, vp, bt, ko, vo, ctx) = _attn_case(3, 8, 2, 128, [0, 17, 300], rope, new, 11)
    _check_attn(got, ref, f"rope={rope} new={new}", rope=bool(rope))
    if new:  # the appended rows landed in the right page slots, rotated and rounded like the oracle's
        kg, vg = gather_paged(kp, bt, ctx), gather_paged(vp, bt, ctx)
        for b, p in enumerate([0, 17, 300]):
            assert np.array_equal(vg[b, p], vo[b, p])
            dk = np.abs(bits_to_f64(kg[b, p]) - bits_to_f64(ko[b, p]))
            assert np.all(dk <= np.abs(bits_to_f64(ko[b, p])) * 2 ** -7 + 1e-30)
            assert np.array_equal(kg[b, :p], ko[b, :p])


@pytest.mark.parametrize("nq,nkv,d,pos", [(16, 16, 128, [300]), (16, 16, 128, [2046]), (16, 1, 64, [300, 999]),
                                          (8, 1, 128, [513]), (4, 2, 128, [1500, 7])])
def test_gqa_decode_group_sizes(nq, nkv, d, pos):
    # groups of 1 (Qwen1.5-MoE shape), 2, 8 and 16 query heads per kv head, over 1 to 16 splits
    got, ref, _ = _attn_case(len(pos), nq, nkv, d, pos, 1, 1, 13)
    _check_attn(got, ref, f"G={nq // nkv} d={d} pos={pos}", rope=True)


def test_gqa_decode_head_dim_64_group_3():
    got, ref, _ = _attn_case(2, 9, 3, 64, [40, 1000], 1, 1, 12)
    _check_attn(got, ref, "d=64 G=3", rope=True)


def test_gqa_decode_mha_and_group_16():
    got, ref, _ = _attn_case(2, 4, 4, 128, [5, 100], 1, 1, 13)
    _check_attn(got, ref, "MHA", rope=True)
    got, ref, _ = _attn_case(1, 32, 2, 128, [777], 1, 1, 14, base=500000.0)
    _check_attn(got, ref, "G=16", rope=True)


def test_gqa_decode_empty_splits_after_another_shape():
    # Split partials live in scratch that keeps an earlier call's contents; a split with no
    # pages must not let those values into the merge (0 * -inf is NaN).
    _attn_case(3, 8, 2, 128, [0, 17, 300], 1, 1, 11)
    for pos in ([40, 1000], [3, 1000], [1000, 0]):
        got, ref, _ = _attn_case(2, 9, 3, 64, pos, 1, 1, 21)
        _check_attn(got, ref, f"d=64 after d=128, pos={pos}", rope=True)


# The attention sweep: B = 64, 32 q / 8 kv heads, d = 128, page 16, at every context of the
# sweep, with the new row appended and q / k rotated in the kernel (rope = 1) or used as
# given (rope = 0). The whole launch runs at full size; the oracle checks every sequence up
# to context 2048, 8 of them at 8192 and 4 at 32768.
SWEEP = [(ctx, rope) for ctx in (512, 2048, 8192, 32768) for rope in (1, 0)]


@pytest.mark.parametrize("ctx,rope", SWEEP)
def test_gqa_decode_sweep(ctx, rope):
    B, nq, nkv, d = 64, 32, 8, 128
    gen = torch.Generator(device="cuda").manual_seed(16 + ctx + rope)  # seeded N(0,1) fill, made on the device
    kpool = torch.randn((B * ctx // 16, nkv, 16, d), device="cuda", generator=gen).to(torch.bfloat16)
    vpool = torch.randn((B * ctx // 16, nkv, 16, d), device="cuda", generator=gen).to(torch.bfloat16)
    rng = np.random.default_rng(ctx + rope)
    bt = rng.permutation(B * ctx // 16).astype(np.int32).reshape(B, ctx // 16)
    q = torch.randn((B, nq, d), device="cuda", generator=gen).to(torch.bfloat16)
    kn = torch.randn((B, nkv, d), device="cuda", generator=gen).to(torch.bfloat16)
    vn = torch.randn((B, nkv, d), device="cuda", generator=gen).to(torch.bfloat16)
    pos = np.full(B, ctx - 1, np.int32)
    sample = tuple(range(B)) if ctx <= 2048 else (0, 9, 21, 30, 42, 50, 57, 63) if ctx <= 8192 else (0, 21, 42, 63)
    local = np.arange(ctx // 16, dtype=np.int32)[None, :]
    before = {}
    for b in sample:  # the oracle's inputs are taken before the kernel runs
        rows = torch.from_numpy(bt[b].astype(np.int64)).cuda()
        before[b] = (from_dev_bf16(kpool[rows].contiguous()), from_dev_bf16(vpool[rows].contiguous()))
    qb, knb, vnb = from_dev_bf16(q), from_dev_bf16(kn), from_dev_bf16(vn)
    out = torch.zeros((B, nq, d), dtype=torch.bfloat16, device="cuda")
    dec.gqa_decode_attn(q, kn, vn, kpool, vpool, torch.from_numpy(bt).cuda(), torch.from_numpy(pos).cuda(), nq, nkv, d,
                        1 / math.sqrt(d), rope, 10000.0, out)
    torch.cuda.synchronize()
    got = bits_to_f64(from_dev_bf16(out))
    for b in sample:
        kc = gather_paged(before[b][0], local, ctx)
        vc = gather_paged(before[b][1], local, ctx)
        ref = oracle.gqa_decode(qb[b:b + 1], knb[b:b + 1], vnb[b:b + 1], kc, vc, pos[b:b + 1], nq, nkv, d,
                                1 / math.sqrt(d), rope, 10000.0)
        _check_attn(got[b:b + 1], ref, f"ctx={ctx} rope={rope} seq {b}", rope=bool(rope))
        rows = torch.from_numpy(bt[b].astype(np.int64)).cuda()
        after_k = gather_paged(from_dev_bf16(kpool[rows].contiguous()), local, ctx)
        after_v = gather_paged(from_dev_bf16(vpool[rows].contiguous()), local, ctx)
        assert np.array_equal(after_v, vc)  # only row ctx-1 changed, and it holds v_new
        assert np.array_equal(after_k[:, :ctx - 1], kc[:, :ctx - 1])
        if not rope:
            assert np.array_equal(after_k, kc)  # the appended key is k_new as given


@pytest.mark.parametrize("T,E,k,renorm", [(64, 60, 4, 0), (64, 60, 4, 1), (7, 8, 8, 0), (33, 256, 16, 1), (5, 3, 1, 0)])
def test_moe_route_topk_bit_exact(T, E, k, renorm):
    logits = synth.route_logits_with_margin(T, E, k, seed=3000 + E)
    ridx, rw, gap = oracle.route_rows(logits, k, renorm)
    assert gap.min() >= 1e-3
    lg = torch.from_numpy(logits).cuda()
    idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    w = torch.zeros((T, k), device="cuda")
    dec.moe_route_topk(lg, k, renorm, idx, w)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), ridx)
    d, r = max_err(w.cpu().numpy(), rw)
    assert d <= 1e-6


def test_synth_device_fill_matches_host():
    n = 1 << 20
    host = synth.bf16_normal((n,), 0, 12345, 0.0, 0.02)
    t = torch.empty(n, dtype=torch.int16, device="cuda")
    rc = synth.dev_lib().syn_dev_fill_bf16(t.data_ptr(), n, 0, 12345, 0.0, 0.02, None)
    assert rc == 0
    torch.cuda.synchronize()
    dev_bits = t.cpu().numpy().view(np.uint16)
    mism = np.count_nonzero(dev_bits != host)
    assert mism <= 2, f"{mism} of {n} elements differ"


@pytest.mark.parametrize("B,I,K,rows", [(1, 344, 256, None), (3, 768, 576, None), (1, 14336, 4096, 600),
                                        (8, 1408, 2048, 300)])
def test_ffn_gate_up_matches_oracle(B, I, K, rows):
    # RMSNorm of the fp32 residual (R1), interleaved gate/up rows, bf16(SiLU(g) u) (R4)
    Wg = synth.bf16_normal((I, K), 8, I + K, 0.0, 0.02)
    Wu = synth.bf16_normal((I, K), 8, I + K + 1, 0.0, 0.02)
    x = (synth.normal_f64(B * K, 9, K) * 3.0).astype(np.float32).reshape(B, K)
    g = synth.bf16_normal_f32(K, 9, K + 1, 1.0, 0.1)
    Wgu = np.stack([Wg, Wu], axis=1).reshape(2 * I, K)
    act = torch.zeros((B, I), dtype=torch.bfloat16, device="cuda")
    dec.ffn_gate_up(to_dev_bf16(Wgu, torch), torch.from_numpy(x).cuda(), torch.from_numpy(g).cuda(), 1e-5, act)
    dec.check_standalone()
    got = bits_to_f64(from_dev_bf16(act))
    sel = np.arange(I) if rows is None else np.linspace(0, I - 1, rows).astype(int)
    for b in range(B):
        xn = np.array([oracle.bf16(v) for v in oracle.rmsnorm(x[b].astype(np.float64), g, 1e-5)])
        ref = oracle.swiglu_act(xn, Wg[sel], Wu[sel])
        assert_parity(got[b, sel], ref, what=f"ffn_gate_up B={B} I={I} K={K}")
        # R1 and R4 are decided in fp32 here and in fp64 in the oracle: a few elements may round
        # the other way (one bf16 quantum, two where an input element also rounded apart)
        q = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
        assert np.mean(np.abs(got[b, sel] - ref) <= 1e-6) > 0.97
        assert np.all(np.abs(got[b, sel] - ref) <= 2 * q + 1e-6)
