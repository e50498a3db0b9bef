"""Pins for the CPU oracle: each test checks it against something other than itself
(a library routine, a closed form, an invariant, brute force, or a value the pages fix),
chosen so that a dropped term, a wrong sign or index, or a transposed operand fails."""
import math
import os
import subprocess
import sys
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import configs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bits(x):
    """fp32/fp64 values that are bf16-representable -> bf16 bits (exact)."""
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def rnd_bf16_bits(shape, seed, std=1.0):
    return synth.bf16_normal(shape, seed, 77, 0.0, std)


def f(b):
    return synth.bits_to_f32(np.asarray(b, np.uint16)).astype(np.float64)


def torch_bf16(x):
    return torch.tensor(np.asarray(x, np.float64)).to(torch.bfloat16).to(torch.float64).numpy()


# ------------------------------------------------------------------ bf16 rounding

def test_bf16_rounding_matches_torch_nearest_even():
    rng = np.random.default_rng(0)
    vals = np.concatenate([rng.standard_normal(20000).astype(np.float32),
                           (rng.standard_normal(2000) * 1e-30).astype(np.float32),
                           (rng.standard_normal(2000) * 1e30).astype(np.float32)])
    # exact ties: bf16 value + half a quantum
    base = rng.standard_normal(2000).astype(np.float32)
    base = synth.bits_to_f32(bits(base) & 0xFFFF)  # truncate to bf16
    ties = (base.view(np.uint32) | 0x8000).view(np.float32)
    vals = np.concatenate([vals, ties])
    ours = np.array([oracle.bf16(float(v)) for v in vals])
    ref = torch.tensor(vals).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)


def test_bf16_rounding_ties_to_even_cases():
    assert oracle.bf16(1.0 + 2.0 ** -8) == 1.0                 # tie -> even mantissa 0
    assert oracle.bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6  # tie -> even mantissa 2
    assert oracle.bf16(-(1.0 + 2.0 ** -8 + 2.0 ** -20)) == -(1.0 + 2.0 ** -7)


def test_generator_rounds_like_torch():
    vals = synth.normal_f64(5000, 5, 1) * 0.02
    b = np.array([synth.lib().syn_round_bf16(float(v)) for v in vals], np.uint16)
    ref = torch.tensor(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    # fp64 -> bf16 directly vs torch's fp64 -> bf16 (both nearest-even from fp64)
    assert np.array_equal(b, ref)


# ------------------------------------------------------------------ RMSNorm

@pytest.mark.parametrize("c", [0.37, -2.5, 1e-3])
def test_rmsnorm_constant_vector_closed_form(c):
    n = 64
    out = oracle.rmsnorm(np.full(n, c), np.ones(n, np.float32), 1e-5)
    assert np.allclose(out, c / math.sqrt(c * c + 1e-5), rtol=1e-15, atol=0)


def test_rmsnorm_unit_gain_gives_unit_rms_and_gain_scales_elementwise():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(576) * 3.0
    out = oracle.rmsnorm(x, np.ones(576, np.float32), 1e-5)
    ms = np.mean(x * x)
    assert math.isclose(np.sqrt(np.mean(out * out)), math.sqrt(ms / (ms + 1e-5)), rel_tol=1e-13)
    g = (1 + 0.1 * rng.standard_normal(576)).astype(np.float32)
    out_g = oracle.rmsnorm(x, g, 1e-5)
    assert np.allclose(out_g, out * g.astype(np.float64), rtol=1e-14)


# ------------------------------------------------------------------ RoPE

def test_rope_position_zero_is_identity():
    v = np.random.default_rng(2).standard_normal((3, 64))
    assert np.array_equal(oracle.rope(v, 0, 10000.0), v)


def test_rope_single_pair_is_textbook_rotation():
    # d = 2: theta_0 = base^0 = 1, so position p rotates by p radians.
    v = np.array([[0.3, -1.2]])
    for p in (1, 5, 1000):
        c, s = math.cos(p), math.sin(p)
        want = [0.3 * c + 1.2 * s, 0.3 * s - 1.2 * c]
        assert np.allclose(oracle.rope(v, p, 10000.0)[0], want, rtol=0, atol=1e-15)


def test_rope_pairs_i_with_i_plus_half():
    # A unit vector on element 1 of d = 8 moves only into element 5 (half-split pairing),
    # at angle p * base^(-2/8).
    d, p, base = 8, 7, 10000.0
    v = np.zeros((1, d))
    v[0, 1] = 1.0
    out = oracle.rope(v, p, base)[0]
    a = p * base ** (-2.0 / d)
    want = np.zeros(d)
    want[1], want[5] = math.cos(a), math.sin(a)
    assert np.allclose(out, want, atol=1e-15)


def test_rope_preserves_norm_per_pair():
    rng = np.random.default_rng(3)
    v = rng.standard_normal((4, 128))
    out = oracle.rope(v, 32767, 500000.0)
    half = 64
    n_in = v[:, :half] ** 2 + v[:, half:] ** 2
    n_out = out[:, :half] ** 2 + out[:, half:] ** 2
    assert np.allclose(n_in, n_out, rtol=1e-13)


def test_rope_dot_product_depends_only_on_relative_position():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 64))
    k = rng.standard_normal((1, 64))
    ref = float(oracle.rope(q, 100, 1e4)[0] @ oracle.rope(k, 37, 1e4)[0])
    for s in (1, 500, 3000):
        got = float(oracle.rope(q, 100 + s, 1e4)[0] @ oracle.rope(k, 37 + s, 1e4)[0])
        assert math.isclose(got, ref, rel_tol=1e-9, abs_tol=1e-10)


# ------------------------------------------------------------------ QK-norm (ANEDVD applyHeadNorm)

def test_head_rmsnorm_normalises_each_head_by_its_own_mean_square():
    # Heads of very different scale: with unit gains every head comes out with RMS
    # sqrt(ms / (ms + eps)) of its OWN mean square ms; one statistic over the whole
    # vector would leave the heads' scale ratio in place.
    rng = np.random.default_rng(40)
    d = 16
    v = rng.standard_normal((3, d)) * np.array([[0.05], [1.0], [40.0]])
    out = oracle.head_rmsnorm(v, np.ones(d, np.float32), 1e-5)
    for h in range(3):
        ms = np.mean(v[h] ** 2)
        assert math.isclose(np.sqrt(np.mean(out[h] ** 2)), math.sqrt(ms / (ms + 1e-5)), rel_tol=1e-13)
        assert np.allclose(out[h], v[h] / math.sqrt(ms + 1e-5), rtol=1e-14)


def test_head_rmsnorm_gain_is_per_element_of_the_head():
    rng = np.random.default_rng(41)
    d = 8
    v = rng.standard_normal((2, d))
    g = np.arange(1, d + 1, dtype=np.float32)
    plain = oracle.head_rmsnorm(v, np.ones(d, np.float32), 1e-5)
    assert np.allclose(oracle.head_rmsnorm(v, g, 1e-5), plain * g[None, :].astype(np.float64), rtol=1e-14)


def _qk_cfg(**over):
    return dict(configs.COMMON, name="qk", hidden=32, layers=1, n_q_heads=2, n_kv_heads=2, head_dim=8,
                ffn_inter=16, vocab=12, max_context=8, qk_norm=1, **over)


def test_qk_norm_keys_in_the_cache_have_unit_rms_per_head():
    # Unit gains, no bias, position 0 (RoPE is the identity there): every cached key head is
    # the bf16 rounding of a unit-RMS vector, even with the second head's projection rows
    # scaled by 64 (a whole-vector norm would leave them 64x apart).
    cfg = _qk_cfg()
    w = synth.make_weights(cfg, seed=42)
    lw = w["layers"][0]
    d, nq, nkv = 8, 2, 2
    wq = f(lw["wqkv"])
    wq[nq * d + d: nq * d + 2 * d] *= 64.0     # k rows of kv head 1 (exact: a power of two)
    lw["wqkv"] = bits(wq)
    lw["q_norm"] = np.ones(d, np.float32)
    lw["k_norm"] = np.ones(d, np.float32)
    m = oracle.Model(cfg, w)
    m.forward(0, 5, 0, want_logits=False)
    k, _ = m.kv_read(0, 0, 0, 1)
    kh = f(k[0]).reshape(nkv, d)
    rms = np.sqrt(np.mean(kh ** 2, axis=1))
    assert np.all(np.abs(rms - 1.0) < 2 ** -7), rms


def test_qk_norm_applies_to_the_biased_projection():
    # With the key projection rows zero, k = bias; the norm must see the bias (added before
    # the norm), so each cached key head is bf16(b_h / sqrt(mean(b_h^2) + eps) * g_k) at p = 0.
    cfg = _qk_cfg(qkv_bias=1)
    w = synth.make_weights(cfg, seed=43)
    lw = w["layers"][0]
    d, nq, nkv = 8, 2, 2
    wq = f(lw["wqkv"])
    wq[nq * d: nq * d + nkv * d] = 0.0
    lw["wqkv"] = bits(wq)
    m = oracle.Model(cfg, w)
    m.forward(0, 3, 0, want_logits=False)
    k, _ = m.kv_read(0, 0, 0, 1)
    b = lw["bqkv"][nq * d: nq * d + nkv * d].astype(np.float64).reshape(nkv, d)
    g = lw["k_norm"].astype(np.float64)
    want = b / np.sqrt(np.mean(b * b, axis=1, keepdims=True) + cfg["rms_eps"]) * g[None, :]
    assert np.array_equal(f(k[0]), torch_bf16(want.reshape(-1)))


def test_qk_norm_comes_before_rope():
    # At p > 0 the cached key is bf16(rope(norm(k))): with a non-uniform gain, normalising
    # after the rotation applies the gain in the rotated frame and gives other values.
    cfg = _qk_cfg()
    w = synth.make_weights(cfg, seed=44)
    lw = w["layers"][0]
    d, nq, nkv = 8, 2, 2
    m = oracle.Model(cfg, w)
    toks = [4, 9, 2]
    m.prefill(0, toks, 0)
    k, _ = m.kv_read(0, 0, 0, 3)
    for p, t in enumerate(toks):
        x = f(w["embed"][t])
        xn = torch_bf16(x / np.sqrt(np.mean(x * x) + cfg["rms_eps"]) * lw["attn_norm"].astype(np.float64))
        kraw = (f(lw["wqkv"])[nq * d: nq * d + nkv * d] @ xn).reshape(nkv, d)
        kn = kraw / np.sqrt(np.mean(kraw ** 2, axis=1, keepdims=True) + cfg["rms_eps"]) \
            * lw["k_norm"].astype(np.float64)[None, :]
        ang = p * cfg["rope_base"] ** (-np.arange(0, d, 2) / d)
        a, bb = kn[:, : d // 2], kn[:, d // 2:]
        rot = np.concatenate([a * np.cos(ang) - bb * np.sin(ang), a * np.sin(ang) + bb * np.cos(ang)], 1)
        assert np.allclose(f(k[p]), torch_bf16(rot.reshape(-1)), rtol=0, atol=1e-12), p


# ------------------------------------------------------------------ attention

def test_attention_single_key_returns_that_value():
    d = 64
    q = np.random.default_rng(5).standard_normal(d)
    K = rnd_bf16_bits((1, d), 1)
    V = rnd_bf16_bits((1, d), 2)
    out = oracle.attend(q, K, V, 1 / math.sqrt(d))
    assert np.array_equal(out, f(V[0]))


def test_attention_equal_scores_average_values():
    d, n = 16, 9
    K = rnd_bf16_bits((n, d), 3)
    V = rnd_bf16_bits((n, d), 4)
    out = oracle.attend(np.zeros(d), K, V, 0.25)
    assert np.allclose(out, f(V).mean(axis=0), rtol=1e-14, atol=1e-15)


def _brute_force_causal(Q, K, V, nq, nkv, scale, window=0, softcap=0.0):
    """Textbook masked-matrix attention for T queries at positions 0..T-1:
    O_h = softmax(mask(cap(Q_h K_g^T * scale))) V_g, g = h // (nq // nkv); the mask hides
    later keys and, with a window W, keys W or more positions back."""
    T, d = Q.shape[0], Q.shape[2]
    out = np.zeros((T, nq, d))
    mask = np.triu(np.ones((T, T), bool), 1)
    if window:
        mask |= np.tril(np.ones((T, T), bool), -window)
    for h in range(nq):
        g = h // (nq // nkv)
        S = Q[:, h, :] @ K[:, g, :].T * scale
        if softcap:
            S = softcap * np.tanh(S / softcap)
        S[mask] = -np.inf
        P = np.exp(S - S.max(axis=1, keepdims=True))
        P /= P.sum(axis=1, keepdims=True)
        out[:, h, :] = P @ V[:, g, :]
    return out


@pytest.mark.parametrize("nq,nkv", [(4, 2), (4, 4), (6, 1)])
def test_causal_gqa_matches_brute_force_masked_matrix(nq, nkv):
    T, d = 8, 4
    Q = rnd_bf16_bits((T, nq, d), 10 + nq)
    Kc = rnd_bf16_bits((1, T, nkv, d), 20 + nkv)
    Vc = rnd_bf16_bits((1, T, nkv, d), 30 + nkv)
    scale = 1 / math.sqrt(d)
    ref = _brute_force_causal(f(Q), f(Kc[0]), f(Vc[0]), nq, nkv, scale)
    for t in range(T):
        kc, vc = Kc.copy(), Vc.copy()
        got = oracle.gqa_decode(Q[t:t + 1], None, None, kc, vc, np.array([t]), nq, nkv, d, scale, 0, 1e4)
        assert np.allclose(got[0], ref[t], rtol=1e-12, atol=1e-14)


def test_decode_append_with_fused_rope_equals_rotating_beforehand():
    nq, nkv, d, ctx = 4, 2, 8, 6
    q = rnd_bf16_bits((1, nq, d), 41)
    kn = rnd_bf16_bits((1, nkv, d), 42)
    vn = rnd_bf16_bits((1, nkv, d), 43)
    Kc = rnd_bf16_bits((1, ctx, nkv, d), 44)
    Vc = rnd_bf16_bits((1, ctx, nkv, d), 45)
    p = 4
    k1, v1 = Kc.copy(), Vc.copy()
    got = oracle.gqa_decode(q, kn, vn, k1, v1, np.array([p]), nq, nkv, d, 0.3, 1, 1e4)
    # by hand: rotate, round, store, attend unrotated path
    qr = np.array([oracle.bf16(x) for x in oracle.rope(f(q[0]), p, 1e4).ravel()]).reshape(nq, d)
    kr = np.array([oracle.bf16(x) for x in oracle.rope(f(kn[0]), p, 1e4).ravel()]).reshape(nkv, d)
    k2, v2 = Kc.copy(), Vc.copy()
    k2[0, p] = bits(kr)
    v2[0, p] = vn[0]
    want = oracle.gqa_decode(bits(qr)[None], None, None, k2, v2, np.array([p]), nq, nkv, d, 0.3, 0, 1e4)
    assert np.array_equal(k1, k2) and np.array_equal(v1, v2)
    assert np.array_equal(got, want)
    # rows after p untouched, rows before p untouched
    assert np.array_equal(k1[0, :p], Kc[0, :p]) and np.array_equal(k1[0, p + 1:], Kc[0, p + 1:])


# ------------------------------------------------------------------ GEMV

def test_matvec_equals_exact_rational_sum():
    N, K = 7, 33
    W = rnd_bf16_bits((N, K), 50)
    x = rnd_bf16_bits((K,), 51)
    got = oracle.matvec(W, f(x))
    Wf, xf = f(W), f(x)
    for n in range(N):
        exact = sum(Fraction(float(Wf[n, k])) * Fraction(float(xf[k])) for k in range(K))
        assert abs(got[n] - float(exact)) <= 1e-15 * max(1.0, abs(float(exact))) + 1e-17


def test_gemv_rows_orientation():
    # y[b][n] = sum_k W[n][k] x[b][k]: a one-hot x row picks one column of W.
    N, K = 5, 16
    W = rnd_bf16_bits((N, K), 52)
    x = np.zeros((2, K), np.uint16)
    x[0, 3] = bits(1.0)
    x[1, 9] = bits(-2.0)
    y = oracle.gemv_rows(W, x)
    assert np.array_equal(y[0], f(W)[:, 3]) and np.array_equal(y[1], -2 * f(W)[:, 9])


# ------------------------------------------------------------------ SwiGLU

def test_swiglu_scalar_closed_form():
    # I = h = 1: out = Wd * bf16(silu(Wg x) * (Wu x)), silu(z) = z / (1 + e^-z).
    x = np.array([1.0])
    Wg, Wu, Wd = bits([[2.0]]), bits([[0.5]]), bits([[1.0]])
    a = 2.0 / (1.0 + math.exp(-2.0)) * 0.5
    want = float(torch.tensor(a, dtype=torch.float64).to(torch.bfloat16).to(torch.float64))
    assert oracle.swiglu(x, Wg, Wu, Wd)[0] == want == 0.87890625


def test_swiglu_zero_gate_or_zero_up_gives_zero():
    h, I = 8, 5
    x = np.random.default_rng(6).standard_normal(h)
    W = rnd_bf16_bits((I, h), 60)
    Wd = rnd_bf16_bits((h, I), 61)
    Z = np.zeros((I, h), np.uint16)
    assert not oracle.swiglu(x, Z, W, Wd).any()
    assert not oracle.swiglu(x, W, Z, Wd).any()


def test_swiglu_is_the_down_projection_of_its_activation():
    rng = np.random.default_rng(70)
    h, I = 24, 40
    x = f(rnd_bf16_bits(h, 71))
    Wg, Wu = rnd_bf16_bits((I, h), 72, 0.3), rnd_bf16_bits((I, h), 73, 0.3)
    Wd = rnd_bf16_bits((h, I), 74, 0.3)
    act = oracle.swiglu_act(x, Wg, Wu)
    assert np.array_equal(act, torch_bf16(act))  # R4: bf16 values
    assert np.allclose(oracle.swiglu(x, Wg, Wu, Wd), f(Wd) @ act, rtol=1e-13, atol=1e-15)
    z = f(Wg) @ x
    u = f(Wu) @ x
    assert np.allclose(act, torch_bf16(z / (1 + np.exp(-z)) * u), rtol=0, atol=1e-12)


def test_swiglu_gate_and_up_are_not_swapped():
    # silu is not symmetric: silu(g) * u != silu(u) * g in general.
    h, I = 8, 4
    x = np.random.default_rng(7).standard_normal(h)
    Wg, Wu = rnd_bf16_bits((I, h), 62), rnd_bf16_bits((I, h), 63)
    Wd = np.eye(h, I, dtype=np.float32)
    Wd = bits(Wd)
    out = oracle.swiglu(x, Wg, Wu, Wd)
    g, u = f(Wg) @ x, f(Wu) @ x
    want = torch_bf16(g / (1 + np.exp(-g)) * u)
    assert np.allclose(out[:I], want, rtol=0, atol=0)


# ------------------------------------------------------------------ routing

def test_route_topk_matches_library_softmax_and_stable_sort():
    rng = np.random.default_rng(8)
    for _ in range(50):
        E, k = 60, 4
        r = rng.standard_normal(E)
        idx, w, gap = oracle.route_topk(r, k, 0)
        p = torch.softmax(torch.tensor(r), 0).numpy()
        order = np.lexsort((np.arange(E), -p))[:k]
        assert np.array_equal(idx, order)
        assert np.allclose(w, p[order], rtol=1e-14)
        srt = np.sort(r)[::-1]
        assert math.isclose(gap, np.min(srt[:k] - srt[1:k + 1]), rel_tol=1e-14)
        idx2, w2, _ = oracle.route_topk(r, k, 1)
        assert np.array_equal(idx2, idx) and math.isclose(w2.sum(), 1.0, rel_tol=1e-14)
        assert np.allclose(w2, p[order] / p[order].sum(), rtol=1e-14)


def test_route_ties_pick_lower_index():
    r = np.array([0.5, 2.0, 2.0, 1.0, 2.0])
    idx, _, gap = oracle.route_topk(r, 3, 0)
    assert list(idx) == [1, 2, 4] and gap == 0.0


def test_route_rows_margin_generator():
    logits = synth.route_logits_with_margin(32, 60, 4)
    _, _, gap = oracle.route_rows(logits, 4, 0)
    assert gap.min() >= 1e-3


# ------------------------------------------------------------------ MoE

def _moe_cfg(E, k, renorm=0, shared_inter=12, shared_gate=1):
    return dict(configs.COMMON, name="moe-pin", hidden=16, layers=1, n_q_heads=2, n_kv_heads=2, head_dim=8,
                vocab=32, n_experts=E, top_k=k, expert_inter=8, shared_inter=shared_inter,
                shared_gate=shared_gate, norm_topk=renorm, max_context=8)


def test_moe_with_k_equal_E_is_dense_softmax_weighted_sum():
    for renorm in (0, 1):
        cfg = _moe_cfg(E=5, k=5, renorm=renorm, shared_inter=0)
        lw = synth.make_layer(cfg, 0, seed=9)
        xn = torch_bf16(np.random.default_rng(9).standard_normal(16))
        out, idx, w, _ = oracle.moe_ffn(cfg, lw, xn)
        p = torch.softmax(torch.tensor(f(lw["w_router"]) @ xn), 0).numpy()
        want = sum(p[e] * oracle.swiglu(xn, lw["e_gate"][e], lw["e_up"][e], lw["e_down"][e]) for e in range(5))
        assert np.allclose(out, want, rtol=1e-12, atol=1e-15)
        assert sorted(idx) == list(range(5))


def test_moe_k1_is_one_expert_times_its_probability():
    cfg = _moe_cfg(E=6, k=1, shared_inter=0)
    lw = synth.make_layer(cfg, 0, seed=10)
    xn = torch_bf16(np.random.default_rng(10).standard_normal(16))
    out, idx, w, _ = oracle.moe_ffn(cfg, lw, xn)
    p = torch.softmax(torch.tensor(f(lw["w_router"]) @ xn), 0).numpy()
    e = int(np.argmax(p))
    assert idx[0] == e
    want = p[e] * oracle.swiglu(xn, lw["e_gate"][e], lw["e_up"][e], lw["e_down"][e])
    assert np.allclose(out, want, rtol=1e-12, atol=1e-15)


def _golden(name):
    vals = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()
            vals[k] = float(v)
    return vals


def test_shared_expert_gate_zero_is_half_weight():
    g = _golden("shared_expert_gate.txt")
    cfg = _moe_cfg(E=2, k=1)
    lw = synth.make_layer(cfg, 0, seed=11)
    # routed experts all zero: whatever comes out is the shared expert
    for n in ("e_gate", "e_up", "e_down"):
        lw[n] = np.zeros_like(lw[n])
    xn = torch_bf16(np.random.default_rng(11).standard_normal(16))
    shared = oracle.swiglu(xn, lw["s_gate"], lw["s_up"], lw["s_down"])
    lw["s_gate_vec"] = np.zeros(16, np.float32)
    out_zero, *_ = oracle.moe_ffn(cfg, lw, xn)
    assert np.array_equal(out_zero, g["gate_zero_scale"] * shared)
    out_nogate, *_ = oracle.moe_ffn(dict(cfg, shared_gate=0), lw, xn)
    assert np.array_equal(out_nogate, g["no_gate_scale"] * shared)


def _lcg_fill(n, seed, scale, base=0.0):
    """The pages' deterministic test fill: s = s*1664525 + 1013904223 (mod 2^32),
    f = (s >> 8) / 2^24 - 0.5, value = base + f * scale."""
    out = np.empty(n)
    s = seed
    for i in range(n):
        s = (s * 1664525 + 1013904223) & 0xFFFFFFFF
        out[i] = base + ((s >> 8) / 16777216.0 - 0.5) * scale
    return out


def test_shared_expert_gate_changes_logits_like_the_pages_fixture():
    # One-layer qwen2moe-style fixture: hidden 32, 4/2 heads of 8, 2 experts top-1 with
    # zero routed experts, shared inter 24, vocab 64; fills as in the pages' test.
    g = _golden("shared_expert_gate.txt")
    cfg = dict(configs.COMMON, name="shared-fixture", hidden=32, layers=1, n_q_heads=4, n_kv_heads=2,
               head_dim=8, vocab=64, n_experts=2, top_k=1, expert_inter=16, shared_inter=24, shared_gate=1,
               max_context=8)

    def b16(a, shape):
        return synth.f32_to_bf16_bits(np.asarray(a, np.float32)).reshape(shape)

    def f32v(a):
        return synth.bits_to_f32(synth.f32_to_bf16_bits(np.asarray(a, np.float32)))

    h, qkv = 32, 4 * 8 + 2 * 2 * 8
    lw = dict(attn_norm=f32v(_lcg_fill(h, 100, 0.1, 1.0)), ffn_norm=f32v(_lcg_fill(h, 200, 0.1, 1.0)),
              wqkv=b16(_lcg_fill(qkv * h, 300, 0.3), (qkv, h)), wo=b16(_lcg_fill(h * 32, 400, 0.3), (h, 32)),
              w_router=b16(_lcg_fill(2 * h, 1100, 0.3), (2, h)),
              e_gate=np.zeros((2, 16, h), np.uint16), e_up=np.zeros((2, 16, h), np.uint16),
              e_down=np.zeros((2, h, 16), np.uint16),
              s_gate=b16(_lcg_fill(24 * h, 1200, 0.3), (24, h)), s_up=b16(_lcg_fill(24 * h, 1300, 0.3), (24, h)),
              s_down=b16(_lcg_fill(h * 24, 1400, 0.3), (h, 24)), s_gate_vec=np.zeros(h, np.float32))
    w = dict(embed=b16(_lcg_fill(64 * h, 1, 1.0), (64, h)), lm_head=b16(_lcg_fill(64 * h, 3, 0.3), (64, h)),
             final_norm=f32v(_lcg_fill(h, 2, 0.1, 1.0)), layers=[lw])
    gated = oracle.Model(cfg, w).prefill(0, [3, 7, 11, 19], 0)
    ungated = oracle.Model(dict(cfg, shared_gate=0), w).prefill(0, [3, 7, 11, 19], 0)
    assert np.max(np.abs(gated - ungated)) > g["min_abs_difference_between_runs"]


# ------------------------------------------------------------------ sliding window, softcaps, sandwich, q8_row

def test_layer_window_schedule_every_pattern_th_layer_is_global():
    base = _small_dense(layers=6, sliding_window=4)
    assert [oracle.layer_window(dict(base, swa_pattern=3), l) for l in range(6)] == [4, 4, 0, 4, 4, 0]
    assert [oracle.layer_window(dict(base, swa_pattern=2), l) for l in range(6)] == [4, 0, 4, 0, 4, 0]
    assert [oracle.layer_window(dict(base, swa_pattern=7), l) for l in range(6)] == [4] * 6
    assert [oracle.layer_window(dict(base, swa_pattern=1), l) for l in range(6)] == [0] * 6
    assert [oracle.layer_window(dict(base, swa_pattern=0), l) for l in range(6)] == [0] * 6
    assert [oracle.layer_window(dict(base, sliding_window=0, swa_pattern=3), l) for l in range(6)] == [0] * 6


def test_window_of_one_returns_the_current_value_and_a_wide_window_changes_nothing():
    rng = np.random.default_rng(60)
    n, d = 9, 16
    q = rng.standard_normal(d)
    K, V = rnd_bf16_bits((n, d), 61), rnd_bf16_bits((n, d), 62)
    assert np.array_equal(oracle.attend_window(q, K, V, 0.25, first=n - 1), f(V[n - 1]))
    full = oracle.attend(q, K, V, 0.25)
    assert np.array_equal(oracle.attend_window(q, K, V, 0.25, first=0), full)
    # a window of 3 is the plain softmax over the last 3 keys only
    s = np.array([q @ f(K[j]) * 0.25 for j in range(n - 3, n)])
    p = np.exp(s - s.max())
    want = (p[:, None] * f(V[n - 3:])).sum(0) / p.sum()
    assert np.allclose(oracle.attend_window(q, K, V, 0.25, first=n - 3), want, rtol=1e-13, atol=1e-15)


def test_attention_softcap_two_keys_closed_form():
    # q . k_0 = 3 and q . k_1 = -1 at scale 1; a cap of 2 turns them into 2 tanh(1.5) and
    # 2 tanh(-0.5), so key 0 weighs 1 / (1 + e^(2 tanh(-0.5) - 2 tanh(1.5)))
    q = np.array([1.0, 0.0])
    K = bits(np.array([[3.0, 0.0], [-1.0, 0.0]]))
    V = bits(np.array([[1.0, 0.0], [0.0, 1.0]]))
    got = oracle.attend_window(q, K, V, 1.0, softcap=2.0)
    w0 = 1.0 / (1.0 + math.exp(2 * math.tanh(-0.5) - 2 * math.tanh(1.5)))
    assert np.allclose(got, [w0, 1.0 - w0], rtol=1e-14)
    # uncapped, the weight is the logistic of the raw score difference
    w0_raw = 1.0 / (1.0 + math.exp(-4.0))
    assert np.allclose(oracle.attend_window(q, K, V, 1.0), [w0_raw, 1 - w0_raw], rtol=1e-14)
    # the cap acts on the scaled score: scale 0.5 with cap 2 is tanh of q.k / 4
    got = oracle.attend_window(q, K, V, 0.5, softcap=2.0)
    w0 = 1.0 / (1.0 + math.exp(2 * math.tanh(-0.25) - 2 * math.tanh(0.75)))
    assert np.allclose(got, [w0, 1.0 - w0], rtol=1e-14)


def test_final_softcap_maps_the_uncapped_logits():
    cfg = _small_dense()
    w = synth.make_weights(cfg, seed=63)
    toks = synth.tokens(6, cfg["vocab"], 1003)
    raw = oracle.Model(cfg, w).prefill(0, toks, 0)
    capped = oracle.Model(dict(cfg, final_softcap=0.25), w).prefill(0, toks, 0)
    assert np.all(np.abs(capped) < 0.25)
    assert np.allclose(capped, 0.25 * np.tanh(raw / 0.25), rtol=1e-14, atol=1e-16)


def test_sandwich_with_zero_post_gains_leaves_only_the_embedding():
    # zero post-norm gains cancel every attention and FFN contribution: the residual stays
    # the embedding row, and the logits are the head applied to its final norm
    cfg = _small_dense(sandwich=1)
    w = synth.make_weights(cfg, seed=64)
    for lw in w["layers"]:
        lw["post_attn_norm"] = np.zeros(cfg["hidden"], np.float32)
        lw["post_ffn_norm"] = np.zeros(cfg["hidden"], np.float32)
    m = oracle.Model(cfg, w)
    got = m.forward(0, 11, 0)
    x = f(w["embed"][11])
    assert np.array_equal(m.last_hidden(), x)
    xn = torch_bf16(x / np.sqrt(np.mean(x * x) + cfg["rms_eps"]) * w["final_norm"].astype(np.float64))
    assert np.allclose(got, f(w["lm_head"]) @ xn, rtol=1e-13, atol=1e-15)


def test_sandwich_post_attention_norm_closed_form_at_position_zero():
    # At p = 0 attention returns the single cached value row, so with a zero post-FFN gain the
    # layer adds exactly rmsnorm(Wo bf16(v)) * g_post to the embedding, v = Wv xn.
    cfg = dict(_small_dense(sandwich=1), layers=1, n_kv_heads=4)
    w = synth.make_weights(cfg, seed=65)
    lw = w["layers"][0]
    lw["post_ffn_norm"] = np.zeros(cfg["hidden"], np.float32)
    m = oracle.Model(cfg, w)
    m.forward(0, 4, 0)
    h, qd, eps = cfg["hidden"], cfg["n_q_heads"] * cfg["head_dim"], cfg["rms_eps"]
    x = f(w["embed"][4])
    xn = torch_bf16(x / np.sqrt(np.mean(x * x) + eps) * lw["attn_norm"].astype(np.float64))
    v = torch_bf16(f(lw["wqkv"])[2 * qd:] @ xn)      # nkv == nq: v has the width of o
    y = f(lw["wo"]) @ v
    want = x + y / np.sqrt(np.mean(y * y) + eps) * lw["post_attn_norm"].astype(np.float64)
    assert np.allclose(m.last_hidden(), want, rtol=1e-12, atol=1e-14)


def test_q8_matvec_equals_exact_rational_sum():
    rng = np.random.default_rng(66)
    N, K = 5, 37
    Q = rng.integers(-127, 128, (N, K)).astype(np.int8)
    S = bits_to_fp32_bf16(rng.uniform(1e-4, 1e-3, N))
    x = f(rnd_bf16_bits(K, 67))
    got = oracle.matvec_q8(Q, S, x)
    for n in range(N):
        exact = Fraction(float(S[n])) * sum(Fraction(int(Q[n, k])) * Fraction(float(x[k])) for k in range(K))
        assert abs(Fraction(float(got[n])) - exact) <= abs(exact) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 80)
    # rows: row n uses scale n only
    e = np.zeros(K)
    e[3] = 1.0
    assert np.array_equal(oracle.matvec_q8(Q, S, e), Q[:, 3].astype(np.float64) * S.astype(np.float64))


def bits_to_fp32_bf16(v):
    return f(bits(torch_bf16(v))).astype(np.float32)


def test_q8_with_power_of_two_scales_is_the_bf16_model():
    # scale 2^-9 times an int8 value is an exact bf16 number: the q8_row model must equal
    # the bf16 model holding those values, bit for bit
    cfg = _small_dense(weight_format=1)
    wq = synth.make_weights(cfg, seed=68)
    wb = synth.make_weights(dict(cfg, weight_format=0), seed=68)
    for lq, lb in zip(wq["layers"], wb["layers"]):
        for name in synth.Q8_MATS:
            lq[name + "_scale"] = np.full(lq[name].shape[0], 2.0 ** -9, np.float32)
            lb[name] = bits(lq[name].astype(np.float64) * 2.0 ** -9)
    wq["lm_head_scale"] = np.full(cfg["vocab"], 2.0 ** -9, np.float32)
    wb["lm_head"] = bits(wq["lm_head"].astype(np.float64) * 2.0 ** -9)
    toks = synth.tokens(7, cfg["vocab"], 1004)
    a = oracle.Model(cfg, wq).prefill(0, toks, 0)
    b = oracle.Model(dict(cfg, weight_format=0), wb).prefill(0, toks, 0)
    assert np.array_equal(a, b)


def test_q8_scales_change_the_result_row_by_row():
    cfg = _small_dense(weight_format=1)
    w = synth.make_weights(cfg, seed=69)
    toks = synth.tokens(5, cfg["vocab"], 1005)
    a = oracle.Model(cfg, w).prefill(0, toks, 0)
    w["lm_head_scale"] = w["lm_head_scale"].copy()
    w["lm_head_scale"][7] *= 2
    b = oracle.Model(cfg, w).prefill(0, toks, 0)
    assert b[7] == 2 * a[7] and np.array_equal(np.delete(a, 7), np.delete(b, 7))


# ------------------------------------------------------------------ whole stack

def _small_dense(**over):
    cfg = dict(configs.COMMON, name="small", hidden=48, layers=2, n_q_heads=4, n_kv_heads=2, head_dim=16,
               ffn_inter=96, vocab=80, max_context=24)
    cfg.update(over)
    return cfg


def test_prefill_equals_sequential_decode_bit_exact():
    cfg = _small_dense()
    w = synth.make_weights(cfg, seed=12)
    toks = synth.tokens(10, cfg["vocab"], 1000)
    a = oracle.Model(cfg, w)
    la = a.prefill(0, toks, 0)
    b = oracle.Model(cfg, w)
    for t, tok in enumerate(toks):
        lb = b.forward(0, tok, t)
    assert np.array_equal(la, lb)
    for l in range(cfg["layers"]):
        assert all(np.array_equal(x, y) for x, y in zip(a.kv_read(0, l, 0, 10), b.kv_read(0, l, 0, 10)))


def test_split_prefill_equals_one_prefill():
    cfg = _small_dense()
    w = synth.make_weights(cfg, seed=13)
    toks = synth.tokens(12, cfg["vocab"], 1001)
    a = oracle.Model(cfg, w)
    la = a.prefill(0, toks, 0)
    b = oracle.Model(cfg, w)
    b.prefill(0, toks[:5], 0)
    lb = b.prefill(0, toks[5:], 5)
    assert np.array_equal(la, lb)


def test_same_seed_same_bits_and_thread_count_does_not_matter():
    code = ("import numpy as np, oracle, synth\n"
            "from synth import configs\n"
            "cfg = dict(configs.TINY)\n"
            "w = synth.make_weights(cfg)\n"
            "m = oracle.Model(cfg, w)\n"
            "l = m.prefill(0, synth.tokens(16, cfg['vocab'], 1000), 0)\n"
            "import sys; sys.stdout.write(l.tobytes().hex()[:4000] + str(hash(l.tobytes())))\n")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    outs = []
    for threads in ("1", "4", "1"):
        env = dict(os.environ, OMP_NUM_THREADS=threads, PYTHONHASHSEED="0")
        outs.append(subprocess.check_output([sys.executable, "-c", code], cwd=root, env=env))
    assert outs[0] == outs[1] == outs[2]


def _textbook_forward(cfg, w, toks):
    """Whole-sequence forward in matrix form (causal mask over all T tokens at once),
    with bf16 rounding at the same four points; independent of the per-token cache loop."""
    T = len(toks)
    h, nq, nkv, d = cfg["hidden"], cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    eps, base = cfg["rms_eps"], cfg["rope_base"]
    X = f(w["embed"])[toks]

    def norm(X, g):
        return torch_bf16(X / np.sqrt(np.mean(X * X, axis=1, keepdims=True) + eps) * g.astype(np.float64))

    inv = base ** (-np.arange(0, d, 2) / d)
    ang = np.arange(T)[:, None] * inv[None, :]
    cos, sin = np.cos(ang), np.sin(ang)

    def rope(M):  # [T][heads][d]
        a, b = M[..., : d // 2], M[..., d // 2:]
        return np.concatenate([a * cos[:, None] - b * sin[:, None], a * sin[:, None] + b * cos[:, None]], -1)

    q8 = cfg.get("weight_format", 0) == 1

    def mat(lw, name):  # the layer's matrix as fp64 values (a q8_row matrix dequantised)
        if q8 and name in synth.Q8_MATS:
            return lw[name].astype(np.float64) * lw[name + "_scale"].astype(np.float64)[:, None]
        return f(lw[name])

    def post(Y, g):  # sandwich norm: RMS-normalised, not rounded
        return Y / np.sqrt(np.mean(Y * Y, axis=1, keepdims=True) + eps) * g.astype(np.float64)

    for li, lw in enumerate(w["layers"]):
        W_l = 0
        if cfg.get("sliding_window", 0) and (li + 1) % max(cfg.get("swa_pattern", 0), 1) != 0:
            W_l = cfg["sliding_window"]
        xn = norm(X, lw["attn_norm"])
        qkv = xn @ mat(lw, "wqkv").T
        if cfg.get("qkv_bias"):
            qkv = qkv + lw["bqkv"].astype(np.float64)
        q = qkv[:, : nq * d].reshape(T, nq, d)
        k = qkv[:, nq * d: nq * d + nkv * d].reshape(T, nkv, d)
        v = qkv[:, nq * d + nkv * d:].reshape(T, nkv, d)
        if cfg.get("qk_norm"):
            def head_norm(M, g):
                return M / np.sqrt(np.mean(M * M, axis=-1, keepdims=True) + eps) * g.astype(np.float64)
            q, k = head_norm(q, lw["q_norm"]), head_norm(k, lw["k_norm"])
        q, k, v = torch_bf16(rope(q)), torch_bf16(rope(k)), torch_bf16(v)
        o = _brute_force_causal(q, k, v, nq, nkv, 1 / math.sqrt(d), W_l, cfg.get("attn_softcap", 0.0))
        ao = torch_bf16(o.reshape(T, nq * d)) @ mat(lw, "wo").T
        X = X + (post(ao, lw["post_attn_norm"]) if cfg.get("sandwich") else ao)
        xn = norm(X, lw["ffn_norm"])
        if cfg.get("n_experts", 0):
            ffn = np.stack([oracle.moe_ffn(cfg, lw, xn[t])[0] for t in range(T)])
        else:
            g, u = xn @ mat(lw, "w_gate").T, xn @ mat(lw, "w_up").T
            ffn = torch_bf16(g / (1 + np.exp(-g)) * u) @ mat(lw, "w_down").T
            if cfg.get("sandwich"):
                ffn = post(ffn, lw["post_ffn_norm"])
        X = X + ffn
    xf = norm(X[-1:], w["final_norm"])
    if cfg.get("tied"):
        head = f(w["embed"])
    elif q8:
        head = w["lm_head"].astype(np.float64) * w["lm_head_scale"].astype(np.float64)[:, None]
    else:
        head = f(w["lm_head"])
    logits = (xf @ head.T)[0]
    cap = cfg.get("final_softcap", 0.0)
    return cap * np.tanh(logits / cap) if cap else logits


@pytest.mark.parametrize("variant", ["dense", "tied_bias", "qknorm", "qknorm_bias", "moe", "moe_qknorm_bias",
                                     "swa_softcaps_sandwich", "swa_every_layer", "q8", "q8_swa_sandwich"])
def test_oracle_matches_whole_sequence_matrix_form(variant):
    if variant == "dense":
        cfg = _small_dense()
    elif variant == "swa_softcaps_sandwich":
        # layers 0 and 2 windowed (3 keys), layer 1 global; scores capped at 0.9 (the scores
        # of this model reach a few units, so the cap bends them); logits capped at 0.5
        cfg = dict(_small_dense(qk_norm=1), layers=3, sliding_window=3, swa_pattern=2, attn_softcap=0.9,
                   final_softcap=0.5, sandwich=1)
    elif variant == "swa_every_layer":
        cfg = _small_dense(sliding_window=4, swa_pattern=5, attn_softcap=2.0)
    elif variant == "q8":
        cfg = _small_dense(weight_format=1)
    elif variant == "q8_swa_sandwich":
        cfg = _small_dense(weight_format=1, sliding_window=2, swa_pattern=2, sandwich=1, final_softcap=3.0)
    elif variant == "tied_bias":
        cfg = _small_dense(tied=1, qkv_bias=1, rope_base=500000.0)
    elif variant == "qknorm":
        cfg = _small_dense(qk_norm=1)
    elif variant == "qknorm_bias":
        cfg = _small_dense(qk_norm=1, qkv_bias=1)
    elif variant == "moe_qknorm_bias":
        cfg = dict(_moe_cfg(E=6, k=2), hidden=32, layers=2, n_q_heads=4, n_kv_heads=2, head_dim=8,
                   qkv_bias=1, qk_norm=1, vocab=48, max_context=16)
    else:
        cfg = dict(_moe_cfg(E=6, k=2), hidden=32, layers=2, n_q_heads=4, n_kv_heads=4, head_dim=8,
                   qkv_bias=1, vocab=48, max_context=16)
    w = synth.make_weights(cfg, seed=14)
    # The matrix form sums in another order (fp64 differences ~1e-16). A value that close to
    # a bf16 rounding boundary rounds the other way and moves the logits by ~1e-4: prompt
    # 1002 meets one such value in the q8 + window + sandwich model, so that model uses 1003.
    toks = synth.tokens(9, cfg["vocab"], 1003 if variant == "q8_swa_sandwich" else 1002)
    got = oracle.Model(cfg, w).prefill(0, toks, 0)
    want = _textbook_forward(cfg, w, toks)
    assert np.allclose(got, want, rtol=1e-9, atol=1e-11)


def test_context_overflow_boundaries_from_the_pages():
    cfg = dict(_small_dense(), layers=1)
    w = synth.make_weights(cfg, seed=15)
    for line in open(os.path.join(GOLDEN, "context_overflow.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        kind, max_ctx, pos0, n, expect = line.split()
        m = oracle.Model(cfg, w, max_ctx=int(max_ctx))
        toks = np.arange(1, int(n) + 1, dtype=np.int32) % cfg["vocab"]
        try:
            if kind == "prefill":
                m.prefill(0, toks, int(pos0))
            else:
                m.forward(0, int(toks[0]), int(pos0))
            got = "ok"
        except oracle.OracleError as e:
            assert e.code == oracle.ERR_CONTEXT_OVERFLOW
            got = "overflow"
        assert got == expect, line


def test_empty_prompt_is_rejected():
    cfg = dict(_small_dense(), layers=1)
    m = oracle.Model(cfg, synth.make_weights(cfg, seed=16))
    with pytest.raises(oracle.OracleError):
        m.prefill(0, np.zeros(0, np.int32), 0)
