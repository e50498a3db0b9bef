"""MoE layers through the C ABI against the CPU oracle: router top-k indices must match
bit-exactly, logits within the parity bar, greedy tokens exact. Inputs are reseeded until
every checked routing decision is at least 1e-3 away from a tie and, past the first layer,
is also left in place when every embedding value moves by one bf16 ulp: fp32 accumulation
lands some bf16 roundings of each layer one ulp from the fp64 oracle's, and a decision that
noise of that size moves is not determined by the arithmetic."""
import numpy as np
import pytest

import oracle
import synth
from synth import configs
import decoder_only_transformer_layer_b200 as dec
from _util import assert_parity, perturb_inputs

pytestmark = pytest.mark.gpu
MARGIN = 1e-3


def tiny_moe(**over):
    cfg = dict(configs.COMMON, name="tiny-moe", hidden=256, layers=2, n_q_heads=4, n_kv_heads=2, head_dim=64,
               vocab=512, n_experts=8, top_k=2, expert_inter=96, shared_inter=128, shared_gate=1, qkv_bias=1,
               max_context=96, prefill_chunk=16)
    cfg.update(over)
    return cfg


def top_gap(v):
    s = np.sort(np.asarray(v, np.float64))
    return s[-1] - s[-2]


def stable(a, b):
    """The oracle's decisions (routes per layer, greedy token) and those of the one-ulp
    perturbed oracle agree."""
    (lga, rta), (lgb, rtb) = a, b
    return np.array_equal(rta[0], rtb[0]) and oracle.argmax(lga) == oracle.argmax(lgb)


def run_gated(cfg, w, n_prompt, n_steps, seed0=1100, tries=60):
    """Oracle prefill + teacher-forced decode; every step's logit gap and every decode
    step's router gaps must clear the margin, and the one-ulp perturbed oracle must make the
    same decisions. Returns prompt, greedy tokens, logits, routes."""
    wp = perturb_inputs(w)
    for t in range(tries):
        toks = synth.tokens(n_prompt, cfg["vocab"], seed0 + t)
        m, mp = oracle.Model(cfg, w), oracle.Model(cfg, wp)
        lg = [m.prefill(0, toks, 0)]
        routes = [m.last_routes()]
        pl = mp.prefill(0, toks, 0)
        ok = top_gap(lg[0]) >= MARGIN and routes[0][2].min() >= MARGIN and stable((lg[0], routes[0]),
                                                                                  (pl, mp.last_routes()))
        greedy = []
        for s in range(n_steps):
            if not ok:
                break
            tok = oracle.argmax(lg[-1])
            greedy.append(tok)
            lg.append(m.forward(0, tok, n_prompt + s))
            routes.append(m.last_routes())
            pl = mp.forward(0, tok, n_prompt + s)
            ok = top_gap(lg[-1]) >= MARGIN and routes[-1][2].min() >= MARGIN and stable((lg[-1], routes[-1]),
                                                                                        (pl, mp.last_routes()))
        mp.close()
        if ok:
            return toks, greedy, lg, routes, m
        m.close()
    pytest.fail("no prompt seed cleared the margins")


@pytest.mark.parametrize("norm_topk", [0, 1])
def test_tiny_moe_prefill_chunks_and_decode(norm_topk):
    cfg = tiny_moe(norm_topk=norm_topk)
    w = synth.make_weights(cfg)
    toks, greedy, lg, routes, m = run_gated(cfg, w, 40, 6)  # prefill chunks 16 + 16 + 8
    d = dec.Decoder(cfg, w)
    got = d.prefill_logits(0, toks, 0)
    assert_parity(got, lg[0], what="moe prefill")
    assert d.last_argmax(1)[0] == oracle.argmax(lg[0])
    for s, t in enumerate(greedy):
        got = d.step_logits([t], [40 + s])[0]
        assert_parity(got, lg[s + 1], what=f"moe decode step {s}")
        assert d.last_argmax(1)[0] == oracle.argmax(lg[s + 1])
        gr = d.last_routes(1)[:, 0, :]
        assert np.array_equal(gr, routes[s + 1][0]), f"step {s}: routes {gr} vs {routes[s + 1][0]}"
    d.close()


def test_tiny_moe_without_shared_gate_and_top1():
    cfg = tiny_moe(top_k=1, shared_gate=0)
    w = synth.make_weights(cfg)
    toks, greedy, lg, routes, m = run_gated(cfg, w, 17, 3, seed0=1200)
    d = dec.Decoder(cfg, w)
    assert_parity(d.prefill_logits(0, toks, 0), lg[0], what="moe top-1 prefill")
    for s, t in enumerate(greedy):
        assert_parity(d.step_logits([t], [17 + s])[0], lg[s + 1], what=f"moe top-1 step {s}")
        assert np.array_equal(d.last_routes(1)[:, 0, :], routes[s + 1][0])


def qwen_moe(layers, B, ctx):
    return configs.with_layers(configs.QWEN15_MOE_A27B, layers, max_context=ctx, max_batch=B)


def test_qwen_moe_shape_batch1_decode():
    cfg = qwen_moe(2, 1, 512)
    w = synth.make_weights(cfg)
    kvd = cfg["n_kv_heads"] * cfg["head_dim"]
    ctx = 300
    fills = [synth.kv_fill(ctx, kvd, 2000, l) for l in range(cfg["layers"])]
    wp = perturb_inputs(w)
    for attempt in range(40):
        toks = synth.tokens(3, cfg["vocab"], 1300 + attempt)
        m, mp = oracle.Model(cfg, w), oracle.Model(cfg, wp)
        for l, (k, v) in enumerate(fills):
            m.kv_write(0, l, 0, k, v)
            mp.kv_write(0, l, 0, k, v)
        lgs, rts, ok = [], [], True
        for s, t in enumerate(toks):
            lgs.append(m.forward(0, int(t), ctx + s))
            rts.append(m.last_routes())
            pl = mp.forward(0, int(t), ctx + s)
            ok = ok and rts[-1][2].min() >= MARGIN and top_gap(lgs[-1]) >= MARGIN and stable(
                (lgs[-1], rts[-1]), (pl, mp.last_routes()))
        mp.close()
        if ok:
            break
    else:
        pytest.fail("no seed cleared the margins")
    d = dec.Decoder(cfg, w)
    for l, (k, v) in enumerate(fills):
        d.kv_write(0, l, 0, k, v)
    for s, t in enumerate(toks):
        got = d.step_logits([int(t)], [ctx + s])[0]
        assert_parity(got, lgs[s], what=f"qwen-moe B=1 step {s}")
        assert np.array_equal(d.last_routes(1)[:, 0, :], rts[s][0])
        assert d.last_argmax(1)[0] == oracle.argmax(lgs[s])


def test_qwen_moe_shape_batch64_decode_sampled():
    # B = 64 sequences on synthetic caches of different lengths; the oracle checks 6 of them.
    B = 64
    cfg = qwen_moe(2, B, 256)
    w = synth.make_weights(cfg)
    kvd = cfg["n_kv_heads"] * cfg["head_dim"]
    lens = [64 + 3 * b for b in range(B)]
    sample = (0, 9, 23, 40, 51, 63)
    toks = synth.tokens(B, cfg["vocab"], 1400)
    ref = {}
    wp = perturb_inputs(w)
    for b in sample:  # reseed the sampled sequences' tokens until their routing clears the margin
        for attempt in range(40):
            tok = int(synth.tokens(1, cfg["vocab"], 1500 + 100 * b + attempt)[0])
            m, mp = oracle.Model(cfg, w), oracle.Model(cfg, wp)
            for l in range(cfg["layers"]):
                k, v = synth.kv_fill(lens[b], kvd, 2000, 100 * b + l)
                m.kv_write(0, l, 0, k, v)
                mp.kv_write(0, l, 0, k, v)
            lg = m.forward(0, tok, lens[b])
            rt = m.last_routes()
            ok = rt[2].min() >= MARGIN and stable((lg, rt), (mp.forward(0, tok, lens[b]), mp.last_routes()))
            m.close()
            mp.close()
            if ok:
                toks[b] = tok
                ref[b] = (lg, rt[0])
                break
        else:
            pytest.fail(f"no seed cleared the router margin for sequence {b}")
    d = dec.Decoder(cfg, w)
    for b in range(B):
        for l in range(cfg["layers"]):
            k, v = synth.kv_fill(lens[b], kvd, 2000, 100 * b + l)
            d.kv_write(b, l, 0, k, v)
    got = d.step_logits(toks, lens)
    routes = d.last_routes(B)
    for b in sample:
        assert_parity(got[b], ref[b][0], what=f"qwen-moe B=64 seq {b}")
        assert np.array_equal(routes[:, b, :], ref[b][1])


# (T, E, k, h, I): groups of 1, 2, 4 (T = 1, 2, 3) and 8 tokens (T >= 5) run on the tensor
# pipe wherever the projection's rows tile into 128-row blocks (2I = 256; h = 256 / 2048),
# else on the CUDA-core grouped GEMV (2I = 192, 272; h = 200): both kernels at every group
# size; K tails of 96, 136 and 200 columns; T * k = 2800 crosses the permutation's tile.
EXPERT_CASES = [(1, 8, 2, 256, 96), (2, 8, 2, 256, 96), (3, 8, 2, 256, 128), (5, 4, 2, 256, 128),
                (2, 8, 2, 200, 96), (3, 8, 2, 200, 128), (9, 8, 2, 200, 128),
                (8, 16, 4, 256, 128), (40, 8, 2, 256, 136),
                (64, 60, 4, 2048, 1408), (700, 16, 4, 256, 96), (33, 8, 8, 256, 128)]


def _experts_case(T, E, k, h, I, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    w = rng.uniform(0.05, 1.0, (T, k)).astype(np.float32)
    x = synth.bf16_normal((T, h), seed, 1, 0.0, 1.0)
    Wg = synth.bf16_normal((E, I, h), seed, 2, 0.0, h ** -0.5)  # unit-scale gate and up
    Wu = synth.bf16_normal((E, I, h), seed, 3, 0.0, h ** -0.5)
    Wd = synth.bf16_normal((E, h, I), seed, 4, 0.0, I ** -0.5)
    return idx, w, x, Wg, Wu, Wd


def _experts_ref(rows, idx, w, x, Wg, Wu, Wd):
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = np.zeros((len(rows), x.shape[1]))
    for i, t in enumerate(rows):
        for j, e in enumerate(idx[t]):
            if 0 <= e < Wg.shape[0]:
                ref[i] += float(w[t, j]) * oracle.swiglu(xf[t], Wg[e], Wu[e], Wd[e])
    return ref


def _experts_run(idx, w, x, Wg, Wu, Wd):
    import torch
    from _util import to_dev_bf16
    E, I, h = Wg.shape
    Wgu = np.stack([Wg, Wu], axis=2).reshape(E, 2 * I, h)  # gate row i at 2i, up row i at 2i + 1
    out = torch.full((x.shape[0], h), float("nan"), device="cuda")
    dec.moe_experts(to_dev_bf16(x, torch), torch.from_numpy(idx).cuda(), torch.from_numpy(w).cuda(),
                    to_dev_bf16(Wgu, torch), to_dev_bf16(Wd, torch), out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("T,E,k,h,I", EXPERT_CASES)
def test_moe_experts_standalone_matches_oracle(T, E, k, h, I):
    idx, w, x, Wg, Wu, Wd = _experts_case(T, E, k, h, I, 5000 + T)
    got = _experts_run(idx, w, x, Wg, Wu, Wd)
    rows = list(range(T)) if T <= 64 and h * I <= 2048 * 128 else sorted({0, 1, T // 3, T // 2, T - 2, T - 1})
    if T > 64:
        rows = sorted(set(rows) | set(range(0, T, 37)))
    ref = _experts_ref(rows, idx, w, x, Wg, Wu, Wd)
    d, r = assert_parity(got[rows], ref, what=f"moe_experts T={T} E={E} k={k} h={h} I={I}")
    # fp32 accumulation; the bf16 rounding of SiLU(g)*u may land one ulp apart on a few elements
    assert r <= 2e-3, f"kernel-level bar: rel={r:.2e}"


def test_moe_experts_drops_out_of_range_entries():
    T, E, k, h, I = 24, 8, 2, 256, 128
    idx, w, x, Wg, Wu, Wd = _experts_case(T, E, k, h, I, 5100)
    idx[3, 1] = -1
    idx[10, 0] = E
    idx[17, :] = E + 5
    got = _experts_run(idx, w, x, Wg, Wu, Wd)
    ref = _experts_ref(range(T), idx, w, x, Wg, Wu, Wd)
    assert_parity(got, ref, what="moe_experts with dropped entries")
    assert np.all(got[17] == 0.0)


def test_tiny_moe_tensor_core_expert_blocks():
    # 2I = 256 and h = 256 tile into 128-row blocks: prefill chunks of 32 tokens (groups of 8)
    # run both expert projections on the tensor pipe inside the model
    cfg = tiny_moe(expert_inter=128, prefill_chunk=32)
    w = synth.make_weights(cfg)
    toks, greedy, lg, routes, m = run_gated(cfg, w, 70, 2, seed0=1700)
    d = dec.Decoder(cfg, w)
    assert_parity(d.prefill_logits(0, toks, 0), lg[0], what="moe tensor-core prefill")
    assert d.last_argmax(1)[0] == oracle.argmax(lg[0])
    for s, t in enumerate(greedy):
        assert_parity(d.step_logits([t], [70 + s])[0], lg[s + 1], what=f"moe tensor-core step {s}")
    d.close()
