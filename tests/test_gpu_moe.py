"""MoE layers through the C ABI against the CPU oracle: router top-k indices must match
bit-exactly (inputs reseeded until every checked routing decision is at least 1e-3 away
from a tie), logits within the parity bar, greedy tokens exact."""
import numpy as np
import pytest

import oracle
import synth
from synth import configs
import decoder_only_transformer_layer_b200 as dec
from _util import assert_parity

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


def run_gated(cfg, w, n_prompt, n_steps, seed0=1100, tries=60):
    """Oracle prefill + teacher-forced decode; every step's logit gap and every decode
    step's router gaps must clear the margin. Returns prompt, greedy tokens, logits, routes."""
    for t in range(tries):
        toks = synth.tokens(n_prompt, cfg["vocab"], seed0 + t)
        m = oracle.Model(cfg, w)
        lg = [m.prefill(0, toks, 0)]
        routes = [m.last_routes()]
        ok = top_gap(lg[0]) >= MARGIN and routes[0][2].min() >= MARGIN
        greedy = []
        for s in range(n_steps):
            if not ok:
                break
            tok = oracle.argmax(lg[-1])
            greedy.append(tok)
            lg.append(m.forward(0, tok, n_prompt + s))
            routes.append(m.last_routes())
            ok = top_gap(lg[-1]) >= MARGIN and routes[-1][2].min() >= MARGIN
        if ok:
            return toks, greedy, lg, routes, m
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
    for attempt in range(40):
        toks = synth.tokens(3, cfg["vocab"], 1300 + attempt)
        m = oracle.Model(cfg, w)
        for l, (k, v) in enumerate(fills):
            m.kv_write(0, l, 0, k, v)
        lgs, rts, ok = [], [], True
        for s, t in enumerate(toks):
            lgs.append(m.forward(0, int(t), ctx + s))
            rts.append(m.last_routes())
            ok = ok and rts[-1][2].min() >= MARGIN and top_gap(lgs[-1]) >= MARGIN
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
    for b in sample:  # reseed the sampled sequences' tokens until their routing clears the margin
        for attempt in range(40):
            tok = int(synth.tokens(1, cfg["vocab"], 1500 + 100 * b + attempt)[0])
            m = oracle.Model(cfg, w)
            for l in range(cfg["layers"]):
                k, v = synth.kv_fill(lens[b], kvd, 2000, 100 * b + l)
                m.kv_write(0, l, 0, k, v)
            lg = m.forward(0, tok, lens[b])
            rt = m.last_routes()
            if rt[2].min() >= MARGIN:
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
