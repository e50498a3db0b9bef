"""Whole-stack parity: dec_prefill / dec_step through the C ABI against the CPU oracle.

Decode parity is teacher-forced (the oracle's greedy token feeds both sides), prompts
are reseeded until every checked step's top-1/top-2 logit gap is >= 1e-3, and greedy
tokens must match bit-exactly."""
import os

import numpy as np
import pytest

import oracle
import synth
from synth import configs
import decoder_only_transformer_layer_b200 as dec
from _util import assert_parity

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def top_gap(logits):
    s = np.sort(np.asarray(logits, np.float64))
    return s[-1] - s[-2]


def gated_run(cfg, w, n_prompt, n_steps, seq_seed=1000, max_tries=40):
    """Oracle prefill + teacher-forced greedy decode, reseeding the prompt until every logit
    gap clears 1e-3. Returns (prompt, greedy tokens, [logits per step], oracle model)."""
    for k in range(max_tries):
        toks = synth.tokens(n_prompt, cfg["vocab"], seq_seed + k)
        m = oracle.Model(cfg, w)
        lg = [m.prefill(0, toks, 0)]
        out = []
        ok = top_gap(lg[0]) >= 1e-3
        for s in range(n_steps):
            if not ok:
                break
            t = oracle.argmax(lg[-1])
            out.append(t)
            lg.append(m.forward(0, t, n_prompt + s))
            ok = top_gap(lg[-1]) >= 1e-3
        if ok:
            return toks, out, lg, m
        m.close()
    pytest.fail("no prompt seed cleared the logit margin")


def check_model(cfg, n_prompt, n_steps):
    w = synth.make_weights(cfg)
    toks, greedy, ref_logits, m = gated_run(cfg, w, n_prompt, n_steps)
    d = dec.Decoder(cfg, w)
    got = d.prefill_logits(0, toks, 0)
    assert_parity(got, ref_logits[0], what=f"{cfg['name']} prefill")
    assert int(np.argmax(got)) == oracle.argmax(ref_logits[0])
    assert d.last_argmax(1)[0] == oracle.argmax(ref_logits[0])
    for s, t in enumerate(greedy):
        got = d.step_logits([t], [n_prompt + s])[0]
        assert_parity(got, ref_logits[s + 1], what=f"{cfg['name']} decode step {s}")
        assert d.last_argmax(1)[0] == oracle.argmax(ref_logits[s + 1])
    check_cache(d, m, cfg["layers"], n_prompt + len(greedy))
    d.close()


def check_cache(d, m, layers, n):
    """Every cache row within the parity bar. Layer 0 rows come straight from the embedding,
    so they must match bit for bit (up to the rare fp32-vs-fp64 rounding flip); deeper layers
    inherit bf16 rounding flips from the layers before them (each flip perturbs every later
    value slightly), so there only the tolerance applies."""
    for li in range(layers):
        gk, gv = d.kv_read(0, li, 0, n)
        rk, rv = m.kv_read(0, li, 0, n)
        for g_, r_ in ((gk, rk), (gv, rv)):
            gf = synth.bits_to_f32(g_).astype(np.float64)
            rf = synth.bits_to_f32(r_).astype(np.float64)
            assert_parity(gf, rf, what=f"cache layer {li}")
            if li == 0:
                assert np.mean(g_ == r_) > 0.99


def test_tiny_dense_prefill16_decode8():
    check_model(dict(configs.TINY), 16, 8)


def test_smollm2_shape_4_layers_ragged_chunks():
    cfg = configs.with_layers(configs.SMOLLM2_135M, 4, max_context=512)
    check_model(cfg, 300, 3)  # chunks 128 + 128 + 44


def test_smollm2_shape_2_layers_chunk512():
    # prefill_chunk 512: tensor-core GEMMs over several 128-token column tiles (N = 512, then
    # a ragged N = 188) and prefill attention over 512-token chunks
    cfg = configs.with_layers(configs.SMOLLM2_135M, 2, max_context=1024, prefill_chunk=512)
    check_model(cfg, 700, 2)  # chunks 512 + 188


def test_llama8b_shape_1_layer_chunk_tail():
    cfg = configs.with_layers(configs.LLAMA3_8B, 1, max_context=256, max_batch=1)
    check_model(cfg, 136, 2)  # chunks 128 + 8


def test_prefill_equals_sequential_steps_on_gpu():
    cfg = dict(configs.TINY)
    w = synth.make_weights(cfg)
    toks = synth.tokens(20, cfg["vocab"], 1005)
    a = dec.Decoder(cfg, w)
    la = a.prefill_logits(0, toks, 0)
    b = dec.Decoder(cfg, w)
    for t, tok in enumerate(toks):
        lb = b.step_logits([tok], [t])[0]
    assert_parity(la, lb, what="prefill vs steps")
    for li in range(cfg["layers"]):
        ka, va = a.kv_read(0, li, 0, 20)
        kb, vb = b.kv_read(0, li, 0, 20)
        for x, y in ((ka, kb), (va, vb)):
            assert_parity(synth.bits_to_f32(x), synth.bits_to_f32(y), what=f"prefill vs steps cache layer {li}")
            if li == 0:
                assert np.mean(x == y) > 0.99


def test_batched_decode_ragged_lengths_gemm_path():
    # B = 32 sequences of different lengths on a synthetic cache (Llama-3-8B shape, 1 layer):
    # the projections run on the tcgen05 GEMM. The oracle checks 6 of the 32 sequences.
    B = 32
    cfg = configs.with_layers(configs.LLAMA3_8B, 1, max_context=512, max_batch=B)
    w = synth.make_weights(cfg)
    kvd = cfg["n_kv_heads"] * cfg["head_dim"]
    lens = [100 + 7 * b for b in range(B)]
    d = dec.Decoder(cfg, w)
    toks = synth.tokens(B, cfg["vocab"], 1010)
    sample = (0, 5, 13, 20, 27, 31)
    models = {}
    for b in range(B):
        k, v = synth.kv_fill(lens[b], kvd, 2000, b)
        d.kv_write(b, 0, 0, k, v)
        if b in sample:
            m = oracle.Model(cfg, w)
            m.kv_write(0, 0, 0, k, v)
            models[b] = m
    got = d.step_logits(toks, lens)
    am = d.last_argmax(B)
    for b in sample:
        ref = models[b].forward(0, int(toks[b]), lens[b])
        assert_parity(got[b], ref, what=f"B=32 seq {b}")
        if top_gap(ref) >= 1e-3:
            assert am[b] == oracle.argmax(ref)
    # second step continues every sequence
    toks2 = am.copy()
    got2 = d.step_logits(toks2, [l + 1 for l in lens])
    for b in sample:
        ref2 = models[b].forward(0, int(toks2[b]), lens[b] + 1)
        assert_parity(got2[b], ref2, what=f"B=32 step 2 seq {b}")


def test_context_overflow_boundaries_from_the_pages():
    cfg = dict(configs.TINY, layers=1)
    w = synth.make_weights(cfg)
    for line in open(os.path.join(GOLDEN, "context_overflow.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        kind, max_ctx, pos0, n, expect = line.split()
        c = dict(cfg, max_context=int(max_ctx))
        d = dec.Decoder(c, w)
        pos0, n = int(pos0), int(n)
        if pos0 > 0 and pos0 < int(max_ctx):
            d.prefill(0, np.arange(pos0, dtype=np.int32) % cfg["vocab"] + 1, 0)
        toks = np.arange(1, n + 1, dtype=np.int32)
        try:
            if kind == "prefill":
                d.prefill(0, toks, pos0)
            else:
                d.step(toks[:1], [pos0])
            got = "ok"
        except dec.DecError as e:
            assert e.status in ("CONTEXT_OVERFLOW",), str(e)
            got = "overflow"
        assert got == expect, line
        d.close()


def test_bad_arguments_are_refused_before_any_launch():
    cfg = dict(configs.TINY, layers=1, max_batch=2, n_pages=3)
    w = synth.make_weights(cfg)
    d = dec.Decoder(cfg, w)
    with pytest.raises(dec.DecError) as e:
        d.prefill(0, np.zeros(0, np.int32), 0)
    assert e.value.status == "INVALID_ARG"
    with pytest.raises(dec.DecError) as e:
        d.prefill(0, [cfg["vocab"]], 0)
    assert e.value.status == "INVALID_ARG"
    with pytest.raises(dec.DecError) as e:
        d.prefill(0, [1, 2], 5)  # pos0 must equal the sequence length (each token enters once)
    assert e.value.status == "INVALID_ARG"
    d.prefill(0, np.arange(40, dtype=np.int32), 0)  # 3 pages: the whole pool
    with pytest.raises(dec.DecError) as e:
        d.prefill(1, [1], 0)
    assert e.value.status == "PAGES_EXHAUSTED"
    d.reset(0)
    d.prefill(1, [1], 0)  # pages returned by reset are reused
    assert d.seq_len(1) == 1 and d.seq_len(0) == 0


def test_decode_splits_of_unequal_length_merge_correctly():
    # SmolLM2 shape at context 1024..1039: the batch-1 decode attention runs 9 context splits
    # per kv head as one thread-block cluster, 8 of 8 pages and the last of 1 page. The short
    # split finishes first and pushes its partial into the other CTAs' shared memory; that
    # must wait until they are done with the page rings the receive area overlaps.
    cfg = configs.with_layers(configs.SMOLLM2_135M, 3, max_context=1040)
    w = synth.make_weights(cfg)
    toks, greedy, ref, m = gated_run(cfg, w, 1024, 14, seq_seed=1900)
    d = dec.Decoder(cfg, w)
    assert_parity(d.prefill_logits(0, toks, 0), ref[0], what="prefill 1024")
    for s, t in enumerate(greedy):
        got = d.step_logits([t], [1024 + s])[0]
        assert_parity(got, ref[s + 1], what=f"step {s} at position {1024 + s}")
    d.close()
