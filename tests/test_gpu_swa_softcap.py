"""Sliding-window attention, attention and final logit softcaps, and sandwich norms (ANEDVD
engine.zig: attentionDecode's .window / .logit_softcap, runHead's final cap, the post-
attention and post-FFN rmsnormFlat; cortiq pipeline.rs: the per-layer window schedule)
through dec_prefill / dec_step against the CPU oracle.

The window is exercised where it crosses prefill key blocks and page boundaries, with
windowed and global layers interleaved; decode is teacher-forced, greedy tokens exact."""
import numpy as np
import pytest

import oracle
import synth
from synth import configs
import decoder_only_transformer_layer_b200 as dec
from _util import assert_parity
from test_gpu_model import check_cache, gated_run

pytestmark = pytest.mark.gpu


def _run(cfg, n_prompt, n_steps, seed):
    w = synth.make_weights(cfg)
    toks, greedy, ref, m = gated_run(cfg, w, n_prompt, n_steps, seq_seed=seed)
    d = dec.Decoder(cfg, w)
    got = d.prefill_logits(0, toks, 0)
    assert_parity(got, ref[0], what=f"{cfg['name']} prefill")
    assert d.last_argmax(1)[0] == oracle.argmax(ref[0])
    for s, t in enumerate(greedy):
        got = d.step_logits([t], [n_prompt + s])[0]
        assert_parity(got, ref[s + 1], what=f"{cfg['name']} step {s}")
        assert d.last_argmax(1)[0] == oracle.argmax(ref[s + 1])
    check_cache(d, m, cfg["layers"], n_prompt + len(greedy))
    d.close()


@pytest.mark.parametrize("window,pattern", [(5, 2), (16, 3), (1, 2), (40, 9)])
def test_tiny_sliding_window(window, pattern):
    # window 5 / 16 cross pages; window 1 attends only the current position; pattern 9 > L
    # makes every layer windowed
    cfg = dict(configs.TINY, layers=3, sliding_window=window, swa_pattern=pattern, prefill_chunk=8, max_context=96)
    _run(cfg, 30, 6, 3700)


def test_tiny_softcaps_and_sandwich():
    # the tiny model's scores are small, so the cap (0.15) is what bends them; logits capped at 0.4
    cfg = dict(configs.TINY, attn_softcap=0.15, final_softcap=0.4, sandwich=1, prefill_chunk=16)
    _run(cfg, 20, 6, 3800)


def test_tiny_everything_at_once():
    cfg = dict(configs.TINY, layers=4, qk_norm=1, sliding_window=7, swa_pattern=2, attn_softcap=0.2,
               final_softcap=0.5, sandwich=1, prefill_chunk=8, max_context=80)
    _run(cfg, 40, 5, 3900)


def test_smollm2_shape_window_across_key_blocks_and_splits():
    # window 100 over 64-key prefill blocks, chunks 128 + 128 + 44, key splits in a cluster
    cfg = configs.with_layers(configs.SMOLLM2_135M, 2, max_context=512, sliding_window=100, swa_pattern=2,
                              attn_softcap=2.0)
    _run(cfg, 300, 3, 4000)


def test_batched_decode_with_a_window_on_ragged_caches():
    # B = 32 sequences, every layer windowed (window 200): the decode kernel's page range
    # starts inside the cache and its context splits cover only the window
    B = 32
    cfg = configs.with_layers(configs.LLAMA3_8B, 1, max_context=512, max_batch=B, sliding_window=200, swa_pattern=2,
                              attn_softcap=5.0)
    w = synth.make_weights(cfg)
    kvd = cfg["n_kv_heads"] * cfg["head_dim"]
    lens = [100 + 9 * b for b in range(B)]
    d = dec.Decoder(cfg, w)
    toks = synth.tokens(B, cfg["vocab"], 4100)
    sample = (0, 7, 11, 19, 26, 31)
    models = {}
    for b in range(B):
        k, v = synth.kv_fill(lens[b], kvd, 2000, b)
        d.kv_write(b, 0, 0, k, v)
        if b in sample:
            m = oracle.Model(cfg, w)
            m.kv_write(0, 0, 0, k, v)
            models[b] = m
    got = d.step_logits(toks, lens)
    for b in sample:
        ref = models[b].forward(0, int(toks[b]), lens[b])
        assert_parity(got[b], ref, what=f"windowed B=32 seq {b}")


def test_window_changes_the_result_only_past_the_window():
    # positions inside the window give the same logits as full attention; later ones do not
    cfg = dict(configs.TINY, layers=1)
    w = synth.make_weights(cfg)
    toks = synth.tokens(20, cfg["vocab"], 1000)
    full = dec.Decoder(cfg, w)
    win = dec.Decoder(dict(cfg, sliding_window=12, swa_pattern=2), w)
    a, b = full.prefill_logits(0, toks[:12], 0), win.prefill_logits(0, toks[:12], 0)
    assert np.array_equal(a, b)
    a, b = full.prefill_logits(0, toks[12:], 12), win.prefill_logits(0, toks[12:], 12)
    assert np.max(np.abs(a - b)) > 1e-3
