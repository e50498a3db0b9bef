"""QK-norm (ANEDVD applyHeadNorm: a per-head RMSNorm of q and k before the rotation)
through dec_prefill / dec_step against the CPU oracle, dense and MoE (with QKV bias).

Prefill runs over several chunks (the prefill kernel that normalises, rotates and appends
a whole chunk), decode is teacher-forced (the decode-attention kernel normalises and
rotates its own row); greedy tokens and routing must match bit-exactly."""
import numpy as np
import pytest

import oracle
import synth
from synth import configs
import decoder_only_transformer_layer_b200 as dec
from _util import assert_parity
from test_gpu_model import check_cache, gated_run
from test_gpu_moe import run_gated, tiny_moe

pytestmark = pytest.mark.gpu


def test_tiny_dense_qk_norm_prefill_chunks_and_decode():
    cfg = dict(configs.TINY, qk_norm=1, prefill_chunk=8)
    w = synth.make_weights(cfg)
    n_prompt, n_steps = 20, 6  # chunks 8 + 8 + 4
    toks, greedy, ref, m = gated_run(cfg, w, n_prompt, n_steps, seq_seed=1600)
    d = dec.Decoder(cfg, w)
    got = d.prefill_logits(0, toks, 0)
    assert_parity(got, ref[0], what="qk-norm prefill")
    assert d.last_argmax(1)[0] == oracle.argmax(ref[0])
    for s, t in enumerate(greedy):
        got = d.step_logits([t], [n_prompt + s])[0]
        assert_parity(got, ref[s + 1], what=f"qk-norm decode step {s}")
        assert d.last_argmax(1)[0] == oracle.argmax(ref[s + 1])
    check_cache(d, m, cfg["layers"], n_prompt + n_steps)
    d.close()


def test_qk_norm_changes_the_result():
    # The same weights without the norm give other logits: the flag is not ignored.
    cfg = dict(configs.TINY, qk_norm=1)
    w = synth.make_weights(cfg)
    toks = synth.tokens(16, cfg["vocab"], 1000)
    a = dec.Decoder(cfg, w).prefill_logits(0, toks, 0)
    b = dec.Decoder(dict(cfg, qk_norm=0), w).prefill_logits(0, toks, 0)
    assert np.max(np.abs(a - b)) > 1e-2


@pytest.mark.parametrize("chunk", [16, 32])
def test_tiny_moe_qk_norm_with_bias(chunk):
    cfg = tiny_moe(qk_norm=1, qkv_bias=1, prefill_chunk=chunk)
    w = synth.make_weights(cfg)
    toks, greedy, lg, routes, m = run_gated(cfg, w, 40, 5, seed0=1800)
    d = dec.Decoder(cfg, w)
    assert_parity(d.prefill_logits(0, toks, 0), lg[0], what="moe qk-norm prefill")
    assert d.last_argmax(1)[0] == oracle.argmax(lg[0])
    for s, t in enumerate(greedy):
        got = d.step_logits([t], [40 + s])[0]
        assert_parity(got, lg[s + 1], what=f"moe qk-norm step {s}")
        assert d.last_argmax(1)[0] == oracle.argmax(lg[s + 1])
        assert np.array_equal(d.last_routes(1)[:, 0, :], routes[s + 1][0])
    check_cache(d, m, cfg["layers"], 40 + len(greedy))
    d.close()
