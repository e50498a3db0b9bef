"""Multi-position verify and rollback (cortiq_engine pipeline.rs: forward_pair streams the
weights once for several positions; truncate_last drops the KV rows of rejected draft
tokens), through the C ABI against the CPU oracle.

In the oracle, N verify positions are N sequential forwards, and a rollback is nothing
at all: a position's cache row is written before anything reads it, so re-stepping after
truncation equals never having stepped."""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import configs
import decoder_only_transformer_layer_b200 as dec
from _util import assert_parity, assert_within_conditioning, perturb_inputs

pytestmark = pytest.mark.gpu


def top_gap(v):
    s = np.sort(np.asarray(v, np.float64))
    return s[-1] - s[-2]


def _gated(cfg, w, n_prompt, drafts, seed0):
    """Oracle prefill then the draft tokens forwarded one by one; reseed the prompt until
    every checked logit row clears the 1e-3 margin. Returns prompt, per-position logits."""
    for k in range(40):
        toks = synth.tokens(n_prompt, cfg["vocab"], seed0 + k)
        m = oracle.Model(cfg, w)
        lg = [m.prefill(0, toks, 0)]
        for i, t in enumerate(drafts):
            lg.append(m.forward(0, int(t), n_prompt + i))
        if min(top_gap(x) for x in lg) >= 1e-3:
            return toks, lg, m
        m.close()
    pytest.fail("no prompt seed cleared the logit margin")


@pytest.mark.parametrize("cfg_name,N", [("tiny", 1), ("tiny", 4), ("tiny", 8), ("llama", 3), ("moe", 5)])
def test_verify_equals_sequential_steps(cfg_name, N):
    if cfg_name == "tiny":
        cfg = dict(configs.TINY)
    elif cfg_name == "llama":
        cfg = configs.with_layers(configs.LLAMA3_8B, 2, max_context=512)
    else:
        cfg = dict(configs.COMMON, name="tiny-moe", hidden=256, layers=2, n_q_heads=4, n_kv_heads=2, head_dim=64,
                   vocab=512, n_experts=8, top_k=2, expert_inter=96, shared_inter=128, shared_gate=1, qkv_bias=1,
                   max_context=96, prefill_chunk=16)
    w = synth.make_weights(cfg)
    drafts = synth.tokens(N, cfg["vocab"], 3100 + N)
    n_prompt = 37
    toks, ref, m = _gated(cfg, w, n_prompt, drafts, 3000)
    d = dec.Decoder(cfg, w)
    d.prefill(0, toks, 0)
    got = d.verify_logits(0, drafts, n_prompt)
    assert d.seq_len(0) == n_prompt + N
    am = d.last_argmax(N)
    if cfg_name == "llama":
        # logits of the 8B shape reach ~6: 3e-2 absolute is 0.5%, at the level of the
        # problem's own response to a one-ulp change of the inputs, so that floor applies
        mp = oracle.Model(cfg, perturb_inputs(w))
        pert = [mp.prefill(0, toks, 0)] + [mp.forward(0, int(t), n_prompt + i) for i, t in enumerate(drafts)]
    for i in range(N):
        if cfg_name == "llama":
            assert_within_conditioning(got[i], ref[i + 1], pert[i + 1], what=f"{cfg_name} verify position {i}")
        else:
            assert_parity(got[i], ref[i + 1], what=f"{cfg_name} verify position {i}")
        assert am[i] == oracle.argmax(ref[i + 1])
    # the verified rows are in the cache, as after N steps
    for li in range(cfg["layers"]):
        gk, gv = d.kv_read(0, li, n_prompt, N)
        rk, rv = m.kv_read(0, li, n_prompt, N)
        for x, y in ((gk, rk), (gv, rv)):
            # 8B-shape rows reach |v| ~ 8, where one bf16 ulp is 0.03: allow a few ulps there
            assert_parity(synth.bits_to_f32(x), synth.bits_to_f32(y), abs_tol=0.1 if cfg_name == "llama" else 3e-2,
                          what=f"verify cache layer {li}")
    d.close()


def test_truncate_then_restep_equals_never_having_stepped():
    # verify 4 drafts, accept 2 (truncate the last 2 rows), step a different token: the result
    # must equal prefill + the 2 accepted tokens + the new token, with no trace of the rest
    cfg = dict(configs.TINY)
    w = synth.make_weights(cfg)
    drafts = synth.tokens(4, cfg["vocab"], 3200)
    for k in range(40):
        alt = int(synth.tokens(1, cfg["vocab"], 3300 + k)[0])
        toks, ref, m = _gated(cfg, w, 20, list(drafts[:2]) + [alt], 3400 + k)
        if alt != drafts[2]:
            break
    d = dec.Decoder(cfg, w)
    d.prefill(0, toks, 0)
    d.verify(0, drafts, 20)
    d.truncate(0, 22)
    assert d.seq_len(0) == 22
    got = d.step_logits([alt], [22])[0]
    assert_parity(got, ref[3], what="re-step after truncate")
    assert d.last_argmax(1)[0] == oracle.argmax(ref[3])
    # truncating across a page boundary returns pages; growing again re-allocates them
    d.truncate(0, 10)
    assert d.seq_len(0) == 10
    m2 = oracle.Model(cfg, w)
    m2.prefill(0, toks[:10], 0)
    tail = synth.tokens(12, cfg["vocab"], 3500)
    ref2 = m2.prefill(0, tail, 10)
    got2 = d.prefill_logits(0, tail, 10)
    assert_parity(got2, ref2, what="prefill after truncating across a page")
    d.close()


def test_verify_device_logits_and_errors():
    cfg = dict(configs.TINY, max_context=40)
    w = synth.make_weights(cfg)
    d = dec.Decoder(cfg, w)
    d.prefill(0, synth.tokens(30, cfg["vocab"], 1000), 0)
    drafts = synth.tokens(4, cfg["vocab"], 3600)
    host = d.verify_logits(0, drafts, 30)
    d.truncate(0, 30)
    buf = torch.full((4, cfg["vocab"]), float("nan"), device="cuda")
    d.verify(0, drafts, 30, buf)
    assert np.array_equal(buf.cpu().numpy(), host)  # same kernels, same order: same bits
    d.truncate(0, 30)
    for bad in (lambda: d.verify(0, np.arange(9), 30),           # more than 8 positions
                lambda: d.verify(0, drafts, 29),                 # not at the sequence length
                lambda: d.verify(0, [cfg["vocab"]], 30),         # token out of range
                lambda: d.truncate(0, 31),                       # longer than the sequence
                lambda: d.truncate(0, -1)):
        with pytest.raises(dec.DecError) as e:
            bad()
        assert e.value.status == "INVALID_ARG"
    with pytest.raises(dec.DecError) as e:
        d.verify(0, np.arange(1, 12), 30)
    assert e.value.status == "INVALID_ARG"
    d.prefill(0, np.arange(1, 11), 30)  # exactly fills the context
    with pytest.raises(dec.DecError) as e:
        d.verify(0, [1], 40)
    assert e.value.status == "CONTEXT_OVERFLOW"
    d.close()
