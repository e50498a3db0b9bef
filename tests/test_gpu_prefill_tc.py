"""The tensor-core prefill attention (head dim 128, power-of-two groups, chunks of at least
one CTA's tokens) against the CPU oracle through the C ABI: chunked prefills of the
Llama-3-8B shape (groups of 4 and 8), of the Qwen1.5-MoE attention (groups of 1) and of
windowed, softcapped layers, each followed by decode steps over the cache it wrote."""
import numpy as np
import pytest

import oracle
import synth
from synth import configs
import decoder_only_transformer_layer_b200 as dec
from _util import assert_parity, assert_within_conditioning, perturb_inputs
from test_gpu_model import check_model, gated_run

pytestmark = pytest.mark.gpu


def check_model_conditioned(cfg, n_prompt, n_steps):
    """check_model for two-layer stacks of the Llama-3-8B shape, whose logits (~6) move by
    about 0.5% when the inputs move by one bf16 ulp: the fixed bar, or twice that floor
    (the oracle run on the perturbed input) measured on the same prompt."""
    w = synth.make_weights(cfg)
    toks, greedy, ref, m = gated_run(cfg, w, n_prompt, n_steps)
    mp = oracle.Model(cfg, perturb_inputs(w))
    pert = [mp.prefill(0, toks, 0)] + [mp.forward(0, int(t), n_prompt + s) for s, t in enumerate(greedy)]
    mp.close()
    d = dec.Decoder(cfg, w)
    assert_within_conditioning(d.prefill_logits(0, toks, 0), ref[0], pert[0], what=f"{cfg['name']} prefill")
    if oracle.argmax(pert[0]) == oracle.argmax(ref[0]):
        assert d.last_argmax(1)[0] == oracle.argmax(ref[0])
    for s, t in enumerate(greedy):
        got = d.step_logits([t], [n_prompt + s])[0]
        assert_within_conditioning(got, ref[s + 1], pert[s + 1], what=f"{cfg['name']} step {s}")
    n = n_prompt + len(greedy)
    for li in range(cfg["layers"]):
        gk, gv = d.kv_read(0, li, 0, n)
        rk, rv = m.kv_read(0, li, 0, n)
        for g_, r_ in ((gk, rk), (gv, rv)):
            # layer 0 straight from the embedding; deeper rows (|v| up to ~8, one bf16 ulp
            # 0.03) carry the first layer's drift: a few ulps at the largest values
            assert_parity(synth.bits_to_f32(g_), synth.bits_to_f32(r_), abs_tol=0.03 if li == 0 else 0.1,
                          what=f"cache layer {li}")
            if li == 0:
                assert np.mean(g_ == r_) > 0.99
    d.close()


def test_llama8b_shape_chunks_of_128_and_a_tail_of_44():
    # 300 tokens: chunks 128 + 128 + 44 (every chunk on the tensor-core kernel: 32 tokens a CTA)
    cfg = configs.with_layers(configs.LLAMA3_8B, 1, max_context=320, max_batch=1)
    check_model(cfg, 300, 2)


def test_group_of_8_one_chunk_of_256():
    # 32 q heads over 4 kv heads (16 tokens a CTA), prefill chunk 256
    cfg = configs.with_layers(configs.LLAMA3_8B, 1, max_context=272, max_batch=1, n_kv_heads=4, prefill_chunk=256)
    check_model(cfg, 256, 2)


def test_group_of_1_qwen_attention_shape():
    # 16 q heads over 16 kv heads with QKV bias (128 tokens a CTA); dense FFN of the same width
    cfg = configs.with_layers(configs.LLAMA3_8B, 1, max_context=272, max_batch=1, hidden=2048, n_q_heads=16,
                              n_kv_heads=16, ffn_inter=5632, qkv_bias=1)
    check_model(cfg, 256, 2)


@pytest.mark.parametrize("window,softcap", [(100, 0.0), (0, 20.0), (200, 10.0)])
def test_window_and_softcap_on_the_tensor_core_path(window, softcap):
    # swa_pattern 2: layer 0 is windowed; 384 tokens in chunks of 128 cross the window's
    # start inside the key blocks, and the softcap bends the scores before the softmax
    cfg = configs.with_layers(configs.LLAMA3_8B, 2, max_context=400, max_batch=1, sliding_window=window,
                              swa_pattern=2 if window else 0, attn_softcap=softcap)
    check_model_conditioned(cfg, 384, 2)
