"""The C ABI's stream contract and error paths, on the GPU.

- dec_step and dec_prefill with device or NULL logits are stream-ordered: they return
  while the device is still busy.
- A device logits buffer is written by the LM head itself; NULL stores no logits and
  keeps the greedy token (the pages' folded head: frink_models decoder.rs FoldedLmHead).
- A bounded device wait that runs out is reported as DEC_ERR_TIMEOUT by the next
  synchronising call, and later calls are correct again. The wait made to run out is the
  tensor-core GEMM's stream-K reduction wait, which a CTA only enters once all its own
  loads and MMAs have completed (test hook dec_test_gemm_wait); nothing faults or traps.
- A failed device allocation inside dec_init is DEC_ERR_OOM and leaks nothing (test hook
  dec_test_fail_alloc)."""
import time

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import configs
import decoder_only_transformer_layer_b200 as dec
from _util import assert_parity, to_dev_bf16
from test_gpu_model import gated_run

pytestmark = pytest.mark.gpu


def _llama_small(layers=2, **over):
    return configs.with_layers(configs.LLAMA3_8B, layers, max_context=512, max_batch=4, **over)


def test_dec_step_returns_before_the_device_finishes():
    cfg = _llama_small()
    w = synth.make_weights(cfg)
    d = dec.Decoder(cfg, w)
    d.prefill(0, synth.tokens(20, cfg["vocab"], 1000), 0)
    d.step([5], [20])  # captures the B = 1 graph (not timed)
    torch.cuda.synchronize()
    for out in (None, torch.empty((1, cfg["vocab"]), device="cuda")):
        n = d.seq_len(0)
        torch.cuda._sleep(int(2e9))  # about a second of spinning queued ahead of the step
        t0 = time.perf_counter()
        d.step([7], [n], out)
        host_s = time.perf_counter() - t0
        busy = not torch.cuda.current_stream().query()
        torch.cuda.synchronize()
        assert busy, "the stream was idle when dec_step returned"
        assert host_s < 0.2, f"dec_step blocked for {host_s:.3f} s"
    t0 = time.perf_counter()
    torch.cuda._sleep(int(2e9))
    d.prefill(1, [3, 4, 5], 0)
    host_s = time.perf_counter() - t0
    assert not torch.cuda.current_stream().query() and host_s < 0.2
    d.check()
    d.close()


def test_device_host_and_no_logits_agree():
    cfg = dict(configs.TINY, max_batch=3)
    w = synth.make_weights(cfg)
    V = cfg["vocab"]
    runs = {}
    for mode in ("host", "device", "none"):
        d = dec.Decoder(cfg, w)
        for b in range(3):
            d.prefill(b, synth.tokens(10 + b, V, 1100 + b), 0)
        toks, pos = [1, 2, 3], [10, 11, 12]
        if mode == "host":
            lg = d.step_logits(toks, pos)
        elif mode == "device":
            buf = torch.full((3, V), float("nan"), device="cuda")
            d.step(toks, pos, buf)
            lg = buf.cpu().numpy()
        else:
            d.step(toks, pos, None)
            lg = None
        runs[mode] = (lg, d.last_argmax(3))
        d.close()
    assert np.array_equal(runs["host"][0], runs["device"][0])  # the same kernels and order: same bits
    assert np.array_equal(runs["host"][1], runs["device"][1])
    assert np.array_equal(runs["host"][1], runs["none"][1])
    assert np.array_equal(runs["host"][1], np.argmax(runs["host"][0], axis=1))


def test_prefill_writes_device_logits_directly():
    cfg = dict(configs.TINY)
    w = synth.make_weights(cfg)
    toks = synth.tokens(16, cfg["vocab"], 1000)
    ref = oracle.Model(cfg, w).prefill(0, toks, 0)
    d = dec.Decoder(cfg, w)
    buf = torch.full((cfg["vocab"],), float("nan"), device="cuda")
    d.prefill(0, toks, 0, buf)
    assert_parity(buf.cpu().numpy(), ref, what="prefill into a device buffer")
    d.close()


def test_greedy_only_decode_loop_matches_the_oracle():
    # logits_out = NULL every step: only the int32 greedy token leaves the device
    cfg = dict(configs.TINY)
    w = synth.make_weights(cfg)
    toks, greedy, ref, m = gated_run(cfg, w, 16, 8)
    d = dec.Decoder(cfg, w)
    d.prefill(0, toks, 0)
    t = int(d.last_argmax(1)[0])
    got = [t]
    for s in range(7):
        d.step([t], [16 + s])
        t = int(d.last_argmax(1)[0])
        got.append(t)
    assert got == [oracle.argmax(r) for r in ref[:8]]
    d.close()


def _gemm_case():
    # B = 16 tokens, N = 20480, K = 1024: 160 row tiles (more than the SMs, so the persistent
    # stream-K GEMM, not the cluster split-K one), tiles shared between CTAs
    B, N, K = 16, 20480, 1024
    W = synth.bf16_normal((N, K), 7, 1, 0.0, 0.02)
    x = synth.bf16_normal((B, K), 7, 2, 0.0, 1.0)
    return W, x, oracle.gemv_rows(W, x)


def test_a_wait_that_runs_out_is_reported_and_the_next_call_is_correct():
    W, x, ref = _gemm_case()
    Wd, xd = to_dev_bf16(W, torch), to_dev_bf16(x, torch)
    y = torch.zeros(ref.shape, device="cuda")
    dec.check_standalone()
    dec.test_gemm_wait(1, 1 << 21)  # about a millisecond, waiting for a piece that never comes
    try:
        dec.weight_gemv(Wd, xd, y)
        with pytest.raises(dec.DecError) as e:
            dec.check_standalone()
        assert e.value.status == "TIMEOUT"
    finally:
        dec.test_gemm_wait(0, 0)
    dec.check_standalone()  # the word was cleared
    for _ in range(2):
        y.zero_()
        dec.weight_gemv(Wd, xd, y)
        dec.check_standalone()
        assert_parity(y.cpu().numpy(), ref, what="GEMM after a timed-out call")


def test_a_timed_out_prefill_is_reported_by_the_context():
    cfg = configs.with_layers(configs.SMOLLM2_135M, 1, max_context=512)
    w = synth.make_weights(cfg)
    toks = synth.tokens(256, cfg["vocab"], 1000)
    ref = oracle.Model(cfg, w).prefill(0, toks, 0)
    d = dec.Decoder(cfg, w)
    dec.test_gemm_wait(1, 1 << 21)
    try:
        d.prefill(0, toks, 0)  # device logits target: no synchronisation, no error yet
        with pytest.raises(dec.DecError) as e:
            d.check()
        assert e.value.status == "TIMEOUT"
    finally:
        dec.test_gemm_wait(0, 0)
    d.check()
    d.reset(0)
    got = d.prefill_logits(0, toks, 0)
    assert_parity(got, ref, what="prefill after a timed-out prefill")
    d.close()


def test_allocation_failure_in_init_is_oom_and_leaks_nothing():
    cfg = dict(configs.TINY, layers=2)
    w = synth.make_weights(cfg)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    try:
        for n in (1, 2, 7, 15, 30):
            dec.test_fail_alloc(n)
            with pytest.raises(dec.DecError) as e:
                dec.Decoder(cfg, w)
            assert e.value.status == "OOM", (n, str(e.value))
    finally:
        dec.test_fail_alloc(0)
    torch.cuda.synchronize()
    assert abs(torch.cuda.mem_get_info()[0] - free0) < (4 << 20)
    d = dec.Decoder(cfg, w)
    toks = synth.tokens(16, cfg["vocab"], 1000)
    assert_parity(d.prefill_logits(0, toks, 0), oracle.Model(cfg, w).prefill(0, toks, 0), what="after OOM")
    d.close()
