"""Benchmark: decode and prefill throughput of a Llama-3-8B-shaped decoder stack on B200.

Default workload (one GPU): random-init bf16 weights of the Llama-3-8B shape (hidden 4096,
32 layers, 32/8 heads of 128, SwiGLU 14336, vocab 128256, RoPE base 5e5); a 4096-token
synthetic prompt is prefilled in chunks of 128 (timed: prefill tok/s), then batch-1 greedy
decode steps run at context 4096+ (timed: the headline decode tok/s). Every decode step
streams 15 GB of weights, far above the 126 MB L2, so no L2 flush is needed between steps.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Multi-GPU: one process per GPU under torchrun; each rank runs an independent replica
(the path has no exchange step), timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from synth import configs  # noqa: E402

METRIC = "decode tok/s + % HBM roofline (8B-shape, b=1); prefill tok/s + % bf16 TC peak"
PROMPT = 4096


def main_config(world, layers):
    """The `config` of the default line, shared by both arms (ours and the reference)."""
    return dict(workload="llama3-8b-shape decode b=1 at context 4096 after a 4096-token prefill (chunk 128)",
                global_batch=world, seq_len=PROMPT, model_shape="llama3-8b", layers=layers,
                parallelism=f"replicas x{world}", l2="inputs larger than L2 (15 GB of weights per step)")


def max_over_ranks(values, device=None):
    """Replicas: every rank times its own copy of the workload; the job's time is the max
    over ranks (a collective on the timings only, never on the data path)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def replica_throughput(units_per_rank, world, ms):
    """Whole-job throughput of N replicas: all ranks' units over the slowest rank's time."""
    return world * units_per_rank / (ms * 1e-3)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return dict(hbm=j["hbm_gbs"], tc=j["bf16_tflops"], tc_sus=j.get("bf16_tflops_sustained", j["bf16_tflops"]),
                    src="measured")
    return dict(hbm=6650.0, tc=1590.0, tc_sus=1400.0, src="fallback")


def measured_traffic():
    """dram read+write bytes per launch of the roofline kernel, from the committed ncu summary;
    None when that summary is missing or the kernel source changed since it was captured."""
    import hashlib
    import re
    try:
        txt = open(os.path.join(ROOT, "profiles", "gemv_llama3-8b_decode_full.md")).read()
        src = open(os.path.join(ROOT, "decoder_only_transformer_layer_b200", "csrc", "gemv.cu"), "rb").read()
    except OSError:
        return None
    m = re.search(r"traffic_bytes_per_launch: (\d+)", txt)
    h = re.search(r"kernel_sha256: ([0-9a-f]+)", txt)
    if not m or not h or h.group(1) != hashlib.sha256(src).hexdigest():
        return None
    return int(m.group(1))


def layer_bytes(cfg):
    """Projection weight bytes of one layer: bf16, or q8_row (1 byte per weight + a 4-byte scale
    per row)."""
    h, d, nq, nkv, I = cfg["hidden"], cfg["head_dim"], cfg["n_q_heads"], cfg["n_kv_heads"], cfg["ffn_inter"]
    qkv_rows = nq * d + 2 * nkv * d
    params = qkv_rows * h + h * nq * d + 3 * I * h
    if cfg.get("weight_format", 0) == 1:
        return params + 4 * (qkv_rows + h + 2 * I + h)
    return 2 * params


def step_bytes(cfg, B, ctx_list):
    """Algorithmic bytes of one decode step: every weight once + each sequence's KV once."""
    L, h, V = cfg["layers"], cfg["hidden"], cfg["vocab"]
    kv_row = 2 * cfg["n_kv_heads"] * cfg["head_dim"] * 2  # k + v, bf16
    head = V * h + 4 * V if cfg.get("weight_format", 0) == 1 else V * h * 2
    weights = L * layer_bytes(cfg) + head + L * 2 * h * 4 + h * 4
    kv = sum(L * c * kv_row for c in ctx_list)
    return weights, kv


def prefill_weight_bytes(cfg):
    """Weight bytes the tensor-core GEMMs read per chunk (bf16: q8_row models keep their
    integers in bf16 for the tensor pipe)."""
    return cfg["layers"] * layer_bytes(dict(cfg, weight_format=0))


def gemm_flops_per_token(cfg):
    return 2 * (layer_bytes(dict(cfg, weight_format=0)) // 2 * cfg["layers"])


def attn_flops_prefill(cfg, T):
    # causal: query t attends t+1 keys; QK and PV each 2*d flops per (head, key)
    return 4 * cfg["head_dim"] * cfg["n_q_heads"] * cfg["layers"] * (T * (T + 1) / 2)


class Clocks:
    """nvidia-smi sampler running during the timed region."""

    def __init__(self, index):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = subprocess.Popen(
            ["nvidia-smi", f"--id={index}",
             "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
             "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)

    def stop(self):
        self.p.terminate()
        try:
            self.p.wait(5)
        except Exception:
            self.p.kill()
        self.f.flush()
        rows = []
        for line in open(self.f.name):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 8:
                rows.append(parts)
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[4:8]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def make_device_weights(cfg, torch, seed=0):
    """Weights of the synthetic recipe generated directly in device memory (same streams as
    synth.make_weights, by the device twin of the generator)."""
    dl = synth.dev_lib()
    st = torch.cuda.current_stream().cuda_stream
    keep = []

    def mat(shape, tid, mean=0.0, std=synth.WEIGHT_STD):
        t = torch.empty(shape, dtype=torch.int16, device="cuda")
        assert dl.syn_dev_fill_bf16(t.data_ptr(), t.numel(), seed, tid, mean, std, st) == 0
        keep.append(t)
        return t

    def vec(n, tid, mean, std):
        t = torch.empty(n, dtype=torch.float32, device="cuda")
        assert dl.syn_dev_fill_bf16_as_f32(t.data_ptr(), n, seed, tid, mean, std, st) == 0
        keep.append(t)
        return t

    q8 = cfg.get("weight_format", 0) == 1

    def q8mat(shape, tid, scale_tid):
        t = torch.empty(shape, dtype=torch.int8, device="cuda")
        assert dl.syn_dev_fill_i8(t.data_ptr(), t.numel(), seed, tid, synth.Q8_STD, st) == 0
        keep.append(t)
        return t, vec(shape[0], scale_tid, synth.WEIGHT_STD / synth.Q8_STD, 0.1 * synth.WEIGHT_STD / synth.Q8_STD)

    h, V = cfg["hidden"], cfg["vocab"]
    w = dict(embed=mat((V, h), 1), lm_head=None if cfg.get("tied") else mat((V, h), 2),
             final_norm=vec(h, 3, 1.0, synth.GAIN_STD), layers=[])
    if q8 and not cfg.get("tied"):
        w["lm_head"], w["lm_head_scale"] = q8mat((V, h), 2, 4)
    for l in range(cfg["layers"]):
        lw = {}
        for name, shape in synth.tensor_shapes(cfg).items():
            if shape is None:
                lw[name] = None
            elif q8 and name in synth.Q8_MATS:
                tid = synth.layer_tid(l, name)
                lw[name], lw[name + "_scale"] = q8mat(shape, tid, tid + 50)
            elif name in synth.GAINS:
                lw[name] = vec(shape[0], synth.layer_tid(l, name), 1.0, synth.GAIN_STD)
            elif name in synth.VECTORS:
                lw[name] = vec(shape[0], synth.layer_tid(l, name), 0.0, synth.WEIGHT_STD)
            elif name in ("e_gate", "e_up", "e_down"):
                part = ("e_gate", "e_up", "e_down").index(name)
                t = torch.empty(shape, dtype=torch.int16, device="cuda")
                for e in range(shape[0]):
                    assert dl.syn_dev_fill_bf16(t[e].data_ptr(), t[e].numel(), seed, synth.expert_tid(l, e, part),
                                                0.0, synth.WEIGHT_STD, st) == 0
                keep.append(t)
                lw[name] = t
            else:
                lw[name] = mat(shape, synth.layer_tid(l, name))
        w["layers"].append(lw)
    torch.cuda.synchronize()
    return w


def _time_launches(torch, call, nbuf, reps):
    """Average device time of `reps` launches of call(i) (CUDA events on the launching stream)."""
    for i in range(3):
        call(i % nbuf)
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(s)
    for i in range(reps):
        call(i % nbuf)
    e1.record(s)
    e1.synchronize()
    return e0.elapsed_time(e1) / reps


def time_gate_up(dec, torch, I, K, reps=20):
    """The decode step's dominant launch, alone: gemv_kernel<1, SWIGLU> with its fused RMSNorm
    prologue (ffn_gate_up) on the interleaved [2I][K] gate/up matrix at B = 1; the weights rotate
    over copies larger than L2. Returns (ms, algorithmic bytes per launch)."""
    nbuf = max(2, int(math.ceil(300e6 / (2 * I * K * 2))))
    Ws = [torch.empty((2 * I, K), dtype=torch.bfloat16, device="cuda").normal_(0, 0.02) for _ in range(nbuf)]
    x = torch.randn((1, K), device="cuda") * 3
    g = torch.ones(K, device="cuda")
    act = torch.empty((1, I), dtype=torch.bfloat16, device="cuda")
    ms = _time_launches(torch, lambda i: dec.ffn_gate_up(Ws[i], x, g, 1e-5, act), nbuf, reps)
    del Ws
    return ms, 2 * I * K * 2 + K * 4 + K * 4 + I * 2


def time_gemv_q8(dec, torch, N, K, reps=20):
    """The q8_row GEMV (weight_gemv_q8, store epilogue) on one int8 [N][K] matrix at B = 1 on
    rotating copies larger than L2. Returns (ms, algorithmic bytes per launch)."""
    nbuf = max(2, int(math.ceil(300e6 / (N * K))))
    Ws = [torch.randint(-127, 128, (N, K), dtype=torch.int8, device="cuda") for _ in range(nbuf)]
    sc = torch.full((N,), 0.02 / 32, device="cuda")
    x = torch.randn((1, K), device="cuda").to(torch.bfloat16)
    y = torch.empty((1, N), device="cuda")
    ms = _time_launches(torch, lambda i: dec.weight_gemv_q8(Ws[i], sc, x, y), nbuf, reps)
    del Ws
    return ms, N * K + N * 4 + K * 2 + N * 4


def cpu_oracle_sample(cfg, ctx):
    """Time the oracle (as it stands) on a bounded sample of the decode workload: layer 0 and
    the LM head of the same model, one token at position ctx over a synthetic cache; the full
    32-layer step time is extrapolated as L * t(layer) + t(head)."""
    import oracle
    c1 = configs.with_layers(cfg, 1, max_context=ctx + 1, max_batch=1)
    w = synth.make_weights(c1)
    m = oracle.Model(c1, w)
    kvd = cfg["n_kv_heads"] * cfg["head_dim"]
    k, v = synth.kv_fill(ctx, kvd, 2000, 0)
    m.kv_write(0, 0, 0, k, v)
    t0 = time.perf_counter()
    m.forward(0, 1, ctx, want_logits=False)
    t_layer = time.perf_counter() - t0
    m.kv_write(0, 0, 0, k, v)
    t0 = time.perf_counter()
    m.forward(0, 1, ctx, want_logits=True)
    t_head = max(0.0, time.perf_counter() - t0 - t_layer)
    step = cfg["layers"] * t_layer + t_head
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return dict(value=1.0 / step, unit="tok/s", cores=threads, kind="oracle",
                sample=f"1 of {cfg['layers']} layers + LM head, one decode token at context {ctx}, fp64 oracle; "
                       f"step extrapolated as {cfg['layers']}*t_layer + t_head "
                       f"(t_layer={t_layer:.3f}s, t_head={t_head:.3f}s)")


def run_reference(args):
    """--impl reference: the CPU oracle timed on this host on a bounded sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cfg = dict(configs.LLAMA3_8B)
    steps = []
    for _ in range(max(1, args.steps)):
        cb = cpu_oracle_sample(cfg, PROMPT)
        steps.append(1.0 / cb["value"])
    val = 1.0 / statistics.median(steps)
    cb["value"] = val
    line = dict(metric=METRIC, value=val, unit="tok/s", n_gpus=args.gpus, steps=args.steps, warmup=args.warmup,
                ms_per_step=1000.0 / val, higher_is_better=True, scaling="weak", vs_baseline=None, dtype="f64",
                data="synthetic", impl="reference",
                config=main_config(args.gpus, cfg["layers"]),
                cpu_baseline=cb, e2e=dict(value=val, unit="tok/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line))
    return 0


WORKLOADS = {
    # decode over synthetic caches (N(0,1) bf16 rows), greedy continuation
    "llama3-8b-b32": dict(model="LLAMA3_8B", B=32, ctx=4096),
    "qwen15-moe-b1": dict(model="QWEN15_MOE_A27B", B=1, ctx=2048),
    "qwen15-moe-b64": dict(model="QWEN15_MOE_A27B", B=64, ctx=2048),
    # prefill a prompt (chunks of 128), then batch-1 decode
    "smollm2-135m": dict(model="SMOLLM2_135M", B=1, ctx=1024, prefill=1024),
    "tiny": dict(model="TINY", B=1, ctx=16, prefill=16),
    # standalone decode attention
    "gqa-sweep": dict(),
    # standalone weight-streaming GEMV on the gate/up matrix of the Llama-3-8B shape (the
    # default line's roofline kernel, launched the way its `achieved` figure is timed)
    "gemv-gate-up": dict(),
    # the headline decode line with q8_row weights (int8 rows, fp32 row scales)
    "llama3-8b-q8": dict(),
    # the CPU oracle's own throughput on the tiny, SmolLM2-135M and Qwen1.5-MoE shapes (B = 1),
    # on this host's cores: a baseline, not the target
    "oracle-baselines": dict(),
    # 4096-token prefill of the Llama-3-8B shape with longer chunks: the projections become
    # compute-bound GEMMs (the chunk-128 line is HBM-bound)
    "llama3-8b-prefill-c512": dict(prefill_chunk=512),
    "llama3-8b-prefill-c4096": dict(prefill_chunk=4096),
}


def decode_step_bytes(cfg, B, ctx_list, experts_touched=None):
    """Weights read once per step (MoE: only the experts some token picked) + every KV row."""
    L, h, V = cfg["layers"], cfg["hidden"], cfg["vocab"]
    d, nq, nkv = cfg["head_dim"], cfg["n_q_heads"], cfg["n_kv_heads"]
    attn = (nq * d + 2 * nkv * d) * h + h * nq * d
    if cfg.get("n_experts", 0):
        Ie, Is, E = cfg["expert_inter"], cfg["shared_inter"], cfg["n_experts"]
        touched = experts_touched if experts_touched is not None else min(E, B * cfg["top_k"])
        ffn = E * h + 3 * Is * h + touched * 3 * Ie * h
    else:
        ffn = 3 * cfg["ffn_inter"] * h
    w = 2 * (L * (attn + ffn) + V * h)  # the LM head (the embedding when tied) is read once
    kv = sum(L * c * 2 * nkv * d * 2 for c in ctx_list)
    return w, kv


def run_prefill_workload(args, torch, dec, P):
    """Prefill of a 4096-token prompt, Llama-3-8B shape, with prefill_chunk C (512 or 4096):
    each timed run is one dec_prefill from position 0 (the sequence is reset between runs,
    outside the timed region)."""
    name = args.workload
    C = WORKLOADS[name]["prefill_chunk"]
    PROMPT = 4096
    runs = max(2, min(args.steps, 4))
    cfg = dict(configs.LLAMA3_8B, max_context=PROMPT + 8, max_batch=1, prefill_chunk=C)
    if args.layers:  # profiling only: fewer layers of the same shape
        cfg = configs.with_layers(cfg, args.layers)
    w = make_device_weights(cfg, torch)
    d = dec.Decoder(cfg, w)
    del w
    torch.cuda.empty_cache()
    stream = torch.cuda.current_stream()
    prompt = synth.tokens(PROMPT, cfg["vocab"], 1000)
    for _ in range(max(1, min(args.warmup, 2))):
        d.prefill(0, prompt, 0)
        d.reset(0)
    torch.cuda.synchronize()
    clk = Clocks(int(os.environ.get("LOCAL_RANK", "0")))
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    times = []
    for _ in range(runs):
        e0.record(stream)
        d.prefill(0, prompt, 0)
        e1.record(stream)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
        d.reset(0)
    clocks = clk.stop()
    ms = statistics.mean(times)
    flops = gemm_flops_per_token(cfg) * PROMPT + attn_flops_prefill(cfg, PROMPT)
    tflops = flops / (ms * 1e-3) / 1e12
    hbm_floor_ms = (PROMPT / C) * (cfg["layers"] * layer_bytes(cfg)) / (P["hbm"] * 1e9) * 1e3
    tc_floor_ms = flops / (P["tc_sus"] * 1e12) * 1e3
    line = dict(metric=f"prefill tok/s ({name}, 4096 tokens, chunk {C})", value=PROMPT / (ms * 1e-3), unit="tok/s",
                n_gpus=1, steps=runs, warmup=max(1, min(args.warmup, 2)), ms_per_step=ms, higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="bf16", data="synthetic",
                config=dict(workload=f"llama3_8b shape, 4096-token prefill, chunk {C}", global_batch=1,
                            seq_len=PROMPT, l2="inputs larger than L2"),
                prefill=dict(tokens=PROMPT, chunk=C, ms=round(ms, 2), tflops=round(tflops, 1),
                             tc_frac=round(tflops / P["tc_sus"], 4), tc_peak_tflops=P["tc_sus"],
                             hbm_floor_ms=round(hbm_floor_ms, 2), tc_floor_ms=round(tc_floor_ms, 2),
                             attainable_frac=round(max(hbm_floor_ms, tc_floor_ms) / ms, 4)),
                clocks=clocks)
    print(json.dumps(line))
    d.close()
    return 0


def run_oracle_baselines(args):
    """The fp64 oracle as it stands, timed on this host: prefill tok/s and batch-1 decode tok/s
    of the tiny, SmolLM2-135M and Qwen1.5-MoE-A2.7B shapes. Prefill is timed on a 128-token
    sample for SmolLM2 (every token costs the same weights; attention grows slowly at these
    lengths); decode at the workload's context over a synthetic cache."""
    import oracle
    rows = []
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    for name, cfg, n_prompt, ctx in (("tiny", dict(configs.TINY), 16, 16),
                                     ("smollm2-135m", dict(configs.SMOLLM2_135M, max_context=1040), 128, 1024),
                                     ("qwen1.5-moe-a2.7b", dict(configs.QWEN15_MOE_A27B, max_context=2056), 0, 2048)):
        w = synth.make_weights(cfg)
        m = oracle.Model(cfg, w)
        row = dict(model=name)
        if n_prompt:
            toks = synth.tokens(n_prompt, cfg["vocab"], 1000)
            t0 = time.perf_counter()
            m.prefill(0, toks, 0)
            row["prefill_tok_s"] = round(n_prompt / (time.perf_counter() - t0), 2)
            row["prefill_tokens"] = n_prompt
        kvd = cfg["n_kv_heads"] * cfg["head_dim"]
        if ctx > n_prompt:
            for l in range(cfg["layers"]):
                k, v = synth.kv_fill(ctx, kvd, 2000, l)
                m.kv_write(0, l, 0, k, v)
        steps = 3
        t0 = time.perf_counter()
        for s in range(steps):
            m.forward(0, 1 + s, ctx + s)
        row["decode_tok_s"] = round(steps / (time.perf_counter() - t0), 3)
        row["decode_ctx"] = ctx
        rows.append(row)
        m.close()
        del w
    print(json.dumps(dict(metric="CPU oracle tok/s (fp64, batch 1)", value=rows[-1]["decode_tok_s"], unit="tok/s",
                          n_gpus=0, steps=3, warmup=0, higher_is_better=True, dtype="f64", data="synthetic",
                          cpu_baseline=dict(kind="oracle", cores=threads), points=rows)))
    return 0


def run_workload(args, torch, dec):
    name = args.workload
    if name == "oracle-baselines":
        return run_oracle_baselines(args)
    P = peaks()
    W, K = max(3, args.warmup), max(1, args.steps)
    if name == "gqa-sweep":
        return run_gqa_sweep(args, torch, dec, P)
    if name == "gemv-gate-up":
        I, Kd = configs.LLAMA3_8B["ffn_inter"], configs.LLAMA3_8B["hidden"]
        ms, byt = time_gate_up(dec, torch, I, Kd, reps=K)
        gbs = byt / (ms * 1e-3) / 1e9
        print(json.dumps(dict(metric=f"fused norm + gate/up + SiLU GEMV GB/s ([{2 * I}][{Kd}] bf16, batch 1)",
                              value=round(gbs, 1), unit="GB/s", n_gpus=1, steps=K, warmup=3, ms_per_step=ms,
                              higher_is_better=True, scaling="weak", vs_baseline=None, dtype="bf16",
                              data="synthetic",
                              config=dict(workload=f"ffn_gate_up [{2 * I}][{Kd}] x [1][{Kd}]",
                                          l2="rotating weights > L2"),
                              roofline=dict(bound="hbm", achieved=round(gbs, 1), peak=P["hbm"], unit="GB/s",
                                            frac=round(gbs / P["hbm"], 4), peak_source=P["src"]))))
        return 0
    if name == "llama3-8b-q8":
        return run_headline(args, torch, dec, q8=True)
    if "prefill_chunk" in WORKLOADS[name]:
        return run_prefill_workload(args, torch, dec, P)
    spec = WORKLOADS[name]
    base = getattr(configs, spec["model"])
    B, ctx = spec["B"], spec["ctx"]
    cfg = dict(base, max_batch=B, max_context=ctx + W + K + 8, prefill_chunk=128)
    if args.layers:  # profiling only: fewer layers of the same shape
        cfg = configs.with_layers(cfg, args.layers)
    w = make_device_weights(cfg, torch)
    d = dec.Decoder(cfg, w)
    del w
    torch.cuda.empty_cache()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    extra = {}
    if "prefill" in spec:
        prompt = synth.tokens(spec["prefill"], cfg["vocab"], 1000)
        d.prefill(0, prompt[:min(128, len(prompt))], 0)
        d.reset(0)
        torch.cuda.synchronize()
        e0.record(stream)
        d.prefill(0, prompt, 0)
        e1.record(stream)
        e1.synchronize()
        pms = e0.elapsed_time(e1)
        extra["prefill"] = dict(tokens=len(prompt), chunk=128, ms=round(pms, 3),
                                tok_s=round(len(prompt) / (pms * 1e-3), 1))
        toks = d.last_argmax(1)
    else:
        # synthetic cache rows made on the device (same rows for every sequence and layer)
        kvd = cfg["n_kv_heads"] * cfg["head_dim"]
        dl, st = synth.dev_lib(), torch.cuda.current_stream().cuda_stream
        kb = torch.empty((ctx, kvd), dtype=torch.int16, device="cuda")
        vb = torch.empty((ctx, kvd), dtype=torch.int16, device="cuda")
        assert dl.syn_dev_fill_bf16(kb.data_ptr(), kb.numel(), 2000, 0, 0.0, 1.0, st) == 0
        assert dl.syn_dev_fill_bf16(vb.data_ptr(), vb.numel(), 2000, 1, 0.0, 1.0, st) == 0
        torch.cuda.synchronize()
        for b in range(B):
            for l in range(cfg["layers"]):
                d.kv_write(b, l, 0, kb, vb)
        del kb, vb
        toks = synth.tokens(B, cfg["vocab"], 1000)
    pos = np.full(B, ctx, np.int32)
    for _ in range(W):
        d.step(toks, pos)
        toks = d.last_argmax(B)
        pos += 1
    torch.cuda.synchronize()
    clk = Clocks(int(os.environ.get("LOCAL_RANK", "0")))
    time.sleep(0.3)
    ctxs = []
    e0.record(stream)
    for _ in range(K):
        d.step(toks, pos)
        ctxs.extend((pos + 1).tolist())
        pos += 1
    e1.record(stream)
    e1.synchronize()
    clocks = clk.stop()
    ms = e0.elapsed_time(e1) / K
    touched = None
    if cfg.get("n_experts", 0):
        r = d.last_routes(B)  # [L][B][k] of the last timed step
        touched = float(np.mean([len(np.unique(r[l])) for l in range(cfg["layers"])]))
        extra["experts_touched_per_layer"] = round(touched, 2)
    wb, kvb = decode_step_bytes(cfg, B, ctxs, touched)
    step_bytes = wb + kvb / K
    gbs = step_bytes / (ms * 1e-3) / 1e9
    line = dict(metric=f"decode tok/s ({name}, b={B}, ctx {ctx})", value=B / (ms * 1e-3), unit="tok/s", n_gpus=1,
                steps=K, warmup=W, ms_per_step=ms, higher_is_better=True, scaling="weak", vs_baseline=None,
                dtype="bf16", data="synthetic",
                config=dict(workload=f"{spec['model'].lower()} shape, batch {B}, context {ctx}", global_batch=B,
                            seq_len=ctx, layers=cfg["layers"], l2="inputs larger than L2"),
                step_roofline=dict(bytes_per_step=step_bytes, achieved_gbs=round(gbs, 1),
                                   frac=round(gbs / P["hbm"], 4), peak=P["hbm"], unit="GB/s", peak_source=P["src"]),
                clocks=clocks, **extra)
    print(json.dumps(line))
    if args.breakdown:  # 4 more steps; the context has room for 8 past the timed ones
        def one_step():
            d.step(toks, pos)
            pos[:] += 1
        kernel_breakdown(torch, one_step, 4, f"{name} (B={B}, ctx {ctx}, {cfg['layers']} layers)")
    d.close()
    return 0


def kernel_breakdown(torch, step, n, title):
    """Per-kernel share of `n` more steps, from the torch profiler's device activity. Kernels
    overlap under programmatic dependent launch, so each one is charged the time from the
    end of everything before it to its own end (its exclusive share of the critical path)."""
    import collections
    from torch.profiler import ProfilerActivity, profile
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        for _ in range(n):
            step()
        torch.cuda.synchronize()
    ev = sorted((e for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA),
                key=lambda e: e.time_range.start)
    agg = collections.defaultdict(lambda: [0, 0.0])
    last = None
    for e in ev:
        name = e.name.replace("(anonymous namespace)::", "").replace("void ", "").split("(")[0][-60:]
        agg[name][0] += 1
        agg[name][1] += max(0.0, e.time_range.end - (e.time_range.start if last is None else max(last, e.time_range.start)))
        last = e.time_range.end if last is None else max(last, e.time_range.end)
    total = sum(v[1] for v in agg.values())
    print(f"kernel breakdown, {title}: {total / n:.0f} us per step (exclusive shares)", file=sys.stderr)
    for name, (c, t) in sorted(agg.items(), key=lambda x: -x[1][1]):
        print(f"  {name:60s} {c // n:4d}/step {t / c:9.2f} us/launch {t / n:9.1f} us/step {100 * t / total:5.1f}%",
              file=sys.stderr)


def run_gqa_sweep(args, torch, dec, P):
    B, nq, nkv, d = 64, 32, 8, 128
    gen = torch.Generator(device="cuda").manual_seed(2000)
    rows = []
    clk = Clocks(int(os.environ.get("LOCAL_RANK", "0")))
    for ctx in (512, 2048, 8192, 32768):
        pages = B * ctx // 16
        kp = torch.randn((pages, nkv, 16, d), device="cuda", generator=gen).to(torch.bfloat16)
        vp = torch.randn((pages, nkv, 16, d), device="cuda", generator=gen).to(torch.bfloat16)
        bt = torch.from_numpy(np.random.default_rng(ctx).permutation(pages).astype(np.int32).reshape(B, -1)).cuda()
        q = torch.randn((B, nq, d), device="cuda", generator=gen).to(torch.bfloat16)
        kn = torch.randn((B, nkv, d), device="cuda", generator=gen).to(torch.bfloat16)
        vn = torch.randn((B, nkv, d), device="cuda", generator=gen).to(torch.bfloat16)
        pos = torch.full((B,), ctx - 1, dtype=torch.int32, device="cuda")
        out = torch.empty((B, nq, d), dtype=torch.bfloat16, device="cuda")
        byts = B * ctx * nkv * d * 2 * 2
        for rope in (0, 1):
            def call():
                dec.gqa_decode_attn(q, kn if rope else None, vn if rope else None, kp, vp, bt, pos, nq, nkv, d,
                                    1 / math.sqrt(d), rope, 10000.0, out)
            for _ in range(max(3, args.warmup)):
                call()
            s = torch.cuda.current_stream()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record(s)
            reps = max(1, args.steps)
            for _ in range(reps):
                call()
            e1.record(s)
            e1.synchronize()
            us = e0.elapsed_time(e1) / reps * 1e3
            gbs = byts / (us * 1e-6) / 1e9
            rows.append(dict(ctx=ctx, fused_rope=rope, us=round(us, 1), gbs=round(gbs, 1),
                             frac=round(gbs / P["hbm"], 4)))
        del kp, vp
        torch.cuda.empty_cache()
    clocks = clk.stop()
    gm = math.exp(sum(math.log(r["gbs"]) for r in rows) / len(rows))
    print(json.dumps(dict(metric="GQA decode attention sweep (B=64, 32q/8kv, d=128, paged 16), GB/s geomean",
                          value=gm, unit="GB/s", n_gpus=1, steps=args.steps, warmup=args.warmup,
                          higher_is_better=True, dtype="bf16", data="synthetic", peak=P["hbm"],
                          peak_source=P["src"], points=rows, clocks=clocks)))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=32)
    ap.add_argument("--warmup", type=int, default=4)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-c4096", action="store_true", help="skip the one-chunk 4096-token prefill sub-object")
    ap.add_argument("--layers", type=int, default=0, help="fewer layers (profiling only; not a bench number)")
    ap.add_argument("--breakdown", action="store_true",
                    help="decode workloads: after the timed region, per-kernel exclusive times of a few more "
                         "steps (torch profiler) on stderr; the JSON line is unchanged")
    ap.add_argument("--workload", default="llama3-8b", choices=["llama3-8b"] + sorted(WORKLOADS),
                    help="llama3-8b: the headline line (prefill 4096 + batch-1 decode); others: one extra line each")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)

    import torch

    import decoder_only_transformer_layer_b200 as dec

    if args.workload != "llama3-8b":
        return run_workload(args, torch, dec)
    return run_headline(args, torch, dec)


def time_prefill_c4096(torch, dec, weights, P, runs=2):
    """The 4096-token prefill in ONE chunk of 4096 (same weights): every projection is a
    compute-bound tcgen05 GEMM, the configuration where the tensor-core target applies."""
    cfg = dict(configs.LLAMA3_8B, max_context=PROMPT + 8, max_batch=1, prefill_chunk=PROMPT)
    d = dec.Decoder(cfg, weights)
    stream = torch.cuda.current_stream()
    prompt = synth.tokens(PROMPT, cfg["vocab"], 1000)
    d.prefill(0, prompt, 0)  # warm-up
    d.reset(0)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    times = []
    for _ in range(runs):
        torch.cuda.synchronize()
        e0.record(stream)
        d.prefill(0, prompt, 0)
        e1.record(stream)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
        d.reset(0)
    d.close()
    ms = statistics.mean(times)
    flops = gemm_flops_per_token(cfg) * PROMPT + attn_flops_prefill(cfg, PROMPT)
    tf = flops / (ms * 1e-3) / 1e12
    return dict(tokens=PROMPT, chunk=PROMPT, ms=round(ms, 2), tok_s=round(PROMPT / (ms * 1e-3), 1),
                tflops=round(tf, 1), tc_frac_sustained=round(tf / P["tc_sus"], 4),
                tc_frac_burst=round(tf / P["tc"], 4), tc_peak_sustained=P["tc_sus"], tc_peak_burst=P["tc"],
                bar_uses="sustained: 64 GEMM launches back to back for tens of ms under the power cap")


def run_headline(args, torch, dec, q8=False):
    """Llama-3-8B shape: 4096-token prefill (chunk 128), then batch-1 greedy decode at context
    4096+. With q8 the projections and the LM head are q8_row (int8 rows, fp32 row scales)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    import torch.distributed as dist
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))

    def barrier():
        if world > 1:
            dist.barrier()

    W = max(3, args.warmup)
    K = max(1, args.steps)
    e2e_steps = min(K, 16)
    cfg = dict(configs.LLAMA3_8B, max_context=PROMPT + W + K + e2e_steps + 16, max_batch=1, prefill_chunk=128,
               weight_format=1 if q8 else 0)
    if args.layers:
        cfg = configs.with_layers(cfg, args.layers)
    weights = make_device_weights(cfg, torch)
    d = dec.Decoder(cfg, weights)
    if q8 or args.layers or args.no_c4096:
        del weights
        weights = None
    torch.cuda.empty_cache()
    stream = torch.cuda.current_stream()
    prompt = synth.tokens(PROMPT, cfg["vocab"], 1000)

    # ---- prefill (timed once, after a warm-up prefill of one chunk on a scratch sequence)
    d.prefill(0, prompt[:128], 0)
    d.reset(0)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    d.prefill(0, prompt, 0)
    e1.record(stream)
    e1.synchronize()
    prefill_ms = e0.elapsed_time(e1)
    tok = int(d.last_argmax(1)[0])

    # ---- decode: W warm-up steps, then K timed steps (greedy, device-resident inputs)
    pos = PROMPT
    for _ in range(W):
        d.step([tok], [pos])
        tok = int(d.last_argmax(1)[0])
        pos += 1
    torch.cuda.synchronize()
    barrier()
    clk = Clocks(local)
    time.sleep(0.3)
    ctx_list = []
    e0.record(stream)
    for _ in range(K):
        d.step([tok], [pos])
        ctx_list.append(pos + 1)
        pos += 1
    e1.record(stream)
    e1.synchronize()
    clocks = clk.stop()
    decode_ms = e0.elapsed_time(e1)
    ms_step = decode_ms / K
    if world > 1:
        ms_step, prefill_ms = max_over_ranks([ms_step, prefill_ms], "cuda")

    # ---- end to end through the C ABI with host buffers (tokens in, logits out per step)
    host_logits = torch.empty((1, cfg["vocab"]), dtype=torch.float32).pin_memory().numpy()
    torch.cuda.synchronize()
    barrier()
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        d.step([tok], [pos], host_logits)
        tok = int(np.argmax(host_logits[0]))
        pos += 1
    e2e_s = (time.perf_counter() - t0) / e2e_steps
    if world > 1:
        (e2e_s,) = max_over_ranks([e2e_s], "cuda")
    if args.breakdown and rank == 0:  # after every timed region: per-kernel shares
        state = dict(tok=tok, pos=pos)

        def one_step():
            d.step([state["tok"]], [state["pos"]])
            state["pos"] += 1
        kernel_breakdown(torch, one_step, 4, f"decode b=1 ({cfg['layers']} layers)")
        d.reset(0)
        kernel_breakdown(torch, lambda: d.prefill(0, prompt, 0), 1, f"prefill {PROMPT} tokens, chunk 128")
    d.close()

    # ---- dominant kernel alone: the decode step's gate/up launch
    P = peaks()
    I, Kd = cfg["ffn_inter"], cfg["hidden"]
    if q8:
        k_ms, k_bytes = time_gemv_q8(dec, torch, 2 * I, Kd)
        k_name = f"gemv_kernel<1,STORE,q8> (weight_gemv_q8) on int8 [{2 * I}][{Kd}] + row scales"
    else:
        k_ms, k_bytes = time_gate_up(dec, torch, I, Kd)
        k_name = (f"gemv_kernel<1,SWIGLU> with the fused RMSNorm prologue (ffn_gate_up: the decode step's "
                  f"gate/up launch) on [{2 * I}][{Kd}] bf16")
    k_gbs = k_bytes / (k_ms * 1e-3) / 1e9

    # ---- the same prompt prefilled in one 4096-token chunk (tensor-core bound GEMMs)
    c4096 = None
    if weights is not None:
        torch.cuda.synchronize()
        c4096 = time_prefill_c4096(torch, dec, weights, P)
        del weights

    wbytes, kvbytes = step_bytes(cfg, 1, ctx_list)
    step_gbs = (wbytes + kvbytes / K) / (ms_step * 1e-3) / 1e9
    value = replica_throughput(1, world, ms_step)
    pf_tok_s = replica_throughput(PROMPT, world, prefill_ms)
    pf_flops = gemm_flops_per_token(cfg) * PROMPT + attn_flops_prefill(cfg, PROMPT)
    pf_tflops = pf_flops / (prefill_ms * 1e-3) / 1e12
    chunk_hbm_floor_ms = (PROMPT / 128) * prefill_weight_bytes(cfg) / (P["hbm"] * 1e9) * 1e3
    launches_per_step = 1 + 5 * cfg["layers"] + 2

    cpu_b = None
    if rank == 0 and not args.no_cpu_baseline and not args.layers and not q8:
        cpu_b = cpu_oracle_sample(dict(configs.LLAMA3_8B), PROMPT)
    if rank == 0:
        metric = METRIC if not q8 else "decode tok/s + % HBM roofline (8B-shape, b=1, q8_row weights)"
        line = dict(
            metric=metric, value=value, unit="tok/s", n_gpus=world, steps=K, warmup=W, ms_per_step=ms_step,
            higher_is_better=True, scaling="weak", vs_baseline=None, dtype="bf16" if not q8 else "int8xbf16",
            data="synthetic",
            config=main_config(world, cfg["layers"]) if not q8 else dict(
                main_config(world, cfg["layers"]), workload="llama3-8b-shape, q8_row projections and LM head, "
                                                            "decode b=1 at context 4096 after a 4096-token prefill"),
            roofline=dict(bound="hbm", achieved=round(k_gbs, 1), peak=P["hbm"], unit="GB/s",
                          frac=round(k_gbs / P["hbm"], 4), traffic=None if q8 else measured_traffic(),
                          traffic_unit="bytes per launch (ncu dram read+write)", kernel=k_name,
                          algorithmic_bytes=k_bytes, launch_us=round(k_ms * 1e3, 2), peak_source=P["src"]),
            step_roofline=dict(bytes_per_step=wbytes + kvbytes / K, achieved_gbs=round(step_gbs, 1),
                               frac=round(step_gbs / P["hbm"], 4), peak=P["hbm"], unit="GB/s"),
            prefill=dict(tokens=PROMPT, chunk=128, ms=round(prefill_ms, 2), tok_s=round(pf_tok_s, 1),
                         tflops=round(pf_tflops, 1), tc_frac=round(pf_tflops / P["tc_sus"], 4),
                         hbm_floor_ms=round(chunk_hbm_floor_ms, 2),
                         attainable_frac=round(chunk_hbm_floor_ms / prefill_ms, 4)),
            cpu_baseline=cpu_b,
            e2e=dict(value=world / e2e_s, unit="tok/s", h2d_bytes_per_step=8, d2h_bytes_per_step=4 * cfg["vocab"]),
            gpu_launches=launches_per_step * K, clocks=clocks)
        if c4096:
            line["prefill_c4096"] = c4096
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
