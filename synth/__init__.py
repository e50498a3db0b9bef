"""Seeded synthetic inputs shared by the CPU oracle and the CUDA path.

This package holds no arithmetic of the method: only the counter-based
generator (SplitMix64 words, Box-Muller normals, nearest-even rounding to
bf16) defined in ``synth.c``, its device twin ``synth_fill.cu``, and the
recipe that names one stream per tensor.

Recipe (seed 0 unless stated):
  * weight matrices, embeddings, LM head, router, experts: N(0, 0.02) -> bf16
  * RMSNorm gains (attention, FFN, final, QK-norm): 1 + N(0, 0.1) -> bf16 value, fp32 storage
  * QKV bias and the shared-expert gate vector: N(0, 0.02) -> bf16 value, fp32 storage
  * prompts: uniform ids in [0, V) from seed 1000 + k
  * synthetic KV fills: N(0, 1) -> bf16 from seed 2000

  * post-attention / post-FFN norm gains (sandwich norms): 1 + N(0, 0.1), like the other gains
  * q8_row models (weight_format 1): each projection and the untied LM head as int8 values
    nearbyint(32 z) clamped to [-127, 127], and one fp32 scale per row, the bf16 value of
    (0.02 / 32)(1 + 0.1 z'): entries of about N(0, 0.02) like the bf16 weights

Stream ids: 1 embed, 2 lm_head, 3 final_norm, 4 lm_head row scales; layer l uses
1000 + 100 l + slot (slots below; a q8_row scale uses its matrix's slot + 50); expert e of
layer l uses 10_000_000 + 10_000 l + 10 e + {0 gate, 1 up, 2 down}.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

from . import configs  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_DEV_SRC = os.path.join(_HERE, "synth_fill.cu")
_DEV_LIB = os.path.join(_HERE, "libsynth_dev.so")

WEIGHT_STD = 0.02
GAIN_STD = 0.1

SLOTS = dict(attn_norm=0, ffn_norm=1, wqkv=2, bqkv=3, q_norm=4, k_norm=5, wo=6, w_gate=7, w_up=8,
             w_down=9, w_router=10, s_gate=11, s_up=12, s_down=13, s_gate_vec=14, post_attn_norm=15,
             post_ffn_norm=16)
GAINS = ("attn_norm", "ffn_norm", "q_norm", "k_norm", "post_attn_norm", "post_ffn_norm")
Q8_MATS = ("wqkv", "wo", "w_gate", "w_up", "w_down")
Q8_STD = 32.0  # int8 values ~ N(0, 32^2); scales ~ WEIGHT_STD / Q8_STD
VECTORS = ("bqkv", "s_gate_vec")


def build(force: bool = False) -> str:
    if (not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                           "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


def build_device(force: bool = False) -> str:
    if (not force and os.path.exists(_DEV_LIB)
            and os.path.getmtime(_DEV_LIB) >= os.path.getmtime(_DEV_SRC)):
        return _DEV_LIB
    tmp = _DEV_LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["nvcc", "-O3", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
                           "-Xcompiler", "-fPIC", "-shared", "-o", tmp, _DEV_SRC])
    os.replace(tmp, _DEV_LIB)
    return _DEV_LIB


_lib = None
_dev = None


def lib():
    global _lib
    if _lib is None:
        L = C.CDLL(build())
        L.syn_stream_key.restype = C.c_uint64
        L.syn_stream_key.argtypes = [C.c_uint64, C.c_uint64]
        L.syn_round_bf16.restype = C.c_uint16
        L.syn_round_bf16.argtypes = [C.c_double]
        L.syn_fill_bf16.argtypes = [C.c_void_p, C.c_int64, C.c_uint64, C.c_uint64, C.c_double, C.c_double]
        L.syn_fill_bf16_as_f32.argtypes = [C.c_void_p, C.c_int64, C.c_uint64, C.c_uint64, C.c_double,
                                           C.c_double]
        L.syn_fill_tokens.argtypes = [C.c_void_p, C.c_int64, C.c_uint64, C.c_uint64, C.c_int32]
        L.syn_fill_normal_f64.argtypes = [C.c_void_p, C.c_int64, C.c_uint64, C.c_uint64]
        L.syn_fill_uniform_f64.argtypes = [C.c_void_p, C.c_int64, C.c_uint64, C.c_uint64]
        L.syn_fill_i8.argtypes = [C.c_void_p, C.c_int64, C.c_uint64, C.c_uint64, C.c_double]
        _lib = L
    return _lib


def dev_lib():
    global _dev
    if _dev is None:
        L = C.CDLL(build_device())
        for f in (L.syn_dev_fill_bf16, L.syn_dev_fill_bf16_as_f32):
            f.restype = C.c_int
            f.argtypes = [C.c_void_p, C.c_int64, C.c_uint64, C.c_uint64, C.c_double, C.c_double, C.c_void_p]
        L.syn_dev_fill_i8.restype = C.c_int
        L.syn_dev_fill_i8.argtypes = [C.c_void_p, C.c_int64, C.c_uint64, C.c_uint64, C.c_double, C.c_void_p]
        _dev = L
    return _dev


# ----------------------------------------------------------------- host generators

def bf16_normal(shape, seed: int, tid: int, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    """bf16 bits (uint16) of mean + std * N(0,1), one stream per (seed, tid)."""
    out = np.empty(shape, np.uint16)
    lib().syn_fill_bf16(out.ctypes.data, out.size, seed, tid, mean, std)
    return out


def bf16_normal_f32(n: int, seed: int, tid: int, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    out = np.empty(n, np.float32)
    lib().syn_fill_bf16_as_f32(out.ctypes.data, n, seed, tid, mean, std)
    return out


def int8_normal(shape, seed: int, tid: int, std: float = Q8_STD) -> np.ndarray:
    """int8 values nearbyint(std * N(0,1)) clamped to [-127, 127], one stream per (seed, tid)."""
    out = np.empty(shape, np.int8)
    lib().syn_fill_i8(out.ctypes.data, out.size, seed, tid, std)
    return out


def q8_rows(shape, seed: int, tid: int, scale_tid: int):
    """A synthetic q8_row matrix: (int8 values [rows][cols], fp32 row scales [rows])."""
    q = int8_normal(shape, seed, tid)
    s = bf16_normal_f32(shape[0], seed, scale_tid, WEIGHT_STD / Q8_STD, 0.1 * WEIGHT_STD / Q8_STD)
    return q, s


def tokens(n: int, vocab: int, seed: int, tid: int = 0) -> np.ndarray:
    out = np.empty(n, np.int32)
    lib().syn_fill_tokens(out.ctypes.data, n, seed, tid, vocab)
    return out


def normal_f64(n: int, seed: int, tid: int) -> np.ndarray:
    out = np.empty(n, np.float64)
    lib().syn_fill_normal_f64(out.ctypes.data, n, seed, tid)
    return out


def uniform_f64(n: int, seed: int, tid: int) -> np.ndarray:
    out = np.empty(n, np.float64)
    lib().syn_fill_uniform_f64(out.ctypes.data, n, seed, tid)
    return out


def bits_to_f32(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Nearest-even rounding of fp32 values to bf16 bits (input preparation only)."""
    u = np.ascontiguousarray(a, np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def layer_tid(layer: int, name: str) -> int:
    return 1000 + 100 * layer + SLOTS[name]


def expert_tid(layer: int, e: int, part: int) -> int:
    return 10_000_000 + 10_000 * layer + 10 * e + part


def tensor_shapes(cfg: dict) -> dict:
    """Shape of every per-layer tensor of a config (None = absent)."""
    h, d, nq, nkv = cfg["hidden"], cfg["head_dim"], cfg["n_q_heads"], cfg["n_kv_heads"]
    qkv = nq * d + 2 * nkv * d
    s = dict(attn_norm=(h,), ffn_norm=(h,), wqkv=(qkv, h), wo=(h, nq * d),
             bqkv=(qkv,) if cfg.get("qkv_bias") else None,
             q_norm=(d,) if cfg.get("qk_norm") else None,
             k_norm=(d,) if cfg.get("qk_norm") else None,
             post_attn_norm=(h,) if cfg.get("sandwich") else None,
             post_ffn_norm=(h,) if cfg.get("sandwich") else None)
    if cfg.get("n_experts", 0) > 0:
        E, Ie, Is = cfg["n_experts"], cfg["expert_inter"], cfg.get("shared_inter", 0)
        s.update(w_router=(E, h), e_gate=(E, Ie, h), e_up=(E, Ie, h), e_down=(E, h, Ie),
                 s_gate=(Is, h) if Is else None, s_up=(Is, h) if Is else None,
                 s_down=(h, Is) if Is else None,
                 s_gate_vec=(h,) if (Is and cfg.get("shared_gate")) else None)
    else:
        I = cfg["ffn_inter"]
        s.update(w_gate=(I, h), w_up=(I, h), w_down=(h, I))
    return s


def make_layer(cfg: dict, layer: int, seed: int = 0) -> dict:
    out = {}
    q8 = cfg.get("weight_format", 0) == 1
    for name, shape in tensor_shapes(cfg).items():
        if shape is None:
            out[name] = None
        elif q8 and name in Q8_MATS:
            tid = layer_tid(layer, name)
            out[name], out[name + "_scale"] = q8_rows(shape, seed, tid, tid + 50)
        elif name in ("e_gate", "e_up", "e_down"):
            part = ("e_gate", "e_up", "e_down").index(name)
            arr = np.empty(shape, np.uint16)
            for e in range(shape[0]):
                lib().syn_fill_bf16(arr[e].ctypes.data, arr[e].size, seed, expert_tid(layer, e, part),
                                    0.0, WEIGHT_STD)
            out[name] = arr
        elif name in GAINS:
            out[name] = bf16_normal_f32(shape[0], seed, layer_tid(layer, name), 1.0, GAIN_STD)
        elif name in VECTORS:
            out[name] = bf16_normal_f32(shape[0], seed, layer_tid(layer, name), 0.0, WEIGHT_STD)
        else:
            out[name] = bf16_normal(shape, seed, layer_tid(layer, name), 0.0, WEIGHT_STD)
    return out


def make_weights(cfg: dict, seed: int = 0) -> dict:
    """All weights of a config on the host: bf16 bits (uint16) and fp32 1-D parameters."""
    h, V = cfg["hidden"], cfg["vocab"]
    w = dict(embed=bf16_normal((V, h), seed, 1, 0.0, WEIGHT_STD),
             lm_head=None if cfg.get("tied") else bf16_normal((V, h), seed, 2, 0.0, WEIGHT_STD),
             final_norm=bf16_normal_f32(h, seed, 3, 1.0, GAIN_STD))
    if cfg.get("weight_format", 0) == 1 and not cfg.get("tied"):
        w["lm_head"], w["lm_head_scale"] = q8_rows((V, h), seed, 2, 4)
    w["layers"] = [make_layer(cfg, l, seed) for l in range(cfg["layers"])]
    return w


def kv_fill(n_rows: int, kv_dim: int, seed: int = 2000, tid: int = 0):
    """Synthetic cache rows: N(0,1) bf16 bits, K and V from two streams."""
    k = bf16_normal((n_rows, kv_dim), seed, 2 * tid, 0.0, 1.0)
    v = bf16_normal((n_rows, kv_dim), seed, 2 * tid + 1, 0.0, 1.0)
    return k, v


def route_logits_with_margin(T: int, E: int, k: int, margin: float = 1e-3, seed: int = 3000):
    """Router logits [T][E] (fp32) whose sorted values differ by at least ``margin`` at every
    step down to rank k+1: draw N(0,1), sort, push consecutive values apart, permute."""
    out = np.empty((T, E), np.float32)
    z = normal_f64(T * E, seed, 0).reshape(T, E)
    u = uniform_f64(T * E, seed, 1).reshape(T, E)
    for t in range(T):
        vals = np.sort(z[t])[::-1].copy()
        for i in range(1, E):
            if vals[i - 1] - vals[i] < 4 * margin:
                vals[i] = vals[i - 1] - 4 * margin
        perm = np.argsort(u[t], kind="stable")
        row = np.empty(E)
        row[perm] = vals
        out[t] = row.astype(np.float32)
    return out
