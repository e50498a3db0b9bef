"""CPU oracle for the decoder-only transformer layer stack (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this package. The product path (the CUDA library and its
binding) never imports, links or calls it.

The arithmetic lives in ``oracle.c`` (plain C, fp64, bf16 rounding only at the
points where the pages store reduced precision). This module compiles it with
gcc and wraps it with ctypes.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

OK, ERR_INVALID_ARG, ERR_CONTEXT_OVERFLOW = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, OpenMP, no FP contraction)."""
    hdr = os.path.join(_HERE, "oracle.h")
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= max(os.path.getmtime(_SRC), os.path.getmtime(hdr))):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                           "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        # ORACLE_LIB points the wrapper at another build of oracle.c (the mutation tests
        # compile deliberately broken copies to show that the pins catch them).
        _lib = C.CDLL(os.environ.get("ORACLE_LIB") or build())
        _declare(_lib)
    return _lib


class Config(C.Structure):
    _fields_ = [(n, C.c_int32) for n in (
        "hidden", "layers", "nq", "nkv", "d", "inter", "vocab",
        "tied", "qkv_bias", "qk_norm",
        "n_experts", "top_k", "expert_inter", "shared_inter", "shared_gate", "norm_topk",
        "max_ctx")] + [("eps", C.c_double), ("rope_base", C.c_double)] + \
        [(n, C.c_int32) for n in ("sliding_window", "swa_pattern", "sandwich", "q8")] + \
        [("attn_softcap", C.c_double), ("final_softcap", C.c_double)]


class Weights(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("lm_head", C.c_void_p), ("final_norm", C.c_void_p),
                ("lm_head_q", C.c_void_p), ("lm_head_s", C.c_void_p)]


_LAYER_FIELDS = ("attn_norm", "ffn_norm", "wqkv", "bqkv", "q_norm", "k_norm", "wo",
                 "w_gate", "w_up", "w_down", "w_router", "e_gate", "e_up", "e_down",
                 "s_gate", "s_up", "s_down", "s_gate_vec", "post_attn_norm", "post_ffn_norm",
                 "wqkv_q", "wqkv_s", "wo_q", "wo_s", "w_gate_q", "w_gate_s", "w_up_q", "w_up_s",
                 "w_down_q", "w_down_s")
# projections that q8_row models hold as int8 [rows][cols] + fp32 row scales
Q8_MATS = ("wqkv", "wo", "w_gate", "w_up", "w_down")


class Layer(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in _LAYER_FIELDS]


_P = C.c_void_p


def _declare(L):
    L.orc_bf16.restype = C.c_double
    L.orc_bf16.argtypes = [C.c_double]
    L.orc_matvec.argtypes = [_P, C.c_int64, C.c_int64, _P, _P]
    L.orc_rmsnorm.argtypes = [_P, _P, C.c_int, C.c_double, _P]
    L.orc_head_rmsnorm.argtypes = [_P, C.c_int, C.c_int, _P, C.c_double]
    L.orc_rope.argtypes = [_P, C.c_int, C.c_int, C.c_int64, C.c_double]
    L.orc_attend.argtypes = [_P, _P, _P, C.c_int64, C.c_int, C.c_int64, C.c_double, _P]
    L.orc_attend_window.argtypes = [_P, _P, _P, C.c_int64, C.c_int, C.c_int64, C.c_int64, C.c_double, C.c_double,
                                    _P]
    L.orc_matvec_q8.argtypes = [_P, _P, C.c_int64, C.c_int64, _P, _P]
    L.orc_layer_window.argtypes = [C.POINTER(Config), C.c_int]
    L.orc_route_topk.argtypes = [_P, C.c_int, C.c_int, C.c_int, _P, _P, _P]
    L.orc_swiglu.argtypes = [_P, _P, _P, _P, C.c_int, C.c_int, _P]
    L.orc_swiglu_act.argtypes = [_P, _P, _P, C.c_int, C.c_int, _P]
    L.orc_moe_ffn.argtypes = [C.POINTER(Config), C.POINTER(Layer), _P, _P, _P, _P, _P]
    L.orc_create.restype = _P
    L.orc_create.argtypes = [C.POINTER(Config), C.POINTER(Weights), C.POINTER(Layer), C.c_int]
    L.orc_destroy.argtypes = [_P]
    L.orc_forward.argtypes = [_P, C.c_int, C.c_int32, C.c_int64, _P]
    L.orc_prefill.argtypes = [_P, C.c_int, _P, C.c_int64, C.c_int64, _P]
    L.orc_argmax.argtypes = [_P, C.c_int64]
    L.orc_kv_write.argtypes = [_P, C.c_int, C.c_int, C.c_int64, C.c_int64, _P, _P]
    L.orc_kv_read.argtypes = [_P, C.c_int, C.c_int, C.c_int64, C.c_int64, _P, _P]
    L.orc_last_routes.argtypes = [_P, _P, _P, _P]
    L.orc_last_hidden.argtypes = [_P, _P]
    L.orc_gqa_decode.argtypes = [_P, _P, _P, _P, _P, C.c_int64, _P, C.c_int, C.c_int, C.c_int, C.c_int,
                                 C.c_double, C.c_int, C.c_double, _P]
    L.orc_route_rows.argtypes = [_P, C.c_int, C.c_int, C.c_int, C.c_int, _P, _P, _P]
    L.orc_gemv_rows.argtypes = [_P, _P, C.c_int, C.c_int64, C.c_int64, _P]


def _p(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=dtype)


# ----------------------------------------------------------------- pieces

def bf16(v: float) -> float:
    return lib().orc_bf16(float(v))


def matvec(W: np.ndarray, x: np.ndarray) -> np.ndarray:
    W = _c(W, np.uint16)
    x = _c(x, np.float64)
    y = np.empty(W.shape[0], np.float64)
    lib().orc_matvec(_p(W), W.shape[0], W.shape[1], _p(x), _p(y))
    return y


def rmsnorm(x, g, eps) -> np.ndarray:
    x = _c(x, np.float64)
    g = _c(g, np.float32)
    out = np.empty_like(x)
    lib().orc_rmsnorm(_p(x), _p(g), x.size, float(eps), _p(out))
    return out


def head_rmsnorm(v: np.ndarray, g, eps) -> np.ndarray:
    """QK-norm of v [heads][d]: each head normalised by its own mean square, times g [d]."""
    v = np.array(v, dtype=np.float64, order="C")
    heads, d = v.shape
    g = _c(g, np.float32)
    lib().orc_head_rmsnorm(_p(v), heads, d, _p(g), float(eps))
    return v


def rope(v: np.ndarray, pos: int, base: float) -> np.ndarray:
    """Rotate v [heads][d] to position pos (returns a new array)."""
    v = np.array(v, dtype=np.float64, order="C")
    heads, d = v.shape
    lib().orc_rope(_p(v), heads, d, int(pos), float(base))
    return v


def attend(q, K, V, scale) -> np.ndarray:
    """One head: q [d] fp64, K/V bf16 bits [n][d]."""
    q = _c(q, np.float64)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    out = np.empty(q.size, np.float64)
    lib().orc_attend(_p(q), _p(K), _p(V), K.shape[1], q.size, K.shape[0], float(scale), _p(out))
    return out


def attend_window(q, K, V, scale, first=0, softcap=0.0) -> np.ndarray:
    """One head over rows first .. n-1 of K/V (bf16 bits [n][d]), optional logit softcap."""
    q = _c(q, np.float64)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    out = np.empty(q.size, np.float64)
    lib().orc_attend_window(_p(q), _p(K), _p(V), K.shape[1], q.size, int(first), K.shape[0], float(scale),
                            float(softcap), _p(out))
    return out


def matvec_q8(Q, S, x) -> np.ndarray:
    """q8_row matrix (int8 [N][K], fp32 scales [N]) times x [K]."""
    Q = _c(Q, np.int8)
    S = _c(S, np.float32)
    x = _c(x, np.float64)
    y = np.empty(Q.shape[0], np.float64)
    lib().orc_matvec_q8(_p(Q), _p(S), Q.shape[0], Q.shape[1], _p(x), _p(y))
    return y


def layer_window(cfg: dict, layer: int) -> int:
    return lib().orc_layer_window(C.byref(_make_config(cfg, 1)), int(layer))


def route_topk(logits, k, renorm):
    logits = _c(logits, np.float64)
    idx = np.empty(k, np.int32)
    w = np.empty(k, np.float64)
    gap = np.empty(1, np.float64)
    lib().orc_route_topk(_p(logits), logits.size, k, int(renorm), _p(idx), _p(w), _p(gap))
    return idx, w, float(gap[0])


def swiglu(x, Wg, Wu, Wd) -> np.ndarray:
    x = _c(x, np.float64)
    Wg, Wu, Wd = (_c(a, np.uint16) for a in (Wg, Wu, Wd))
    out = np.empty(Wd.shape[0], np.float64)
    lib().orc_swiglu(_p(x), _p(Wg), _p(Wu), _p(Wd), Wg.shape[0], Wg.shape[1], _p(out))
    return out


def swiglu_act(x, Wg, Wu) -> np.ndarray:
    """The SwiGLU activation R4(silu(Wg x) * (Wu x)) [I] (before the down projection)."""
    x = _c(x, np.float64)
    Wg, Wu = _c(Wg, np.uint16), _c(Wu, np.uint16)
    out = np.empty(Wg.shape[0], np.float64)
    lib().orc_swiglu_act(_p(x), _p(Wg), _p(Wu), Wg.shape[0], Wg.shape[1], _p(out))
    return out


def gqa_decode(q, k_new, v_new, kcache, vcache, pos, nq, nkv, d, scale, fused_rope, rope_base):
    """Standalone decode attention. kcache/vcache: bf16 bits [B][ctx][nkv][d], updated in place
    with the appended row. q: [B][nq][d] bf16 bits. Returns out [B][nq][d] fp64."""
    B = q.shape[0]
    q = _c(q, np.uint16)
    k_new = _c(k_new, np.uint16)
    v_new = _c(v_new, np.uint16)
    assert kcache.flags.c_contiguous and vcache.flags.c_contiguous
    pos = _c(pos, np.int32)
    out = np.empty((B, nq, d), np.float64)
    lib().orc_gqa_decode(_p(q), _p(k_new), _p(v_new), _p(kcache), _p(vcache), kcache.shape[1], _p(pos),
                         B, nq, nkv, d, float(scale), int(fused_rope), float(rope_base), _p(out))
    return out


def route_rows(logits, k, renorm):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    gap = np.empty(T, np.float64)
    lib().orc_route_rows(_p(logits), T, E, k, int(renorm), _p(idx), _p(w), _p(gap))
    return idx, w, gap


def gemv_rows(W, x) -> np.ndarray:
    W = _c(W, np.uint16)
    x = _c(x, np.uint16)
    B = x.shape[0]
    y = np.empty((B, W.shape[0]), np.float64)
    lib().orc_gemv_rows(_p(W), _p(x), B, W.shape[0], W.shape[1], _p(y))
    return y


# ----------------------------------------------------------------- model

_F32_FIELDS = ("attn_norm", "ffn_norm", "bqkv", "q_norm", "k_norm", "s_gate_vec", "post_attn_norm",
               "post_ffn_norm")


def _make_config(cfg: dict, max_ctx: int) -> Config:
    c = Config()
    c.hidden, c.layers, c.nq, c.nkv, c.d = (cfg["hidden"], cfg["layers"], cfg["n_q_heads"],
                                             cfg["n_kv_heads"], cfg["head_dim"])
    c.inter, c.vocab = cfg.get("ffn_inter", 0), cfg["vocab"]
    c.tied, c.qkv_bias, c.qk_norm = cfg.get("tied", 0), cfg.get("qkv_bias", 0), cfg.get("qk_norm", 0)
    c.n_experts, c.top_k = cfg.get("n_experts", 0), cfg.get("top_k", 0)
    c.expert_inter, c.shared_inter = cfg.get("expert_inter", 0), cfg.get("shared_inter", 0)
    c.shared_gate, c.norm_topk = cfg.get("shared_gate", 0), cfg.get("norm_topk", 0)
    c.max_ctx = int(max_ctx)
    c.eps, c.rope_base = float(cfg["rms_eps"]), float(cfg["rope_base"])
    c.sliding_window, c.swa_pattern = cfg.get("sliding_window", 0), cfg.get("swa_pattern", 0)
    c.sandwich, c.q8 = cfg.get("sandwich", 0), int(cfg.get("weight_format", 0) == 1)
    c.attn_softcap, c.final_softcap = float(cfg.get("attn_softcap", 0.0)), float(cfg.get("final_softcap", 0.0))
    return c


def _fill_layer(dst: Layer, lw: dict, keep: list, q8: bool = False) -> None:
    """Point a Layer at the arrays of a synth layer dict. In a q8_row model the projection
    entries (Q8_MATS) are int8 and their row scales sit under '<name>_scale'."""
    for f in _LAYER_FIELDS:
        setattr(dst, f, None)
    for f, a in lw.items():
        if a is None or f.endswith("_scale") or f not in _LAYER_FIELDS:
            continue
        if q8 and f in Q8_MATS:
            qa = np.ascontiguousarray(a, dtype=np.int8)
            sa = np.ascontiguousarray(lw[f + "_scale"], dtype=np.float32)
            keep += [qa, sa]
            setattr(dst, f + "_q", qa.ctypes.data)
            setattr(dst, f + "_s", sa.ctypes.data)
            continue
        a = np.ascontiguousarray(a, dtype=np.float32 if f in _F32_FIELDS else np.uint16)
        keep.append(a)
        setattr(dst, f, a.ctypes.data)


def moe_ffn(cfg: dict, lw: dict, xn):
    """MoE FFN of one layer on one normalised input row; returns (out, idx, w, gap)."""
    keep = []
    c = _make_config(cfg, 1)
    L = Layer()
    _fill_layer(L, lw, keep, cfg.get("weight_format", 0) == 1)
    xn = _c(xn, np.float64)
    k = max(1, cfg.get("top_k", 0))
    out = np.empty(cfg["hidden"], np.float64)
    idx = np.zeros(k, np.int32)
    w = np.zeros(k, np.float64)
    gap = np.zeros(1, np.float64)
    lib().orc_moe_ffn(C.byref(c), C.byref(L), _p(xn), _p(out), _p(idx), _p(w), _p(gap))
    return out, idx[:cfg.get("top_k", 0)], w[:cfg.get("top_k", 0)], float(gap[0])


@dataclass
class _Keep:
    arrays: list


class Model:
    """A whole decoder stack on the CPU, with its own contiguous KV cache per sequence.

    ``weights`` is the dict made by ``synth.make_weights`` (bf16 bits as uint16,
    1-D parameters as fp32)."""

    def __init__(self, cfg: dict, weights: dict, n_seqs: int = 1, max_ctx: int | None = None):
        self.cfg = dict(cfg)
        self.max_ctx = int(max_ctx or cfg["max_context"])
        c = _make_config(cfg, self.max_ctx)
        keep = []

        def ptr(a, dtype):
            if a is None:
                return None
            a = np.ascontiguousarray(a, dtype=dtype)
            keep.append(a)
            return a.ctypes.data

        q8 = cfg.get("weight_format", 0) == 1
        w = Weights()
        w.embed = ptr(weights["embed"], np.uint16)
        if q8 and weights.get("lm_head") is not None:
            w.lm_head_q = ptr(weights["lm_head"], np.int8)
            w.lm_head_s = ptr(weights["lm_head_scale"], np.float32)
        else:
            w.lm_head = ptr(weights.get("lm_head"), np.uint16)
        w.final_norm = ptr(weights["final_norm"], np.float32)
        layers = (Layer * cfg["layers"])()
        for i, lw in enumerate(weights["layers"]):
            _fill_layer(layers[i], lw, keep, q8)
        self._keep = _Keep(keep)
        self._c = c
        self.n_seqs = n_seqs
        self.h = lib().orc_create(C.byref(c), C.byref(w), layers, n_seqs)
        if not self.h:
            raise MemoryError("oracle: cache allocation failed")

    def close(self):
        if getattr(self, "h", None):
            lib().orc_destroy(self.h)
            self.h = None

    def __del__(self):
        self.close()

    def forward(self, seq: int, token: int, pos: int, want_logits: bool = True):
        logits = np.empty(self.cfg["vocab"], np.float64) if want_logits else None
        rc = lib().orc_forward(self.h, seq, int(token), int(pos), _p(logits))
        if rc != OK:
            raise OracleError(rc)
        return logits

    def prefill(self, seq: int, tokens, pos0: int):
        toks = np.ascontiguousarray(tokens, np.int32)
        logits = np.empty(self.cfg["vocab"], np.float64)
        rc = lib().orc_prefill(self.h, seq, _p(toks), toks.size, int(pos0), _p(logits))
        if rc != OK:
            raise OracleError(rc)
        return logits

    def kv_write(self, seq, layer, pos0, k, v):
        k = _c(k, np.uint16)
        v = _c(v, np.uint16)
        rc = lib().orc_kv_write(self.h, seq, layer, pos0, k.shape[0], _p(k), _p(v))
        if rc != OK:
            raise OracleError(rc)

    def kv_read(self, seq, layer, pos0, n):
        kvd = self.cfg["n_kv_heads"] * self.cfg["head_dim"]
        k = np.empty((n, kvd), np.uint16)
        v = np.empty((n, kvd), np.uint16)
        rc = lib().orc_kv_read(self.h, seq, layer, pos0, n, _p(k), _p(v))
        if rc != OK:
            raise OracleError(rc)
        return k, v

    def last_routes(self):
        L, k = self.cfg["layers"], max(1, self.cfg.get("top_k", 0))
        idx = np.empty((L, k), np.int32)
        w = np.empty((L, k), np.float64)
        gap = np.empty(L, np.float64)
        lib().orc_last_routes(self.h, _p(idx), _p(w), _p(gap))
        return idx, w, gap

    def last_hidden(self):
        out = np.empty(self.cfg["hidden"], np.float64)
        lib().orc_last_hidden(self.h, _p(out))
        return out


class OracleError(RuntimeError):
    def __init__(self, code):
        super().__init__({1: "invalid argument", 2: "context overflow"}.get(code, f"error {code}"))
        self.code = code


def argmax(v) -> int:
    v = _c(v, np.float64)
    return lib().orc_argmax(_p(v), v.size)
