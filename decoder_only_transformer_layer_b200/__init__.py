"""B200 (sm_100a) decoder-only transformer layer stack: Python binding of libdec.so.

This module only marshals arguments for the C ABI declared in include/dec_api.h.
Every step of the forward runs in the library's CUDA kernels; there is no CPU
path. Importing works without a GPU (the library loads and its symbols can be
inspected), but calls need a CUDA device and fail loudly otherwise.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from ._build import LIB, build, stale  # noqa: F401

__all__ = ["lib", "Decoder", "DecError", "gqa_decode_attn", "moe_route_topk", "moe_experts", "weight_gemv",
           "weight_gemv_q8", "ffn_gate_up", "check_standalone", "STATUS"]

STATUS = {0: "OK", 1: "INVALID_ARG", 2: "CONTEXT_OVERFLOW", 3: "PAGES_EXHAUSTED", 4: "OOM", 5: "CUDA",
          6: "TIMEOUT", 7: "UNSUPPORTED"}


class DecError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code
        self.status = STATUS.get(code, str(code))


class Config(C.Structure):
    _fields_ = [(n, C.c_int32) for n in (
        "hidden", "layers", "n_q_heads", "n_kv_heads", "head_dim", "ffn_inter", "vocab",
        "tied_embeddings", "qkv_bias", "qk_norm", "n_experts", "top_k", "expert_inter", "shared_inter",
        "shared_gate", "norm_topk_prob")] + [("rms_eps", C.c_float), ("rope_base", C.c_float)] + \
        [(n, C.c_int32) for n in ("max_batch", "max_context", "page_size", "prefill_chunk", "n_pages",
                                  "sliding_window", "swa_pattern")] + \
        [("attn_softcap", C.c_float), ("final_softcap", C.c_float), ("sandwich_norms", C.c_int32),
         ("weight_format", C.c_int32)]


LAYER_FIELDS = ("attn_norm", "ffn_norm", "wqkv", "bqkv", "q_norm", "k_norm", "wo", "w_gate", "w_up", "w_down",
                "w_router", "e_gate", "e_up", "e_down", "s_gate", "s_up", "s_down", "s_gate_vec",
                "post_attn_norm", "post_ffn_norm", "wqkv_scale", "wo_scale", "w_gate_scale", "w_up_scale",
                "w_down_scale")


class LayerWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in LAYER_FIELDS]


class Weights(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("lm_head", C.c_void_p), ("final_norm", C.c_void_p),
                ("layers", C.POINTER(LayerWeights)), ("lm_head_scale", C.c_void_p)]


_P = C.c_void_p
_I = C.c_int32
_lib = None


def lib():
    """The loaded libdec.so (built on first use if the sources are newer)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB) or stale():
            build()
        L = C.CDLL(LIB)
        L.dec_last_error.restype = C.c_char_p
        L.dec_init.argtypes = [C.POINTER(Config), C.POINTER(Weights), _P, C.POINTER(_P)]
        L.dec_free.argtypes = [_P]
        L.dec_reset.argtypes = [_P, _I]
        L.dec_prefill.argtypes = [_P, _I, _P, _I, _I, _P]
        L.dec_step.argtypes = [_P, _P, _P, _I, _P]
        L.dec_last_argmax.argtypes = [_P, _P, _I]
        L.dec_kv_read.argtypes = [_P, _I, _I, _I, _I, _P, _P]
        L.dec_kv_write.argtypes = [_P, _I, _I, _I, _I, _P, _P]
        L.dec_last_routes.argtypes = [_P, _P, _I]
        L.dec_last_hidden.argtypes = [_P, _P, _I]
        L.dec_seq_len.argtypes = [_P, _I, _P]
        L.gqa_decode_attn.argtypes = [_P, _P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, C.c_float, _I,
                                      C.c_float, _P, _P]
        L.gqa_decode_attn_noalloc.argtypes = L.gqa_decode_attn.argtypes
        L.moe_route_topk.argtypes = [_P, _I, _I, _I, _I, _P, _P, _P]
        L.weight_gemv.argtypes = [_P, _P, _I, _I, _I, _P, _P]
        L.weight_gemv_q8.argtypes = [_P, _P, _P, _I, _I, _I, _P, _P]
        L.ffn_gate_up.argtypes = [_P, _P, _P, C.c_float, _I, _I, _I, _P, _P]
        L.moe_experts.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P]
        L.dec_check.argtypes = [_P]
        L.dec_verify.argtypes = [_P, _I, _P, _I, _I, _P]
        L.dec_truncate.argtypes = [_P, _I, _I]
        L.dec_check_standalone.argtypes = [_P]
        L.dec_test_fail_alloc.argtypes = [_I]
        L.dec_test_gemm_wait.argtypes = [_I, C.c_int64]
        L.dec_test_streamk_check.argtypes = [_I, _I, _I, _I]
        L.dec_test_streamk_check.restype = C.c_int
        for f in ("dec_init", "dec_free", "dec_reset", "dec_prefill", "dec_step", "dec_last_argmax", "dec_kv_read",
                  "dec_kv_write", "dec_last_routes", "dec_last_hidden", "dec_seq_len", "gqa_decode_attn",
                  "gqa_decode_attn_noalloc", "moe_route_topk", "moe_experts", "weight_gemv", "dec_check",
                  "dec_check_standalone", "dec_test_fail_alloc", "dec_test_gemm_wait", "dec_verify", "dec_truncate", "weight_gemv_q8", "ffn_gate_up"):
            getattr(L, f).restype = C.c_int
        _lib = L
    return _lib


def _check(rc: int):
    if rc != 0:
        raise DecError(rc, lib().dec_last_error().decode())


def _ptr(a):
    """Device or host address of a torch tensor or numpy array (None -> NULL)."""
    if a is None:
        return None
    if hasattr(a, "data_ptr"):
        return a.data_ptr()
    if isinstance(a, np.ndarray):
        if not a.flags.c_contiguous:
            raise ValueError("array must be C-contiguous")
        return a.ctypes.data
    raise TypeError(f"unsupported buffer type {type(a)}")


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return int(stream)


def make_config(cfg: dict) -> Config:
    c = Config()
    c.hidden, c.layers = cfg["hidden"], cfg["layers"]
    c.n_q_heads, c.n_kv_heads, c.head_dim = cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    c.ffn_inter, c.vocab = cfg.get("ffn_inter", 0), cfg["vocab"]
    c.tied_embeddings, c.qkv_bias, c.qk_norm = cfg.get("tied", 0), cfg.get("qkv_bias", 0), cfg.get("qk_norm", 0)
    c.n_experts, c.top_k = cfg.get("n_experts", 0), cfg.get("top_k", 0)
    c.expert_inter, c.shared_inter = cfg.get("expert_inter", 0), cfg.get("shared_inter", 0)
    c.shared_gate, c.norm_topk_prob = cfg.get("shared_gate", 0), cfg.get("norm_topk", 0)
    c.rms_eps, c.rope_base = cfg["rms_eps"], cfg["rope_base"]
    c.max_batch, c.max_context = cfg.get("max_batch", 1), cfg["max_context"]
    c.page_size, c.prefill_chunk = cfg.get("page_size", 16), cfg.get("prefill_chunk", 128)
    c.n_pages = cfg.get("n_pages", 0)
    c.sliding_window, c.swa_pattern = cfg.get("sliding_window", 0), cfg.get("swa_pattern", 0)
    c.attn_softcap, c.final_softcap = cfg.get("attn_softcap", 0.0), cfg.get("final_softcap", 0.0)
    c.sandwich_norms, c.weight_format = cfg.get("sandwich", 0), cfg.get("weight_format", 0)
    return c


class Decoder:
    """A model context on the current CUDA device (dec_init ... dec_free).

    ``weights``: dict with ``embed``, ``lm_head`` (or None when tied), ``final_norm`` and
    ``layers`` (list of dicts keyed like dec_layer_weights), each a numpy array (host) or a
    torch tensor (host or device): bf16 matrices as uint16 / bfloat16 / int16 storage, 1-D
    parameters as float32. The library copies and repacks them; they may be freed after."""

    def __init__(self, cfg: dict, weights: dict, stream=None):
        self.cfg = dict(cfg)
        self._cfg_c = make_config(cfg)
        self.stream = _stream(stream)
        layers = (LayerWeights * cfg["layers"])()
        for i, lw in enumerate(weights["layers"]):
            for f in LAYER_FIELDS:
                setattr(layers[i], f, _ptr(lw.get(f)))
        w = Weights()
        w.embed = _ptr(weights["embed"])
        w.lm_head = _ptr(weights.get("lm_head"))
        w.final_norm = _ptr(weights["final_norm"])
        w.layers = layers
        w.lm_head_scale = _ptr(weights.get("lm_head_scale"))
        h = _P()
        _check(lib().dec_init(C.byref(self._cfg_c), C.byref(w), self.stream, C.byref(h)))
        self.h = h

    def close(self):
        if getattr(self, "h", None):
            lib().dec_free(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ------------------------------------------------------------------ forward
    def prefill(self, seq: int, tokens, pos0: int, logits_out=None):
        toks = np.ascontiguousarray(tokens, dtype=np.int32)
        _check(lib().dec_prefill(self.h, seq, toks.ctypes.data if toks.size else None, toks.size, pos0,
                                 _ptr(logits_out)))
        return logits_out

    def step(self, tokens, pos, logits_out=None):
        toks = np.ascontiguousarray(tokens, dtype=np.int32)
        ps = np.ascontiguousarray(pos, dtype=np.int32)
        if toks.size != ps.size:
            raise ValueError("tokens and pos differ in length")
        _check(lib().dec_step(self.h, toks.ctypes.data, ps.ctypes.data, toks.size, _ptr(logits_out)))
        return logits_out

    def prefill_logits(self, seq: int, tokens, pos0: int) -> np.ndarray:
        out = np.empty(self.cfg["vocab"], np.float32)
        self.prefill(seq, tokens, pos0, out)
        return out

    def step_logits(self, tokens, pos) -> np.ndarray:
        out = np.empty((len(tokens), self.cfg["vocab"]), np.float32)
        self.step(tokens, pos, out)
        return out

    def verify(self, seq: int, tokens, pos0: int, logits_out=None):
        toks = np.ascontiguousarray(tokens, dtype=np.int32)
        _check(lib().dec_verify(self.h, seq, toks.ctypes.data if toks.size else None, toks.size, pos0,
                                _ptr(logits_out)))
        return logits_out

    def verify_logits(self, seq: int, tokens, pos0: int) -> np.ndarray:
        out = np.empty((len(tokens), self.cfg["vocab"]), np.float32)
        self.verify(seq, tokens, pos0, out)
        return out

    def truncate(self, seq: int, length: int):
        _check(lib().dec_truncate(self.h, seq, length))

    def last_argmax(self, B: int) -> np.ndarray:
        out = np.empty(B, np.int32)
        _check(lib().dec_last_argmax(self.h, out.ctypes.data, B))
        return out

    def check(self):
        """Synchronise and raise DecError(TIMEOUT) if a device wait of an earlier call ran out."""
        _check(lib().dec_check(self.h))

    def reset(self, seq: int = -1):
        _check(lib().dec_reset(self.h, seq))

    def seq_len(self, seq: int) -> int:
        n = C.c_int32()
        _check(lib().dec_seq_len(self.h, seq, C.byref(n)))
        return n.value

    # ------------------------------------------------------------------ test hooks
    def kv_write(self, seq, layer, pos0, k, v):
        """k, v: bf16 rows [n][nkv*d] as uint16 numpy arrays (host) or 16-bit torch tensors."""
        if not hasattr(k, "data_ptr"):
            k = np.ascontiguousarray(k, np.uint16)
            v = np.ascontiguousarray(v, np.uint16)
        _check(lib().dec_kv_write(self.h, seq, layer, pos0, k.shape[0], _ptr(k), _ptr(v)))

    def kv_read(self, seq, layer, pos0, n):
        kvd = self.cfg["n_kv_heads"] * self.cfg["head_dim"]
        k = np.empty((n, kvd), np.uint16)
        v = np.empty((n, kvd), np.uint16)
        _check(lib().dec_kv_read(self.h, seq, layer, pos0, n, k.ctypes.data, v.ctypes.data))
        return k, v

    def last_routes(self, B):
        out = np.empty((self.cfg["layers"], B, self.cfg["top_k"]), np.int32)
        _check(lib().dec_last_routes(self.h, out.ctypes.data, B))
        return out

    def last_hidden(self, B):
        out = np.empty((B, self.cfg["hidden"]), np.float32)
        _check(lib().dec_last_hidden(self.h, out.ctypes.data, B))
        return out


# ---------------------------------------------------------------------- standalone calls

def gqa_decode_attn(q, k_new, v_new, k_pool, v_pool, block_table, pos, nq, nkv, d, scale, fused_rope,
                    rope_base, out, page_size=16, stream=None):
    """Device tensors: q bf16 [B][nq][d]; k_new/v_new bf16 [B][nkv][d] or None; pools bf16
    [n_pages][nkv][page][d]; block_table int32 [B][max_pages]; pos int32 [B]; out bf16 [B][nq][d]."""
    B, max_pages = block_table.shape
    _check(lib().gqa_decode_attn(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_pool), _ptr(v_pool), _ptr(block_table),
                                 max_pages, _ptr(pos), B, nq, nkv, d, page_size, float(scale), int(fused_rope),
                                 float(rope_base), _ptr(out), _stream(stream)))
    return out


def gqa_decode_attn_noalloc(q, k_new, v_new, k_pool, v_pool, block_table, pos, nq, nkv, d, scale, fused_rope,
                            rope_base, out, page_size=16, stream=None):
    """gqa_decode_attn for callers that must not let the library allocate device memory:
    the scratch is a fixed array built into the library (same arguments and results)."""
    B, max_pages = block_table.shape
    _check(lib().gqa_decode_attn_noalloc(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_pool), _ptr(v_pool),
                                         _ptr(block_table), max_pages, _ptr(pos), B, nq, nkv, d, page_size,
                                         float(scale), int(fused_rope), float(rope_base), _ptr(out),
                                         _stream(stream)))
    return out


def moe_route_topk(logits, k, renorm, idx_out, w_out, stream=None):
    """Device tensors: logits fp32 [T][E]; idx_out int32 [T][k]; w_out fp32 [T][k]."""
    T, E = logits.shape
    _check(lib().moe_route_topk(_ptr(logits), T, E, k, int(renorm), _ptr(idx_out), _ptr(w_out), _stream(stream)))
    return idx_out, w_out


def moe_experts(x, idx, w, Wgu, Wd, out, stream=None):
    """Device tensors: x bf16 [T][h]; idx int32 [T][k]; w fp32 [T][k]; Wgu bf16 [E][2I][h]
    (gate row i at 2i, up row i at 2i+1); Wd bf16 [E][h][I]; out fp32 [T][h]."""
    T, h = x.shape
    k = idx.shape[1]
    E, I2, _ = Wgu.shape
    _check(lib().moe_experts(_ptr(x), _ptr(idx), _ptr(w), T, h, E, k, I2 // 2, _ptr(Wgu), _ptr(Wd), _ptr(out),
                             _stream(stream)))
    return out


def weight_gemv(W, x, y, stream=None):
    """Device tensors: W bf16 [N][K]; x bf16 [B][K]; y fp32 [B][N]."""
    N, K = W.shape
    B = x.shape[0]
    _check(lib().weight_gemv(_ptr(W), _ptr(x), B, N, K, _ptr(y), _stream(stream)))
    return y


def ffn_gate_up(Wgu, x, gain, eps, act, stream=None):
    """Device tensors: Wgu bf16 [2I][K] (gate row i at 2i, up row i at 2i+1); x fp32 [B][K];
    gain fp32 [K]; act bf16 [B][I] = bf16(SiLU(gate . xn) * (up . xn)), xn the RMS-normed x."""
    I2, K = Wgu.shape
    B = x.shape[0]
    _check(lib().ffn_gate_up(_ptr(Wgu), _ptr(x), _ptr(gain), float(eps), B, I2 // 2, K, _ptr(act), _stream(stream)))
    return act


def weight_gemv_q8(Wq, scale, x, y, stream=None):
    """Device tensors: Wq int8 [N][K]; scale fp32 [N]; x bf16 [B][K]; y fp32 [B][N]."""
    N, K = Wq.shape
    B = x.shape[0]
    _check(lib().weight_gemv_q8(_ptr(Wq), _ptr(scale), _ptr(x), B, N, K, _ptr(y), _stream(stream)))
    return y


def check_standalone(stream=None):
    """Synchronise `stream`; raise DecError(TIMEOUT) if a bounded device wait of a standalone
    call on the current device ran out since the last check."""
    _check(lib().dec_check_standalone(_stream(stream)))


def test_fail_alloc(n: int):
    """Test hook: the n-th device allocation of the library from now on fails (0 = off)."""
    _check(lib().dec_test_fail_alloc(int(n)))


def test_streamk_check(M: int, N: int, K: int, ctas: int) -> int:
    """Test hook: violations of the persistent GEMM's work-split invariants for an
    M x N x K product over `ctas` CTAs, checked on the host (0 = sound)."""
    return int(lib().dec_test_streamk_check(int(M), int(N), int(K), int(ctas)))


def test_gemm_wait(extra_pieces: int, limit_cycles: int):
    """Test hook: later tensor-core GEMM launches wait for pieces that never arrive and give
    up after limit_cycles; (0, 0) restores normal operation."""
    _check(lib().dec_test_gemm_wait(int(extra_pieces), int(limit_cycles)))
