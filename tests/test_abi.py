"""The C-ABI library loads on the CPU host and exports every entry point the header declares.
Only argument validation is exercised here: those calls return before any CUDA call."""
import ctypes as C
import os
import re

import decoder_only_transformer_layer_b200 as dec

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "dec_api.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:dec_status|const char\*)\s+(\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("dec_init", "dec_prefill", "dec_step", "gqa_decode_attn", "moe_route_topk", "weight_gemv",
                     "dec_free", "dec_reset", "dec_kv_read", "dec_kv_write", "dec_last_error"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = dec.lib()
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_validation_errors_need_no_gpu():
    lib = dec.lib()
    assert lib.moe_route_topk(None, 4, 60, 4, 0, None, None, None) == 1
    assert lib.weight_gemv(None, None, 1, 8, 8, None, None) == 1
    assert lib.moe_experts(None, None, None, 4, 256, 8, 2, 128, None, None, None, None) == 1
    assert b"NULL" in lib.dec_last_error()
    h = C.c_void_p()
    assert lib.dec_init(None, None, None, C.byref(h)) == 1
    assert lib.dec_prefill(None, 0, None, 0, 0, None) == 1
    assert lib.dec_step(None, None, None, 1, None) == 1
    assert lib.dec_check(None) == 1
    assert lib.dec_test_gemm_wait(-1, 0) == 1
    assert lib.dec_test_gemm_wait(0, 0) == 0
    assert lib.dec_test_fail_alloc(0) == 0


def test_config_struct_matches_header():
    src = open(os.path.join(ROOT, "include", "dec_api.h")).read()
    body = re.search(r"typedef struct dec_config \{(.*?)\} dec_config;", src, re.S).group(1)
    fields = re.findall(r"^\s*(?:int32_t|float)\s+(\w+);", body, re.M)
    assert fields == [f for f, _ in dec.Config._fields_]
    lbody = re.search(r"typedef struct dec_layer_weights \{(.*?)\} dec_layer_weights;", src, re.S).group(1)
    lfields = re.findall(r"\*\s*(\w+);", lbody)
    assert tuple(lfields) == dec.LAYER_FIELDS
