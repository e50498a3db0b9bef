"""The persistent tensor-core GEMM's work split, checked on the host (no GPU).

A tile shared between CTAs is finished by the CTA holding its last k blocks; the others
publish their fp32 pieces and never wait. Two invariants of the split keep that protocol
sound: every unit is computed exactly once, and every piece some other CTA finishes is the
first segment its CTA processes, so it is published before its CTA could wait on anything
(the finishers' waits can form no cycle). The library's own plan arithmetic is run on the
host over the products the model launches and a spread of others."""
import pytest

import decoder_only_transformer_layer_b200 as dec


def launched_ctas(M, N, K, sms):
    # the launcher's rule: one CTA per SM, each with at least 8 units
    bn = 32 if N <= 32 else 64 if N <= 64 else 128 if N <= 128 else 256
    units = ((M + 127) // 128) * ((N + bn - 1) // bn) * ((K + 63) // 64)
    return max(1, min(sms, units // 8))


MODEL_PRODUCTS = [  # (M, K): QKV, o_proj, gate/up, down of the Llama-3-8B and SmolLM2 shapes; Qwen1.5-MoE dense parts
    (6144, 4096), (4096, 4096), (28672, 4096), (4096, 14336),
    (960, 576), (576, 576), (3072, 576), (576, 1536),
    (6144, 2048), (2048, 2048), (128256, 4096),
]


@pytest.mark.parametrize("N", [9, 16, 32, 44, 64, 100, 128, 188, 256, 512, 4096])
@pytest.mark.parametrize("sms", [148, 132, 114])
def test_model_products_split_soundly(N, sms):
    for M, K in MODEL_PRODUCTS:
        nc = launched_ctas(M, N, K, sms)
        assert dec.test_streamk_check(M, N, K, nc) == 0, (M, N, K, nc)


def test_a_spread_of_shapes_splits_soundly():
    for M in (128, 384, 1000, 4096, 20480):
        for K in (64, 1024, 3000, 4096):
            for N in (1, 33, 129, 600):
                for sms in (1, 7, 148):
                    nc = launched_ctas(M, N, K, sms)
                    assert dec.test_streamk_check(M, N, K, nc) == 0, (M, N, K, nc)


def test_the_check_flags_a_split_with_empty_ranges():
    # more CTAs than units: some ranges are empty, so a finisher would count pieces that
    # do not exist; the launcher's rule never asks for this, and the check must see it
    M, N, K = 512, 128, 256  # 4 tiles x 4 k blocks = 16 units
    assert dec.test_streamk_check(M, N, K, launched_ctas(M, N, K, 148)) == 0
    assert dec.test_streamk_check(M, N, K, 40) > 0
    assert dec.test_streamk_check(M, N, K, 0) == -1
