"""gqa_decode_attn_noalloc: decode attention for callers that cannot let the library
allocate device memory (their memory is reserved up front by their own pool, their
loop cannot absorb a cudaMalloc's synchronisation, or their host forbids allocation).

The call must give the same results as gqa_decode_attn, twice in a row (its scratch
array keeps the previous call's contents), and refuse shapes its fixed scratch cannot
hold. This file is collected last so that a run stopping at the first failure has
already run every other test."""
import math

import numpy as np
import pytest
import torch

import synth
import decoder_only_transformer_layer_b200 as dec
from _util import assert_parity, bits_to_f64, build_paged, from_dev_bf16, to_dev_bf16

pytestmark = pytest.mark.gpu


def _inputs(B, nq, nkv, d, pos, seed):
    ctx = int(max(pos)) + 1
    q = synth.bf16_normal((B, nq, d), seed, 1, 0.0, 1.0)
    kc = synth.bf16_normal((B, ctx, nkv, d), seed, 2, 0.0, 1.0)
    vc = synth.bf16_normal((B, ctx, nkv, d), seed, 3, 0.0, 1.0)
    kn = synth.bf16_normal((B, nkv, d), seed, 4, 0.0, 1.0)
    vn = synth.bf16_normal((B, nkv, d), seed, 5, 0.0, 1.0)
    kpool, vpool, bt = build_paged(kc, vc, 16, seed)
    return q, kn, vn, kpool, vpool, bt, np.asarray(pos, np.int32)


def _run(fn, inp, nq, nkv, d):
    q, kn, vn, kpool, vpool, bt, pos = inp
    kp, vp = to_dev_bf16(kpool, torch), to_dev_bf16(vpool, torch)  # fresh pools: the call appends to them
    out = torch.zeros((q.shape[0], nq, d), dtype=torch.bfloat16, device="cuda")
    fn(to_dev_bf16(q, torch), to_dev_bf16(kn, torch), to_dev_bf16(vn, torch), kp, vp, torch.from_numpy(bt).cuda(),
       torch.from_numpy(pos).cuda(), nq, nkv, d, 1.0 / math.sqrt(d), 1, 10000.0, out)
    torch.cuda.synchronize()
    return bits_to_f64(from_dev_bf16(out)), from_dev_bf16(kp), from_dev_bf16(vp)


@pytest.mark.parametrize("B,nq,nkv,d,pos", [
    (3, 8, 2, 128, [0, 17, 300]),        # splits > 1: partials and merge counters in the fixed array
    (2, 9, 3, 64, [40, 1000]),
    (1, 32, 8, 128, [4095]),             # the 8B decode shape at context 4096
    (64, 32, 8, 128, [511] * 64),        # the sweep shape: one split per CTA
])
def test_matches_allocating_entry_point_twice_in_a_row(B, nq, nkv, d, pos):
    inp = _inputs(B, nq, nkv, d, pos, seed=21)
    ref, kref, vref = _run(dec.gqa_decode_attn, inp, nq, nkv, d)
    for _ in range(2):
        got, kgot, vgot = _run(dec.gqa_decode_attn_noalloc, inp, nq, nkv, d)
        assert_parity(got, ref, what="noalloc vs gqa_decode_attn")
        # same split choice and summation order as the allocating call
        assert np.array_equal(got, ref)
        assert np.array_equal(kgot, kref) and np.array_equal(vgot, vref)


def test_refuses_shapes_beyond_the_fixed_scratch():
    B, nq, nkv, d = 4096, 8, 8, 64  # 32768 (sequence, kv head) pairs > 16384
    q = torch.zeros((B, nq, d), dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros((B, nkv, 16, d), dtype=torch.bfloat16, device="cuda")
    bt = torch.arange(B, dtype=torch.int32, device="cuda").reshape(B, 1)
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    out = torch.zeros((B, nq, d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dec.DecError) as e:
        dec.gqa_decode_attn_noalloc(q, None, None, pool, pool, bt, pos, nq, nkv, d, 0.125, 0, 1e4, out)
    assert e.value.status == "UNSUPPORTED" and "fixed scratch" in str(e.value)
