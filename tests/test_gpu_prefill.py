"""Chunked prefill on the GPU against the fp64 oracle: multi-token RoPE, the multi-token
KV append through the slot mapping, and the causal paged prefill attention.
Tolerance: |gpu - ref| <= 1e-3 + 1e-2 |ref| (RoPE/attention); the append bit-exact."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
import paged_kv_cache_460_b200 as pkv
from tests.gpu_cases import to_bits, to_dev, tolerance_report

pytestmark = pytest.mark.gpu

CASES = [
    # d, P, Hq, Hkv, dtype, cached tokens before the chunk, chunk lengths
    (128, 16, 8, 8, "f16", [0, 30, 100], [17, 1, 40]),
    (128, 32, 8, 2, "bf16", [5, 0, 64, 200], [16, 33, 15, 3]),
    (64, 16, 4, 4, "bf16", [0, 0], [64, 1]),
    (64, 32, 8, 1, "f16", [31, 90], [2, 70]),
    (128, 16, 16, 2, "bf16", [300], [24]),
    (128, 16, 4, 2, "f16", [47, 0, 13], [5, 0, 16]),
]


@pytest.mark.parametrize("d,P,Hq,Hkv,dtype,cached,chunk", CASES)
def test_prefill_chunk_matches_oracle(d, P, Hq, Hkv, dtype, cached, chunk):
    L = [c + n for c, n in zip(cached, chunk)]
    s = synth.random_spec(1000 + d + P + Hq, len(L), Hq, Hkv, d, P, [x - 1 for x in L], dtype=dtype)
    kp, vp = synth.pool_values_numpy(s)
    r = np.random.Generator(np.random.PCG64(1001 + sum(L)))
    total = sum(chunk)
    q = synth.round_f32(r.standard_normal((total, Hq, d), dtype=np.float32), dtype)
    k = synth.round_f32(r.standard_normal((total, Hkv, d), dtype=np.float32), dtype)
    v = synth.round_f32(r.standard_normal((total, Hkv, d), dtype=np.float32), dtype)
    cu_q = np.concatenate([[0], np.cumsum(chunk)]).astype(np.int32)
    pos = np.concatenate([np.arange(c, c + n) for c, n in zip(cached, chunk)]).astype(np.int32)
    seq = np.concatenate([np.full(n, b) for b, n in enumerate(chunk)]).astype(np.int64)
    bt_rows = s.block_tables[seq]
    slots = pkv.pkv_slot_mapping(bt_rows, pos, P)
    ctx = np.array(L, np.int32)
    scale = 1.0 / math.sqrt(d)

    kp_t, vp_t = to_dev(kp, dtype), to_dev(vp, dtype)
    pool = pkv.KVPool(kp_t, vp_t)
    q_t, k_t, v_t = to_dev(q, dtype), to_dev(k, dtype), to_dev(v, dtype)
    pkv.rope_apply(q_t, k_t, torch.from_numpy(pos).cuda(), s.theta)
    pkv.paged_kv_append(pool, 0, k_t, v_t, torch.from_numpy(slots).cuda())
    out = torch.full_like(q_t, float("nan"))
    pkv.paged_prefill_attention(pool, 0, out, q_t, torch.from_numpy(cu_q).cuda(),
                                torch.from_numpy(s.block_tables).cuda(), torch.from_numpy(ctx).cuda(), scale)

    q_rot, _ = oracle.rope(q, pos, s.theta, dtype)
    k_rot, _ = oracle.rope(k, pos, s.theta, dtype)
    kp2, vp2 = oracle.kv_append(kp[0], vp[0], k_rot, v, bt_rows, pos)
    assert np.array_equal(to_bits(kp_t)[0], kp2) and np.array_equal(to_bits(vp_t)[0], vp2)
    ref = oracle.prefill_attention(q_rot, kp2, vp2, s.block_tables, cu_q, ctx, scale, dtype)
    ok, maxerr, ratio = tolerance_report(to_bits(out), ref, dtype)
    assert ok, "max |err| %.3g, err/bound %.3g" % (maxerr, ratio)
    assert pkv.kv_get_device_error() == 0


@pytest.mark.parametrize("scale", [-0.2, 0.0])
def test_prefill_with_negative_and_zero_scale(scale):
    """A negative scale puts the softmax weight on the smallest scores; zero gives every visible
    key the same weight."""
    d, P, Hq, Hkv, dtype, cached, chunk = 128, 16, 8, 2, "bf16", [40, 3], [70, 9]
    L = [c + n for c, n in zip(cached, chunk)]
    s = synth.random_spec(1200, len(L), Hq, Hkv, d, P, [x - 1 for x in L], dtype=dtype)
    kp, vp = synth.pool_values_numpy(s)
    r = np.random.Generator(np.random.PCG64(1201))
    q = synth.round_f32(r.standard_normal((sum(chunk), Hq, d), dtype=np.float32), dtype)
    cu_q = np.concatenate([[0], np.cumsum(chunk)]).astype(np.int32)
    ctx = np.array(L, np.int32)
    pool = pkv.KVPool(to_dev(kp, dtype), to_dev(vp, dtype))
    q_t = to_dev(q, dtype)
    out = torch.full_like(q_t, float("nan"))
    pkv.paged_prefill_attention(pool, 0, out, q_t, torch.from_numpy(cu_q).cuda(),
                                torch.from_numpy(s.block_tables).cuda(), torch.from_numpy(ctx).cuda(), scale)
    ref = oracle.prefill_attention(q, kp[0], vp[0], s.block_tables, cu_q, ctx, scale, dtype)
    ok, maxerr, ratio = tolerance_report(to_bits(out), ref, dtype)
    assert ok, "scale %g: max |err| %.3g, err/bound %.3g" % (scale, maxerr, ratio)
    assert pkv.kv_get_device_error() == 0


def test_prefill_of_single_tokens_equals_decode():
    """A chunk of one token per sequence is the decode step; both kernels agree within the
    tolerance (their reduction orders differ)."""
    s = synth.random_spec(1100, 4, 8, 2, 128, 16, [700, 33, 0, 129], dtype="bf16")
    kp, vp = synth.pool_values_numpy(s)
    kp_t, vp_t = to_dev(kp, "bf16"), to_dev(vp, "bf16")
    pool = pkv.KVPool(kp_t, vp_t)
    q, _, _ = synth.step_values(s)
    q_t = to_dev(q[0], "bf16")
    bt = torch.from_numpy(s.block_tables).cuda()
    cl = torch.from_numpy(s.context_lens).cuda()
    dec = torch.empty_like(q_t)
    pkv.paged_decode_attention(pool, 0, dec, q_t, bt, cl, 0.125)
    pre = torch.empty_like(q_t)
    pkv.paged_prefill_attention(pool, 0, pre, q_t, torch.arange(5, dtype=torch.int32, device="cuda"), bt, cl, 0.125)
    ref = oracle.decode_attention(q[0], kp[0], vp[0], s.block_tables, s.context_lens, 0.125, "bf16")
    for got in (dec, pre):
        ok, maxerr, ratio = tolerance_report(to_bits(got), ref, "bf16")
        assert ok, "max |err| %.3g" % maxerr
