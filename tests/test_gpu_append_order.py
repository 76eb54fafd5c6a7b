"""Appends of several tokens per sequence, directly followed by decode attention on the
same stream with no host synchronisation in between.

The decode kernels read cached pages before they wait on the kernel ahead of them, so
a call that appends must not let them start until its rows are written.  These tests
append three tokens per sequence -- crossing page boundaries, so that pages other than
each sequence's last one are written -- and check the attention that follows against
the fp64 oracle applied to the appended cache ("为什么要自己动手写一个LLM推理引擎"
(wzjinhao.cn/news/61427) s4.3: the new k, v join the cache, then attention reads it).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
import paged_kv_cache_460_b200 as pkv
from tests.gpu_cases import TDT, to_bits, to_dev, tolerance_report

pytestmark = pytest.mark.gpu

NEW = 3        # tokens appended per sequence


def _setup(seed, before, Hq, Hkv, d, P, dtype):
    """Sequences holding `before[b]` tokens get NEW more; the spec's tables cover the result."""
    before = np.asarray(before, np.int32)
    s = synth.random_spec(seed, len(before), Hq, Hkv, d, P, before + NEW - 1, dtype=dtype)
    r = np.random.Generator(np.random.PCG64(seed + 1))
    n = s.batch * NEW
    k = synth.round_f32(r.standard_normal((n, Hkv, d), dtype=np.float32), dtype)
    v = synth.round_f32(r.standard_normal((n, Hkv, d), dtype=np.float32), dtype)
    q = synth.round_f32(r.standard_normal((s.batch, Hq, d), dtype=np.float32), dtype)
    tok_seq = np.repeat(np.arange(s.batch), NEW)
    tok_pos = (before[tok_seq] + np.tile(np.arange(NEW), s.batch)).astype(np.int32)
    tok_tables = s.block_tables[tok_seq]
    return s, q, k, v, tok_pos, tok_tables


def _boundary_mix(P):
    # before + NEW crosses a page boundary for most rows; some start a fresh page
    return [P - 2, P - 1, P, 2 * P - 1, 3 * P - 2, 1, 0, 5 * P + 14, 40 * P - 1, 7 * P + 15, 100 * P + P - 2,
            2 * P - 2] * 6


@pytest.mark.parametrize("how", ["paged_kv_append", "rope_append"])
@pytest.mark.parametrize("d,P,Hq,Hkv,dtype", [(128, 16, 8, 8, "f16"), (128, 32, 32, 8, "bf16"),
                                               (64, 16, 4, 1, "f16")])
def test_multi_token_append_then_decode_without_sync(how, d, P, Hq, Hkv, dtype):
    s, q, k, v, tok_pos, tok_tables = _setup(700 + d + P + Hq, _boundary_mix(P), Hq, Hkv, d, P, dtype)
    kp, vp = synth.pool_values_numpy(s)
    kp_t, vp_t = to_dev(kp, dtype), to_dev(vp, dtype)
    pool = pkv.KVPool(kp_t, vp_t)
    slots = pkv.pkv_slot_mapping(tok_tables, tok_pos, P)
    slots_t = torch.from_numpy(slots).cuda()
    k_t, v_t, q_t = to_dev(k, dtype), to_dev(v, dtype), to_dev(q, dtype)
    bt_t = torch.from_numpy(s.block_tables).cuda()
    cl_t = torch.from_numpy(s.context_lens).cuda()
    scale = 1.0 / math.sqrt(d)
    ws = pkv.DecodeWorkspace(s.batch, Hq, Hkv, d, P, q_t.dtype)
    out = torch.full_like(q_t, float("nan"))
    torch.cuda.synchronize()
    if how == "paged_kv_append":
        pkv.paged_kv_append(pool, 0, k_t, v_t, slots_t)
        k_in = k
    else:
        # rope_append turns k (and a throwaway q) at each token's position before appending
        q_dummy = torch.zeros((k_t.shape[0], Hq, d), dtype=q_t.dtype, device="cuda")
        pkv.rope_append(pool, 0, q_dummy, k_t, v_t, torch.from_numpy(tok_pos).cuda(), slots_t, s.theta)
        k_in, _ = oracle.rope(k, tok_pos, s.theta, dtype)
    pkv.paged_decode_attention(pool, 0, out, q_t, bt_t, cl_t, scale, workspace=ws)
    torch.cuda.synchronize()
    kp2, vp2 = oracle.kv_append(kp[0], vp[0], k_in, v, tok_tables, tok_pos)
    assert np.array_equal(to_bits(kp_t[0]), kp2) and np.array_equal(to_bits(vp_t[0]), vp2)
    ref = oracle.decode_attention(q, kp2, vp2, s.block_tables, s.context_lens, scale, dtype)
    ok, maxerr, ratio = tolerance_report(to_bits(out), ref, dtype)
    assert ok, "%s: max |err| %.3g (%.3g of the bound)" % (how, maxerr, ratio)
    assert pkv.kv_get_device_error() == 0


STEP_SHAPES = [
    # d, P, Hq, Hkv, dtype, cached lengths (-1 = padded row), int8 pages
    (128, 16, 32, 32, "f16", [0, 14, 15, 16, 47, 300, -1, 1000], False),
    (128, 32, 32, 8, "bf16", [30, 31, 32, 33, 500, 1, 0, 95], False),
    (64, 16, 4, 4, "f16", [40, 15, 16, 17, 63, 64, 65, 800], True),
    (128, 32, 32, 8, "bf16", [255, 256, 257, 511, -1], True),
]


@pytest.mark.parametrize("d,P,Hq,Hkv,dtype,cached,i8", STEP_SHAPES)
def test_rope_append_step_is_rope_append_with_positions_from_the_lengths(d, P, Hq, Hkv, dtype, cached, i8):
    """rope_append_step (position context_lens[b] - 1, slot from the page table) gives the
    bits of rope_append with the host's positions and slot mapping: turned q and k, pool
    pages (int8 pools: codes and row scales); then decode attention, issued right after it
    with no synchronisation, matches the oracle."""
    s = synth.random_spec(760 + d + P + Hq, len(cached), Hq, Hkv, d, P, cached, dtype=dtype)
    q, k, v = synth.step_values(s)
    bt_t = torch.from_numpy(s.block_tables).cuda()
    cl_t = torch.from_numpy(s.context_lens).cuda()
    pos_t = torch.from_numpy(s.positions).cuda()
    slots_t = torch.from_numpy(pkv.pkv_slot_mapping(s.block_tables, s.positions, P)).cuda()
    tdt = TDT[dtype]
    if i8:
        pools_np = synth.pool_values_i8_numpy(s)
        sets = [[torch.from_numpy(x).cuda() for x in pools_np] for _ in range(2)]
        pools = [pkv.KVPool(*t, dtype=tdt) for t in sets]
    else:
        kp, vp = synth.pool_values_numpy(s)
        sets = [[to_dev(kp, dtype), to_dev(vp, dtype)] for _ in range(2)]
        pools = [pkv.KVPool(*t) for t in sets]
    qs = [to_dev(q[0], dtype) for _ in range(2)]
    ks = [to_dev(k[0], dtype) for _ in range(2)]
    v_t = to_dev(v[0], dtype)
    out = torch.full_like(qs[1], float("nan"))
    pkv.rope_append(pools[0], 0, qs[0], ks[0], v_t, pos_t, slots_t, s.theta)
    torch.cuda.synchronize()
    pkv.rope_append_step(pools[1], 0, qs[1], ks[1], v_t, bt_t, cl_t, s.theta)
    pkv.paged_decode_attention(pools[1], 0, out, qs[1], bt_t, cl_t, 1.0 / math.sqrt(d))
    torch.cuda.synchronize()
    assert torch.equal(qs[0].view(torch.int16), qs[1].view(torch.int16))
    assert torch.equal(ks[0].view(torch.int16), ks[1].view(torch.int16))
    for a, b in zip(sets[0], sets[1]):
        assert torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8))
    assert pkv.kv_get_device_error() == 0
    q_rot, _ = oracle.rope(q[0], s.positions, s.theta, dtype)
    k_rot, _ = oracle.rope(k[0], s.positions, s.theta, dtype)
    scale = 1.0 / math.sqrt(d)
    if i8:
        kc, vc, ksc, vsc = oracle.kv_append_i8(*(x[0] for x in pools_np), k_rot, v[0], s.block_tables, s.positions,
                                               dtype)
        pairs = [(b, h) for b in range(s.batch) for h in range(Hq)]
        ref = oracle.decode_attention_i8_pairs(q_rot, kc, vc, ksc, vsc, s.block_tables, s.context_lens, scale,
                                               dtype, pairs).reshape(s.batch, Hq, d)
    else:
        kp2, vp2 = oracle.kv_append(kp[0], vp[0], k_rot, v[0], s.block_tables, s.positions)
        ref = oracle.decode_attention(q_rot, kp2, vp2, s.block_tables, s.context_lens, scale, dtype)
    ok, maxerr, ratio = tolerance_report(to_bits(out), ref, dtype)
    assert ok, "max |err| %.3g (%.3g of the bound)" % (maxerr, ratio)


def test_rope_append_step_skips_and_flags_a_bad_table_entry():
    s = synth.random_spec(790, 3, 8, 8, 128, 16, [20, 40, 7], dtype="f16")
    bt = s.block_tables.copy()
    bt[1, 40 // 16] = s.num_pages + 5          # the page of sequence 1's new token: out of range
    kp, vp = synth.pool_values_numpy(s)
    kp_t, vp_t = to_dev(kp, "f16"), to_dev(vp, "f16")
    pool = pkv.KVPool(kp_t, vp_t)
    q, k, v = synth.step_values(s)
    pkv.kv_get_device_error()
    pkv.rope_append_step(pool, 0, to_dev(q[0], "f16"), to_dev(k[0], "f16"), to_dev(v[0], "f16"),
                         torch.from_numpy(bt).cuda(), torch.from_numpy(s.context_lens).cuda(), s.theta)
    assert pkv.kv_get_device_error() == pkv.PKV_DEVERR_BAD_PAGE
    k_rot, _ = oracle.rope(k[0], s.positions, s.theta, "f16")
    keep = np.array([0, 2])
    kp2, vp2 = oracle.kv_append(kp[0], vp[0], k_rot[keep], v[0][keep], s.block_tables[keep], s.positions[keep])
    assert np.array_equal(to_bits(kp_t[0]), kp2) and np.array_equal(to_bits(vp_t[0]), vp2)
