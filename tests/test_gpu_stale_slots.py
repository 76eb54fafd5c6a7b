"""Slots no sequence covers may hold anything: a page's rows past its sequence's length, and
pages no table names.  The attention kernels must not let them reach the output -- their
softmax weights are zero, but 0 * NaN is NaN in a product or an MMA.  Every uncovered slot
of the pools is set to NaN here (int8 pages: NaN row scales and codes of 127), and each
path is compared with the fp64 oracle, which reads covered slots only.
Bar: |gpu - ref| <= 1e-3 + 1e-2 |ref|, no NaN anywhere in the output."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
import paged_kv_cache_460_b200 as pkv
from tests.gpu_cases import Case, to_bits, to_dev, tolerance_report

pytestmark = pytest.mark.gpu

NAN16 = {"f16": 0x7E00, "bf16": 0x7FC0}


@pytest.fixture(autouse=True)
def _clean_error_word():
    pkv.kv_get_device_error()
    yield


def _uncovered(block_tables, lens, num_pages, page_size):
    """Boolean [pages, P]: True where no sequence's first lens[b] tokens live."""
    covered = np.zeros((num_pages, page_size), bool)
    for b, n in enumerate(lens):
        for t in range(int(n)):
            covered[block_tables[b][t // page_size], t % page_size] = True
    return ~covered


def _slots_view(pool):
    """[layers, pages, Hkv, P, ...] -> a view [layers, pages, P, Hkv, ...] for (page, slot) masks."""
    axes = list(range(pool.ndim))
    axes[2], axes[3] = 3, 2
    return pool.transpose(axes)


def _poison16(kp, vp, mask, dtype):
    """NaN into every uncovered (page, slot) of every layer and head (uint16 pools, in place)."""
    _slots_view(kp)[:, mask] = NAN16[dtype]
    _slots_view(vp)[:, mask] = NAN16[dtype]


def _check(out_bits, ref, dtype, what):
    ok, maxerr, ratio = tolerance_report(out_bits, ref, dtype)
    assert ok, "%s: max |err| %.3g, err/bound %.3g" % (what, maxerr, ratio)
    assert pkv.kv_get_device_error() == 0


DECODE = [
    # d, P, Hq, Hkv, dtype, cached lengths (-1 = padded row)
    (128, 16, 8, 8, "f16", [0, 14, 15, 16, 47, 300, -1, 1000]),
    (64, 32, 4, 4, "bf16", [30, 31, 32, 33, 1]),
    (128, 32, 8, 2, "bf16", [5, 63, 64, 200]),
    (128, 16, 16, 2, "f16", [100, 15, 2, 900]),
]


def _poisoned_case(d, P, Hq, Hkv, dtype, cached, seed):
    s = synth.random_spec(seed, len(cached), Hq, Hkv, d, P, cached, dtype=dtype)
    c = Case(s)
    mask = _uncovered(s.block_tables, s.context_lens, c.kp.shape[1], P)
    _poison16(c.kp, c.vp, mask, dtype)
    c.kp_t.copy_(to_dev(c.kp, dtype))
    c.vp_t.copy_(to_dev(c.vp, dtype))
    return s, c


@pytest.mark.parametrize("d,P,Hq,Hkv,dtype,cached", DECODE)
def test_decode_ignores_uncovered_slots(d, P, Hq, Hkv, dtype, cached):
    s, c = _poisoned_case(d, P, Hq, Hkv, dtype, cached, 2100 + d + P + Hq)
    out = c.gpu_layer(0)
    _check(to_bits(out), c.oracle_layer(0), dtype, "decode")
    assert (to_bits(out)[s.context_lens == 0] == 0).all()


@pytest.mark.parametrize("d,P,Hq,Hkv,dtype,cached", [x for x in DECODE if x[2] == x[3]])
def test_fused_layer_ignores_uncovered_slots(d, P, Hq, Hkv, dtype, cached):
    s, c = _poisoned_case(d, P, Hq, Hkv, dtype, cached, 2200 + d + P + Hq)
    q_t, k_t, v_t = (to_dev(x[0], dtype) for x in (c.q, c.k, c.v))
    rope = pkv.rope_table(c.cl_t, d, s.theta)
    out = torch.full_like(q_t, float("nan"))
    pkv.paged_decode_layer(c.pool, 0, out, q_t, k_t, v_t, rope, c.bt_t, c.cl_t, c.scale)
    _check(to_bits(out), c.oracle_layer(0), dtype, "fused layer")


@pytest.mark.parametrize("d,P,Hq,Hkv,dtype,cached", DECODE)
def test_int8_decode_ignores_uncovered_slots(d, P, Hq, Hkv, dtype, cached):
    from tests.test_gpu_int8 import I8Case
    s = synth.random_spec(2300 + d + P + Hq, len(cached), Hq, Hkv, d, P, cached, dtype=dtype)
    c = I8Case(s)
    mask = _uncovered(s.block_tables, s.context_lens, c.kc.shape[1], P)
    for codes, scales in ((c.kc, c.ks), (c.vc, c.vs)):
        _slots_view(codes)[:, mask] = 127
        _slots_view(scales)[:, mask] = np.nan
    for dst, src in zip(c.t, (c.kc, c.vc, c.ks, c.vs)):
        dst.copy_(torch.from_numpy(src).cuda())
    out = c.gpu_layer(0)
    _check(to_bits(out), c.oracle_layer(0), dtype, "int8 decode")


PREFILL = [
    # d, P, Hq, Hkv, dtype, cached tokens before the chunk, chunk lengths
    (128, 16, 8, 8, "f16", [0, 30, 100], [17, 1, 40]),
    (128, 32, 8, 2, "bf16", [5, 0, 64, 200], [16, 33, 15, 3]),
    (64, 16, 4, 4, "bf16", [0, 7], [64, 1]),
    (64, 32, 8, 1, "f16", [31, 90], [2, 70]),
]


@pytest.mark.parametrize("d,P,Hq,Hkv,dtype,cached,chunk", PREFILL)
def test_prefill_ignores_uncovered_slots(d, P, Hq, Hkv, dtype, cached, chunk):
    L = [a + n for a, n in zip(cached, chunk)]
    s = synth.random_spec(2400 + d + P + Hq, len(L), Hq, Hkv, d, P, [x - 1 for x in L], dtype=dtype)
    kp, vp = synth.pool_values_numpy(s)
    _poison16(kp, vp, _uncovered(s.block_tables, np.array(L), kp.shape[1], P), dtype)
    r = np.random.Generator(np.random.PCG64(2401 + sum(L)))
    total = sum(chunk)
    q = synth.round_f32(r.standard_normal((total, Hq, d), dtype=np.float32), dtype)
    # the chunk's rows are already in the pool (covered): attention alone is under test
    cu_q = np.concatenate([[0], np.cumsum(chunk)]).astype(np.int32)
    ctx = np.array(L, np.int32)
    scale = 1.0 / math.sqrt(d)
    pool = pkv.KVPool(to_dev(kp, dtype), to_dev(vp, dtype))
    q_t = to_dev(q, dtype)
    out = torch.full_like(q_t, float("nan"))
    pkv.paged_prefill_attention(pool, 0, out, q_t, torch.from_numpy(cu_q).cuda(),
                                torch.from_numpy(s.block_tables).cuda(), torch.from_numpy(ctx).cuda(), scale)
    ref = oracle.prefill_attention(q, kp[0], vp[0], s.block_tables, cu_q, ctx, scale, dtype)
    _check(to_bits(out), ref, dtype, "prefill")
