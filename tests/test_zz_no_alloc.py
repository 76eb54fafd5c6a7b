"""paged_decode_attention_noalloc: decode attention for callers that cannot allocate.

Some callers cannot obtain device memory themselves -- a plugin whose host program
owns every allocation, a runtime whose caching allocator already holds the whole
GPU, a serving loop that must not call cudaMalloc because it synchronises the
device.  For them the library keeps its scratch in one fixed 4 MiB device array.
These tests call that entry point through the C ABI and hold it to the result of
the ordinary entry point (which takes a caller workspace) and to the oracle, on
calls in a row that share the array, with split counts that rise from call to call.

The file is named so that pytest collects it last: if one of its tests fails, a run
that stops at the first failure has already run every other test, and when the whole
suite runs, the shared array has already seen the other tests' calls.  Each test also
passes on its own in a fresh process.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import synth
import paged_kv_cache_460_b200 as pkv
from paged_kv_cache_460_b200 import _lib
from tests.gpu_cases import Case, TDT, to_bits, tolerance_report


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_rejects_scratch_beyond_its_limit():
    """A split count whose scratch would not fit in the fixed array is refused before
    any device work (no GPU needed for this check)."""
    L = _lib.lib()
    h = ctypes.c_void_p()
    fake = ctypes.c_void_p(0x10000)
    assert L.kv_pool_create(1, 8, 16, 8, 128, 0, fake, fake, ctypes.byref(h)) == 0
    # 16 KiB of counters + 2 x 4000 partitions x 8 heads x 130 fp32 values is far above 4 MiB
    st = L.paged_decode_attention_noalloc(h, 0, fake, fake, fake, 4, fake, 1, 64, 8, 0.1, 4000, None)
    assert st == _lib.PKV_ERR_NO_SPACE
    L.kv_pool_destroy(h)


def _case(seed, cached, Hq, Hkv, d, P, dtype):
    s = synth.random_spec(seed, len(cached), Hq, Hkv, d, P, cached, dtype=dtype)
    kp, vp = synth.pool_values_numpy(s)
    q, _, _ = synth.step_values(s)
    tdt = torch.float16 if dtype == "f16" else torch.bfloat16

    def dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy()).view(tdt).cuda()

    kp_t, vp_t = dev(kp), dev(vp)
    return dict(s=s, pool=pkv.KVPool(kp_t, vp_t), keep=(kp_t, vp_t), q=dev(q[0]),
                bt=torch.from_numpy(s.block_tables).cuda(), cl=torch.from_numpy(s.context_lens).cuda(),
                scale=1.0 / math.sqrt(d))


def _with_workspace(c, num_splits=0):
    out = torch.empty_like(c["q"])
    pkv.paged_decode_attention(c["pool"], 0, out, c["q"], c["bt"], c["cl"], c["scale"], num_splits=num_splits)
    return out


def _noalloc_raw(pool, q, bt, cl, batch, q_heads, kv_heads, scale, num_splits):
    out = torch.full_like(q, float("nan"))
    st = _lib.lib().paged_decode_attention_noalloc(
        pool.handle, 0, _ptr(out), _ptr(q), _ptr(bt), bt.shape[1], _ptr(cl), batch, q_heads, kv_heads,
        ctypes.c_float(scale), num_splits, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == _lib.PKV_OK, _lib.status_string(st)
    return out


def _noalloc(c, num_splits=0):
    s = c["s"]
    return _noalloc_raw(c["pool"], c["q"], c["bt"], c["cl"], s.batch, s.q_heads, s.kv_heads, c["scale"],
                        num_splits)


def _close(a, b):
    a, b = a.double().cpu().numpy(), b.double().cpu().numpy()
    return np.all(np.abs(a - b) <= 1e-3 + 1e-2 * np.abs(b))


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    # the first call leaves its partial results in the shared array; the second,
    # a different and smaller problem, must not be affected by them
    first = _case(901, [700, 3, 1500, 0, 257, 64], 32, 8, 128, 16, "bf16")
    second = _case(902, [40, 511], 8, 8, 64, 32, "f16")
    ref1, ref2 = _with_workspace(first), _with_workspace(second)
    got1 = _noalloc(first)
    got2 = _noalloc(second)
    torch.cuda.synchronize()
    assert _close(got1, ref1)
    assert _close(got2, ref2)
    # and again on the first problem, after the second changed the array
    got1b = _noalloc(first)
    torch.cuda.synchronize()
    assert _close(got1b, ref1)
    assert pkv.kv_get_device_error() == 0


@pytest.mark.gpu
def test_noalloc_explicit_split_counts_match_workspace_entry_point():
    """Explicit split counts that fit in the array, on calls in a row, each against the
    ordinary entry point given the same split count."""
    c = _case(903, [700, 3, 1500, 0, 257, 64], 32, 8, 128, 16, "bf16")
    for ns in (148, 5, 296, 1):
        ref = _with_workspace(c, ns)
        got = _noalloc(c, ns)
        torch.cuda.synchronize()
        assert _close(got, ref), "num_splits=%d" % ns
    assert pkv.kv_get_device_error() == 0


# Split counts that rise from call to call on one scratch: with 7 partitions the first
# (sequence, kv head) is cut by CTA 0's range, so that call leaves CTA 0's partial right
# behind the counter region; the calls with 444 and then 1000 partitions use counters
# far beyond the first call's 7.
RISING = (7, 444, 1000)


def _rising_case():
    s = synth.random_spec(911, 3, 4, 4, 64, 16, [1500, 20, 900], dtype="f16")
    pages = (s.context_lens + s.page_size - 1) // s.page_size
    W = s.kv_heads * int(pages.sum())
    assert pages[0] > -(-W // RISING[0])          # CTA 0's first segment is cut
    return s


@pytest.mark.gpu
@pytest.mark.parametrize("entry", ["noalloc", "workspace"])
def test_rising_split_counts_on_one_scratch_match_the_oracle(entry):
    s = _rising_case()
    c = Case(s)
    c.gpu_layer(0, num_splits=1)       # RoPE + append once; c.last_q holds the turned q
    ref = c.oracle_layer(0)
    ws = None
    if entry == "workspace":
        ws = pkv.DecodeWorkspace(s.batch, s.q_heads, s.kv_heads, s.head_dim, s.page_size, TDT[s.dtype],
                                 max(RISING))
    for ns in RISING + RISING:
        if entry == "noalloc":
            out = _noalloc_raw(c.pool, c.last_q, c.bt_t, c.cl_t, s.batch, s.q_heads, s.kv_heads, c.scale, ns)
        else:
            out = torch.full_like(c.last_q, float("nan"))
            pkv.paged_decode_attention(c.pool, 0, out, c.last_q, c.bt_t, c.cl_t, c.scale, num_splits=ns,
                                       workspace=ws)
        ok, maxerr, ratio = tolerance_report(to_bits(out), ref, s.dtype)
        assert ok, "%s, num_splits=%d: max |err| %.3g (%.3g of the bound)" % (entry, ns, maxerr, ratio)
    if ws is not None:
        counters = ws.buffer[:4 * pkv.PKV_MAX_DECODE_SPLITS].view(torch.int32)
        assert int((counters != 0).sum().item()) == 0
    assert pkv.kv_get_device_error() == 0


@pytest.mark.gpu
def test_noalloc_on_int8_pages_matches_workspace_entry_point_and_oracle():
    """An int8 pool with eight query heads per kv head: the int8 kernel keeps its counters
    and partials in the same shared array."""
    from tests.test_gpu_int8 import I8Case
    s = synth.random_spec(921, 4, 64, 8, 128, 16, [700, 3, 1500, 257], dtype="bf16")
    c = I8Case(s)
    ref_ws = c.gpu_layer(0, fused=False, num_splits=300)     # append, then the ordinary entry point
    ref = c.oracle_layer(0)
    q_rot = torch.from_numpy(pkv_q_rot(c)).view(TDT[s.dtype]).cuda()
    for ns in (300, 0, 300):
        got = _noalloc_raw(c.pool, q_rot, c.bt_t, c.cl_t, s.batch, s.q_heads, s.kv_heads, c.scale, ns)
        torch.cuda.synchronize()
        assert _close(got, ref_ws), "num_splits=%d" % ns
        ok, maxerr, ratio = tolerance_report(to_bits(got), ref, s.dtype)
        assert ok, "num_splits=%d: max |err| %.3g (%.3g of the bound)" % (ns, maxerr, ratio)
    assert pkv.kv_get_device_error() == 0


def pkv_q_rot(c):
    """The turned q of layer 0, computed by the library's RoPE kernel on a fresh copy."""
    s = c.s
    q_t = torch.from_numpy(np.ascontiguousarray(c.q[0]).view(np.int16).copy()).view(TDT[s.dtype]).cuda()
    pkv.rope_apply(q_t, None, c.pos_t, s.theta)
    torch.cuda.synchronize()
    return q_t.cpu().view(torch.int16).numpy()
