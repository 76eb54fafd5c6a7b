"""paged_decode_attention_noalloc: decode attention for callers that cannot allocate.

Some callers cannot obtain device memory themselves -- a plugin whose host program
owns every allocation, a runtime whose caching allocator already holds the whole
GPU, a serving loop that must not call cudaMalloc because it synchronises the
device.  For them the library keeps its scratch in one fixed 4 MiB device array.
These tests call that entry point through the C ABI and hold it to the result of
the ordinary entry point (which takes a caller workspace), on two calls in a row
that share the array.  This file is collected last on purpose.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import synth
import paged_kv_cache_460_b200 as pkv
from paged_kv_cache_460_b200 import _lib


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_rejects_scratch_beyond_its_limit():
    """A split count whose scratch would not fit in the fixed array is refused before
    any device work (no GPU needed for this check)."""
    L = _lib.lib()
    h = ctypes.c_void_p()
    fake = ctypes.c_void_p(0x10000)
    assert L.kv_pool_create(1, 8, 16, 8, 128, 0, fake, fake, ctypes.byref(h)) == 0
    # 2 x 100000 partitions x 8 heads x 130 fp32 values is far above 4 MiB
    st = L.paged_decode_attention_noalloc(h, 0, fake, fake, fake, 4, fake, 1, 64, 8, 0.1, 100000, None)
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


def _with_workspace(c):
    s = c["s"]
    out = torch.empty_like(c["q"])
    pkv.paged_decode_attention(c["pool"], 0, out, c["q"], c["bt"], c["cl"], c["scale"])
    return out


def _noalloc(c):
    s = c["s"]
    out = torch.full_like(c["q"], float("nan"))
    st = _lib.lib().paged_decode_attention_noalloc(
        c["pool"].handle, 0, _ptr(out), _ptr(c["q"]), _ptr(c["bt"]), s.max_pages, _ptr(c["cl"]), s.batch,
        s.q_heads, s.kv_heads, ctypes.c_float(c["scale"]), 0,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == _lib.PKV_OK, _lib.status_string(st)
    return out


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
