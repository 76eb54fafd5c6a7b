"""The bounded waits of the chunked-prefill kernel, made to run out.

Every wait through which one warp of the tensor-core prefill kernel consumes another's
work (K/V stage full, S full, P ready, O done, stage empty) gives up after a cycle limit,
sets PKV_DEVERR_TIMEOUT and makes every role stop; the copy warp then waits for its copies
in flight and the MMA warp for its MMAs (both with the normal one-second limit) before the
CTA frees its tensor memory and returns.  A test build of the library shortens only the
consumer limit, to one cycle, and polls those barriers without suspending, so that the
first consumer wait that is not already satisfied gives up.  The call must return, the
device error word must carry PKV_DEVERR_TIMEOUT, and the normal library must then compute
the same prefill correctly in the same process.
"""
import ctypes
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth
import paged_kv_cache_460_b200 as pkv
from paged_kv_cache_460_b200 import _lib
from paged_kv_cache_460_b200 import build as pkv_build
from tests.gpu_cases import to_bits, to_dev, tolerance_report

pytestmark = pytest.mark.gpu

SHORT_WAIT_DEFINES = ["PKV_CONSUMER_WAIT_LIMIT_CYCLES=1LL", "PKV_CONSUMER_WAIT_POLL=1"]


@pytest.fixture(scope="module")
def short_wait_lib(tmp_path_factory):
    path = os.environ.get("PKV_SHORTWAIT_LIB", "")      # a build made beforehand with the same defines
    if not os.path.exists(path):
        path = str(tmp_path_factory.mktemp("shortwait") / "libpagedkv_shortwait.so")
        pkv_build.build(out=path, defines=SHORT_WAIT_DEFINES)
    h = ctypes.CDLL(path)                       # its own symbols, kernels and error word
    for name in ("kv_get_device_error", "kv_pool_create", "kv_pool_destroy", "paged_prefill_attention"):
        res, args = _lib.SIGNATURES[name]
        fn = getattr(h, name)
        fn.restype = res
        fn.argtypes = args
    return h


def _case():
    d, P, Hq, Hkv, dtype, cached, chunk = 128, 16, 8, 2, "f16", [30, 100, 0], [40, 17, 64]
    L = [c + n for c, n in zip(cached, chunk)]
    s = synth.random_spec(1300, len(L), Hq, Hkv, d, P, [x - 1 for x in L], dtype=dtype)
    kp, vp = synth.pool_values_numpy(s)
    r = np.random.Generator(np.random.PCG64(1301))
    q = synth.round_f32(r.standard_normal((sum(chunk), Hq, d), dtype=np.float32), dtype)
    cu_q = np.concatenate([[0], np.cumsum(chunk)]).astype(np.int32)
    return s, kp, vp, q, cu_q, np.array(L, np.int32)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def test_consumer_wait_runs_out_and_the_kernel_returns(short_wait_lib):
    s, kp, vp, q, cu_q, ctx = _case()
    kp_t, vp_t = to_dev(kp, s.dtype), to_dev(vp, s.dtype)
    q_t = to_dev(q, s.dtype)
    cu_t = torch.from_numpy(cu_q).cuda()
    bt_t = torch.from_numpy(s.block_tables).cuda()
    cl_t = torch.from_numpy(ctx).cuda()
    scale = 1.0 / math.sqrt(s.head_dim)
    T = short_wait_lib
    err = ctypes.c_uint32()
    assert T.kv_get_device_error(ctypes.byref(err)) == 0          # start from a clear word
    h = ctypes.c_void_p()
    assert T.kv_pool_create(1, s.num_pages, s.page_size, s.kv_heads, s.head_dim, pkv.PKV_F16, _ptr(kp_t), _ptr(vp_t),
                            ctypes.byref(h)) == 0
    out = torch.full_like(q_t, float("nan"))
    st = T.paged_prefill_attention(h, 0, _ptr(out), _ptr(q_t), _ptr(cu_t), q_t.shape[0], _ptr(bt_t), s.max_pages,
                                   _ptr(cl_t), s.batch, s.q_heads, s.kv_heads, ctypes.c_float(scale),
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, _lib.status_string(st)
    assert T.kv_get_device_error(ctypes.byref(err)) == 0          # synchronises: the kernel has returned
    assert err.value & pkv.PKV_DEVERR_TIMEOUT
    T.kv_pool_destroy(h)

    # the normal library, same process, same inputs: correct, and its error word clear
    pkv.kv_get_device_error()
    pool = pkv.KVPool(kp_t, vp_t)
    out2 = torch.full_like(q_t, float("nan"))
    pkv.paged_prefill_attention(pool, 0, out2, q_t, cu_t, bt_t, cl_t, scale)
    ref = oracle.prefill_attention(q, kp[0], vp[0], s.block_tables, cu_q, ctx, scale, s.dtype)
    ok, maxerr, ratio = tolerance_report(to_bits(out2), ref, s.dtype)
    assert ok, "max |err| %.3g (%.3g of the bound)" % (maxerr, ratio)
    assert pkv.kv_get_device_error() == 0
