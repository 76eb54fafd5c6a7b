"""The fused decode layer (RoPE + append + attention in one launch) on the GPU.

Bars: the output is within |gpu - ref| <= 1e-3 + 1e-2 |ref| of the fp64 oracle, the appended
rows are bit-exact, and both are bit-identical to the two-launch path (rope_append, then
paged_decode_attention), whose kernels compute the same thing in the same order.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
import paged_kv_cache_460_b200 as pkv
from paged_kv_cache_460_b200.step import DecodeStep
from tests.gpu_cases import Case, TDT, to_bits, to_dev, tolerance_report

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_error_word():
    pkv.kv_get_device_error()
    yield


def _fused_layer(c, layer, num_splits=0):
    s = c.s
    q_t, k_t, v_t = (to_dev(x[layer], s.dtype) for x in (c.q, c.k, c.v))
    rope = pkv.rope_table(c.cl_t, s.head_dim, s.theta)
    out = torch.full_like(q_t, float("nan"))
    pkv.paged_decode_layer(c.pool, layer, out, q_t, k_t, v_t, rope, c.bt_t, c.cl_t, c.scale, num_splits=num_splits)
    return out, q_t, k_t


SHAPES = [
    # d, P, H, dtype, cached lengths (-1 = padded row)
    (128, 16, 8, "f16", [0, 14, 15, 16, 47, 300, -1, 1000]),
    (128, 32, 4, "bf16", [30, 31, 32, 33, 500, 1]),
    (64, 16, 4, "f16", [40, 15, 16, 17, 63, 64, 65, 800]),
    (64, 32, 2, "bf16", [3, 700, 31]),
]


@pytest.mark.parametrize("d,P,H,dtype,cached", SHAPES)
def test_fused_layer_matches_oracle_and_two_launch_path(d, P, H, dtype, cached):
    s = synth.random_spec(1300 + d + P + H, len(cached), H, H, d, P, cached, dtype=dtype)
    fused, split = Case(s), Case(s)
    out, q_t, k_t = _fused_layer(fused, 0)
    ref_out = split.gpu_layer(0, fused=True)            # rope_append, then paged_decode_attention
    ok, maxerr, ratio = tolerance_report(to_bits(out), fused.oracle_layer(0), dtype)
    assert ok, "max |err| %.3g, err/bound %.3g" % (maxerr, ratio)
    assert np.array_equal(to_bits(out), to_bits(ref_out))
    assert np.array_equal(to_bits(fused.kp_t), to_bits(split.kp_t))
    assert np.array_equal(to_bits(fused.vp_t), to_bits(split.vp_t))
    # inputs untouched; the pool holds the turned k and the v at each new token's slot
    assert np.array_equal(to_bits(q_t), fused.q[0]) and np.array_equal(to_bits(k_t), fused.k[0])
    k_rot, _ = oracle.rope(fused.k[0], s.positions, s.theta, dtype)
    kp2, vp2 = oracle.kv_append(fused.kp[0], fused.vp[0], k_rot, fused.v[0], s.block_tables, s.positions)
    assert np.array_equal(to_bits(fused.kp_t)[0], kp2) and np.array_equal(to_bits(fused.vp_t)[0], vp2)
    assert (to_bits(out)[s.context_lens == 0] == 0).all()
    assert pkv.kv_get_device_error() == 0


def test_fused_layer_split_sweep():
    s = synth.random_spec(1400, 5, 8, 8, 128, 16, [1000, 17, 300, 0, 2000])
    ref = None
    for splits in (1, 7, 148, 444, 2000):
        c = Case(s)
        out, _, _ = _fused_layer(c, 0, num_splits=splits)
        if ref is None:
            ref = c.oracle_layer(0)
        ok, maxerr, _ = tolerance_report(to_bits(out), ref, s.dtype)
        assert ok, "splits %d: max |err| %.3g" % (splits, maxerr)
    assert pkv.kv_get_device_error() == 0


def test_fused_step_is_bit_identical_to_two_launch_step_at_full_size():
    """batch10, 32 layers, through DecodeStep: the fused step (1 + 32 launches) and the
    two-launch step (64 launches) on copies of the same pool give the same output and pool bits."""
    s = synth.spec("batch10")
    kp, vp = synth.pool_values_torch(s, "cuda")
    pools = [pkv.KVPool(kp, vp), pkv.KVPool(kp.clone(), vp.clone())]
    qs, ks, vs = synth.step_values_torch(s, 1, "cuda")
    outs = []
    for pool, fused in zip(pools, (False, True)):
        st = DecodeStep(pool, s.batch, s.q_heads, s.max_pages, theta=s.theta, fused=fused)
        st.set_metadata(s.block_tables, s.context_lens, non_blocking=False)
        st.q.copy_(qs[0])
        st.k.copy_(ks[0])
        st.v.copy_(vs[0])
        st.eager()                  # once: the two-launch path turns q and k in place
        torch.cuda.synchronize()
        outs.append(st.out.clone())
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    assert torch.equal(pools[0].k_cache.view(torch.int16), pools[1].k_cache.view(torch.int16))
    assert torch.equal(pools[0].v_cache.view(torch.int16), pools[1].v_cache.view(torch.int16))
    assert pkv.kv_get_device_error() == 0


def test_fused_layer_rejects_what_it_does_not_serve():
    s = synth.random_spec(1500, 2, 8, 2, 128, 16, [40, 3])
    c = Case(s)
    q_t, k_t, v_t = (to_dev(x[0], s.dtype) for x in (c.q, c.k, c.v))
    rope = pkv.rope_table(c.cl_t, s.head_dim, s.theta)
    with pytest.raises(pkv.PagedKVError):
        pkv.paged_decode_layer(c.pool, 0, torch.empty_like(q_t), q_t, k_t, v_t, rope, c.bt_t, c.cl_t, c.scale)


@pytest.mark.parametrize("fused,workload,layers,kv", [(True, "batch10", 6, "f16"), (False, "batch10", 3, "f16"),
                                                  (True, "cbatch", 2, "f16"), (True, "batch10", 6, "int8"),
                                                  (False, "cbatch", 2, "int8")])
def test_step_with_pinned_host_buffers_matches_copy_then_replay(fused, workload, layers, kv):
    """DecodeStep.run with pinned host buffers captures the host copies into the step's graph
    (the layers' rows copied in by chunks on their own stream, the outputs copied back as their
    kernels finish) and must give the bits of the plain path: copy everything in, replay the
    step graph, copy everything out -- output and pool, on the first run and on replays; 16-bit
    and int8 pages, the fused layer and the two-launch step."""
    s = synth.spec(workload, num_layers=layers)
    if s.q_heads != s.kv_heads and fused:
        fused = False                     # the fused layer takes one query head per kv head
    if kv == "int8":
        kc, vc, ksc, vsc = synth.pool_values_i8_torch(s, "cuda")
        tdt = torch.float16 if s.dtype == "f16" else torch.bfloat16
        pools = [pkv.KVPool(kc, vc, ksc, vsc, dtype=tdt),
                 pkv.KVPool(kc.clone(), vc.clone(), ksc.clone(), vsc.clone(), dtype=tdt)]
    else:
        kp, vp = synth.pool_values_torch(s, "cuda")
        pools = [pkv.KVPool(kp, vp), pkv.KVPool(kp.clone(), vp.clone())]
    qs, ks, vs = synth.step_values_torch(s, 2, "cuda")
    outs = []
    for pool, pinned in zip(pools, (False, True)):
        st = DecodeStep(pool, s.batch, s.q_heads, s.max_pages, theta=s.theta, fused=fused)
        st.set_metadata(s.block_tables, s.context_lens, non_blocking=False)
        host = [(x[j].cpu().pin_memory() if pinned else x[j].cpu()) for j in range(2) for x in (qs, ks, vs)]
        hout = torch.empty(st.out.shape, dtype=st.out.dtype)
        hout = hout.pin_memory() if pinned else hout
        res = []
        for it in range(3):               # set 0, set 1, set 0 again: capture, second graph, replay
            j = it % 2
            st.run(host[3 * j], host[3 * j + 1], host[3 * j + 2], hout)
            torch.cuda.synchronize()
            res.append(hout.clone())
        assert len(st.host_graphs) == (2 if pinned else 0)
        outs.append(res)
    for a, b in zip(*outs):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    for x, y in ((pools[0].k_cache, pools[1].k_cache), (pools[0].v_cache, pools[1].v_cache)):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))
    if kv == "int8":
        assert torch.equal(pools[0].k_scales, pools[1].k_scales)
        assert torch.equal(pools[0].v_scales, pools[1].v_scales)
    assert pkv.kv_get_device_error() == 0
