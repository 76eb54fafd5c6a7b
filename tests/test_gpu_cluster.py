"""The cluster variant of decode attention against the fp64 oracle and the partitioned kernel.

For 16-bit pools with one query head per kv head and few (sequence, kv head) pairs, a call
with num_splits = 0 runs one thread-block cluster per pair, each CTA taking an equal share of
the pair's pages, and merges the shares through distributed shared memory.  These cases
cover a long single sequence, ragged and empty sequences, a pair with fewer pages than the
cluster has CTAs, a single token, both element types, both page sizes and head dims, and the
fused layer; each output is held to the oracle ("为什么要自己动手写一个LLM推理引擎"
(wzjinhao.cn/news/61427) s4.3) and to the partitioned kernel given an explicit split count.
"""
import math

import numpy as np
import pytest
import torch

import synth
import paged_kv_cache_460_b200 as pkv
from tests.gpu_cases import Case, TDT, to_bits, to_dev, tolerance_report

pytestmark = pytest.mark.gpu

SHAPES = [
    # d, P, H (query = kv heads), dtype, cached lengths (-1 = padded row)
    (128, 16, 32, "f16", [2048]),
    (64, 32, 8, "bf16", [700, 3]),
    (128, 16, 4, "f16", [0, 15, -1, 1000, 16]),
    (128, 32, 2, "bf16", [5000, 31, 32, 33]),
    (64, 16, 16, "f16", [100, 257, 40]),
]


def _expect_close(gpu, ref, dtype, what):
    ok, maxerr, ratio = tolerance_report(to_bits(gpu), ref, dtype)
    assert ok, "%s: max |err| %.3g (%.3g of the bound)" % (what, maxerr, ratio)


@pytest.mark.parametrize("d,P,H,dtype,cached", SHAPES)
def test_cluster_variant_matches_oracle_and_partitioned_kernel(d, P, H, dtype, cached):
    s = synth.random_spec(1900 + d + P + H, len(cached), H, H, d, P, cached, dtype=dtype)
    c = Case(s)
    C = pkv.pkv_decode_cluster_size(c.pool, s.batch, s.max_pages, H)
    assert C >= 2, "the shape should take the cluster variant"
    out = c.gpu_layer(0)                      # RoPE + append, then num_splits = 0: the cluster variant
    ref = c.oracle_layer(0)
    _expect_close(out, ref, dtype, "cluster variant (C = %d)" % C)
    assert (to_bits(out)[s.context_lens == 0] == 0).all()
    part = torch.empty_like(c.last_q)
    pkv.paged_decode_attention(c.pool, 0, part, c.last_q, c.bt_t, c.cl_t, c.scale, num_splits=37)
    _expect_close(part, ref, dtype, "partitioned kernel")
    again = torch.empty_like(c.last_q)
    pkv.paged_decode_attention(c.pool, 0, again, c.last_q, c.bt_t, c.cl_t, c.scale)
    assert np.array_equal(to_bits(again), to_bits(out))          # deterministic
    assert pkv.kv_get_device_error() == 0


@pytest.mark.parametrize("d,P,H,dtype,cached", [SHAPES[0], SHAPES[2], SHAPES[3]])
def test_fused_layer_cluster_variant_matches_two_launch_path(d, P, H, dtype, cached):
    """paged_decode_layer with num_splits = 0 on these shapes runs the fused cluster variant:
    the appended pool rows are bit-identical to rope_append's, the output within tolerance of
    rope_append + the partitioned attention kernel, and of the oracle."""
    s = synth.random_spec(1950 + d + P + H, len(cached), H, H, d, P, cached, dtype=dtype)
    fused, split = Case(s), Case(s)
    ref_out = split.gpu_layer(0, num_splits=29)
    q_t, k_t, v_t = (to_dev(x[0], s.dtype) for x in (fused.q, fused.k, fused.v))
    rope = pkv.rope_table(fused.cl_t, s.head_dim, s.theta)
    out = torch.empty_like(q_t)
    pkv.paged_decode_layer(fused.pool, 0, out, q_t, k_t, v_t, rope, fused.bt_t, fused.cl_t, fused.scale)
    torch.cuda.synchronize()
    assert torch.equal(fused.kp_t.view(torch.int16), split.kp_t.view(torch.int16))
    assert torch.equal(fused.vp_t.view(torch.int16), split.vp_t.view(torch.int16))
    ok, maxerr, _ = tolerance_report(to_bits(out), split.oracle_layer(0), s.dtype)
    assert ok, "fused cluster variant: max |err| %.3g" % maxerr
    a, b = out.double().cpu().numpy(), ref_out.double().cpu().numpy()
    assert np.all(np.abs(a - b) <= 1e-3 + 1e-2 * np.abs(b))
    assert pkv.kv_get_device_error() == 0


def test_cluster_size_rule():
    """Large batches keep the partitioned kernel; a long single sequence and a few heads take
    clusters of at most eight CTAs, and never more CTAs per pair than the table has pages."""
    full = pkv.pkv_decode_default_splits(32, 32, 128, 16, pkv.PKV_F16)
    big = synth.spec("batch10", num_layers=1)
    cb = Case(synth.random_spec(1990, 10, 32, 32, 128, 16, [100] * 10))
    assert pkv.pkv_decode_cluster_size(cb.pool, 10, big.max_pages, 32) == 0        # 320 pairs
    one = Case(synth.random_spec(1991, 1, 32, 32, 128, 16, [2048]))
    assert pkv.pkv_decode_cluster_size(one.pool, 1, one.s.max_pages, 32) == min(8, full // 32, one.s.max_pages)
    tiny = Case(synth.spec("tiny"))
    assert pkv.pkv_decode_cluster_size(tiny.pool, 1, tiny.s.max_pages, 4) == min(8, tiny.s.max_pages)
    gqa = Case(synth.random_spec(1992, 1, 8, 2, 128, 16, [500]))
    assert pkv.pkv_decode_cluster_size(gqa.pool, 1, gqa.s.max_pages, 8) == 0        # grouped heads
