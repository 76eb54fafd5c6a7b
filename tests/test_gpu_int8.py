"""int8 KV pages on the GPU against the fp64 oracle.

Bars: the quantising append is bit-exact (codes and the per-row fp32 scales; the
quantiser's decisions are fp32 on both sides); attention over the dequantised cache is
within |gpu - ref| <= 1e-3 + 1e-2 |ref| of the oracle, which dequantises in fp64.
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


@pytest.fixture(autouse=True)
def _clean_error_word():
    pkv.kv_get_device_error()
    yield


class I8Case:
    """Device state of one workload on an int8 pool."""

    def __init__(self, s, backend="numpy"):
        self.s = s
        self.q, self.k, self.v = synth.step_values(s)
        if backend == "numpy":
            self.kc, self.vc, self.ks, self.vs = synth.pool_values_i8_numpy(s)
            self.t = [torch.from_numpy(x).cuda() for x in (self.kc, self.vc, self.ks, self.vs)]
        else:
            self.kc = self.vc = self.ks = self.vs = None
            self.t = list(synth.pool_values_i8_torch(s, "cuda"))
        self.pool = pkv.KVPool(self.t[0], self.t[1], self.t[2], self.t[3], dtype=TDT[s.dtype])
        self.bt_t = torch.from_numpy(s.block_tables).cuda()
        self.cl_t = torch.from_numpy(s.context_lens).cuda()
        self.pos_t = torch.from_numpy(s.positions).cuda()
        self.slots_t = torch.from_numpy(pkv.pkv_slot_mapping(s.block_tables, s.positions, s.page_size)).cuda()
        self.scale = 1.0 / math.sqrt(s.head_dim)

    def gpu_layer(self, layer, fused=True, num_splits=0, workspace=None, v_override=None):
        s = self.s
        q_t = to_dev(self.q[layer], s.dtype)
        k_t = to_dev(self.k[layer], s.dtype)
        v_t = to_dev(self.v[layer] if v_override is None else v_override, s.dtype)
        if fused:
            pkv.rope_append(self.pool, layer, q_t, k_t, v_t, self.pos_t, self.slots_t, s.theta)
        else:
            pkv.rope_apply(q_t, k_t, self.pos_t, s.theta)
            pkv.paged_kv_append(self.pool, layer, k_t, v_t, self.slots_t)
        out = torch.full_like(q_t, float("nan"))
        pkv.paged_decode_attention(self.pool, layer, out, q_t, self.bt_t, self.cl_t, self.scale,
                                   num_splits=num_splits, workspace=workspace)
        return out

    def oracle_append(self, layer, v=None):
        s = self.s
        k_rot, _ = oracle.rope(self.k[layer], s.positions, s.theta, s.dtype)
        v = self.v[layer] if v is None else v
        return oracle.kv_append_i8(self.kc[layer], self.vc[layer], self.ks[layer], self.vs[layer], k_rot, v,
                                   s.block_tables, s.positions, s.dtype)

    def oracle_layer(self, layer, v=None):
        s = self.s
        q_rot, _ = oracle.rope(self.q[layer], s.positions, s.theta, s.dtype)
        kc, vc, ks, vs = self.oracle_append(layer, v)
        pairs = [(b, h) for b in range(s.batch) for h in range(s.q_heads)]
        out = oracle.decode_attention_i8_pairs(q_rot, kc, vc, ks, vs, s.block_tables, s.context_lens, self.scale,
                                               s.dtype, pairs)
        return out.reshape(s.batch, s.q_heads, s.head_dim)


def _expect_close(gpu, ref, dtype, what):
    ok, maxerr, ratio = tolerance_report(to_bits(gpu) if torch.is_tensor(gpu) else gpu, ref, dtype)
    assert ok, "%s: max |err| %.3g, max err/bound %.3g" % (what, maxerr, ratio)


SHAPES = [
    # d, P, Hq, Hkv, dtype, cached lengths (-1 = padded row)
    (128, 16, 8, 8, "f16", [0, 14, 15, 16, 47, 300, -1, 1000]),
    (128, 32, 8, 2, "bf16", [30, 31, 32, 33, 500, 1, 0, 95]),
    (64, 16, 4, 4, "f16", [40, 15, 16, 17, 63, 64, 65, 800]),
    (64, 32, 8, 1, "bf16", [31, 32, 33, 200, 64, 5]),
    (128, 16, 16, 2, "f16", [100, 15, 2, 900]),
    (128, 32, 32, 8, "bf16", [255, 256, 257, 511]),
    (64, 16, 2, 1, "f16", [3, 700]),
    (128, 16, 32, 32, "bf16", [129, 2047]),
]


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("d,P,Hq,Hkv,dtype,cached", SHAPES[:4])
def test_int8_append_is_bit_exact(d, P, Hq, Hkv, dtype, cached, fused):
    s = synth.random_spec(500 + d + P + Hq, len(cached), Hq, Hkv, d, P, cached, dtype=dtype)
    c = I8Case(s)
    v = c.v[0].copy()
    v[0, 0, :] = 0                 # an all-zero row: scale 0, codes 0
    c.gpu_layer(0, fused=fused, v_override=v)
    kc, vc, ks, vs = c.oracle_append(0, v)
    assert np.array_equal(c.t[0][0].cpu().numpy(), kc)
    assert np.array_equal(c.t[1][0].cpu().numpy(), vc)
    assert np.array_equal(c.t[2][0].cpu().numpy().view(np.uint32), ks.view(np.uint32))
    assert np.array_equal(c.t[3][0].cpu().numpy().view(np.uint32), vs.view(np.uint32))
    assert pkv.kv_get_device_error() == 0


@pytest.mark.parametrize("d,P,Hq,Hkv,dtype,cached", SHAPES)
def test_int8_step_matches_oracle_on_random_shapes(d, P, Hq, Hkv, dtype, cached):
    s = synth.random_spec(600 + d + P + Hq, len(cached), Hq, Hkv, d, P, cached, dtype=dtype)
    c = I8Case(s)
    out = c.gpu_layer(0)
    _expect_close(out, c.oracle_layer(0), dtype, "int8 shape %s" % ((d, P, Hq, Hkv, dtype),))
    assert (to_bits(out)[s.context_lens == 0] == 0).all()
    assert pkv.kv_get_device_error() == 0


@pytest.mark.parametrize("name", ["tiny", "layer7b"])
def test_int8_step_matches_oracle_on_workload(name):
    c = I8Case(synth.spec(name))
    _expect_close(c.gpu_layer(0), c.oracle_layer(0), c.s.dtype, "int8 " + name)
    assert pkv.kv_get_device_error() == 0


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_int8_row_scales_spanning_many_binades(dtype):
    """Row scales drawn log-uniformly over 2^-10 .. 2^2 (and a few all-zero V rows), so that
    the largest V scale of consecutive 16-token units changes binade all the time.  (The
    kernel keeps each unit's P * s_V in fp16 relative to the unit's largest V scale: rows
    more than 2^14 below it lose relative precision; 12 binades stay inside that range.)"""
    s = synth.random_spec(650, 4, 16, 4, 128, 16, [700, 33, 129, 2047], dtype=dtype)
    c = I8Case(s)
    r = np.random.Generator(np.random.PCG64(651))
    for arr, t in ((c.ks, c.t[2]), (c.vs, c.t[3])):
        arr[...] = (2.0 ** r.uniform(-10, 2, size=arr.shape) / 127.0).astype(np.float32)
        t.copy_(torch.from_numpy(arr))
    zero = r.random(c.vs.shape) < 0.02
    c.vs[zero] = 0
    c.t[3].copy_(torch.from_numpy(c.vs))
    _expect_close(c.gpu_layer(0), c.oracle_layer(0), dtype, "int8 wide scales")
    assert pkv.kv_get_device_error() == 0


@pytest.mark.parametrize("dtype,mean,mag", [("f16", 4.0, 1.0), ("bf16", 0.0, 2.0 ** 17), ("bf16", 3.0, 1.0)])
def test_int8_biased_and_large_queries(dtype, mean, mag):
    """q with a large common offset (sum_d q_d far from 0, which the K side subtracts after
    the MMA) and bf16 q beyond fp16's range (scaled by a power of two per head row)."""
    s = synth.random_spec(660, 3, 8, 2, 128, 16, [300, 47, 1500], dtype=dtype)
    c = I8Case(s)
    r = np.random.Generator(np.random.PCG64(661))
    q = (r.standard_normal(c.q.shape, dtype=np.float32) + np.float32(mean)) * np.float32(mag / 8.0)
    c.q = synth.round_f32(q, dtype)
    _expect_close(c.gpu_layer(0), c.oracle_layer(0), dtype, "int8 q mean %g mag %g" % (mean, mag))
    assert pkv.kv_get_device_error() == 0


def test_int8_split_count_sweep():
    s = synth.random_spec(700, 5, 8, 8, 128, 16, [1000, 17, 300, 0, 2000])
    ref = None
    for splits in (1, 3, 64, 148, 444, 2000):
        c = I8Case(s)
        out = c.gpu_layer(0, num_splits=splits)
        if ref is None:
            ref = c.oracle_layer(0)
        _expect_close(out, ref, s.dtype, "int8 splits=%d" % splits)
    assert pkv.kv_get_device_error() == 0


def _sample_pairs(s, n, seed):
    r = np.random.Generator(np.random.PCG64(seed))
    live = [b for b in range(s.batch) if s.context_lens[b] > 0]
    longest = int(np.argmax(s.context_lens))
    pairs = {(longest, 0), (longest, s.kv_heads - 1)}
    while len(pairs) < min(n, len(live) * s.kv_heads):
        pairs.add((int(r.choice(live)), int(r.integers(s.kv_heads))))
    return sorted(pairs)


@pytest.mark.parametrize("name,layers,check_layers",
                         [("batch10", 32, (0, 31)), ("cbatch", 1, (0,)), ("longctx", 1, (0,))])
def test_int8_full_size_workload_sampled(name, layers, check_layers):
    """The benchmark's int8 configuration at full size; sampled (sequence, kv head) pairs
    are recomputed by the oracle from page snapshots taken before any kernel runs."""
    s = synth.spec(name, num_layers=layers)
    c = I8Case(s, backend="torch")
    G = s.q_heads // s.kv_heads
    snaps = {}
    for L in check_layers:
        snaps[L] = []
        for b, g in _sample_pairs(s, 10, 900 + L):
            np_b = (int(s.context_lens[b]) + s.page_size - 1) // s.page_size
            pages = torch.from_numpy(s.block_tables[b, :np_b].astype(np.int64)).cuda()
            mini = [t[L].index_select(0, pages)[:, g:g + 1].contiguous().cpu().numpy() for t in c.t]
            snaps[L].append((b, g, mini))
    ws = pkv.DecodeWorkspace(s.batch, s.q_heads, s.kv_heads, s.head_dim, s.page_size, TDT[s.dtype],
                             storage=pkv.PKV_I8)
    outs = {}
    for L in range(layers):
        out = c.gpu_layer(L, workspace=ws)
        if L in snaps:
            outs[L] = to_bits(out)
    for L, sn in snaps.items():
        q_rot, _ = oracle.rope(c.q[L], s.positions, s.theta, s.dtype)
        k_rot, _ = oracle.rope(c.k[L], s.positions, s.theta, s.dtype)
        refs, gots = [], []
        for b, g, (kc, vc, ks, vs) in sn:
            table = np.arange(kc.shape[0], dtype=np.int32)[None, :]
            pos = np.array([s.positions[b]], np.int32)
            kc2, vc2, ks2, vs2 = oracle.kv_append_i8(kc, vc, ks, vs, k_rot[b:b + 1, g:g + 1],
                                                     c.v[L][b:b + 1, g:g + 1], table, pos, s.dtype)
            refs.append(oracle.decode_attention_i8_pairs(q_rot[b:b + 1, g * G:(g + 1) * G], kc2, vc2, ks2, vs2,
                                                         table, np.array([s.context_lens[b]], np.int32),
                                                         c.scale, s.dtype, [(0, j) for j in range(G)]))
            gots.append(outs[L][b, g * G:(g + 1) * G])
        _expect_close(np.stack(gots), np.stack(refs), s.dtype, "int8 %s layer %d" % (name, L))
    assert pkv.kv_get_device_error() == 0


@pytest.mark.parametrize("d,P,Hq,Hkv,dtype,cached", [SHAPES[0], SHAPES[1], SHAPES[3], SHAPES[4], SHAPES[7]])
def test_int8_fused_layer_matches_two_launch_path(d, P, Hq, Hkv, dtype, cached):
    """paged_decode_layer on an int8 pool: the new rows quantised in-kernel exactly as the
    append kernel does; output, codes and scales bit-identical to rope_append + attention."""
    s = synth.random_spec(1700 + d + P + Hq, len(cached), Hq, Hkv, d, P, cached, dtype=dtype)
    fused, split = I8Case(s), I8Case(s)
    ref_out = split.gpu_layer(0)
    q_t, k_t, v_t = (to_dev(x[0], s.dtype) for x in (fused.q, fused.k, fused.v))
    rope = pkv.rope_table(fused.cl_t, s.head_dim, s.theta)
    out = torch.full_like(q_t, float("nan"))
    pkv.paged_decode_layer(fused.pool, 0, out, q_t, k_t, v_t, rope, fused.bt_t, fused.cl_t, fused.scale)
    assert np.array_equal(to_bits(out), to_bits(ref_out))
    for a, b in zip(fused.t, split.t):
        assert torch.equal(a, b)
    _expect_close(out, fused.oracle_layer(0), dtype, "int8 fused %s" % ((d, P, Hq, Hkv, dtype),))
    assert pkv.kv_get_device_error() == 0
