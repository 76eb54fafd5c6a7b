"""Parity of the CUDA path (called through the C ABI) with the fp64 oracle.

Bars: KV append bit-exact; RoPE and attention within |gpu - ref| <= 1e-3 + 1e-2 |ref|
(the tolerance the decode step is specified with); the attention output must also be
bit-identical under any permutation of physical pages and across repeated runs.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
import paged_kv_cache_460_b200 as pkv
from tests.gpu_cases import ATOL, RTOL, Case, TDT, to_bits, to_dev, tolerance_report

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_error_word():
    pkv.kv_get_device_error()
    yield


def _expect_close(gpu, ref, dtype, what):
    ok, maxerr, ratio = tolerance_report(to_bits(gpu) if torch.is_tensor(gpu) else gpu, ref, dtype)
    assert ok, "%s: max |err| %.3g, max err/bound %.3g" % (what, maxerr, ratio)


# ------------------------------------------------------------------ RoPE
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
def test_rope_matches_oracle(dtype, d):
    r = np.random.Generator(np.random.PCG64(100 + d))
    pos = np.array([0, 1, 15, 16, 17, 2048, 32768, 65535, 123456, -1, 5, 999], np.int32)
    n, hq, hk = len(pos), 8, 2
    q = synth.round_f32(r.standard_normal((n, hq, d), dtype=np.float32), dtype)
    k = synth.round_f32(r.standard_normal((n, hk, d), dtype=np.float32), dtype)
    q_t, k_t = to_dev(q, dtype), to_dev(k, dtype)
    pkv.rope_apply(q_t, k_t, torch.from_numpy(pos).cuda(), 10000.0)
    torch.cuda.synchronize()
    live = pos >= 0
    for x, xt in ((q, q_t), (k, k_t)):
        got = to_bits(xt)
        ref_bits, ref_exact = oracle.rope(x[live], pos[live], 10000.0, dtype)
        _expect_close(got[live], ref_exact, dtype, "rope")
        # one rounding of an fp64 rotation on both sides: equal bits but for rare ties
        assert (got[live] == ref_bits).mean() > 0.999
        assert np.array_equal(got[~live], x[~live])               # padded rows untouched
        assert np.array_equal(got[pos == 0], x[pos == 0])          # position 0 is the identity


# ------------------------------------------------------------------ append
@pytest.mark.parametrize("P,d,dtype", [(16, 128, "f16"), (32, 128, "bf16"), (16, 64, "f16")])
def test_append_is_bit_exact(P, d, dtype):
    s = synth.random_spec(200 + P + d, 9, 4, 4, d, P, [0, 5, P - 1, P, P + 1, 3 * P, 7 * P + 5, -1, 2])
    r = np.random.Generator(np.random.PCG64(201))
    kp = r.integers(0, 65536, (s.num_pages, 4, P, d), dtype=np.uint16)   # sentinel: random bits
    vp = r.integers(0, 65536, (s.num_pages, 4, P, d), dtype=np.uint16)
    k = r.integers(0, 65536, (9, 4, d), dtype=np.uint16)
    v = r.integers(0, 65536, (9, 4, d), dtype=np.uint16)
    kp_t, vp_t = to_dev(kp[None], dtype), to_dev(vp[None], dtype)
    pool = pkv.KVPool(kp_t, vp_t)
    slots = torch.from_numpy(pkv.pkv_slot_mapping(s.block_tables, s.positions, P)).cuda()
    pkv.paged_kv_append(pool, 0, to_dev(k, dtype), to_dev(v, dtype), slots)
    kref, vref = oracle.kv_append(kp, vp, k, v, s.block_tables, s.positions)
    assert np.array_equal(to_bits(kp_t)[0], kref)
    assert np.array_equal(to_bits(vp_t)[0], vref)
    assert pkv.kv_get_device_error() == 0


def test_append_out_of_range_slot_is_skipped_and_flagged():
    P, d = 16, 64
    kp = np.zeros((1, 4, 2, P, d), np.uint16)
    kp_t, vp_t = to_dev(kp, "f16"), to_dev(kp, "f16")
    pool = pkv.KVPool(kp_t, vp_t)
    k = to_dev(np.full((2, 2, d), 0x3C00, np.uint16), "f16")
    slots = torch.tensor([4 * P, 3], dtype=torch.int64, device="cuda")   # first is past the pool
    pkv.paged_kv_append(pool, 0, k, k, slots)
    err = pkv.kv_get_device_error()
    assert err & pkv.PKV_DEVERR_BAD_SLOT
    got = to_bits(kp_t)
    assert (got[0, 0, :, 3] == 0x3C00).all() and got.sum() == 2 * d * 0x3C00


@pytest.mark.parametrize("d,P,Hq,Hkv,dtype", [(128, 16, 8, 8, "f16"), (128, 32, 8, 2, "bf16"), (64, 16, 4, 1, "f16")])
def test_fused_rope_append_equals_separate_calls(d, P, Hq, Hkv, dtype):
    cached = [0, 5, P - 1, P, 3 * P + 2, -1, 100]
    s = synth.random_spec(250 + d + P, len(cached), Hq, Hkv, d, P, cached, dtype=dtype)
    a, b = Case(s), Case(s)
    out_a = to_bits(a.gpu_layer(0))
    out_b = to_bits(b.gpu_layer(0, fused=True))
    assert np.array_equal(to_bits(a.kp_t), to_bits(b.kp_t))
    assert np.array_equal(to_bits(a.vp_t), to_bits(b.vp_t))
    assert np.array_equal(to_bits(a.last_q), to_bits(b.last_q))
    assert np.array_equal(out_a, out_b)
    _expect_close(out_b, b.oracle_layer(0), dtype, "fused step")
    assert pkv.kv_get_device_error() == 0


# ------------------------------------------------------------------ whole step, small workloads
@pytest.mark.parametrize("name", ["tiny", "layer7b"])
def test_step_matches_oracle_on_workload(name):
    c = Case(synth.spec(name))
    out = c.gpu_layer(0)
    _expect_close(out, c.oracle_layer(0), c.s.dtype, name)
    assert pkv.kv_get_device_error() == 0


SHAPES = [
    # d, P, Hq, Hkv, dtype, cached lengths (-1 = padded row)
    (128, 16, 8, 8, "f16", [0, 14, 15, 16, 47, 300, -1, 1000]),
    (128, 32, 8, 2, "bf16", [30, 31, 32, 33, 500, 1, 0, 95]),
    (64, 16, 4, 4, "f16", [40, 15, 16, 17, 63, 64, 65, 800]),
    (64, 32, 8, 1, "bf16", [31, 32, 33, 200, 64, 5]),
    (128, 16, 16, 2, "f16", [100, 15, 2, 900]),
    (128, 16, 4, 2, "bf16", [255, 256, 257, 511]),
    (64, 16, 2, 1, "f16", [3, 700]),
]


@pytest.mark.parametrize("d,P,Hq,Hkv,dtype,cached", SHAPES)
def test_step_matches_oracle_on_random_shapes(d, P, Hq, Hkv, dtype, cached):
    s = synth.random_spec(300 + d + P + Hq, len(cached), Hq, Hkv, d, P, cached, dtype=dtype)
    c = Case(s)
    out = c.gpu_layer(0)
    ref = c.oracle_layer(0)
    _expect_close(out, ref, dtype, "shape %s" % ((d, P, Hq, Hkv, dtype),))
    assert (to_bits(out)[s.context_lens == 0] == 0).all()
    assert pkv.kv_get_device_error() == 0


def test_split_count_sweep():
    s = synth.random_spec(400, 6, 8, 8, 128, 16, [700, 3, 129, 0, 64, 333])
    c = Case(s)
    base = c.oracle_layer(0)
    outs = []
    for ns in (1, 2, 3, 7, 16, 64, 148, 296, 1000):
        c2 = Case(s)                        # fresh pools: the step appends in place
        out = c2.gpu_layer(0, num_splits=ns)
        _expect_close(out, base, "f16", "num_splits=%d" % ns)
        outs.append(to_bits(out))
    # a fixed split count is deterministic
    c3 = Case(s)
    assert np.array_equal(to_bits(c3.gpu_layer(0, num_splits=7)), outs[3])


def test_reused_workspace_gives_identical_bits():
    """The merge counters in the workspace are back at zero after every call."""
    s = synth.random_spec(450, 5, 8, 4, 128, 16, [900, 33, 0, 300, 1500], dtype="bf16")
    c = Case(s)
    c.gpu_layer(0)                               # the append has happened; now attention only
    ws = pkv.DecodeWorkspace(s.batch, s.q_heads, s.kv_heads, s.head_dim, s.page_size, TDT[s.dtype], 7)
    q = c.last_q
    outs = []
    for _ in range(3):
        out = torch.empty_like(q)
        pkv.paged_decode_attention(c.pool, 0, out, q, c.bt_t, c.cl_t, c.scale, num_splits=7, workspace=ws)
        outs.append(to_bits(out))
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[1], outs[2])
    assert (ws.buffer[:7 * 4].view(torch.int32) == 0).all().item()
    _expect_close(outs[0], c.oracle_layer(0), "bf16", "reused workspace")


def test_physical_page_permutation_gives_identical_bits():
    s = synth.random_spec(500, 4, 8, 4, 128, 16, [500, 77, 16, 1200], dtype="bf16")
    c = Case(s)
    out1 = to_bits(c.gpu_layer(0))
    # move every physical page to a new home; same logical content
    r = np.random.Generator(np.random.PCG64(501))
    perm = r.permutation(s.num_pages)
    s2 = synth.random_spec(500, 4, 8, 4, 128, 16, [500, 77, 16, 1200], dtype="bf16")
    s2.block_tables = np.where(s.block_tables >= 0, perm[np.maximum(s.block_tables, 0)], -1).astype(np.int32)
    c2 = Case(s2)
    kp2 = np.empty_like(c.kp)
    vp2 = np.empty_like(c.vp)
    kp2[:, perm] = c.kp
    vp2[:, perm] = c.vp
    c2.kp_t.copy_(to_dev(kp2, "bf16"))
    c2.vp_t.copy_(to_dev(vp2, "bf16"))
    out2 = to_bits(c2.gpu_layer(0))
    assert np.array_equal(out1, out2)


def test_single_token_context_returns_v_bits():
    # cached length 0: the step appends one token and attends to it alone
    s = synth.random_spec(600, 3, 8, 2, 128, 16, [0, 0, 0], dtype="f16")
    c = Case(s)
    out = to_bits(c.gpu_layer(0))
    v = c.v[0]                                   # [B, Hkv, d]
    for h in range(8):
        assert np.array_equal(out[:, h], v[:, h // 4])


def test_bad_page_is_flagged_not_read():
    s = synth.random_spec(700, 2, 4, 4, 64, 16, [40, 20])
    c = Case(s)
    bad = s.block_tables.copy()
    bad[0, 1] = s.num_pages + 5                  # never dereferenced: skipped and flagged
    c.bt_t = torch.from_numpy(bad).cuda()
    c.gpu_layer(0)
    assert pkv.kv_get_device_error() & pkv.PKV_DEVERR_BAD_PAGE


# ------------------------------------------------------------------ full-size workloads, sampled
def _sample_pairs(s, n, seed):
    r = np.random.Generator(np.random.PCG64(seed))
    live = np.nonzero(s.context_lens > 0)[0]
    longest, shortest = live[np.argmax(s.context_lens[live])], live[np.argmin(s.context_lens[live])]
    pairs = {(int(longest), 0), (int(shortest), s.kv_heads - 1), (int(live[0]), 0), (int(live[-1]), s.kv_heads - 1)}
    while len(pairs) < n:
        pairs.add((int(r.choice(live)), int(r.integers(0, s.kv_heads))))
    return sorted(pairs)


@pytest.mark.parametrize("name,layers,check_layers", [
    ("batch10", 32, (0, 17, 31)),
    ("cbatch", 1, (0,)),
    ("longctx", 1, (0,)),
])
def test_full_size_workload_sampled(name, layers, check_layers):
    s = synth.spec(name, num_layers=layers)
    c = Case(s, pool_backend="torch")
    G = s.q_heads // s.kv_heads
    snaps = {L: c.snapshot_pairs(L, _sample_pairs(s, 12, 800 + L)) for L in check_layers}
    ws = pkv.DecodeWorkspace(s.batch, s.q_heads, s.kv_heads, s.head_dim, s.page_size, TDT[s.dtype])
    outs = {}
    for L in range(layers):                      # the step as the benchmark runs it
        out = c.gpu_layer(L, workspace=ws, fused=True)
        if L in snaps:
            outs[L] = to_bits(out)
    for L, sn in snaps.items():
        ref = c.oracle_pairs(L, sn)
        got = np.stack([outs[L][b, g * G:(g + 1) * G] for b, g, _, _ in sn])
        _expect_close(got, ref, s.dtype, "%s layer %d" % (name, L))
    assert pkv.kv_get_device_error() == 0


# ------------------------------------------------------------------ RMSNorm
@pytest.mark.parametrize("dtype,rows,hidden,fused", [("f16", 10, 4096, False), ("bf16", 64, 4096, True),
                                                     ("f16", 3, 4104, True), ("bf16", 1, 16384, False)])
def test_rms_norm_matches_oracle(dtype, rows, hidden, fused):
    r = np.random.Generator(np.random.PCG64(900 + hidden + rows))
    x = synth.round_f32(r.standard_normal((rows, hidden), dtype=np.float32) * 3, dtype)
    w = synth.round_f32(1 + 0.1 * r.standard_normal(hidden, dtype=np.float32), dtype)
    res = synth.round_f32(r.standard_normal((rows, hidden), dtype=np.float32), dtype) if fused else None
    x_t, w_t = to_dev(x, dtype), to_dev(w, dtype)
    res_t = to_dev(res, dtype) if fused else None
    out = torch.empty_like(x_t)
    pkv.rms_norm(out, x_t, w_t, 1e-6, residual=res_t)
    ref_bits, ref_exact, ref_res = oracle.rms_norm(x, w, 1e-6, dtype, residual=res)
    _expect_close(out, ref_exact, dtype, "rms_norm")
    if fused:
        assert np.array_equal(to_bits(res_t), ref_res)        # the rounded sum is bit-exact
    assert (to_bits(out) == ref_bits).mean() > 0.99


def test_automatic_split_count_follows_the_work_bound():
    """num_splits = 0 takes a full wave of CTAs unless the work bound (kv heads x batch x units
    of the table's pages) would leave a CTA fewer than 16 units; where the cluster variant does
    not apply, the automatic call gives the bits of the explicit call with that count."""
    full = pkv.pkv_decode_default_splits(32, 32, 128, 16, pkv.PKV_F16)
    s = synth.random_spec(610, 8, 32, 32, 128, 16, [20] * 8)    # 256 short (sequence, head) pairs
    c = Case(s)
    assert pkv.pkv_decode_cluster_size(c.pool, s.batch, s.max_pages, s.q_heads) == 0
    auto = pkv.pkv_decode_auto_splits(c.pool, s.batch, s.max_pages, s.q_heads)
    assert auto == min(full, -(-(32 * s.batch * s.max_pages) // 16)) and auto < full
    out_auto = c.gpu_layer(0)
    q = c.last_q
    out_expl = torch.empty_like(q)
    pkv.paged_decode_attention(c.pool, 0, out_expl, q, c.bt_t, c.cl_t, c.scale, num_splits=auto)
    assert np.array_equal(to_bits(out_auto), to_bits(out_expl))
    _expect_close(out_auto, c.oracle_layer(0), "f16", "automatic splits")
    one = Case(synth.random_spec(611, 1, 32, 32, 128, 16, [2048]))   # the single long sequence
    assert pkv.pkv_decode_auto_splits(one.pool, 1, one.s.max_pages, 32) == min(full, -(-(32 * one.s.max_pages) // 16))
    big = synth.spec("batch10", num_layers=1)
    assert pkv.pkv_decode_auto_splits(pkv.KVPool(*synth.pool_values_torch(big, "cuda")), big.batch, big.max_pages,
                                      big.q_heads) == full
    tiny = synth.spec("tiny")
    ct = Case(tiny)
    assert pkv.pkv_decode_auto_splits(ct.pool, 1, tiny.max_pages, 4) == 1
