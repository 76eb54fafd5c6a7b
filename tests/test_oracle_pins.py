"""Pins of the fp64 oracle to things other than itself (CPU only).

Each test checks the oracle against what the pages or the mathematics fix:
library codecs on every bit pattern, brute force on tiny inputs, the
no-cache full recompute, closed forms, invariants and worked numbers.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ formats
def test_half_decode_matches_numpy_on_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.decode(bits, "f16")
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_bf16_decode_matches_torch_on_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.decode(bits, "bf16")
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def _edge_doubles():
    r = np.random.Generator(np.random.PCG64(1))
    vals = [0.0, -0.0, 1.0, -1.0, 65504.0, 65519.99, 65520.0, 1e6, -1e6, 2.0 ** -24, 2.0 ** -25,
            3 * 2.0 ** -26, 2.0 ** -14, 2.0 ** -14 - 2.0 ** -25, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11,
            1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 3.0e38, 3.5e38, 1e-40, 1e-45, math.inf, -math.inf]
    vals += list(r.standard_normal(20000) * 10.0 ** r.integers(-9, 6, 20000))
    # exact midpoints between neighbouring halfs (ties)
    h = np.arange(0, 0x7BFF, 37, dtype=np.uint16).view(np.float16).astype(np.float64)
    h2 = (np.arange(0, 0x7BFF, 37, dtype=np.uint16) + 1).view(np.float16).astype(np.float64)
    vals += list((h + h2) / 2)
    return np.array(vals, np.float64)


def test_half_encode_matches_numpy_rne():
    x = _edge_doubles()
    ours = oracle.encode(x, "f16")
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)  # numpy: one RNE step from double
    assert np.array_equal(ours, ref)


def test_bf16_encode_is_nearest_even_by_brute_force():
    bits = np.arange(0, 0x7F80, dtype=np.uint16)       # every finite non-negative bf16
    vals = oracle.decode(bits, "bf16")
    x = _edge_doubles()
    x = x[np.isfinite(x) & (np.abs(x) < 3.3e38)]
    ours = oracle.encode(x, "bf16")
    a = np.abs(x)
    hi = np.searchsorted(vals, a, side="left")
    hi = np.minimum(hi, len(vals) - 1)
    lo = np.maximum(hi - 1, 0)
    dlo, dhi = a - vals[lo], vals[hi] - a
    pick = np.where(dlo < dhi, lo, hi)
    tie = dlo == dhi
    pick = np.where(tie, np.where(bits[lo] % 2 == 0, lo, hi), pick)
    pick = np.where(vals[hi] == a, hi, pick)
    exp = bits[pick] | np.where(np.signbit(x), 0x8000, 0).astype(np.uint16)
    assert np.array_equal(ours, exp)


def test_bf16_encode_matches_torch_on_float_values():
    r = np.random.Generator(np.random.PCG64(2))
    f = (r.standard_normal(50000) * 10.0 ** r.integers(-30, 30, 50000)).astype(np.float32)
    ours = oracle.encode(f.astype(np.float64), "bf16")
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


# ------------------------------------------------------------------ helpers
def _logical_case(seed, B, Hq, Hkv, d, P, lens, dtype="f16", scale=None):
    """Random logical caches, scattered into a shuffled paged pool by the test."""
    r = np.random.Generator(np.random.PCG64(seed))
    sp = synth.random_spec(seed, B, Hq, Hkv, d, P, [l - 1 for l in lens], dtype=dtype)
    q = synth.round_f32(r.standard_normal((B, Hq, d), dtype=np.float32), dtype)
    kp = synth.round_f32(r.standard_normal((sp.num_pages, Hkv, P, d), dtype=np.float32), dtype)
    vp = synth.round_f32(r.standard_normal((sp.num_pages, Hkv, P, d), dtype=np.float32), dtype)
    Kl, Vl = [], []
    dec = lambda a: oracle.decode(a, dtype)
    for b, L in enumerate(lens):
        ks, vs = [], []
        for t in range(L):
            page = sp.block_tables[b][t // P]
            ks.append([list(dec(kp[page, g, t % P])) for g in range(Hkv)])
            vs.append([list(dec(vp[page, g, t % P])) for g in range(Hkv)])
        Kl.append(ks)
        Vl.append(vs)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    return sp, q, kp, vp, Kl, Vl, scale


# ------------------------------------------------------------------ attention
@pytest.mark.parametrize("Hq,Hkv,d,P,lens,dtype", [
    (2, 2, 8, 4, [1, 7], "f16"),
    (4, 2, 8, 4, [13, 40], "f16"),
    (4, 1, 6, 3, [40, 9], "bf16"),
    (3, 3, 4, 16, [17, 0], "f16"),
])
def test_attention_matches_brute_force(Hq, Hkv, d, P, lens, dtype):
    sp, q, kp, vp, Kl, Vl, scale = _logical_case(11 + len(lens) + d, len(lens), Hq, Hkv, d, P, lens,
                                                 dtype)
    cl = np.array(lens, np.int32)
    ours = oracle.decode_attention(q, kp, vp, sp.block_tables, cl, scale, dtype)
    qd = [[list(oracle.decode(q[b, h], dtype)) for h in range(Hq)] for b in range(len(lens))]
    ref = np.array(brute.decode_logical(qd, Kl, Vl, lens, Hq, Hkv, scale))
    assert np.allclose(ours, ref, rtol=1e-12, atol=1e-14)


def test_plausible_mistakes_fail_brute_force():
    """The brute-force comparison distinguishes a dropped scale, a wrong GQA map and
    a page-table row read for the wrong sequence (planted in copies of the inputs,
    on the CPU).  Reordering one sequence's own pages is invisible by design:
    attention over the cached tokens does not depend on their order."""
    sp, q, kp, vp, Kl, Vl, scale = _logical_case(5, 2, 4, 2, 8, 4, [21, 30])
    cl = np.array([21, 30], np.int32)
    qd = [[list(oracle.decode(q[b, h], "f16")) for h in range(4)] for b in range(2)]
    ref = np.array(brute.decode_logical(qd, Kl, Vl, [21, 30], 4, 2, scale))
    good = oracle.decode_attention(q, kp, vp, sp.block_tables, cl, scale, "f16")
    assert np.allclose(good, ref, rtol=1e-12, atol=1e-14)
    no_scale = oracle.decode_attention(q, kp, vp, sp.block_tables, cl, 1.0, "f16")
    assert not np.allclose(no_scale, ref, rtol=1e-6, atol=1e-6)
    # query head h reading kv head h % Hkv (interleaved groups) instead of h // group
    wrong_map = oracle.decode_attention(q[:, [0, 2, 1, 3]], kp, vp, sp.block_tables, cl, scale, "f16")
    assert not np.allclose(wrong_map[:, [0, 2, 1, 3]], ref, rtol=1e-6, atol=1e-6)
    bt = sp.block_tables[[1, 0]].copy()
    swapped = oracle.decode_attention(q, kp, vp, bt, cl, scale, "f16")
    assert not np.allclose(swapped, ref, rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("T,Hq,Hkv", [(9, 2, 2), (33, 4, 2), (20, 8, 1)])
def test_decode_equals_last_row_of_full_causal_recompute(T, Hq, Hkv):
    """The cache check of the pages (s5.2): disable the cache, recompute the whole
    sequence with the causal mask, and compare with the cached decode step."""
    d, P = 8, 4
    r = np.random.Generator(np.random.PCG64(T))
    qs = synth.round_f32(r.standard_normal((T, Hq, d), dtype=np.float32), "f16")
    ks = synth.round_f32(r.standard_normal((T, Hkv, d), dtype=np.float32), "f16")
    vs = synth.round_f32(r.standard_normal((T, Hkv, d), dtype=np.float32), "f16")
    full = oracle.causal_attention_full(oracle.decode(qs, "f16"), oracle.decode(ks, "f16"),
                                        oracle.decode(vs, "f16"), 1 / math.sqrt(d))
    sp = synth.random_spec(T, 1, Hq, Hkv, d, P, [T - 1])
    kp = np.zeros((sp.num_pages, Hkv, P, d), np.uint16)
    vp = np.zeros_like(kp)
    for t in range(T):
        page = sp.block_tables[0][t // P]
        kp[page, :, t % P] = ks[t]
        vp[page, :, t % P] = vs[t]
    dec = oracle.decode_attention(qs[T - 1:T], kp, vp, sp.block_tables, np.array([T], np.int32),
                                  1 / math.sqrt(d), "f16")
    assert np.allclose(dec[0], full[T - 1], rtol=1e-12, atol=1e-14)
    # and the first row of the full form sees only token 0
    assert np.allclose(full[0], np.repeat(oracle.decode(vs[0], "f16"), Hq // Hkv, axis=0),
                       rtol=0, atol=1e-15)


def test_softmax_rows_sum_to_one():
    sp, q, kp, vp, _, _, scale = _logical_case(3, 3, 4, 4, 16, 4, [1, 17, 64])
    _, w = oracle.decode_attention(q, kp, vp, sp.block_tables, np.array([1, 17, 64], np.int32),
                                   scale, "f16", return_weights=True)
    for b, L in enumerate([1, 17, 64]):
        assert np.all(np.abs(w[b, :, :L].sum(-1) - 1.0) < 1e-12)
        assert np.all(w[b, :, L:] == 0)
        assert np.all(w[b, :, :L] > 0)


def test_single_token_context_returns_v_exactly():
    sp, q, kp, vp, _, Vl, scale = _logical_case(4, 2, 4, 2, 16, 16, [1, 1], dtype="bf16")
    out = oracle.decode_attention(q, kp, vp, sp.block_tables, np.array([1, 1], np.int32), scale,
                                  "bf16")
    for b in range(2):
        for h in range(4):
            assert np.array_equal(out[b, h], np.array(Vl[b][0][h // 2]))


def test_identical_keys_give_mean_of_v():
    sp, q, kp, vp, _, Vl, scale = _logical_case(6, 1, 2, 2, 8, 4, [23])
    for t in range(23):                     # every key of the sequence := key 0
        page = sp.block_tables[0][t // 4]
        p0 = sp.block_tables[0][0]
        kp[page, :, t % 4] = kp[p0, :, 0]
    out = oracle.decode_attention(q, kp, vp, sp.block_tables, np.array([23], np.int32), scale, "f16")
    mean = np.array(Vl[0]).mean(axis=0)      # [Hkv, d]
    assert np.allclose(out[0], mean, rtol=1e-12, atol=1e-14)


def test_invariant_under_physical_page_permutation():
    sp, q, kp, vp, _, _, scale = _logical_case(8, 2, 4, 4, 8, 4, [29, 14])
    cl = np.array([29, 14], np.int32)
    ref = oracle.decode_attention(q, kp, vp, sp.block_tables, cl, scale, "f16")
    r = np.random.Generator(np.random.PCG64(9))
    perm = r.permutation(sp.num_pages)            # new home of every physical page
    kp2 = np.empty_like(kp)
    vp2 = np.empty_like(vp)
    kp2[perm] = kp
    vp2[perm] = vp
    bt2 = np.where(sp.block_tables >= 0, perm[np.maximum(sp.block_tables, 0)], -1).astype(np.int32)
    out = oracle.decode_attention(q, kp2, vp2, bt2, cl, scale, "f16")
    assert np.array_equal(out, ref)


def test_peaked_key_selects_its_value():
    sp, q, kp, vp, _, Vl, _ = _logical_case(10, 1, 1, 1, 8, 4, [19])
    qv = oracle.decode(q[0, 0], "f16")
    t_hot = 11
    page = sp.block_tables[0][t_hot // 4]
    kp[page, 0, t_hot % 4] = oracle.encode(qv * 100.0, "f16")
    out = oracle.decode_attention(q, kp, vp, sp.block_tables, np.array([19], np.int32), 1.0, "f16")
    assert np.allclose(out[0, 0], Vl[0][t_hot][0], atol=1e-9)


def test_pairs_routine_equals_full_routine():
    sp, q, kp, vp, _, _, scale = _logical_case(12, 3, 4, 2, 16, 4, [5, 0, 37])
    cl = np.array([5, 0, 37], np.int32)
    full = oracle.decode_attention(q, kp, vp, sp.block_tables, cl, scale, "f16")
    pairs = [(b, h) for b in range(3) for h in range(4)]
    part = oracle.decode_attention_pairs(q, kp, vp, sp.block_tables, cl, scale, "f16", pairs)
    assert np.array_equal(part, full.reshape(-1, 16))


def test_empty_context_gives_zeros():
    sp, q, kp, vp, _, _, scale = _logical_case(13, 2, 2, 2, 8, 4, [0, 3])
    out = oracle.decode_attention(q, kp, vp, sp.block_tables, np.array([0, 3], np.int32), scale, "f16")
    assert np.all(out[0] == 0)
    assert np.all(np.isfinite(out))


# ------------------------------------------------------------------ RoPE
def test_rope_position_zero_is_identity_bit_exact():
    r = np.random.Generator(np.random.PCG64(20))
    for dtype in ("f16", "bf16"):
        x = synth.round_f32(r.standard_normal((5, 3, 64), dtype=np.float32), dtype)
        y, _ = oracle.rope(x, np.zeros(5, np.int32), 10000.0, dtype)
        assert np.array_equal(x, y)


def test_rope_unit_vectors_closed_form():
    """e_{2i} turns into (cos a_i, sin a_i) on the pair (2i, 2i+1) and nowhere else,
    a_i = pos * theta^(-2i/d); e_{2i+1} into (-sin a_i, cos a_i)."""
    d, pos, theta = 16, 7, 10000.0
    for i in range(d // 2):
        for odd in (0, 1):
            x = np.zeros((1, 1, d))
            x[0, 0, 2 * i + odd] = 1.0
            y = oracle.rope_f64(x, [pos], theta)[0, 0]
            a = pos * theta ** (-2.0 * i / d)
            exp = np.zeros(d)
            if odd == 0:
                exp[2 * i], exp[2 * i + 1] = math.cos(a), math.sin(a)
            else:
                exp[2 * i], exp[2 * i + 1] = -math.sin(a), math.cos(a)
            assert np.allclose(y, exp, rtol=0, atol=1e-15)


def test_rope_preserves_pair_norms_and_inverts():
    r = np.random.Generator(np.random.PCG64(21))
    x = r.standard_normal((6, 4, 128))
    pos = np.array([0, 1, 17, 2048, 32768, 12345], np.int32)
    y = oracle.rope_f64(x, pos, 10000.0)
    n0 = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    n1 = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    assert np.allclose(n0, n1, rtol=1e-12, atol=0)
    back = oracle.rope_f64(y, -pos, 10000.0)
    assert np.allclose(back, x, rtol=0, atol=1e-11)


def test_rope_scores_depend_only_on_relative_position():
    r = np.random.Generator(np.random.PCG64(22))
    q = r.standard_normal((1, 1, 64))
    k = r.standard_normal((1, 1, 64))
    base = None
    for p in (0, 5, 100, 4000):
        qr = oracle.rope_f64(q, [p + 9], 10000.0)
        kr = oracle.rope_f64(k, [p], 10000.0)
        s = float((qr * kr).sum())
        base = s if base is None else base
        assert abs(s - base) < 1e-9


def test_rope_storage_rounding_is_one_step():
    """Storage RoPE = one nearest-even rounding of the exact fp64 rotation."""
    r = np.random.Generator(np.random.PCG64(23))
    x = synth.round_f32(r.standard_normal((4, 2, 128), dtype=np.float32), "f16")
    pos = np.array([3, 999, 20000, 32768], np.int32)
    y, exact = oracle.rope(x, pos, 10000.0, "f16")
    assert np.array_equal(y, exact.astype(np.float16).view(np.uint16))


# ------------------------------------------------------------------ page table and append
def _golden_slots():
    rows = []
    with open(os.path.join(GOLDEN, "slot_mapping.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            P, table, pos, slot = [s.strip() for s in line.split("|")]
            rows.append((int(P), [int(x) for x in table.split(",")], int(pos), int(slot)))
    return rows


def test_slot_mapping_golden():
    for P, table, pos, slot in _golden_slots():
        bt = np.array([table], np.int32)
        assert oracle.slot_mapping(bt, np.array([pos], np.int32), P)[0] == slot


def test_append_changes_exactly_the_mapped_rows():
    sp = synth.random_spec(30, 3, 4, 2, 16, 4, [5, 8, -1])
    r = np.random.Generator(np.random.PCG64(31))
    kp = r.integers(0, 65536, (sp.num_pages, 2, 4, 16), dtype=np.uint16)
    vp = r.integers(0, 65536, (sp.num_pages, 2, 4, 16), dtype=np.uint16)
    k = r.integers(0, 65536, (3, 2, 16), dtype=np.uint16)
    v = r.integers(0, 65536, (3, 2, 16), dtype=np.uint16)
    kp2, vp2 = oracle.kv_append(kp, vp, k, v, sp.block_tables, sp.positions)
    changed = set()
    for b, pos in enumerate(sp.positions):
        if pos < 0:
            continue
        page, row = sp.block_tables[b][pos // 4], pos % 4
        assert np.array_equal(kp2[page, :, row], k[b]) and np.array_equal(vp2[page, :, row], v[b])
        changed.add((page, row))
    mask = np.ones((sp.num_pages, 4), bool)
    for page, row in changed:
        mask[page, row] = False
    assert np.array_equal(kp2.transpose(0, 2, 1, 3)[mask], kp.transpose(0, 2, 1, 3)[mask])
    assert np.array_equal(vp2.transpose(0, 2, 1, 3)[mask], vp.transpose(0, 2, 1, 3)[mask])


# ------------------------------------------------------------------ KV size
def test_kv_cache_size_worked_example():
    with open(os.path.join(GOLDEN, "kv_cache_size.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    for layers, heads, hd, tokens, eb, req, approx in rows:
        n = oracle.kv_cache_bytes(int(layers), int(heads), int(hd), int(tokens), int(eb)) * int(req)
        assert round(n / 2 ** 30) == int(approx)
    assert oracle.kv_cache_bytes(32, 32, 128, 2048, 2) == 2 ** 30


def test_workload_kv_bytes_match_size_model():
    s = synth.spec("layer7b")
    assert s.kv_bytes_read() == 2049 * 2 * 32 * 128 * 2
    assert oracle.kv_cache_bytes(1, 32, 128, 2049, 2) == s.kv_bytes_read()


# ------------------------------------------------------------------ RMSNorm
def test_rms_norm_eps_sits_inside_the_root():
    """[ENGINE] s4.2: eps is added to the mean square, then the root is taken.  A constant
    row c makes both placements closed forms that differ clearly for small c."""
    c, eps, hidden = 1e-3, 1e-6, 64
    x = np.full((1, hidden), c)
    bits = oracle.encode(x, "f16")
    cd = oracle.decode(bits[0, :1], "f16")[0]
    w = oracle.encode(np.ones(hidden), "f16")
    _, exact, _ = oracle.rms_norm(bits, w, eps, "f16")
    inside = cd / math.sqrt(cd * cd + eps)
    outside = cd / (math.sqrt(cd * cd) + eps)
    assert np.allclose(exact, inside, rtol=1e-12, atol=0)
    assert abs(inside - outside) > 0.2


def test_rms_norm_brute_force_and_unit_rms():
    r = np.random.Generator(np.random.PCG64(70))
    x = synth.round_f32(r.standard_normal((3, 24), dtype=np.float32), "bf16")
    w = synth.round_f32(r.standard_normal(24, dtype=np.float32), "bf16")
    _, exact, _ = oracle.rms_norm(x, w, 1e-6, "bf16")
    xd, wd = oracle.decode(x, "bf16"), oracle.decode(w, "bf16")
    for i in range(3):
        row = [float(v) for v in xd[i]]
        inv = 1.0 / math.sqrt(math.fsum(v * v for v in row) / len(row) + 1e-6)
        ref = [row[k] * inv * float(wd[k]) for k in range(24)]
        assert np.allclose(exact[i], ref, rtol=1e-12, atol=1e-15)
    ones = oracle.encode(np.ones(24), "bf16")
    _, unit, _ = oracle.rms_norm(x, ones, 0.0, "bf16")
    assert np.allclose((unit ** 2).mean(axis=1), 1.0, rtol=1e-12)


def test_rms_norm_residual_is_summed_and_rounded_first():
    r = np.random.Generator(np.random.PCG64(71))
    x = synth.round_f32(r.standard_normal((2, 16), dtype=np.float32), "f16")
    res = synth.round_f32(r.standard_normal((2, 16), dtype=np.float32), "f16")
    w = oracle.encode(np.ones(16), "f16")
    y, exact, summed = oracle.rms_norm(x, w, 1e-6, "f16", residual=res)
    expect_sum = (oracle.decode(x, "f16") + oracle.decode(res, "f16")).astype(np.float16).view(np.uint16)
    assert np.array_equal(summed, expect_sum)
    y2, exact2, _ = oracle.rms_norm(summed, w, 1e-6, "f16")
    assert np.array_equal(y, y2) and np.array_equal(exact, exact2)


# ------------------------------------------------------------------ chunked prefill
def test_prefill_of_one_token_is_the_decode_step():
    sp, q, kp, vp, _, _, scale = _logical_case(80, 3, 8, 2, 16, 4, [9, 30, 1])
    cl = np.array([9, 30, 1], np.int32)
    dec = oracle.decode_attention(q, kp, vp, sp.block_tables, cl, scale, "f16")
    pre = oracle.prefill_attention(q, kp, vp, sp.block_tables, np.arange(4, dtype=np.int32), cl, scale, "f16")
    assert np.array_equal(pre, dec)


@pytest.mark.parametrize("T,chunk,Hq,Hkv", [(23, 23, 2, 2), (40, 9, 4, 2), (17, 5, 8, 1)])
def test_prefill_equals_full_causal_recompute(T, chunk, Hq, Hkv):
    """The cache check of s5.2 for a chunk: the last `chunk` rows of the full causal
    recompute, computed from the paged cache with the mask slice [T-chunk, T)."""
    d, P = 8, 4
    r = np.random.Generator(np.random.PCG64(T + chunk))
    qs = synth.round_f32(r.standard_normal((T, Hq, d), dtype=np.float32), "bf16")
    ks = synth.round_f32(r.standard_normal((T, Hkv, d), dtype=np.float32), "bf16")
    vs = synth.round_f32(r.standard_normal((T, Hkv, d), dtype=np.float32), "bf16")
    full = oracle.causal_attention_full(oracle.decode(qs, "bf16"), oracle.decode(ks, "bf16"),
                                        oracle.decode(vs, "bf16"), 1 / math.sqrt(d))
    sp = synth.random_spec(T, 1, Hq, Hkv, d, P, [T - 1])
    kp = np.zeros((sp.num_pages, Hkv, P, d), np.uint16)
    vp = np.zeros_like(kp)
    for t in range(T):
        page = sp.block_tables[0][t // P]
        kp[page, :, t % P] = ks[t]
        vp[page, :, t % P] = vs[t]
    pre = oracle.prefill_attention(qs[T - chunk:], kp, vp, sp.block_tables, np.array([0, chunk], np.int32),
                                   np.array([T], np.int32), 1 / math.sqrt(d), "bf16")
    assert np.allclose(pre, full[T - chunk:], rtol=1e-12, atol=1e-14)


def test_prefill_matches_brute_force():
    sp, q, kp, vp, Kl, Vl, scale = _logical_case(81, 2, 4, 2, 8, 4, [13, 7])
    cq = np.array([0, 3, 5], np.int32)                     # 3 new tokens of seq 0, 2 of seq 1
    qq = np.concatenate([q, q[:1], q[1:], q[:1]])[:5]      # any 5 query rows
    pre = oracle.prefill_attention(qq, kp, vp, sp.block_tables, cq, np.array([13, 7], np.int32), scale, "f16")
    for b, (lo, hi, L) in enumerate([(0, 3, 13), (3, 5, 7)]):
        for i in range(hi - lo):
            pos = L - (hi - lo) + i
            for h in range(4):
                qv = list(oracle.decode(qq[lo + i, h], "f16"))
                ref = brute.attention_one(qv, [Kl[b][t][h // 2] for t in range(pos + 1)],
                                          [Vl[b][t][h // 2] for t in range(pos + 1)], scale)
                assert np.allclose(pre[lo + i, h], ref, rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------ int8 KV pages
def test_int8_codes_match_a_float32_reference():
    """The quantiser's fp32 steps, redone with numpy float32 (each op rounded to nearest)."""
    r = np.random.Generator(np.random.PCG64(90))
    for dtype in ("f16", "bf16"):
        x = synth.round_f32(r.standard_normal((50, 128), dtype=np.float32) * 2, dtype)
        codes, scales = oracle.quantize_rows_i8(x, dtype)
        xf = oracle.decode(x, dtype).astype(np.float32)
        amax = np.abs(xf).max(axis=1)
        inv = (np.float32(127.0) / amax).astype(np.float32)
        ref = np.clip(np.rint((xf * inv[:, None]).astype(np.float32)), -127, 127).astype(np.int8)
        assert np.array_equal(codes, ref)
        assert np.array_equal(scales, (amax / np.float32(127.0)).astype(np.float32))
        # the largest element maps to +-127 and every element is within half a step, plus the
        # fp32 roundings of the scale and of x * inv (each 2^-24 relative, times |code| <= 127)
        assert np.all(np.abs(codes).max(axis=1) == 127)
        err = np.abs(codes.astype(np.float64) * scales[:, None] - oracle.decode(x, dtype))
        assert np.all(err <= scales[:, None] * (0.5 + 2 * 127 * 2.0 ** -24))


def test_int8_zero_row_and_attention_on_dequantised_values():
    codes, scales = oracle.quantize_rows_i8(np.zeros((1, 16), np.uint16), "f16")
    assert np.all(codes == 0) and scales[0] == 0
    sp, q, kp, vp, _, _, scale = _logical_case(91, 2, 4, 2, 16, 4, [19, 6])
    kc, ks = oracle.quantize_rows_i8(kp, "f16")
    vc, vs = oracle.quantize_rows_i8(vp, "f16")
    cl = np.array([19, 6], np.int32)
    pairs = [(b, h) for b in range(2) for h in range(4)]
    got = oracle.decode_attention_i8_pairs(q, kc, vc, ks, vs, sp.block_tables, cl, scale, "f16", pairs)
    # brute force on the dequantised cache (exact products code * scale in double)
    kd = kc.astype(np.float64) * ks[..., None].astype(np.float64)
    vd = vc.astype(np.float64) * vs[..., None].astype(np.float64)
    for n, (b, h) in enumerate(pairs):
        keys, vals = [], []
        for t in range(cl[b]):
            page = sp.block_tables[b][t // 4]
            keys.append(list(kd[page, h // 2, t % 4]))
            vals.append(list(vd[page, h // 2, t % 4]))
        ref = brute.attention_one(list(oracle.decode(q[b, h], "f16")), keys, vals, scale)
        assert np.allclose(got[n], ref, rtol=1e-12, atol=1e-14)


def test_int8_append_lands_where_the_fp16_append_does():
    """Quantising append == plain append (pinned above) followed by row-wise quantisation of
    the written rows; untouched rows keep their codes and scales."""
    r = np.random.Generator(np.random.PCG64(92))
    pages, kvh, P, d, n = 6, 2, 4, 16, 3
    kp = synth.round_f32(r.standard_normal((pages, kvh, P, d), dtype=np.float32), "f16")
    vp = synth.round_f32(r.standard_normal((pages, kvh, P, d), dtype=np.float32), "f16")
    k = synth.round_f32(r.standard_normal((n, kvh, d), dtype=np.float32), "f16")
    v = synth.round_f32(r.standard_normal((n, kvh, d), dtype=np.float32), "f16")
    bt = np.array([[5, 2], [0, 1], [3, 4]], np.int32)
    pos = np.array([6, 0, -1], np.int32)
    kc, ks = oracle.quantize_rows_i8(kp, "f16")
    vc, vs = oracle.quantize_rows_i8(vp, "f16")
    kc2, vc2, ks2, vs2 = oracle.kv_append_i8(kc, vc, ks, vs, k, v, bt, pos, "f16")
    kp2, vp2 = oracle.kv_append(kp, vp, k, v, bt, pos)
    kc_ref, ks_ref = oracle.quantize_rows_i8(kp2, "f16")
    vc_ref, vs_ref = oracle.quantize_rows_i8(vp2, "f16")
    assert np.array_equal(kc2, kc_ref) and np.array_equal(ks2, ks_ref)
    assert np.array_equal(vc2, vc_ref) and np.array_equal(vs2, vs_ref)
    assert not np.array_equal(kc2, kc)                  # something was written
    assert np.array_equal(kc2[2, :, 2], kc_ref[2, :, 2])  # page 2 row 2 (token 6 of seq 0)


def test_openmp_build_gives_the_same_bits_as_the_plain_build():
    """The all-core build of the pair routines only spreads independent pairs over threads:
    every output bit equals the single-thread build's."""
    sp = synth.random_spec(88, 5, 8, 2, 64, 16, [300, 1, 47, 0, 129], dtype="bf16")
    pairs = [(b, h) for b in range(sp.batch) for h in range(sp.q_heads)]
    m = synth.pair_batch_numpy(sp, [(b, g) for b in range(sp.batch) for g in range(sp.kv_heads)], 9)
    G = sp.q_heads // sp.kv_heads
    hp = [(i, h) for i in range(m["q"].shape[0]) for h in range(G)]
    oracle.set_threads(4)
    a = oracle.decode_attention_pairs(m["q"], m["k"], m["v"], m["block_tables"], m["context_lens"], 0.125, "bf16", hp)
    b = oracle.decode_attention_pairs(m["q"], m["k"], m["v"], m["block_tables"], m["context_lens"], 0.125, "bf16", hp,
                                      omp=True)
    assert np.array_equal(a.view(np.uint64), b.view(np.uint64))
    m8 = synth.pair_batch_numpy(sp, [(b, g) for b in range(sp.batch) for g in range(sp.kv_heads)], 10, kv="int8")
    args = (m8["q"], m8["k_codes"], m8["v_codes"], m8["k_scales"], m8["v_scales"], m8["block_tables"],
            m8["context_lens"], 0.125, "bf16", hp)
    a8 = oracle.decode_attention_i8_pairs(*args)
    b8 = oracle.decode_attention_i8_pairs(*args, omp=True)
    assert np.array_equal(a8.view(np.uint64), b8.view(np.uint64))
    assert len(pairs) == sp.batch * sp.q_heads

