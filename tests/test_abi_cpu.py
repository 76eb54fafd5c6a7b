"""The C ABI without a GPU: the library loads, exports every declared entry point,
and its host-side logic (argument checks, free list, slot mapping, sizes) is right.
No call here launches device work."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import synth
import paged_kv_cache_460_b200 as pkv
from paged_kv_cache_460_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedkv.h")
GOLDEN = os.path.join(ROOT, "tests", "golden")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w \*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("defined",)))


@pytest.fixture(scope="module")
def L():
    from paged_kv_cache_460_b200 import build
    build.build()
    return _lib.lib()


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("kv_pool_create", "rope_apply", "paged_kv_append", "paged_decode_attention",
                 "kv_get_device_error", "pkv_slot_mapping"):
        assert must in names


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), name
        assert name in _lib.SIGNATURES, "binding lacks a signature for %s" % name


def test_status_strings(L):
    for s in range(5):
        assert pkv._lib.status_string(s)
    assert pkv._lib.status_string(99) == "unknown status"


def _fake_ptr(v=0x10000):
    return ctypes.c_void_p(v)


def _pool(L, num_pages=8, page_size=16, kv_heads=2, head_dim=64, dtype=0, layers=1):
    h = ctypes.c_void_p()
    st = L.kv_pool_create(layers, num_pages, page_size, kv_heads, head_dim, dtype, _fake_ptr(), _fake_ptr(0x20000),
                          ctypes.byref(h))
    assert st == 0
    return h


def test_pool_create_validates(L):
    h = ctypes.c_void_p()
    assert L.kv_pool_create(1, 8, 16, 2, 64, 0, None, _fake_ptr(), ctypes.byref(h)) == _lib.PKV_ERR_INVALID_ARG
    assert L.kv_pool_create(1, 8, 16, 2, 64, 0, _fake_ptr(0x10008), _fake_ptr(), ctypes.byref(h)) == \
        _lib.PKV_ERR_INVALID_ARG
    assert L.kv_pool_create(0, 8, 16, 2, 64, 0, _fake_ptr(), _fake_ptr(), ctypes.byref(h)) == _lib.PKV_ERR_INVALID_ARG
    assert L.kv_pool_create(1, 8, 8, 2, 64, 0, _fake_ptr(), _fake_ptr(), ctypes.byref(h)) == _lib.PKV_ERR_UNSUPPORTED
    assert L.kv_pool_create(1, 8, 16, 2, 96, 0, _fake_ptr(), _fake_ptr(), ctypes.byref(h)) == _lib.PKV_ERR_UNSUPPORTED
    assert L.kv_pool_create(1, 8, 16, 2, 64, 7, _fake_ptr(), _fake_ptr(), ctypes.byref(h)) == _lib.PKV_ERR_UNSUPPORTED
    assert L.kv_pool_create(1, 8, 16, 2, 64, 0, _fake_ptr(), _fake_ptr(), None) == _lib.PKV_ERR_INVALID_ARG
    # 16-token blocks of a layer past the kernels' 32-bit index: rejected before any allocation
    assert L.kv_pool_create(1, 1 << 30, 32, 1, 64, 0, _fake_ptr(), _fake_ptr(), ctypes.byref(h)) == \
        _lib.PKV_ERR_INVALID_ARG
    assert L.kv_pool_create(1, 1 << 27, 16, 16, 64, 0, _fake_ptr(), _fake_ptr(), ctypes.byref(h)) == \
        _lib.PKV_ERR_INVALID_ARG


def test_free_list_properties(L):
    h = _pool(L, num_pages=10)
    buf = np.empty(10, np.int32)
    p = buf.ctypes.data_as(ctypes.c_void_p)
    assert L.kv_pool_free_count(h) == 10
    assert L.kv_pool_alloc(h, 4, p) == 0
    assert list(buf[:4]) == [0, 1, 2, 3]                      # increasing order at first
    assert L.kv_pool_alloc(h, 7, p) == _lib.PKV_ERR_NO_SPACE  # all or nothing
    assert L.kv_pool_free_count(h) == 6
    two = np.array([2, 0], np.int32)
    assert L.kv_pool_free(h, 2, two.ctypes.data_as(ctypes.c_void_p)) == 0
    # double free, repeated id and out-of-range id are rejected and change nothing
    assert L.kv_pool_free(h, 1, two.ctypes.data_as(ctypes.c_void_p)) == _lib.PKV_ERR_INVALID_ARG
    rep = np.array([1, 1], np.int32)
    assert L.kv_pool_free(h, 2, rep.ctypes.data_as(ctypes.c_void_p)) == _lib.PKV_ERR_INVALID_ARG
    bad = np.array([3, 10], np.int32)
    assert L.kv_pool_free(h, 2, bad.ctypes.data_as(ctypes.c_void_p)) == _lib.PKV_ERR_INVALID_ARG
    assert L.kv_pool_free_count(h) == 8
    assert L.kv_pool_alloc(h, 2, p) == 0
    assert list(buf[:2]) == [0, 2]                            # most recently freed first
    L.kv_pool_destroy(h)


def test_free_list_random_walk_conserves_pages(L):
    h = _pool(L, num_pages=64)
    r = np.random.Generator(np.random.PCG64(5))
    owned = []
    for _ in range(400):
        if owned and r.random() < 0.45:
            k = int(r.integers(1, len(owned) + 1))
            idx = r.permutation(len(owned))[:k]
            ids = np.array([owned[i] for i in idx], np.int32)
            assert L.kv_pool_free(h, k, ids.ctypes.data_as(ctypes.c_void_p)) == 0
            owned = [o for i, o in enumerate(owned) if i not in set(idx.tolist())]
        else:
            n = int(r.integers(1, 9))
            out = np.empty(n, np.int32)
            st = L.kv_pool_alloc(h, n, out.ctypes.data_as(ctypes.c_void_p))
            if st == _lib.PKV_ERR_NO_SPACE:
                assert L.kv_pool_free_count(h) < n
                continue
            assert st == 0
            assert not set(out.tolist()) & set(owned)           # never handed out twice
            owned += out.tolist()
        assert L.kv_pool_free_count(h) + len(owned) == 64
        assert all(0 <= o < 64 for o in owned)
    L.kv_pool_destroy(h)


def test_pool_info(L):
    h = _pool(L, num_pages=12, page_size=32, kv_heads=8, head_dim=128, dtype=1, layers=3)
    vals = [ctypes.c_int() for _ in range(6)]
    assert L.kv_pool_info(h, *[ctypes.byref(v) for v in vals]) == 0
    assert [v.value for v in vals] == [3, 12, 32, 8, 128, 1]
    L.kv_pool_destroy(h)


def test_slot_mapping_matches_oracle_and_golden(L):
    for P in (16, 32):
        s = synth.random_spec(3 + P, 7, 4, 4, 64, P, [0, 1, P - 1, P, P + 1, 5 * P + 3, -1])
        ours = pkv.pkv_slot_mapping(s.block_tables, s.positions, P)
        ref = oracle.slot_mapping(s.block_tables, s.positions, P)
        assert np.array_equal(ours, ref)
    with open(os.path.join(GOLDEN, "slot_mapping.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            P, table, pos, slot = [x.strip() for x in line.split("|")]
            bt = np.array([[int(t) for t in table.split(",")]], np.int32)
            assert pkv.pkv_slot_mapping(bt, np.array([int(pos)], np.int32), int(P))[0] == int(slot)


def test_slot_mapping_rejects_bad_tables(L):
    bt = np.array([[3, -1]], np.int32)
    with pytest.raises(pkv.PagedKVError):
        pkv.pkv_slot_mapping(bt, np.array([20], np.int32), 16)      # entry -1
    with pytest.raises(pkv.PagedKVError):
        pkv.pkv_slot_mapping(bt, np.array([40], np.int32), 16)      # beyond the table


def test_kv_cache_bytes_worked_example(L):
    assert pkv.pkv_kv_cache_bytes(32, 32, 128, 2048, pkv.PKV_F16) == 2 ** 30
    assert pkv.pkv_kv_cache_bytes(32, 32, 128, 2048, pkv.PKV_F16) == oracle.kv_cache_bytes(32, 32, 128, 2048, 2)


def test_workspace_size_and_host_validation(L):
    ws = L.pkv_decode_workspace_size(10, 32, 32, 128, 296)
    assert ws >= 2 * 296 * 128 * 4 and ws % 256 == 0
    assert L.pkv_decode_workspace_size(10, 32, 5, 128, 296) == 0       # heads do not divide
    assert L.pkv_decode_workspace_size(10, 32, 32, 128, 0) == 0
    h = _pool(L, num_pages=8, page_size=16, kv_heads=2, head_dim=64)
    f = _fake_ptr
    # every call below fails validation before any CUDA call
    assert L.paged_decode_attention(None, 0, f(), f(), f(), 4, f(), 1, 2, 2, 0.1, 1, f(0x100000), 1 << 20, None) \
        == _lib.PKV_ERR_INVALID_ARG
    assert L.paged_decode_attention(h, 1, f(), f(), f(), 4, f(), 1, 2, 2, 0.1, 1, f(0x100000), 1 << 20, None) \
        == _lib.PKV_ERR_INVALID_ARG                                      # layer out of range
    assert L.paged_decode_attention(h, 0, f(), f(), f(), 4, f(), 1, 3, 2, 0.1, 1, f(0x100000), 1 << 20, None) \
        == _lib.PKV_ERR_INVALID_ARG                                      # q_heads % kv_heads
    assert L.paged_decode_attention(h, 0, f(), f(), f(), 4, f(), 1, 2, 1, 0.1, 1, f(0x100000), 1 << 20, None) \
        == _lib.PKV_ERR_INVALID_ARG                                      # kv_heads != pool's
    assert L.paged_decode_attention(h, 0, f(), f(), f(), 4, f(), 1, 32, 2, 0.1, 1, f(0x100000), 1 << 20, None) \
        == _lib.PKV_ERR_UNSUPPORTED                                      # group 16
    assert L.paged_decode_attention(h, 0, f(), f(), f(), 4, f(), 1, 2, 2, 0.1, 1, f(0x100000), 16, None) \
        == _lib.PKV_ERR_NO_SPACE                                         # workspace too small
    assert L.paged_decode_attention(h, 0, f(), f(), f(), 4, f(), 1, 2, 2, 0.1, 1, f(0x100010), 1 << 20, None) \
        == _lib.PKV_ERR_INVALID_ARG                                      # workspace misaligned
    assert L.paged_decode_attention(h, 0, None, f(), f(), 4, f(), 1, 2, 2, 0.1, 1, f(0x100000), 1 << 20, None) \
        == _lib.PKV_ERR_INVALID_ARG
    assert L.paged_decode_attention(h, 0, f(), f(), f(), 4, f(), 0, 2, 2, 0.1, 1, f(0x100000), 1 << 20, None) == 0
    assert L.paged_kv_append(h, 2, f(), f(), f(), 1, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.paged_kv_append(h, 0, f(0x10008), f(), f(), 1, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.paged_kv_append(h, 0, None, f(), f(), 1, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.paged_kv_append(h, 0, f(), f(), f(), 0, None) == 0
    assert L.rope_apply(f(), f(), f(), 1, 2, 2, 96, 10000.0, 0, None) == _lib.PKV_ERR_UNSUPPORTED
    assert L.rope_apply(f(), f(), f(), 1, 2, 2, 64, -1.0, 0, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.rope_apply(None, f(), f(), 1, 2, 2, 64, 10000.0, 0, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.rope_apply(f(), f(), f(), 0, 2, 2, 64, 10000.0, 0, None) == 0
    L.kv_pool_destroy(h)


def test_header_constants_match_the_binding():
    text = open(HEADER).read()
    for name in ("PKV_MAX_DECODE_SPLITS", "PKV_ERR_NO_SPACE", "PKV_DEVERR_TIMEOUT", "PKV_I8"):
        m = re.search(r"#define\s+%s\s+(0x[0-9a-fA-F]+|\d+)" % name, text)
        assert m, name
        assert int(m.group(1), 0) == getattr(_lib, name), name


def test_workspace_counter_region_is_fixed(L):
    """The counters occupy the same 16 KiB at the start of every workspace, whatever the split
    count: only the partials after them grow with num_splits."""
    cap = _lib.PKV_MAX_DECODE_SPLITS
    sizes = {n: L.pkv_decode_workspace_size(4, 8, 8, 64, n) for n in (1, 7, 444, 1000, cap)}
    assert sizes[1] >= 4 * cap + 2 * 1 * 64 * 4
    for n, ws in sizes.items():
        parts = 2 * n * 64 * 4 + 2 * n * 2 * 4             # o and (m, l) of both slots of every CTA
        assert ws >= 4 * cap + parts and ws % 256 == 0, n
        assert ws <= 4 * cap + parts + 3 * 256, n
    assert L.pkv_decode_workspace_size(4, 8, 8, 64, cap + 1) == 0
    h = _pool(L, num_pages=8, page_size=16, kv_heads=2, head_dim=64)
    f = _fake_ptr
    assert L.paged_decode_attention(h, 0, f(), f(), f(), 4, f(), 1, 2, 2, 0.1, cap + 1, f(0x100000), 1 << 30,
                                    None) == _lib.PKV_ERR_INVALID_ARG
    assert L.paged_decode_layer(h, 0, f(), f(), f(), f(), f(), f(), 4, f(), 1, 2, 2, 0.1, cap + 1, f(0x100000),
                                1 << 30, None) == _lib.PKV_ERR_INVALID_ARG
    L.kv_pool_destroy(h)


def test_noalloc_checks_arguments_before_its_scratch_limit(L):
    """The no-alloc entry point refuses a bad layer or kv-head count as paged_decode_attention
    does (INVALID_ARG), even with a split count whose scratch would not fit; with valid
    arguments that split count gets NO_SPACE.  No device work is launched."""
    h = _pool(L, num_pages=8, page_size=16, kv_heads=8, head_dim=128)
    f = _fake_ptr
    too_many = 4000           # 16 KiB + 2 x 4000 x 8 x 130 fp32 values: far above 4 MiB at group 8
    assert L.paged_decode_attention_noalloc(h, 1, f(), f(), f(), 4, f(), 1, 64, 8, 0.1, too_many, None) \
        == _lib.PKV_ERR_INVALID_ARG                                      # layer out of range
    assert L.paged_decode_attention_noalloc(h, 0, f(), f(), f(), 4, f(), 1, 64, 4, 0.1, too_many, None) \
        == _lib.PKV_ERR_INVALID_ARG                                      # kv_heads != pool's
    assert L.paged_decode_attention_noalloc(h, 0, f(), f(), f(), 4, f(), 1, 64, 8, 0.1,
                                            _lib.PKV_MAX_DECODE_SPLITS + 1, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.paged_decode_attention_noalloc(h, 0, f(), f(), f(), 4, f(), 1, 64, 8, 0.1, too_many, None) \
        == _lib.PKV_ERR_NO_SPACE
    L.kv_pool_destroy(h)


def test_rope_append_step_validates(L):
    h = _pool(L, num_pages=8, page_size=16, kv_heads=2, head_dim=64)
    f = _fake_ptr
    assert L.rope_append_step(None, 0, f(), f(), f(), f(), 4, f(), 1, 2, 10000.0, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.rope_append_step(h, 1, f(), f(), f(), f(), 4, f(), 1, 2, 10000.0, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.rope_append_step(h, 0, f(), f(), f(), f(), 0, f(), 1, 2, 10000.0, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.rope_append_step(h, 0, f(), f(), f(), f(), 4, f(), 1, 2, 0.0, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.rope_append_step(h, 0, f(), None, f(), f(), 4, f(), 1, 2, 10000.0, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.rope_append_step(h, 0, f(), f(), f(), None, 4, f(), 1, 2, 10000.0, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.rope_append_step(h, 0, f(0x10008), f(), f(), f(), 4, f(), 1, 2, 10000.0, None) \
        == _lib.PKV_ERR_INVALID_ARG                                      # q misaligned
    assert L.rope_append_step(h, 0, f(), f(), f(), f(), 4, f(), 0, 2, 10000.0, None) == 0
    L.kv_pool_destroy(h)


def test_rope_append_validates(L):
    h = _pool(L, num_pages=8, page_size=16, kv_heads=2, head_dim=64)
    f = _fake_ptr
    assert L.rope_append(h, 1, f(), f(), f(), f(), f(), 1, 2, 10000.0, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.rope_append(h, 0, f(), f(), f(), None, f(), 1, 2, 10000.0, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.rope_append(h, 0, f(0x10004), f(), f(), f(), f(), 1, 2, 10000.0, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.rope_append(h, 0, f(), f(), f(), f(), f(), 1, 2, 0.0, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.rope_append(h, 0, f(), f(), f(), f(), f(), 0, 2, 10000.0, None) == 0
    L.kv_pool_destroy(h)


def test_rms_norm_validates(L):
    f = _fake_ptr
    assert L.rms_norm(f(), f(), None, f(), 2, 4100, 1e-6, 0, None) == _lib.PKV_ERR_INVALID_ARG    # hidden % 8
    assert L.rms_norm(f(), f(), None, f(), 2, 32768, 1e-6, 0, None) == _lib.PKV_ERR_UNSUPPORTED
    assert L.rms_norm(f(), f(), None, f(), 2, 4096, -1.0, 0, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.rms_norm(None, f(), None, f(), 2, 4096, 1e-6, 0, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.rms_norm(f(), f(), f(0x10004), f(), 2, 4096, 1e-6, 0, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.rms_norm(f(), f(), None, f(), 0, 4096, 1e-6, 0, None) == 0


def test_prefill_validates(L):
    h = _pool(L, num_pages=8, page_size=16, kv_heads=2, head_dim=64)
    f = _fake_ptr
    assert L.paged_prefill_attention(h, 0, f(), f(), f(), 4, f(), 4, f(), 1, 3, 2, 0.1, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.paged_prefill_attention(h, 0, f(), f(), f(), 4, f(), 4, f(), 1, 32, 2, 0.1, None) == _lib.PKV_ERR_UNSUPPORTED
    assert L.paged_prefill_attention(h, 1, f(), f(), f(), 4, f(), 4, f(), 1, 2, 2, 0.1, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.paged_prefill_attention(h, 0, None, f(), f(), 4, f(), 4, f(), 1, 2, 2, 0.1, None) == _lib.PKV_ERR_INVALID_ARG
    assert L.paged_prefill_attention(h, 0, f(), f(), f(), 0, f(), 4, f(), 1, 2, 2, 0.1, None) == 0
    # the per-sequence work prefix no longer fits beside the tiles in one CTA's shared memory
    assert L.paged_prefill_attention(h, 0, f(), f(), f(), 30000, f(), 4, f(), 30000, 2, 2, 0.1, None) == \
        _lib.PKV_ERR_UNSUPPORTED
    L.kv_pool_destroy(h)


def _pool_i8(L, num_pages=8, page_size=16, kv_heads=2, head_dim=64, dtype=0, layers=1):
    h = ctypes.c_void_p()
    f = _fake_ptr
    st = L.kv_pool_create_i8(layers, num_pages, page_size, kv_heads, head_dim, dtype, f(), f(0x20000), f(0x30000),
                             f(0x40000), ctypes.byref(h))
    assert st == 0
    return h


def test_int8_pool_create_validates_and_reports_its_storage(L):
    h = ctypes.c_void_p()
    f = _fake_ptr
    assert L.kv_pool_create_i8(1, 8, 16, 2, 64, 0, f(), f(), None, f(), ctypes.byref(h)) == _lib.PKV_ERR_INVALID_ARG
    assert L.kv_pool_create_i8(1, 8, 16, 2, 64, 0, f(), f(), f(), f(0x10004), ctypes.byref(h)) == \
        _lib.PKV_ERR_INVALID_ARG
    assert L.kv_pool_create_i8(1, 8, 16, 2, 64, _lib.PKV_I8, f(), f(), f(), f(), ctypes.byref(h)) == \
        _lib.PKV_ERR_UNSUPPORTED          # the activation type must be fp16 or bf16
    assert L.kv_pool_create_i8(1, 8, 8, 2, 64, 0, f(), f(), f(), f(), ctypes.byref(h)) == _lib.PKV_ERR_UNSUPPORTED
    h = _pool_i8(L, dtype=1, layers=2)
    storage, dt = ctypes.c_int(), ctypes.c_int()
    assert L.kv_pool_storage(h, ctypes.byref(storage)) == 0 and storage.value == _lib.PKV_I8
    assert L.kv_pool_info(h, None, None, None, None, None, ctypes.byref(dt)) == 0 and dt.value == 1
    assert L.kv_pool_storage(None, ctypes.byref(storage)) == _lib.PKV_ERR_INVALID_ARG
    # chunked prefill reads 16-bit pages only
    assert L.paged_prefill_attention(h, 0, f(), f(), f(), 4, f(), 4, f(), 1, 2, 2, 0.1, None) == \
        _lib.PKV_ERR_UNSUPPORTED
    L.kv_pool_destroy(h)
    h = _pool(L)
    assert L.kv_pool_storage(h, ctypes.byref(storage)) == 0 and storage.value == 0
    L.kv_pool_destroy(h)


def test_int8_kv_cache_bytes():
    # 7B shape, 2048 tokens: each (token, head) row is 128 code bytes plus a 4-byte scale, for K and V
    assert pkv.pkv_kv_cache_bytes(32, 32, 128, 2048, pkv.PKV_I8) == 32 * 2 * 32 * 2048 * 132
    assert pkv.pkv_kv_cache_bytes(32, 32, 128, 2048, pkv.PKV_I8) * 2 < \
        pkv.pkv_kv_cache_bytes(32, 32, 128, 2048, pkv.PKV_F16) * 1.04


def test_fused_layer_and_rope_table_validate(L):
    f = _fake_ptr
    assert L.rope_table(f(), 4, 96, 10000.0, f(), None) == _lib.PKV_ERR_UNSUPPORTED
    assert L.rope_table(f(), 4, 128, 0.0, f(), None) == _lib.PKV_ERR_INVALID_ARG
    assert L.rope_table(f(), 4, 128, 10000.0, f(0x10008), None) == _lib.PKV_ERR_INVALID_ARG
    assert L.rope_table(None, 0, 128, 10000.0, None, None) == 0
    h = _pool(L, num_pages=8, page_size=16, kv_heads=2, head_dim=64)
    args = lambda hq, hkv: (h, 0, f(), f(), f(), f(), f(), f(), 4, f(), 1, hq, hkv, 0.1, 0, f(0x20000), 1 << 20, None)
    assert L.paged_decode_layer(*args(4, 2)) == _lib.PKV_ERR_UNSUPPORTED        # grouped heads: not fused
    assert L.paged_decode_layer(*args(3, 2)) == _lib.PKV_ERR_INVALID_ARG
    a = list(args(2, 2))
    a[5] = None                                                                  # no v
    assert L.paged_decode_layer(*a) == _lib.PKV_ERR_INVALID_ARG
    a = list(args(2, 2))
    a[1] = 1                                                                     # layer out of range
    assert L.paged_decode_layer(*a) == _lib.PKV_ERR_INVALID_ARG
    L.kv_pool_destroy(h)
    h = _pool_i8(L)
    assert L.paged_decode_layer(h, 0, f(), f(), f(), f(), f(), f(), 4, f(), 1, 32, 2, 0.1, 0, f(0x20000), 1 << 20,
                                None) == _lib.PKV_ERR_UNSUPPORTED                 # group 16: no kernel
    L.kv_pool_destroy(h)
