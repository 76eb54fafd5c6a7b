"""fp64 CPU oracle for the paged decode step -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does, and this
package imports nothing from the product: both sides meet only in the seeded
input generator (``synth``), which holds none of the method's arithmetic.

Every function takes and returns numpy arrays.  Storage tensors are uint16 bit
patterns (IEEE binary16 or bfloat16, selected by ``dtype`` = "f16" / "bf16");
results are float64 before any rounding.  The arithmetic lives in oracle.c,
each routine there citing the page and section it follows.

Pins (tests/test_oracle_pins.py): format codecs against numpy/torch on all 2^16
patterns and brute-force nearest search; attention against a pure-Python brute
force, the last row of full causal recompute, softmax row sums, the one-token
and identical-key closed forms, page-permutation invariance and a peaked-key
limit; RoPE against its identity/closed-form/relative-position properties;
append and slot mapping against a brute-force scan; KV bytes against the
figure the pages print.
"""
import ctypes
import numpy as np

from . import build as _build

_DT = {"f16": 0, "bf16": 1}

_libs = {}


def _load(omp=False):
    """The plain build, or (omp=True) the OpenMP build whose pair routines use every core."""
    if omp not in _libs:
        path = _build.build(omp=omp)
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        I64 = ctypes.c_int64
        lib.ora_half_to_double.argtypes = [ctypes.c_uint16]
        lib.ora_half_to_double.restype = D
        lib.ora_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.ora_bf16_to_double.restype = D
        lib.ora_double_to_half.argtypes = [D]
        lib.ora_double_to_half.restype = ctypes.c_uint16
        lib.ora_double_to_bf16.argtypes = [D]
        lib.ora_double_to_bf16.restype = ctypes.c_uint16
        lib.ora_decode_array.argtypes = [P, P, I64, I]
        lib.ora_encode_array.argtypes = [P, P, I64, I]
        lib.ora_rope_f64.argtypes = [P, P, P, I, I, I, D]
        lib.ora_rope.argtypes = [P, P, P, P, I, I, I, D, I]
        lib.ora_slot_mapping.argtypes = [P, I, P, I, I, P]
        lib.ora_kv_append.argtypes = [P, P, P, P, P, I, P, I, I, I, I]
        lib.ora_decode_attention.argtypes = [P, P, P, P, I, P, I, I, I, I, I, D, I, P, P, I]
        lib.ora_decode_attention_pairs.argtypes = [P, P, P, P, I, P, I, I, I, I, D, I, P, P, I, P]
        lib.ora_causal_attention_full.argtypes = [P, P, P, I, I, I, I, D, P]
        lib.ora_rms_norm.argtypes = [P, P, P, I, I, D, I, P, P, P]
        lib.ora_prefill_attention.argtypes = [P, P, P, P, I, P, P, I, I, I, I, I, D, I, P]
        lib.ora_quantize_row_i8.argtypes = [P, I, I, P, P]
        lib.ora_kv_append_i8.argtypes = [P, P, P, P, P, P, P, I, P, I, I, I, I, I]
        lib.ora_decode_attention_i8_pairs.argtypes = [P, P, P, P, P, P, I, P, I, I, I, I, D, I, P, P, I, P]
        lib.ora_kv_cache_bytes.argtypes = [I, I, I, I64, I]
        lib.ora_kv_cache_bytes.restype = I64
        lib.ora_set_threads.argtypes = [I]
        lib.ora_set_threads.restype = I
        _libs[omp] = lib
    return _libs[omp]


def set_threads(n):
    """Threads of the OpenMP build's pair routines (n >= 1); returns the count in force."""
    return int(_load(omp=True).ora_set_threads(int(n)))


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ----------------------------------------------------------------- formats
def decode(bits, dtype):
    """uint16 storage bits -> float64 values."""
    bits = _c(bits, np.uint16)
    out = np.empty(bits.shape, np.float64)
    _load().ora_decode_array(_p(bits), _p(out), bits.size, _DT[dtype])
    return out


def encode(values, dtype):
    """float64 -> uint16 storage bits, one round-to-nearest-even step."""
    values = _c(values, np.float64)
    out = np.empty(values.shape, np.uint16)
    _load().ora_encode_array(_p(values), _p(out), values.size, _DT[dtype])
    return out


# ----------------------------------------------------------------- RoPE
def rope_f64(x, positions, theta):
    """x: float64 [n, heads, d] -> rotated float64, no rounding."""
    x = _c(x, np.float64)
    n, heads, d = x.shape
    pos = _c(positions, np.int32)
    y = np.empty_like(x)
    _load().ora_rope_f64(_p(x), _p(y), _p(pos), n, heads, d, float(theta))
    return y


def rope(x_bits, positions, theta, dtype):
    """Storage-level RoPE: returns (rounded uint16 bits, exact float64)."""
    x_bits = _c(x_bits, np.uint16)
    n, heads, d = x_bits.shape
    pos = _c(positions, np.int32)
    y = np.empty_like(x_bits)
    exact = np.empty(x_bits.shape, np.float64)
    _load().ora_rope(_p(x_bits), _p(y), _p(exact), _p(pos), n, heads, d, float(theta), _DT[dtype])
    return y, exact


# ----------------------------------------------------------------- page table
def slot_mapping(block_tables, positions, page_size):
    bt = _c(block_tables, np.int32)
    pos = _c(positions, np.int32)
    out = np.empty(pos.shape[0], np.int64)
    _load().ora_slot_mapping(_p(bt), bt.shape[1], _p(pos), pos.shape[0], page_size, _p(out))
    return out


def kv_append(k_pool, v_pool, k, v, block_tables, positions):
    """Returns updated copies of the one-layer pools [pages, kvh, P, d] (uint16)."""
    kp = np.array(k_pool, dtype=np.uint16, copy=True, order="C")
    vp = np.array(v_pool, dtype=np.uint16, copy=True, order="C")
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    bt = _c(block_tables, np.int32)
    pos = _c(positions, np.int32)
    _, kvh, P, d = kp.shape
    _load().ora_kv_append(_p(kp), _p(vp), _p(k), _p(v), _p(bt), bt.shape[1], _p(pos),
                          pos.shape[0], kvh, P, d)
    return kp, vp


# ----------------------------------------------------------------- attention
def decode_attention(q, k_pool, v_pool, block_tables, context_lens, scale, dtype,
                     return_weights=False):
    """q: uint16 [B, Hq, d]; pools: uint16 [pages, Hkv, P, d] (one layer).

    Returns float64 [B, Hq, d] (and the softmax weights [B, Hq, max_len] when asked).
    """
    q = _c(q, np.uint16)
    kp = _c(k_pool, np.uint16)
    vp = _c(v_pool, np.uint16)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    B, Hq, d = q.shape
    _, Hkv, P, _ = kp.shape
    out = np.empty((B, Hq, d), np.float64)
    max_len = int(cl.max()) if (return_weights and cl.size) else 0
    w = np.empty((B, Hq, max(max_len, 1)), np.float64) if return_weights else None
    _load().ora_decode_attention(_p(q), _p(kp), _p(vp), _p(bt), bt.shape[1], _p(cl), B, Hq, Hkv,
                                 d, P, float(scale), _DT[dtype], _p(out),
                                 _p(w) if w is not None else None, max_len)
    if return_weights:
        return out, w[:, :, :max_len]
    return out


def decode_attention_pairs(q, k_pool, v_pool, block_tables, context_lens, scale, dtype, pairs, omp=False):
    """Same arithmetic for selected (b, h) pairs only; returns float64 [n_pairs, d].
    omp=True runs the pairs on all cores (OpenMP build; each pair's arithmetic unchanged)."""
    q = _c(q, np.uint16)
    kp = _c(k_pool, np.uint16)
    vp = _c(v_pool, np.uint16)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    _, Hq, d = q.shape
    _, Hkv, P, _ = kp.shape
    pairs = np.asarray(pairs, dtype=np.int64).reshape(-1, 2)
    pb = _c(pairs[:, 0], np.int32)
    ph = _c(pairs[:, 1], np.int32)
    out = np.empty((pairs.shape[0], d), np.float64)
    _load(omp).ora_decode_attention_pairs(_p(q), _p(kp), _p(vp), _p(bt), bt.shape[1], _p(cl), Hq, Hkv,
                                       d, P, float(scale), _DT[dtype], _p(pb), _p(ph),
                                       pairs.shape[0], _p(out))
    return out


def causal_attention_full(q, k, v, scale):
    """q: float64 [T, Hq, d], k/v: float64 [T, Hkv, d] -> float64 [T, Hq, d]."""
    q = _c(q, np.float64)
    k = _c(k, np.float64)
    v = _c(v, np.float64)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    out = np.empty((T, Hq, d), np.float64)
    _load().ora_causal_attention_full(_p(q), _p(k), _p(v), T, Hq, Hkv, d, float(scale), _p(out))
    return out


def kv_cache_bytes(layers, heads, head_dim, tokens, elt_bytes):
    return int(_load().ora_kv_cache_bytes(layers, heads, head_dim, tokens, elt_bytes))


# ----------------------------------------------------------------- RMSNorm
def rms_norm(x, w, eps, dtype, residual=None):
    """x: uint16 [rows, hidden]; w: uint16 [hidden].  Returns (rounded bits, exact float64,
    rounded residual sums or None)."""
    x = _c(x, np.uint16)
    w = _c(w, np.uint16)
    rows, hidden = x.shape
    out = np.empty_like(x)
    exact = np.empty(x.shape, np.float64)
    res = _c(residual, np.uint16) if residual is not None else None
    res_out = np.empty_like(x) if residual is not None else None
    _load().ora_rms_norm(_p(x), _p(res) if res is not None else None, _p(w), rows, hidden, float(eps),
                         _DT[dtype], _p(out), _p(exact), _p(res_out) if res_out is not None else None)
    return out, exact, res_out


# ----------------------------------------------------------------- chunked prefill
def prefill_attention(q, k_pool, v_pool, block_tables, cu_q, context_lens, scale, dtype):
    """q: uint16 [total_q, Hq, d]; query rows of sequence b are cu_q[b] .. cu_q[b+1]-1 and
    sit at positions context_lens[b] - n_b ... context_lens[b] - 1.  Returns float64."""
    q = _c(q, np.uint16)
    kp = _c(k_pool, np.uint16)
    vp = _c(v_pool, np.uint16)
    bt = _c(block_tables, np.int32)
    cq = _c(cu_q, np.int32)
    cl = _c(context_lens, np.int32)
    total, Hq, d = q.shape
    _, Hkv, P, _ = kp.shape
    out = np.zeros((total, Hq, d), np.float64)
    _load().ora_prefill_attention(_p(q), _p(kp), _p(vp), _p(bt), bt.shape[1], _p(cq), _p(cl), cl.shape[0], Hq,
                                  Hkv, d, P, float(scale), _DT[dtype], _p(out))
    return out


# ----------------------------------------------------------------- int8 KV pages
def quantize_rows_i8(x, dtype):
    """x: uint16 [..., d] storage rows -> (int8 codes [..., d], float32 scales [...])."""
    x = _c(x, np.uint16)
    d = x.shape[-1]
    flat = x.reshape(-1, d)
    codes = np.empty(flat.shape, np.int8)
    scales = np.empty(flat.shape[0], np.float32)
    lib = _load()
    for r in range(flat.shape[0]):
        lib.ora_quantize_row_i8(_p(flat[r]), d, _DT[dtype], _p(codes[r]), _p(scales[r:r + 1]))
    return codes.reshape(x.shape), scales.reshape(x.shape[:-1])


def kv_append_i8(k_codes, v_codes, k_scales, v_scales, k, v, block_tables, positions, dtype):
    """Quantising append into copies of one layer's int8 pool (codes [pages, Hkv, P, d],
    scales [pages, Hkv, P])."""
    kc = np.array(k_codes, dtype=np.int8, copy=True, order="C")
    vc = np.array(v_codes, dtype=np.int8, copy=True, order="C")
    ks = np.array(k_scales, dtype=np.float32, copy=True, order="C")
    vs = np.array(v_scales, dtype=np.float32, copy=True, order="C")
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    bt = _c(block_tables, np.int32)
    pos = _c(positions, np.int32)
    _, kvh, P, d = kc.shape
    _load().ora_kv_append_i8(_p(kc), _p(vc), _p(ks), _p(vs), _p(k), _p(v), _p(bt), bt.shape[1], _p(pos),
                             pos.shape[0], kvh, P, d, _DT[dtype])
    return kc, vc, ks, vs


def decode_attention_i8_pairs(q, k_codes, v_codes, k_scales, v_scales, block_tables, context_lens, scale, dtype,
                              pairs, omp=False):
    """Decode attention of selected (b, h) pairs over an int8 pool (k = code * scale exactly
    in fp64); omp=True runs the pairs on all cores.  Returns float64 [n_pairs, d]."""
    q = _c(q, np.uint16)
    kc = _c(k_codes, np.int8)
    vc = _c(v_codes, np.int8)
    ks = _c(k_scales, np.float32)
    vs = _c(v_scales, np.float32)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    _, Hq, d = q.shape
    _, Hkv, P, _ = kc.shape
    pairs = np.asarray(pairs, dtype=np.int64).reshape(-1, 2)
    pb = _c(pairs[:, 0], np.int32)
    ph = _c(pairs[:, 1], np.int32)
    out = np.empty((pairs.shape[0], d), np.float64)
    _load(omp).ora_decode_attention_i8_pairs(_p(q), _p(kc), _p(vc), _p(ks), _p(vs), _p(bt), bt.shape[1], _p(cl), Hq,
                                          Hkv, d, P, float(scale), _DT[dtype], _p(pb), _p(ph), pairs.shape[0],
                                          _p(out))
    return out
