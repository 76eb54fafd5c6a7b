"""Paged KV cache decode step on B200 (sm_100a): thin Python binding of libpagedkv.

One autoregressive decode step of LLaMA-style attention against a paged KV cache
("为什么要自己动手写一个LLM推理引擎", wzjinhao.cn/news/61427, s3.4 paging, s4.2 RoPE,
s4.3 forward with a cache):

    rope_apply              RoPE on the new token's q and k (in place)
    pkv_slot_mapping        slot of each new token from the page table (host)
    paged_kv_append         write the new k, v into their slots
    paged_decode_attention  softmax(scale q.K^T) V over each sequence's pages

Every function here only marshals arguments (torch tensors -> raw pointers, the
current CUDA stream) and calls the C ABI of libpagedkv.so; all arithmetic of the
step runs in the library's CUDA kernels.  PyTorch provides device memory and
streams only.  Errors raise PagedKVError.
"""
import ctypes

import numpy as np

from . import _lib
from ._lib import (PKV_BF16, PKV_DEVERR_BAD_PAGE, PKV_DEVERR_BAD_SLOT, PKV_DEVERR_TIMEOUT, PKV_F16, PKV_I8,
                   PKV_MAX_DECODE_SPLITS, PagedKVError, lib)

__all__ = [
    "KVPool", "rope_apply", "paged_kv_append", "rope_append", "rope_append_step", "paged_decode_attention", "rope_table",
    "paged_decode_layer", "paged_prefill_attention", "rms_norm", "pkv_slot_mapping",
    "pkv_kv_cache_bytes", "pkv_decode_workspace_size", "pkv_decode_default_splits", "pkv_decode_auto_splits",
    "pkv_decode_cluster_size",
    "kv_get_device_error", "DecodeWorkspace", "PagedKVError", "PKV_F16", "PKV_BF16", "PKV_I8",
    "PKV_DEVERR_BAD_PAGE", "PKV_DEVERR_BAD_SLOT", "PKV_DEVERR_TIMEOUT", "PKV_MAX_DECODE_SPLITS",
]


def _torch():
    import torch
    return torch


def dtype_code(dt):
    torch = _torch()
    if dt == torch.float16:
        return PKV_F16
    if dt == torch.bfloat16:
        return PKV_BF16
    raise PagedKVError("dtype", _lib.PKV_ERR_UNSUPPORTED)


def _stream(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _need(t, name, dtype=None, cuda=True):
    if t is None:
        return
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if cuda and not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))


# ------------------------------------------------------------------ pool
class KVPool:
    """A paged KV pool over caller-owned device tensors.

    k_cache, v_cache: [num_layers, num_pages, kv_heads, page_size, head_dim], fp16 or bf16.
    For int8 pages pass int8 code tensors of that shape, fp32 scales k_scales, v_scales
    [num_layers, num_pages, kv_heads, page_size] and the activation dtype (fp16 or bf16)
    of q, k, v and the outputs.
    The host free list hands page ids out with ``alloc`` and takes them back with ``free``.
    """

    def __init__(self, k_cache, v_cache, k_scales=None, v_scales=None, dtype=None):
        torch = _torch()
        if k_cache.shape != v_cache.shape or k_cache.dtype != v_cache.dtype or k_cache.dim() != 5:
            raise ValueError("k_cache and v_cache must both be [layers, pages, kv_heads, page, head_dim]")
        _need(k_cache, "k_cache", cuda=False)
        _need(v_cache, "v_cache", cuda=False)
        self.k_cache, self.v_cache = k_cache, v_cache
        self.k_scales, self.v_scales = k_scales, v_scales
        L, N, H, P, D = k_cache.shape
        self.num_layers, self.num_pages, self.kv_heads, self.page_size, self.head_dim = L, N, H, P, D
        h = ctypes.c_void_p()
        if k_cache.dtype == torch.int8:
            if k_scales is None or v_scales is None or dtype is None:
                raise ValueError("int8 pages need k_scales, v_scales and the activation dtype")
            for t, n in ((k_scales, "k_scales"), (v_scales, "v_scales")):
                _need(t, n, torch.float32, cuda=False)
                if tuple(t.shape) != (L, N, H, P):
                    raise ValueError("%s must be [layers, pages, kv_heads, page]" % n)
            self.dtype = dtype
            self.storage = PKV_I8
            st = lib().kv_pool_create_i8(L, N, P, H, D, dtype_code(dtype), _ptr(k_cache), _ptr(v_cache),
                                         _ptr(k_scales), _ptr(v_scales), ctypes.byref(h))
            _lib.check("kv_pool_create_i8", st)
        else:
            self.dtype = k_cache.dtype
            self.storage = dtype_code(k_cache.dtype)
            st = lib().kv_pool_create(L, N, P, H, D, dtype_code(k_cache.dtype), _ptr(k_cache), _ptr(v_cache),
                                      ctypes.byref(h))
            _lib.check("kv_pool_create", st)
        self.handle = h
        del torch

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            lib().kv_pool_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def alloc(self, n):
        out = np.empty(n, np.int32)
        _lib.check("kv_pool_alloc", lib().kv_pool_alloc(self.handle, n, out.ctypes.data_as(ctypes.c_void_p)))
        return out

    def free(self, ids):
        ids = np.ascontiguousarray(ids, np.int32)
        _lib.check("kv_pool_free", lib().kv_pool_free(self.handle, ids.size, ids.ctypes.data_as(ctypes.c_void_p)))

    @property
    def free_count(self):
        return lib().kv_pool_free_count(self.handle)

    def info(self):
        vals = [ctypes.c_int() for _ in range(6)]
        _lib.check("kv_pool_info", lib().kv_pool_info(self.handle, *[ctypes.byref(v) for v in vals]))
        return tuple(v.value for v in vals)


# ------------------------------------------------------------------ host helpers
def pkv_kv_cache_bytes(num_layers, kv_heads, head_dim, tokens, dtype=PKV_F16):
    return int(lib().pkv_kv_cache_bytes(num_layers, kv_heads, head_dim, tokens, dtype))


def pkv_slot_mapping(block_tables, positions, page_size):
    """Host: int32 [n, max_pages] table and int32 [n] positions -> int64 [n] slots."""
    bt = np.ascontiguousarray(block_tables, np.int32)
    pos = np.ascontiguousarray(positions, np.int32)
    out = np.empty(pos.shape[0], np.int64)
    st = lib().pkv_slot_mapping(bt.ctypes.data_as(ctypes.c_void_p), bt.shape[1], pos.ctypes.data_as(ctypes.c_void_p),
                                pos.shape[0], page_size, out.ctypes.data_as(ctypes.c_void_p))
    _lib.check("pkv_slot_mapping", st)
    return out


def pkv_decode_default_splits(q_heads, kv_heads, head_dim, page_size, dtype=PKV_F16):
    n = ctypes.c_int()
    _lib.check("pkv_decode_default_splits",
               lib().pkv_decode_default_splits(q_heads, kv_heads, head_dim, page_size, dtype, ctypes.byref(n)))
    return n.value


def pkv_decode_auto_splits(pool, batch, max_pages_per_seq, q_heads, kv_heads=None):
    """The split count a decode call with num_splits = 0 uses on this pool and shape."""
    n = ctypes.c_int()
    _lib.check("pkv_decode_auto_splits",
               lib().pkv_decode_auto_splits(pool.handle, batch, max_pages_per_seq, q_heads,
                                            pool.kv_heads if kv_heads is None else kv_heads, ctypes.byref(n)))
    return n.value


def pkv_decode_cluster_size(pool, batch, max_pages_per_seq, q_heads, kv_heads=None):
    """Cluster size of the cluster variant that num_splits = 0 runs on this pool and shape
    (0: the partitioned kernel)."""
    n = ctypes.c_int()
    _lib.check("pkv_decode_cluster_size",
               lib().pkv_decode_cluster_size(pool.handle, batch, max_pages_per_seq, q_heads,
                                             pool.kv_heads if kv_heads is None else kv_heads, ctypes.byref(n)))
    return n.value


def pkv_decode_workspace_size(batch, q_heads, kv_heads, head_dim, num_splits):
    return int(lib().pkv_decode_workspace_size(batch, q_heads, kv_heads, head_dim, num_splits))


def kv_get_device_error():
    v = ctypes.c_uint32()
    _lib.check("kv_get_device_error", lib().kv_get_device_error(ctypes.byref(v)))
    return v.value


# ------------------------------------------------------------------ kernels
def rope_apply(q, k, positions, theta=10000.0, stream=None):
    """In-place RoPE of q [n, q_heads, d] and k [n, kv_heads, d] at positions (int32 [n])."""
    torch = _torch()
    ref = q if q is not None else k
    _need(q, "q", ref.dtype)
    _need(k, "k", ref.dtype)
    _need(positions, "positions", torch.int32)
    n = ref.shape[0]
    qh = q.shape[1] if q is not None else 0
    kh = k.shape[1] if k is not None else 0
    st = lib().rope_apply(_ptr(q), _ptr(k), _ptr(positions), n, qh, kh, ref.shape[2], float(theta),
                          dtype_code(ref.dtype), _stream(stream))
    _lib.check("rope_apply", st)


def paged_kv_append(pool, layer, k, v, slot_mapping, stream=None):
    """Write k, v [n, kv_heads, d] into the pool's slots (int64 [n], negative = skip)."""
    torch = _torch()
    _need(k, "k", pool.dtype)
    _need(v, "v", pool.dtype)
    _need(slot_mapping, "slot_mapping", torch.int64)
    st = lib().paged_kv_append(pool.handle, layer, _ptr(k), _ptr(v), _ptr(slot_mapping), k.shape[0],
                               _stream(stream))
    _lib.check("paged_kv_append", st)


def rope_append(pool, layer, q, k, v, positions, slot_mapping, theta=10000.0, stream=None):
    """RoPE on q [n, q_heads, d] and k [n, kv_heads, d] (in place), then append k and v
    into the pool's slots -- one launch, same results as rope_apply + paged_kv_append."""
    torch = _torch()
    _need(q, "q", pool.dtype)
    _need(k, "k", pool.dtype)
    _need(v, "v", pool.dtype)
    _need(positions, "positions", torch.int32)
    _need(slot_mapping, "slot_mapping", torch.int64)
    st = lib().rope_append(pool.handle, layer, _ptr(q), _ptr(k), _ptr(v), _ptr(positions), _ptr(slot_mapping),
                           k.shape[0], q.shape[1], float(theta), _stream(stream))
    _lib.check("rope_append", st)


def rope_append_step(pool, layer, q, k, v, block_tables, context_lens, theta=10000.0, stream=None):
    """The decode step's RoPE + append: sequence b's new token sits at position
    context_lens[b] - 1; q [B, q_heads, d] and k [B, kv_heads, d] are turned in place there
    and k, v written into that position's slot of the page table -- the results of
    rope_append with those positions and slots, in one launch that lets the next decode
    call (same lengths and tables) start while it runs."""
    torch = _torch()
    _need(q, "q", pool.dtype)
    _need(k, "k", pool.dtype)
    _need(v, "v", pool.dtype)
    _need(block_tables, "block_tables", torch.int32)
    _need(context_lens, "context_lens", torch.int32)
    st = lib().rope_append_step(pool.handle, layer, _ptr(q), _ptr(k), _ptr(v), _ptr(block_tables),
                                block_tables.shape[1], _ptr(context_lens), k.shape[0], q.shape[1], float(theta),
                                _stream(stream))
    _lib.check("rope_append_step", st)


def paged_prefill_attention(pool, layer, out, q, cu_q, block_tables, context_lens, scale, kv_heads=None,
                            stream=None):
    """Chunked prefill: rows cu_q[b] .. cu_q[b+1]-1 of q [total_q, q_heads, d] are the new tokens
    of sequence b at positions context_lens[b] - n_b ...; each attends causally over the pages."""
    torch = _torch()
    _need(out, "out", pool.dtype)
    _need(q, "q", pool.dtype)
    _need(cu_q, "cu_q", torch.int32)
    _need(block_tables, "block_tables", torch.int32)
    _need(context_lens, "context_lens", torch.int32)
    total_q, Hq, _ = q.shape
    st = lib().paged_prefill_attention(pool.handle, layer, _ptr(out), _ptr(q), _ptr(cu_q), total_q, _ptr(block_tables),
                                       block_tables.shape[1], _ptr(context_lens), context_lens.shape[0], Hq,
                                       pool.kv_heads if kv_heads is None else kv_heads, float(scale), _stream(stream))
    _lib.check("paged_prefill_attention", st)
    return out


def rms_norm(out, x, weight, eps=1e-6, residual=None, stream=None):
    """out = x * rsqrt(mean(x^2) + eps) * weight per row of x [rows, hidden]; with a residual,
    x + residual (rounded) is written back to the residual and normalised instead."""
    _need(out, "out", x.dtype)
    _need(x, "x", x.dtype)
    _need(weight, "weight", x.dtype)
    _need(residual, "residual", x.dtype)
    rows, hidden = x.shape
    st = lib().rms_norm(_ptr(out), _ptr(x), _ptr(residual), _ptr(weight), rows, hidden, float(eps),
                        dtype_code(x.dtype), _stream(stream))
    _lib.check("rms_norm", st)
    return out


class DecodeWorkspace:
    """Device scratch for paged_decode_attention, sized for a batch and a split count.
    Allocated zero-filled, as the kernel's per-partition counters require; every call
    leaves them at zero, and they sit in a fixed region that no call's partial results
    overlap, so the workspace serves any split count up to the one it was sized for."""

    def __init__(self, batch, q_heads, kv_heads, head_dim, page_size, dtype, num_splits=0, device=None,
                 storage=None):
        torch = _torch()
        # auto: sized for the full wave, which bounds every automatic split count, so calls
        # may pass num_splits = 0 and let the library choose
        self.auto = num_splits == 0
        if num_splits == 0:
            code = dtype_code(dtype) if storage is None else storage
            num_splits = pkv_decode_default_splits(q_heads, kv_heads, head_dim, page_size, code)
        self.num_splits = num_splits
        self.nbytes = pkv_decode_workspace_size(batch, q_heads, kv_heads, head_dim, num_splits)
        self.buffer = torch.zeros(self.nbytes, dtype=torch.uint8, device=device or "cuda")


def paged_decode_attention(pool, layer, out, q, block_tables, context_lens, scale, kv_heads=None,
                           num_splits=0, workspace=None, stream=None):
    """out[b, h] = softmax(scale * q[b, h] . K_b^T) V_b over context_lens[b] paged tokens."""
    torch = _torch()
    _need(out, "out", pool.dtype)
    _need(q, "q", pool.dtype)
    _need(block_tables, "block_tables", torch.int32)
    _need(context_lens, "context_lens", torch.int32)
    B, Hq, _ = q.shape
    if kv_heads is None:
        kv_heads = pool.kv_heads
    if workspace is None:
        workspace = DecodeWorkspace(B, Hq, kv_heads, pool.head_dim, pool.page_size, pool.dtype, num_splits,
                                    device=q.device, storage=pool.storage)
    if num_splits == 0 and not workspace.auto:
        num_splits = workspace.num_splits
    st = lib().paged_decode_attention(pool.handle, layer, _ptr(out), _ptr(q), _ptr(block_tables),
                                      block_tables.shape[1], _ptr(context_lens), B, Hq, kv_heads, float(scale),
                                      num_splits, _ptr(workspace.buffer), workspace.nbytes, _stream(stream))
    _lib.check("paged_decode_attention", st)
    return out


def rope_table(context_lens, head_dim, theta=10000.0, table=None, stream=None):
    """(cos, sin) of each sequence's new-token angles, float64 [batch, head_dim / 2, 2] on the
    device, for paged_decode_layer (position = context_lens[b] - 1)."""
    torch = _torch()
    _need(context_lens, "context_lens", torch.int32)
    B = context_lens.shape[0]
    if table is None:
        table = torch.empty((B, head_dim // 2, 2), dtype=torch.float64, device=context_lens.device)
    _need(table, "table", torch.float64)
    _lib.check("rope_table", lib().rope_table(_ptr(context_lens), B, head_dim, float(theta), _ptr(table),
                                              _stream(stream)))
    return table


def paged_decode_layer(pool, layer, out, q, k, v, rope, block_tables, context_lens, scale, num_splits=0,
                       workspace=None, stream=None):
    """One decode layer in one launch: RoPE on q [B, Hq, d] and k [B, Hkv, d] (inputs left
    unchanged), k and v appended at position context_lens[b] - 1, and out = attention over the
    context_lens[b] tokens.  rope: the step's rope_table."""
    torch = _torch()
    for t, n in ((out, "out"), (q, "q"), (k, "k"), (v, "v")):
        _need(t, n, pool.dtype)
    _need(rope, "rope", torch.float64)
    _need(block_tables, "block_tables", torch.int32)
    _need(context_lens, "context_lens", torch.int32)
    B, Hq, _ = q.shape
    if workspace is None:
        workspace = DecodeWorkspace(B, Hq, pool.kv_heads, pool.head_dim, pool.page_size, pool.dtype, num_splits,
                                    device=q.device, storage=pool.storage)
    if num_splits == 0 and not workspace.auto:
        num_splits = workspace.num_splits
    st = lib().paged_decode_layer(pool.handle, layer, _ptr(out), _ptr(q), _ptr(k), _ptr(v), _ptr(rope),
                                  _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), B, Hq, pool.kv_heads,
                                  float(scale), num_splits, _ptr(workspace.buffer), workspace.nbytes, _stream(stream))
    _lib.check("paged_decode_layer", st)
    return out
