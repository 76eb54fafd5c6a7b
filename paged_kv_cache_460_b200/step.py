"""A whole decode step over all layers, captured once in a CUDA graph.

"为什么要自己动手写一个LLM推理引擎" (wzjinhao.cn/news/61427) s5.3 names per-call launch
and CPU-sync overhead as a decode bottleneck.  DecodeStep issues every layer's
RoPE + KV append (one fused kernel) and paged attention (one kernel) from one
CUDA graph, so a step costs one graph launch instead of two kernel launches per
layer from Python.  The graph
reads fixed device buffers; `run` copies a step's inputs from (pinned) host memory
into them, replays the graph and copies the outputs back.  All arithmetic stays in
the library's kernels; this module only orders the calls.
"""
import math

import torch

from . import (DecodeWorkspace, KVPool, paged_decode_attention, paged_decode_layer, rope_append_step, rope_table)


class DecodeStep:
    """One decode step (all layers) of a fixed batch shape on a paged pool.

    pool: KVPool over [layers, pages, kv_heads, page_size, head_dim] caches.
    batch, q_heads: the step's shape; the kv heads and head_dim are the pool's.
    Device buffers (fill them, or pass host tensors to ``run``):
      q [layers, batch, q_heads, d], k and v [layers, batch, kv_heads, d],
      block_tables [batch, max_pages] int32, context_lens [batch] int32 (the new token
      included: it sits at position context_lens[b] - 1, in the slot the page table gives
      that position), out [layers, batch, q_heads, d].
    """

    def __init__(self, pool: KVPool, batch, q_heads, max_pages, scale=None, theta=10000.0, num_splits=0,
                 device=None, fused=False):
        self.pool = pool
        dev = torch.device(device) if device is not None else pool.k_cache.device
        L, d, Hkv = pool.num_layers, pool.head_dim, pool.kv_heads
        dt = pool.dtype
        self.q = torch.zeros((L, batch, q_heads, d), dtype=dt, device=dev)
        self.k = torch.zeros((L, batch, Hkv, d), dtype=dt, device=dev)
        self.v = torch.zeros((L, batch, Hkv, d), dtype=dt, device=dev)
        self.out = torch.empty((L, batch, q_heads, d), dtype=dt, device=dev)
        self.block_tables = torch.full((batch, max_pages), -1, dtype=torch.int32, device=dev)
        self.context_lens = torch.zeros(batch, dtype=torch.int32, device=dev)
        self.scale = 1.0 / math.sqrt(d) if scale is None else scale
        self.theta = theta
        self.num_splits = num_splits          # 0: the library's automatic choice for the shape
        self.workspace = DecodeWorkspace(batch, q_heads, Hkv, d, pool.page_size, dt, num_splits, device=dev,
                                         storage=pool.storage)
        self.graph = None
        # fused: one angle-table launch per step, then one launch per layer (RoPE, append and
        # attention together); otherwise RoPE + append and attention, two launches per layer
        self.fused = fused
        self.rope = torch.zeros((batch, d // 2, 2), dtype=torch.float64, device=dev) if fused else None
        self.kernels_per_step = (1 + L) if fused else 2 * L

    def layer(self, i, stream=None):
        """Enqueue layer i of the step on the current stream: RoPE + KV append (one
        kernel, each sequence's new token at position context_lens[b] - 1 and its slot
        taken from the page table), then attention (one kernel); fused: the whole layer in
        one kernel (the step's angle table must be current)."""
        if self.fused:
            paged_decode_layer(self.pool, i, self.out[i], self.q[i], self.k[i], self.v[i], self.rope,
                               self.block_tables, self.context_lens, self.scale,
                               num_splits=self.num_splits, workspace=self.workspace, stream=stream)
            return
        rope_append_step(self.pool, i, self.q[i], self.k[i], self.v[i], self.block_tables, self.context_lens,
                         self.theta, stream)
        paged_decode_attention(self.pool, i, self.out[i], self.q[i], self.block_tables, self.context_lens,
                               self.scale, num_splits=self.num_splits, workspace=self.workspace,
                               stream=stream)

    def eager(self):
        if self.fused:
            rope_table(self.context_lens, self.pool.head_dim, self.theta, table=self.rope)
        for i in range(self.pool.num_layers):
            self.layer(i)

    def capture(self):
        """Record the step into a CUDA graph (run it eagerly once first, outside any capture)."""
        self.eager()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                self.eager()
        torch.cuda.current_stream().wait_stream(s)
        self.graph = g
        return g

    def replay(self):
        if self.graph is None:
            self.capture()
        self.graph.replay()

    def set_metadata(self, block_tables, context_lens, non_blocking=True):
        """Copy the page tables and lengths in (host or device tensors); each sequence's new
        token position and its slot follow from them on the device."""
        self.block_tables.copy_(torch.as_tensor(block_tables), non_blocking=non_blocking)
        self.context_lens.copy_(torch.as_tensor(context_lens), non_blocking=non_blocking)

    def run(self, q, k, v, out_host=None):
        """Copy the step's q, k, v (host, ideally pinned) in, replay, copy out to out_host."""
        self.q.copy_(q, non_blocking=True)
        self.k.copy_(k, non_blocking=True)
        self.v.copy_(v, non_blocking=True)
        self.replay()
        if out_host is not None:
            out_host.copy_(self.out, non_blocking=True)
        return out_host
