"""A whole decode step over all layers, captured once in a CUDA graph.

"为什么要自己动手写一个LLM推理引擎" (wzjinhao.cn/news/61427) s5.3 names per-call launch
and CPU-sync overhead as a decode bottleneck.  DecodeStep issues every layer's
RoPE + KV append (one fused kernel) and paged attention (one kernel) from one
CUDA graph, so a step costs one graph launch instead of two kernel launches per
layer from Python.  The graph
reads fixed device buffers; `run` copies a step's inputs from (pinned) host memory
into them, replays the graph and copies the outputs back.  With pinned host buffers
the copies are part of a second graph and overlap the kernels: the layers' q, k, v go
in on a copy stream in chunks ahead of the compute, and the outputs go back on another
stream in chunks as their kernels finish.  All arithmetic stays in the library's kernels; this module only orders the
calls and copies.
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
        self.host_graphs = {}                 # pinned host buffers (data pointers) -> pipelined graph

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

    def _pinned(self, *ts):
        return all(isinstance(t, torch.Tensor) and t.device.type == "cpu" and t.is_pinned() and t.is_contiguous()
                   for t in ts)

    @staticmethod
    def _chunks(L, growth=4):
        """Layer ranges [lo, hi) of growing length: 1, 4, 16, ... layers (a layer's rows copy
        several times faster than its kernels run, so each chunk lands before its first layer)."""
        out, lo, n = [], 0, 1
        while lo < L:
            out.append((lo, min(L, lo + n)))
            lo, n = lo + n, growth * n
        return out

    def capture_host(self, q, k, v, out_host):
        """Record the step with its host copies (pinned q, k, v, out_host of the device
        buffers' shapes) into one graph.  A copy stream brings the layers' rows in by chunks of
        growing length (layer 0, then 1-4, 5-20, ...), each chunk's copy running while the
        kernels of the chunks before it work, and the compute stream waits for a chunk only at
        its first layer; the outputs go back on a third stream in chunks that shrink toward the
        last layer, each once its last kernel is done.  Few waits keep most of the layer
        kernels' programmatic launches chained.  Run the step once outside any capture first
        (`eager` or `capture`)."""
        L = self.pool.num_layers
        if self.graph is None:
            self.capture()
        torch.cuda.synchronize()
        main, h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ins = self._chunks(L)
        outs = [(L - hi, L - lo) for lo, hi in reversed(self._chunks(L))]
        got = {lo: torch.cuda.Event() for lo, _ in ins}
        g = torch.cuda.CUDAGraph()
        main.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(main):
            with torch.cuda.graph(g, stream=main):
                h2d.wait_stream(main)                       # fork the copy streams into the capture
                d2h.wait_stream(main)
                with torch.cuda.stream(h2d):
                    for lo, hi in ins:
                        self.q[lo:hi].copy_(q[lo:hi], non_blocking=True)
                        self.k[lo:hi].copy_(k[lo:hi], non_blocking=True)
                        self.v[lo:hi].copy_(v[lo:hi], non_blocking=True)
                        got[lo].record(h2d)
                if self.fused:
                    rope_table(self.context_lens, self.pool.head_dim, self.theta, table=self.rope)
                ends = {hi - 1: (lo, hi) for lo, hi in outs}
                for i in range(L):
                    if i in got:
                        main.wait_event(got[i])
                    self.layer(i)
                    if i in ends:
                        lo, hi = ends[i]
                        done = torch.cuda.Event()
                        done.record(main)
                        d2h.wait_event(done)
                        with torch.cuda.stream(d2h):
                            out_host[lo:hi].copy_(self.out[lo:hi], non_blocking=True)
                main.wait_stream(h2d)                       # join
                main.wait_stream(d2h)
        torch.cuda.current_stream().wait_stream(main)
        key = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out_host.data_ptr())
        self.host_graphs[key] = g
        return g

    def run(self, q, k, v, out_host=None):
        """Copy the step's q, k, v (host, ideally pinned) in, replay, copy out to out_host.
        Pinned host buffers of the step's shapes (all four) take the pipelined graph, captured
        on their first use; other inputs are copied in, then the step graph replays."""
        if out_host is not None and self._pinned(q, k, v, out_host) and q.shape == self.q.shape and \
                k.shape == self.k.shape and v.shape == self.v.shape and out_host.shape == self.out.shape and \
                q.dtype == k.dtype == v.dtype == out_host.dtype == self.q.dtype:
            key = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out_host.data_ptr())
            g = self.host_graphs.get(key)
            if g is None:
                g = self.capture_host(q, k, v, out_host)
            g.replay()
            return out_host
        if self.graph is None:
            # capture first: its eager pass runs on the buffers as they are, so this step's
            # inputs go through the kernels once (the two-launch path turns q in place)
            self.capture()
        self.q.copy_(q, non_blocking=True)
        self.k.copy_(k, non_blocking=True)
        self.v.copy_(v, non_blocking=True)
        self.graph.replay()
        if out_host is not None:
            out_host.copy_(self.out, non_blocking=True)
        return out_host
