"""Seeded synthetic inputs for one paged decode step.

This module is shared by the tests, the smoke check and the benchmark, and by
both sides of every parity check: it feeds the same bits to the CUDA library
and to the fp64 oracle.  It holds none of the method's arithmetic -- no RoPE,
no slot computation, no attention -- only the shapes, value distributions and
page-allocation structure of the five decode workloads:

  tiny      batch 1, 4 heads, head_dim 64, 40 cached tokens, 16-token pages drawn
            from a seeded permutation of an 8-page pool, fp16
  layer7b   batch 1, 32 q/kv heads, head_dim 128, 2048 cached tokens, 16-token
            pages from a shuffled 256-page pool, fp16
  batch10   batch 10, 32 layers each with its own cache, 32 heads, head_dim 128,
            cached lengths uniform in [128, 2048], 16-token pages handed out
            round-robin across the requests (interleaved), fp16
  cbatch    batch 64, 32 q heads / 8 kv heads, head_dim 128, cached lengths
            lognormal (median 1024, sigma 1, capped at 8192), 32-token pages;
            every request is allocated, a seeded 30% are freed, the free list is
            shuffled and replacements are allocated from it, bf16
  longctx   batch 4, 32768 cached tokens each, 32 heads, head_dim 128, 16-token
            pages from a shuffled pool, fp16, 1% of (sequence, token) keys scaled x8

Every value is drawn in fp32 from N(0, 1) and rounded once, to nearest-even,
to the storage type.  Seeds: values PCG64(460 + index), allocation
PCG64(1460 + index), index = position of the workload in the list above.
Large pools (a few GB) are filled on the GPU by torch's seeded Philox
generator (``pool_backend="torch"``); small ones by numpy PCG64.

"cached" lengths count the tokens already in the cache; the decode step
appends one token at position cached_len, so the attention then covers
cached_len + 1 tokens.  Block-table entries past a sequence's pages are -1.
"""
from dataclasses import dataclass, field
import math

import numpy as np

WORKLOADS = ("tiny", "layer7b", "batch10", "cbatch", "longctx")
DT_BYTES = {"f16": 2, "bf16": 2}


@dataclass
class DecodeSpec:
    name: str
    index: int
    batch: int
    q_heads: int
    kv_heads: int
    head_dim: int
    page_size: int
    num_layers: int
    num_pages: int
    dtype: str
    theta: float
    cached_lens: np.ndarray          # int32 [B]
    block_tables: np.ndarray         # int32 [B, max_pages], -1 padded
    peaky_keys: float = 0.0          # fraction of (b, token) keys scaled x8
    notes: dict = field(default_factory=dict)

    @property
    def context_lens(self):
        """Tokens attended after the append (cached + the new one); 0 for empty rows."""
        cl = self.cached_lens.astype(np.int64) + 1
        cl[self.cached_lens < 0] = 0
        return cl.astype(np.int32)

    @property
    def positions(self):
        """Position of the new token of each row (-1 for a padded row)."""
        return self.cached_lens.astype(np.int32)

    @property
    def max_pages(self):
        return self.block_tables.shape[1]

    @property
    def elt_bytes(self):
        return DT_BYTES[self.dtype]

    def kv_bytes_read(self):
        """Algorithmic K+V bytes one attention call over one layer must read."""
        return int(self.context_lens.astype(np.int64).sum()) * 2 * self.kv_heads * self.head_dim * self.elt_bytes

    def pool_shape(self):
        return (self.num_layers, self.num_pages, self.kv_heads, self.page_size, self.head_dim)


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _pages_needed(cached, P):
    return (cached + 1 + P - 1) // P      # after the append


def _table(lists, width):
    bt = np.full((len(lists), width), -1, np.int32)
    for b, pages in enumerate(lists):
        bt[b, :len(pages)] = pages
    return bt


def _round_robin(need, free_list, order_rng):
    """Hand out pages from the head of free_list, one per request per round, the
    requests taking turns in a seeded order each round."""
    owned = [[] for _ in need]
    head = 0
    while any(len(o) < n for o, n in zip(owned, need)):
        for b in order_rng.permutation(len(need)):
            if len(owned[b]) < need[b]:
                owned[b].append(int(free_list[head]))
                head += 1
    return owned, head


def spec(name, num_layers=None):
    """Shapes, lengths and page tables of one named workload (no values)."""
    idx = WORKLOADS.index(name)
    arng = _rng(1460 + idx)
    if name == "tiny":
        P, cached = 16, np.array([40], np.int32)
        perm = arng.permutation(8)
        n = _pages_needed(40, P)
        s = DecodeSpec(name, idx, 1, 4, 4, 64, P, 1, 8, "f16", 10000.0, cached,
                       _table([perm[:n]], n))
    elif name == "layer7b":
        P, cached = 16, np.array([2048], np.int32)
        perm = arng.permutation(256)
        n = _pages_needed(2048, P)
        s = DecodeSpec(name, idx, 1, 32, 32, 128, P, 1, 256, "f16", 10000.0, cached,
                       _table([perm[:n]], n))
    elif name == "batch10":
        P, B = 16, 10
        cached = arng.integers(128, 2048, size=B, endpoint=True).astype(np.int32)
        need = [_pages_needed(int(c), P) for c in cached]
        num_pages = int(sum(need))
        owned, _ = _round_robin(need, np.arange(num_pages), arng)
        s = DecodeSpec(name, idx, B, 32, 32, 128, P, 32 if num_layers is None else num_layers,
                       num_pages, "f16", 10000.0, cached, _table(owned, max(need)))
    elif name == "cbatch":
        P, B = 32, 64

        def draw(n):
            x = np.rint(arng.lognormal(mean=math.log(1024.0), sigma=1.0, size=n))
            return np.clip(x, 1, 8192).astype(np.int32)

        first = draw(B)
        need0 = [_pages_needed(int(c), P) for c in first]
        freed = np.sort(arng.choice(B, size=int(round(0.3 * B)), replace=False))
        repl = draw(len(freed))
        need_r = [_pages_needed(int(c), P) for c in repl]
        num_pages = int(sum(need0) + sum(need_r))
        owned, head = _round_robin(need0, np.arange(num_pages), arng)
        free_list = [p for b in freed for p in owned[b]] + list(range(head, num_pages))
        free_list = list(arng.permutation(np.array(free_list, np.int64)))
        cached = first.copy()
        for k, b in enumerate(freed):
            cached[b] = repl[k]
            owned[b] = [int(free_list.pop(0)) for _ in range(need_r[k])]
        width = max(len(o) for o in owned)
        s = DecodeSpec(name, idx, B, 32, 8, 128, P, 1, num_pages, "bf16", 10000.0, cached,
                       _table(owned, width), notes={"freed_and_reallocated": [int(b) for b in freed]})
    elif name == "longctx":
        P, B = 16, 4
        cached = np.full(B, 32768, np.int32)
        n = _pages_needed(32768, P)
        num_pages = B * n + 4
        perm = arng.permutation(num_pages)
        s = DecodeSpec(name, idx, B, 32, 32, 128, P, 1, num_pages, "f16", 10000.0, cached,
                       _table([perm[b * n:(b + 1) * n] for b in range(B)], n), peaky_keys=0.01)
    else:
        raise ValueError(name)
    if num_layers is not None:
        s.num_layers = num_layers
    return s


def random_spec(seed, batch, q_heads, kv_heads, head_dim, page_size, cached_lens, dtype="f16",
                extra_pages=3, num_layers=1, table_slack=1, theta=10000.0):
    """A small case with the given cached lengths (-1 = padded row); pages are a
    seeded permutation of a pool slightly larger than needed."""
    rng = _rng(seed)
    cached = np.asarray(cached_lens, np.int32)
    need = [0 if c < 0 else _pages_needed(int(c), page_size) for c in cached]
    num_pages = int(sum(need)) + extra_pages
    perm = rng.permutation(num_pages)
    lists, o = [], 0
    for n in need:
        lists.append(perm[o:o + n])
        o += n
    width = max(max(need) if need else 1, 1) + table_slack
    return DecodeSpec("random", -1, len(cached), q_heads, kv_heads, head_dim, page_size,
                      num_layers, num_pages, dtype, theta, cached, _table(lists, width))


# ----------------------------------------------------------------- values
def round_f32(x, dtype):
    """fp32 array -> uint16 storage bits, round to nearest-even."""
    x = np.ascontiguousarray(x, np.float32)
    if dtype == "f16":
        return x.astype(np.float16).view(np.uint16)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def value_seed(s):
    return 460 + s.index if s.index >= 0 else 7919


def step_values(s, seed=None):
    """q, k, v of the new token for every layer: uint16 [layers, B, H, d]."""
    rng = _rng(value_seed(s) if seed is None else seed)
    L, B, d = s.num_layers, s.batch, s.head_dim
    q = round_f32(rng.standard_normal((L, B, s.q_heads, d), dtype=np.float32), s.dtype)
    k = round_f32(rng.standard_normal((L, B, s.kv_heads, d), dtype=np.float32), s.dtype)
    v = round_f32(rng.standard_normal((L, B, s.kv_heads, d), dtype=np.float32), s.dtype)
    return q, k, v


def _peaky_rows(s, rng):
    """(b, token) pairs whose keys are scaled x8, and where they live."""
    rows = []
    for b in range(s.batch):
        L = int(s.cached_lens[b])
        if L <= 0:
            continue
        hit = np.nonzero(rng.random(L) < s.peaky_keys)[0]
        for t in hit:
            rows.append((b, int(t), int(s.block_tables[b, t // s.page_size]), int(t % s.page_size)))
    return rows


def pool_values_numpy(s, seed=None):
    """K and V pools, uint16 [layers, pages, Hkv, P, d], numpy PCG64."""
    rng = _rng((value_seed(s) if seed is None else seed) + 1_000_000)
    shape = s.pool_shape()
    kf = rng.standard_normal(shape, dtype=np.float32)
    vf = rng.standard_normal(shape, dtype=np.float32)
    if s.peaky_keys > 0:
        for (_, _, page, row) in _peaky_rows(s, rng):
            kf[:, page, :, row, :] *= 8.0
    return round_f32(kf, s.dtype), round_f32(vf, s.dtype)


def pool_values_torch(s, device, seed=None):
    """K and V pools as torch tensors on `device` ([layers, pages, Hkv, P, d],
    fp16/bf16), filled layer by layer from torch's seeded generator."""
    import torch
    tdt = torch.float16 if s.dtype == "f16" else torch.bfloat16
    base = (value_seed(s) if seed is None else seed) + 2_000_000
    shape = s.pool_shape()
    kp = torch.empty(shape, dtype=tdt, device=device)
    vp = torch.empty(shape, dtype=tdt, device=device)
    g = torch.Generator(device=device)
    for layer in range(shape[0]):
        for t, off in ((kp, 0), (vp, 1)):
            g.manual_seed(base + 2 * layer + off)
            tmp = torch.randn(shape[1:], generator=g, device=device, dtype=torch.float32)
            t[layer].copy_(tmp)           # one round-to-nearest-even step
            del tmp
    if s.peaky_keys > 0:
        rng = _rng(base)
        rows = _peaky_rows(s, rng)
        if rows:
            pages = torch.tensor([r[2] for r in rows], device=device)
            prow = torch.tensor([r[3] for r in rows], device=device)
            for layer in range(shape[0]):
                sel = kp[layer][pages, :, prow, :].float() * 8.0
                kp[layer][pages, :, prow, :] = sel.to(tdt)
    return kp, vp


def step_values_torch(s, n_sets, device, seed=None):
    """n_sets independent (q, k, v) inputs for every layer, generated on `device`
    by torch's seeded generator: tensors [n_sets, layers, B, H, d] of the storage type."""
    import torch
    tdt = torch.float16 if s.dtype == "f16" else torch.bfloat16
    g = torch.Generator(device=device)
    g.manual_seed((value_seed(s) if seed is None else seed) + 3_000_000)
    out = []
    for heads in (s.q_heads, s.kv_heads, s.kv_heads):
        x = torch.randn((n_sets, s.num_layers, s.batch, heads, s.head_dim), generator=g, device=device,
                        dtype=torch.float32)
        out.append(x.to(tdt))
    return tuple(out)


def mini_pool_numpy(s, b, g, seed):
    """K and V pages of one (sequence, kv head) as a standalone pool
    [pages(b), 1, P, d] with an identity page table, numpy PCG64 (host-only runs)."""
    rng = _rng(seed)
    np_b = (int(s.context_lens[b]) + s.page_size - 1) // s.page_size
    shape = (np_b, 1, s.page_size, s.head_dim)
    k = round_f32(rng.standard_normal(shape, dtype=np.float32), s.dtype)
    v = round_f32(rng.standard_normal(shape, dtype=np.float32), s.dtype)
    return k, v


def pair_batch_numpy(s, pairs, seed, kv="native"):
    """A standalone batch of (sequence, kv head) pairs of workload `s` for host-only runs:
    pair i becomes sequence i with one kv head and the group's q heads, its own pages
    (identity-ordered, numpy PCG64) and the workload's length of its sequence.
    Returns dict(q [n, G, d] storage bits, block_tables [n, max_pages], context_lens [n],
    k, v [pages, 1, P, d] storage bits -- or, kv="int8", k_codes, v_codes int8 and k_scales,
    v_scales fp32 [pages, 1, P] drawn as pool_values_i8_numpy draws them)."""
    rng = _rng(seed)
    G = s.q_heads // s.kv_heads
    lens = np.array([int(s.context_lens[b]) for b, _ in pairs], np.int32)
    npages = (lens.astype(np.int64) + s.page_size - 1) // s.page_size
    total = int(npages.sum())
    width = max(1, int(npages.max()) if len(pairs) else 1)
    table = np.full((len(pairs), width), -1, np.int32)
    off = 0
    for i, n in enumerate(npages):
        table[i, :n] = np.arange(off, off + n, dtype=np.int32)
        off += int(n)
    shape = (total, 1, s.page_size, s.head_dim)
    out = dict(block_tables=table, context_lens=lens,
               q=round_f32(rng.standard_normal((len(pairs), G, s.head_dim), dtype=np.float32), s.dtype))
    if kv == "int8":
        out["k_codes"] = rng.integers(-127, 128, size=shape, dtype=np.int8)
        out["v_codes"] = rng.integers(-127, 128, size=shape, dtype=np.int8)
        out["k_scales"] = (rng.uniform(1.5, 2.5, size=shape[:-1]) / 127.0).astype(np.float32)
        out["v_scales"] = (rng.uniform(1.5, 2.5, size=shape[:-1]) / 127.0).astype(np.float32)
    else:
        out["k"] = round_f32(rng.standard_normal(shape, dtype=np.float32), s.dtype)
        out["v"] = round_f32(rng.standard_normal(shape, dtype=np.float32), s.dtype)
    return out


# ----------------------------------------------------------------- int8 pages
# Stored int8 pages are drawn directly: codes uniform in [-127, 127], per-row fp32 scales
# uniform in [1.5, 2.5] / 127 (values within about +-2, like the fp16 pools' N(0, 1)), the
# keys of the long-context mix's peaky rows with an 8x scale.

def pool_values_i8_numpy(s, seed=None):
    """(k_codes, v_codes) int8 [layers, pages, Hkv, P, d] and (k_scales, v_scales) fp32
    [layers, pages, Hkv, P], numpy PCG64."""
    rng = _rng((value_seed(s) if seed is None else seed) + 4_000_000)
    shape = s.pool_shape()
    kc = rng.integers(-127, 128, size=shape, dtype=np.int8)
    vc = rng.integers(-127, 128, size=shape, dtype=np.int8)
    ks = (rng.uniform(1.5, 2.5, size=shape[:-1]) / 127.0).astype(np.float32)
    vs = (rng.uniform(1.5, 2.5, size=shape[:-1]) / 127.0).astype(np.float32)
    if s.peaky_keys > 0:
        for (_, _, page, row) in _peaky_rows(s, rng):
            ks[:, page, :, row] *= np.float32(8.0)
    return kc, vc, ks, vs


def pool_values_i8_torch(s, device, seed=None):
    """The same kind of int8 pages as torch tensors on `device`, filled layer by layer from
    torch's seeded generator: (k_codes, v_codes, k_scales, v_scales)."""
    import torch
    base = (value_seed(s) if seed is None else seed) + 5_000_000
    shape = s.pool_shape()
    codes = [torch.empty(shape, dtype=torch.int8, device=device) for _ in range(2)]
    scales = [torch.empty(shape[:-1], dtype=torch.float32, device=device) for _ in range(2)]
    g = torch.Generator(device=device)
    for layer in range(shape[0]):
        for i in range(2):
            g.manual_seed(base + 4 * layer + 2 * i)
            codes[i][layer].random_(-127, 128, generator=g)
            g.manual_seed(base + 4 * layer + 2 * i + 1)
            scales[i][layer].uniform_(1.5 / 127.0, 2.5 / 127.0, generator=g)
    if s.peaky_keys > 0:
        rows = _peaky_rows(s, _rng(base))
        if rows:
            pages = torch.tensor([r[2] for r in rows], device=device)
            prow = torch.tensor([r[3] for r in rows], device=device)
            for layer in range(shape[0]):
                scales[0][layer][pages, :, prow] *= 8.0
    return codes[0], codes[1], scales[0], scales[1]
