"""Chunked prefill at the benchmark's full size, sampled against the fp64 oracle.

The benchmark times 512-token chunks over the batch-10 contexts (fp16, one query head per
kv head) and over the continuous-batching mix (bf16, four query heads per kv head): the
last min(L_b, 512) tokens of each context are the chunk, causal over the whole cached
prefix ("为什么要自己动手写一个LLM推理引擎" (wzjinhao.cn/news/61427) s4.3, the mask slice
[start_pos : start_pos + seq_len]).  The kernel runs on the whole batch in the launch
configuration the benchmark uses; the pages of sampled (sequence, kv head) pairs are copied
off the device before it runs, and every row of those pairs' chunks is compared with
oracle.prefill_attention element by element.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
import paged_kv_cache_460_b200 as pkv
from tests.gpu_cases import TDT, to_bits, tolerance_report

pytestmark = pytest.mark.gpu

CHUNK = 512


def _pick_pairs(s, start, n, seed, max_keys):
    """Sampled (b, kv head) pairs: the longest context, a chunk that starts mid-page, a
    context that ends mid-page, then seeded picks, keeping the oracle's work bounded."""
    r = np.random.Generator(np.random.PCG64(seed))
    L = s.context_lens.astype(np.int64)
    P = s.page_size
    chosen = [int(np.argmax(L))]
    mid_start = [b for b in range(s.batch) if start[b] % P != 0 and L[b] % P != 0]
    aligned = [b for b in range(s.batch) if start[b] % P == 0 or L[b] % P == 0]
    chosen += mid_start[:1] + aligned[:1]
    order = r.permutation(s.batch)
    cost = lambda b: int(L[b]) * int(min(L[b], CHUNK))
    budget = max_keys
    pairs = []
    for b in chosen + [int(x) for x in order]:
        if len(pairs) >= n:
            break
        if any(pb == b for pb, _ in pairs) or cost(b) > budget:
            continue
        budget -= cost(b)
        pairs.append((b, int(r.integers(s.kv_heads))))
    assert any(start[b] % P != 0 for b, _ in pairs), "no chunk starting mid-page was sampled"
    assert any(L[b] % P != 0 for b, _ in pairs), "no context ending mid-page was sampled"
    return pairs


@pytest.mark.parametrize("name,n_pairs,max_keys", [("batch10", 10, 8_000_000), ("cbatch", 8, 7_000_000)])
def test_prefill_full_size_sampled(name, n_pairs, max_keys):
    s = synth.spec(name, num_layers=1)
    dev = torch.device("cuda")
    tdt = TDT[s.dtype]
    kp, vp = synth.pool_values_torch(s, dev)
    ctx = s.context_lens.astype(np.int64)
    chunk = np.minimum(ctx, CHUNK)
    start = ctx - chunk
    cu_q = np.concatenate([[0], np.cumsum(chunk)]).astype(np.int32)
    total = int(cu_q[-1])
    G = s.q_heads // s.kv_heads
    r = np.random.Generator(np.random.PCG64(5151 + s.index))
    q = synth.round_f32(r.standard_normal((total, s.q_heads, s.head_dim), dtype=np.float32), s.dtype)
    pairs = _pick_pairs(s, start, n_pairs, 77 + s.index, max_keys)

    # page snapshots of the sampled pairs, before any library kernel runs
    snaps = []
    for b, g in pairs:
        np_b = (int(ctx[b]) + s.page_size - 1) // s.page_size
        pages = torch.from_numpy(s.block_tables[b, :np_b].astype(np.int64)).to(dev)
        kmini = to_bits(kp[0].index_select(0, pages)[:, g:g + 1])
        vmini = to_bits(vp[0].index_select(0, pages)[:, g:g + 1])
        snaps.append((b, g, kmini, vmini))

    pool = pkv.KVPool(kp, vp)
    q_t = torch.from_numpy(q.view(np.int16)).view(tdt).to(dev)
    out = torch.full_like(q_t, float("nan"))
    pkv.paged_prefill_attention(pool, 0, out, q_t, torch.from_numpy(cu_q).to(dev),
                                torch.from_numpy(s.block_tables).to(dev), torch.from_numpy(s.context_lens).to(dev),
                                1.0 / math.sqrt(s.head_dim))
    got_all = to_bits(out)
    assert pkv.kv_get_device_error() == 0

    scale = 1.0 / math.sqrt(s.head_dim)
    for b, g, kmini, vmini in snaps:
        rows = slice(int(cu_q[b]), int(cu_q[b + 1]))
        n_b = int(chunk[b])
        q_b = q[rows, g * G:(g + 1) * G]
        table = np.arange(kmini.shape[0], dtype=np.int32)[None, :]
        ref = oracle.prefill_attention(q_b, kmini, vmini, table, np.array([0, n_b], np.int32),
                                       np.array([ctx[b]], np.int32), scale, s.dtype)
        got = got_all[rows, g * G:(g + 1) * G]
        ok, maxerr, ratio = tolerance_report(got, ref, s.dtype)
        assert ok, "%s sequence %d (L %d, chunk from %d), kv head %d: max |err| %.3g (%.3g of the bound)" % (
            name, b, ctx[b], start[b], g, maxerr, ratio)
    assert np.isfinite(oracle.decode(got_all, s.dtype)).all()
