"""Pure-Python brute force for tiny inputs: the definitions, written out with
Python floats, math.exp and math.fsum, no max subtraction and no paging.

Decode attention ("大模型推理全流程解析", s2.2.2; "为什么要自己动手写一个LLM推理引擎",
s4.3): the single new query is dotted with every cached key, scaled, passed
through softmax, and the weights average the cached values.
"""
import math


def attention_one(q, keys, values, scale):
    """q: [d]; keys, values: [L][d] (Python floats) -> [d]."""
    scores = [scale * math.fsum(a * b for a, b in zip(q, k)) for k in keys]
    e = [math.exp(s) for s in scores]
    z = math.fsum(e)
    d = len(values[0])
    return [math.fsum(e[t] * values[t][i] for t in range(len(values))) / z for i in range(d)]


def softmax_weights(q, keys, scale):
    scores = [scale * math.fsum(a * b for a, b in zip(q, k)) for k in keys]
    e = [math.exp(s) for s in scores]
    z = math.fsum(e)
    return [x / z for x in e]


def decode_logical(q, K, V, context_lens, q_heads, kv_heads, scale):
    """q: [B][Hq][d]; K, V: [B][L][Hkv][d] logical (contiguous) caches.
    Query head h reads kv head h // (q_heads // kv_heads)."""
    group = q_heads // kv_heads
    out = []
    for b, L in enumerate(context_lens):
        rows = []
        for h in range(q_heads):
            g = h // group
            if L == 0:
                rows.append([0.0] * len(q[b][h]))
                continue
            keys = [K[b][t][g] for t in range(L)]
            vals = [V[b][t][g] for t in range(L)]
            rows.append(attention_one(q[b][h], keys, vals, scale))
        out.append(rows)
    return out
