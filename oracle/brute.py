"""Pure-Python paged decode attention for tiny cases.

TEST INFRASTRUCTURE ONLY (tests and the smoke check).  A second, independent
spelling of the definition the C oracle follows ("pagedattention vllm"
§Attention Computation: attention over blocks gathered through the table equals
attention over the contiguous cache): first rebuild each sequence's contiguous
key and value lists by walking its block table in logical order, then run
textbook softmax attention on them with ``math.exp``.  Inputs are float64
arrays already decoded from storage.
"""
from __future__ import annotations

import math


def contiguous_kv(k_cache, v_cache, table_row, L, kv_head, block_size):
    """Keys and values of one sequence and KV head, in token order."""
    ks, vs = [], []
    for j in range((L + block_size - 1) // block_size):
        phys = int(table_row[j])
        for o in range(block_size):
            if j * block_size + o >= L:
                break
            ks.append([float(x) for x in k_cache[phys][kv_head][o]])
            vs.append([float(x) for x in v_cache[phys][kv_head][o]])
    return ks, vs


def attention_row(qrow, ks, vs, scale):
    """softmax(q . k_t * scale) weighted sum of v_t; zero row when empty."""
    D = len(qrow)
    if not ks:
        return [0.0] * D
    logits = [scale * sum(qrow[d] * k[d] for d in range(D)) for k in ks]
    top = max(logits)
    weights = [math.exp(x - top) for x in logits]
    z = sum(weights)
    return [sum(w * v[d] for w, v in zip(weights, vs)) / z for d in range(D)]


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, scale, window=0):
    """q [B][Hq][D], caches [N][Hkv][bs][D] (float64 values) -> [B][Hq][D];
    window > 0: only each sequence's last `window` tokens."""
    B = len(q)
    Hq = len(q[0])
    Hkv = len(k_cache[0])
    bs = len(k_cache[0][0])
    G = Hq // Hkv
    out = []
    for b in range(B):
        L = int(context_lens[b])
        rows = []
        for h in range(Hq):
            ks, vs = contiguous_kv(k_cache, v_cache, block_tables[b], L, h // G, bs)
            if window > 0:
                ks, vs = ks[-window:], vs[-window:]
            rows.append(attention_row([float(x) for x in q[b][h]], ks, vs, scale))
        out.append(rows)
    return out
