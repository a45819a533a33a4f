"""Pure-Python brute force for tiny paged decode cases (test infrastructure).

A second, independent restatement of the oracle's definition, written with
Python floats and loops only, for inputs small enough to check by hand
(head_dim of a few elements, a handful of tokens).  It widens fp16 / bf16 bit
patterns with the standard library's ``struct`` codecs rather than by hand, so
the C oracle's own widening is checked against a library routine.

Definition followed: "vLLM PagedAttention 大模型推理架构深度实战" section 2.2
(logical block i of a sequence lives in the physical block its block table
names; 16-token blocks) and section 5.1 (attention is exact); "vLLM：重塑大模型
推理性能的关键引擎", PagedAttention section, kernel sketch (ceil(len / BLOCK_SIZE)
blocks, table row stride MAX_BLOCKS).
"""
from __future__ import annotations

import math
import struct


def widen_bits(bits: int, dtype: str) -> float:
    """fp16 via struct's IEEE half codec; bf16 as the high half of a float32."""
    if dtype in ("f16", "fp16", "float16"):
        return struct.unpack("<e", struct.pack("<H", bits & 0xFFFF))[0]
    return struct.unpack("<f", struct.pack("<I", (bits & 0xFFFF) << 16))[0]


def attention(q, keys, values, scale):
    """softmax(scale * q . k_j) weighted sum of v_j, by loops (lists of floats)."""
    n = len(keys)
    if n == 0:
        return [0.0] * len(q)
    logits = [scale * sum(qi * ki for qi, ki in zip(q, k)) for k in keys]
    top = max(logits)
    weights = [math.exp(x - top) for x in logits]
    total = sum(weights)
    out = [0.0] * len(values[0])
    for w, v in zip(weights, values):
        for d in range(len(v)):
            out[d] += (w / total) * v[d]
    return out


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, scale, dtype):
    """Nested-list / numpy-indexable inputs of bit patterns; returns nested lists.

    q[s][h][d]; cache[block][kv_head][slot][d]; block_tables[s][i]; the KV head
    of query head h is h // (H // Hk).
    """
    S = len(q)
    H = len(q[0])
    Hk = len(k_cache[0])
    B = len(k_cache[0][0])
    group = H // Hk
    out = []
    for s in range(S):
        n = int(context_lens[s])
        rows = []
        for h in range(H):
            kvh = h // group
            keys, vals = [], []
            for j in range(n):
                blk = int(block_tables[s][j // B])
                keys.append([widen_bits(int(x), dtype) for x in k_cache[blk][kvh][j % B]])
                vals.append([widen_bits(int(x), dtype) for x in v_cache[blk][kvh][j % B]])
            qv = [widen_bits(int(x), dtype) for x in q[s][h]]
            rows.append(attention(qv, keys, vals, scale))
        out.append(rows)
    return out
