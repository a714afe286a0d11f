"""Pure-Python brute force for tiny inputs (TEST INFRASTRUCTURE ONLY).

A second, independent statement of the same definition as ``oracle.c``
("大模型推理加速实战…PagedAttention分页管理方案" (yunthe.com), PagedAttention
section: look up each token's physical block through the block table, then
standard attention; GQA grouping from "LLM推理显存优化KV Cache管理3大策略"
(mlqm.cn) §3).  Plain Python floats (IEEE double), nested loops, no numpy
arithmetic.  Used only on inputs small enough for interpreted loops.
"""
from __future__ import annotations

import math


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, softmax_scale):
    """q: nested [B][n_q][d]; caches nested [NB][bs][n_kv][d]; returns [B][n_q][d]."""
    B = len(q)
    n_q = len(q[0])
    d = len(q[0][0])
    bs = len(k_cache[0])
    n_kv = len(k_cache[0][0])
    group = n_q // n_kv
    out = []
    for s in range(B):
        ctx = context_lens[s]
        rows_k = []
        rows_v = []
        for t in range(ctx):
            phys = block_tables[s][t // bs]
            rows_k.append(k_cache[phys][t % bs])
            rows_v.append(v_cache[phys][t % bs])
        seq_out = []
        for h in range(n_q):
            kvh = h // group
            if ctx == 0:
                seq_out.append([0.0] * d)
                continue
            logits = []
            for t in range(ctx):
                acc = 0.0
                for i in range(d):
                    acc += float(q[s][h][i]) * float(rows_k[t][kvh][i])
                logits.append(softmax_scale * acc)
            top = max(logits)
            weights = [math.exp(z - top) for z in logits]
            total = sum(weights)
            o = [0.0] * d
            for t in range(ctx):
                w = weights[t] / total
                for i in range(d):
                    o[i] += w * float(rows_v[t][kvh][i])
            seq_out.append(o)
        out.append(seq_out)
    return out
