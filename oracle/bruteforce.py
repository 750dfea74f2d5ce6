"""Pure-Python brute force for tiny decode cases (test infrastructure).

A second, independent statement of the decode definition used to pin the numpy
oracle: plain loops, correctly rounded sums (``math.fsum``), and softmax without
the max shift, ``p_t = exp(s_t) / sum_u exp(s_u)``.  The bf16 inputs are decoded
with ``struct`` rather than numpy.  Only for inputs small enough that Python loops
finish in seconds and ``exp(s)`` neither overflows nor underflows.
"""
from __future__ import annotations

import math
import struct


def _bf16(bits: int) -> float:
    return struct.unpack("<f", struct.pack("<I", (int(bits) & 0xFFFF) << 16))[0]


def _val(x) -> float:
    # uint16 numpy scalars are bf16 bit patterns; anything else is a number.
    if getattr(x, "dtype", None) is not None and str(x.dtype) == "uint16":
        return _bf16(int(x))
    return float(x)


def decode_bruteforce(q, kv_cache, block_table, cache_seqlens, softmax_scale, d_v, page_size=64):
    """Returns nested lists ``out[b][h][j]`` and ``lse[b][h]``."""
    B, H, D = len(q), len(q[0]), len(q[0][0])
    outs, lses = [], []
    for b in range(B):
        T = int(cache_seqlens[b])
        rows = []
        for t in range(T):
            if block_table is None:
                row = kv_cache[b][t]
            else:
                row = kv_cache[int(block_table[b][t // page_size])][t % page_size]
            rows.append([_val(row[d]) for d in range(D)])
        ob, lb = [], []
        for h in range(H):
            qh = [_val(q[b][h][d]) for d in range(D)]
            w = []
            for t in range(T):
                s = softmax_scale * math.fsum(qh[d] * rows[t][d] for d in range(D))
                w.append(math.exp(s))
            if T == 0:
                ob.append([0.0] * d_v)
                lb.append(-math.inf)
                continue
            Z = math.fsum(w)
            ob.append([math.fsum(w[t] * rows[t][j] for t in range(T)) / Z for j in range(d_v)])
            lb.append(math.log(Z))
        outs.append(ob)
        lses.append(lb)
    return outs, lses


def decode_multi_bruteforce(q, kv_cache, block_table, cache_seqlens, softmax_scale, d_v, page_size=64):
    """Several causal query tokens per sequence, as plain loops with an explicit mask.

    ``q[b][i][h]`` is query token i of sequence b; it sits at position T - s_q + i and
    a cached token t takes part iff t <= T - s_q + i.  Returns ``out[b][i][h][j]`` and
    ``lse[b][i][h]``; a query with no visible token gets zeros and -inf.
    """
    B, SQ, H, D = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    outs, lses = [], []
    for b in range(B):
        T = int(cache_seqlens[b])
        rows = []
        for t in range(T):
            if block_table is None:
                row = kv_cache[b][t]
            else:
                row = kv_cache[int(block_table[b][t // page_size])][t % page_size]
            rows.append([_val(row[d]) for d in range(D)])
        ob, lb = [], []
        for i in range(SQ):
            pos = T - SQ + i
            oi, li = [], []
            for h in range(H):
                qh = [_val(q[b][i][h][d]) for d in range(D)]
                vis = [t for t in range(T) if t <= pos]
                if not vis:
                    oi.append([0.0] * d_v)
                    li.append(-math.inf)
                    continue
                w = {t: math.exp(softmax_scale * math.fsum(qh[d] * rows[t][d] for d in range(D))) for t in vis}
                Z = math.fsum(w.values())
                oi.append([math.fsum(w[t] * rows[t][j] for t in vis) / Z for j in range(d_v)])
                li.append(math.log(Z))
            ob.append(oi)
            lb.append(li)
        outs.append(ob)
        lses.append(lb)
    return outs, lses
