"""Pure-Python brute force for tiny cases -- TEST INFRASTRUCTURE ONLY.

A second, independent statement of the oracle's decode attention
("PagedAttention", "How attention reads paged memory"): no C, no numpy
arithmetic.  16-bit floats are decoded with the standard library's IEEE
binary16 codec (``struct`` format 'e') and, for bfloat16, by placing the bits
in the upper half of a binary32 word.  Sums use ``math.fsum`` (exactly rounded),
so the result is within a few ulps of the exact value.  Meant for inputs of a
few hundred tokens at most.
"""
from __future__ import annotations

import math
import struct


def decode16(bits: int, dtype: str) -> float:
    if dtype in ("bf16", "bfloat16"):
        return struct.unpack("<f", struct.pack("<I", (int(bits) & 0xFFFF) << 16))[0]
    return struct.unpack("<e", struct.pack("<H", int(bits) & 0xFFFF))[0]


def decode_attention(q, key_cache, value_cache, block_tables, seq_lens, scale, dtype):
    """q: nested lists / arrays [B][Hq][D] of uint16 bits; pools [nb][bs][Hkv][D].

    Returns [B][Hq][D] Python floats.  Token t of sequence b is read from
    physical block block_tables[b][t // bs] at offset t % bs; query head h
    reads KV head h // (Hq // Hkv); a sequence of length 0 yields zeros."""
    B = len(q)
    Hq = len(q[0])
    D = len(q[0][0])
    bs = len(key_cache[0])
    Hkv = len(key_cache[0][0])
    group = Hq // Hkv
    out = []
    for b in range(B):
        L = int(seq_lens[b])
        rows = []
        for h in range(Hq):
            if L == 0:
                rows.append([0.0] * D)
                continue
            g = h // group
            qv = [decode16(x, dtype) for x in q[b][h]]
            keys, vals = [], []
            for t in range(L):
                blk = int(block_tables[b][t // bs])
                off = t % bs
                keys.append([decode16(x, dtype) for x in key_cache[blk][off][g]])
                vals.append([decode16(x, dtype) for x in value_cache[blk][off][g]])
            s = [scale * math.fsum(qv[d] * k[d] for d in range(D)) for k in keys]
            m = max(s)
            p = [math.exp(x - m) for x in s]
            den = math.fsum(p)
            rows.append([math.fsum(p[t] * vals[t][d] for t in range(L)) / den
                         for d in range(D)])
        out.append(rows)
    return out


def decode_attention_multi(q, q_start, key_cache, value_cache, block_tables, seq_lens, scale,
                           dtype):
    """Several query tokens per sequence: q rows q_start[b] .. q_start[b+1]-1
    are sequence b's last n tokens; query i of them attends tokens
    0 .. seq_lens[b] - n + i (itself and everything before it).  Returns
    [T][Hq][D] Python floats; a query that attends nothing yields zeros."""
    T = len(q)
    Hq = len(q[0])
    D = len(q[0][0])
    bs = len(key_cache[0])
    Hkv = len(key_cache[0][0])
    group = Hq // Hkv
    out = [None] * T
    for b in range(len(seq_lens)):
        L = int(seq_lens[b])
        r0, r1 = int(q_start[b]), int(q_start[b + 1])
        n = r1 - r0
        for i in range(n):
            r = r0 + i
            last = min(L - n + i, L - 1)  # the last position this query sees
            rows = []
            for h in range(Hq):
                if last < 0:
                    rows.append([0.0] * D)
                    continue
                g = h // group
                qv = [decode16(x, dtype) for x in q[r][h]]
                s, vals = [], []
                for t in range(last + 1):
                    blk = int(block_tables[b][t // bs])
                    off = t % bs
                    k = [decode16(x, dtype) for x in key_cache[blk][off][g]]
                    vals.append([decode16(x, dtype) for x in value_cache[blk][off][g]])
                    s.append(scale * math.fsum(qv[d] * k[d] for d in range(D)))
                m = max(s)
                p = [math.exp(x - m) for x in s]
                den = math.fsum(p)
                rows.append([math.fsum(p[t] * vals[t][d] for t in range(len(p))) / den
                             for d in range(D)])
            out[r] = rows
    return out
