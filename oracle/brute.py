"""Brute-force attention over CONTIGUOUS K/V with pure-Python loops.

TEST INFRASTRUCTURE ONLY (tiny inputs). It never sees the pool or a block table:
it works on the per-sequence K/V rows as the input generator drew them, so it
checks the numpy oracle's gather, GQA mapping, causal mask and softmax by an
independent route. Scores are scale * sum_d q_d k_d; weights exp(z - max) / sum;
output sum_j w_j v_j (the textbook definition of softmax attention).
"""
from __future__ import annotations

import math


def _f(bits: int) -> float:
    """One bf16 bit pattern -> Python float (exact)."""
    import struct
    return struct.unpack("<f", struct.pack("<I", (int(bits) & 0xFFFF) << 16))[0]


def attend(q, keys, values, scale):
    """q: list[D]; keys, values: list[n][D] of floats -> list[D]."""
    n = len(keys)
    D = len(q)
    if n == 0:
        return [0.0] * D
    z = []
    for j in range(n):
        acc = 0.0
        for d in range(D):
            acc += q[d] * keys[j][d]
        z.append(scale * acc)
    m = max(z)
    w = [math.exp(zj - m) for zj in z]
    tot = math.fsum(w)
    out = []
    for d in range(D):
        out.append(math.fsum(w[j] * values[j][d] for j in range(n)) / tot)
    return out


def decode_contiguous(q_bits, k_rows, v_rows, scale):
    """q_bits [B][Hq][D]; k_rows[s], v_rows[s]: [ctx_s][Hkv][D] bf16 bits.

    Returns nested lists [B][Hq][D]. Query head h uses kv head h // (Hq // Hkv).
    """
    out = []
    for s in range(len(q_bits)):
        Hq = len(q_bits[s])
        ks, vs = k_rows[s], v_rows[s]
        Hkv = len(ks[0]) if len(ks) else 1
        group = Hq // Hkv
        row = []
        for h in range(Hq):
            g = h // group
            q = [_f(x) for x in q_bits[s][h]]
            keys = [[_f(x) for x in ks[j][g]] for j in range(len(ks))]
            vals = [[_f(x) for x in vs[j][g]] for j in range(len(vs))]
            row.append(attend(q, keys, vals, scale))
        out.append(row)
    return out


def prefill_contiguous(q_bits, cu_seqlens, k_rows, v_rows, scale):
    """Causal prefill: query i of sequence s (n_new_s queries, ctx_s keys) sits at
    position ctx_s - n_new_s + i and sees keys 0..that position."""
    out = [None] * int(cu_seqlens[-1])
    for s in range(len(k_rows)):
        q0, q1 = int(cu_seqlens[s]), int(cu_seqlens[s + 1])
        ks, vs = k_rows[s], v_rows[s]
        ctx = len(ks)
        n_new = q1 - q0
        for i in range(n_new):
            pos = ctx - n_new + i
            Hq = len(q_bits[q0 + i])
            Hkv = len(ks[0])
            group = Hq // Hkv
            row = []
            for h in range(Hq):
                g = h // group
                q = [_f(x) for x in q_bits[q0 + i][h]]
                keys = [[_f(x) for x in ks[j][g]] for j in range(pos + 1)]
                vals = [[_f(x) for x in vs[j][g]] for j in range(pos + 1)]
                row.append(attend(q, keys, vals, scale))
            out[q0 + i] = row
    return out
