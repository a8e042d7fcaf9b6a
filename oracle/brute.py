"""Brute-force attention in pure Python (tiny inputs only).

TEST INFRASTRUCTURE, used to pin the NumPy oracle. Every sum is an exactly
rounded ``math.fsum``; nothing is vectorised, so each step can be checked
against the definition by eye: score, mask, max, exponentials, their sum,
the weighted sum of values, and the log-sum-exp ("推理加速" interview notes,
section FlashAttention: FlashAttention keeps the mathematical definition of
attention; GQA mapping h -> h // G from "5.2 推理加速的未来趋势").
"""
from __future__ import annotations

import math


def brute_attention(q, k, v, scale, causal):
    """q [B][Hq][Sq][D], k/v [B][Hkv][Sk][D] as nested lists of floats.

    Returns (O, LSE) as nested lists. Bottom-right causal alignment.
    """
    B = len(q)
    Hq = len(q[0])
    Sq = len(q[0][0])
    Hkv = len(k[0])
    Sk = len(k[0][0])
    G = Hq // Hkv
    O = []
    L = []
    for b in range(B):
        Ob, Lb = [], []
        for h in range(Hq):
            kv = h // G
            Oh, Lh = [], []
            for i in range(Sq):
                scores = []
                for j in range(Sk):
                    if causal and j > i + (Sk - Sq):
                        continue
                    dot = math.fsum(q[b][h][i][d] * k[b][kv][j][d] for d in range(len(q[b][h][i])))
                    scores.append((j, scale * dot))
                if not scores:
                    Oh.append([0.0] * len(q[b][h][i]))
                    Lh.append(-math.inf)
                    continue
                m = max(s for _, s in scores)
                w = [(j, math.exp(s - m)) for j, s in scores]
                denom = math.fsum(e for _, e in w)
                row = []
                for d in range(len(v[b][kv][0])):
                    row.append(math.fsum(e * v[b][kv][j][d] for j, e in w) / denom)
                Oh.append(row)
                Lh.append(m + math.log(denom))
            Ob.append(Oh)
            Lb.append(Lh)
        O.append(Ob)
        L.append(Lb)
    return O, L
