"""Pure-Python brute force of attention for tiny inputs -- TEST INFRASTRUCTURE.

An independent second statement of the definition on the ai6s.net
"ops-transformer FlashAttention" article, section "标准注意力的致命伤不在算力，
在搬运" (Q·Kᵀ -> scale -> softmax -> ·V), written term by term with
``math.exp`` and ``math.fsum`` and no arrays, so that it shares nothing with
``attn_oracle.c``.  Used only to pin the C oracle on inputs of a few rows.
"""
from __future__ import annotations

import math


def attention_rows(q, k, v, scale, causal=False, lk=None, window_left=None, blocks=None,
                   block=(1, 1)):
    """q: list of Nq rows, k/v: lists of Nk rows (lists of floats).

    Returns (o, lse): o is a list of Nq output rows, lse a list of Nq floats.
    Key j is visible to query i iff j < lk and (not causal or j <= i + lk - Nq)
    and (window_left is None or j >= i + lk - Nq - window_left) and (blocks
    is None or blocks[i // block[0]][j // block[1]] is true).
    """
    nq = len(q)
    nk = len(k) if lk is None else lk
    d = len(q[0])
    o, lse = [], []
    for i in range(nq):
        scores = []
        for j in range(nk):
            if causal and j > i + nk - nq:
                continue
            if window_left is not None and j < i + nk - nq - window_left:
                continue
            if blocks is not None and not blocks[i // block[0]][j // block[1]]:
                continue
            s = 0.0
            for t in range(d):
                s = s + q[i][t] * k[j][t]
            scores.append((j, scale * s))
        if not scores:
            o.append([0.0] * d)
            lse.append(-math.inf)
            continue
        m = max(s for _, s in scores)
        e = [(j, math.exp(s - m)) for j, s in scores]
        denom = math.fsum(w for _, w in e)
        row = []
        for t in range(d):
            row.append(math.fsum((w / denom) * v[j][t] for j, w in e))
        o.append(row)
        lse.append(m + math.log(denom))
    return o, lse
