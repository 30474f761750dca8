"""Pure-Python brute force for tiny sliding-window attention cases.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).  Nothing here calls the C
oracle: it rebuilds the visible set of every query from scratch by walking the
whole token history, and evaluates the softmax with ``math.exp`` on Python
floats, one (row, head) at a time.  Meant for a few dozen tokens at most.

Mistral 7B, section 2: token i sees tokens j in (i - W, i], at most W of them
(Figure 1 caption); query head h reads kv head h // (Hq // Hkv).
"""
from __future__ import annotations

import math
from typing import List


def window_members(i: int, W: int) -> List[int]:
    """Positions a token at position i attends to: the W most recent, itself included."""
    members = []
    j = i
    while j >= 0 and len(members) < W:
        members.append(j)
        j -= 1
    return sorted(members)


def attention(q, k, v, W: int, scale: float):
    """q [L][Hq][d], k/v [L][Hkv][d] as nested lists -> out [L][Hq][d]."""
    L = len(q)
    Hq = len(q[0])
    Hkv = len(k[0])
    d = len(q[0][0])
    group = Hq // Hkv
    out = []
    for i in range(L):
        row = []
        for h in range(Hq):
            g = h // group
            js = window_members(i, W)
            scores = [scale * sum(q[i][h][c] * k[j][g][c] for c in range(d)) for j in js]
            top = max(scores)
            w = [math.exp(s - top) for s in scores]
            tot = sum(w)
            row.append([sum(w[n] * v[js[n]][g][c] for n in range(len(js))) / tot
                        for c in range(d)])
        out.append(row)
    return out
