"""Pure-Python brute force for tiny inputs (test infrastructure only).

Written independently of ``hisa_oracle.c``: exact rational arithmetic
(``fractions.Fraction``) and selection by counting ranks instead of sorting.
A candidate's rank is the number of candidates that beat it (higher score, or
equal score and lower index); the element of rank r lands at output slot r.

Sources: aitrends.kr, "HISA: 세밀한 희소 어텐션을 위한 효율적인 계층적 인덱싱" —
the paragraphs on block pooling, stage 1 (block filtering with forced first /
last-two blocks) and stage 2 (token refinement); idea.jsleekr.com, section
"DSA: 딥시크의 희소 어텐션" (flat scan of every earlier key).
"""

from __future__ import annotations

from fractions import Fraction
from typing import List, Sequence, Tuple

import numpy as np


def _vals(rows_u16: np.ndarray) -> List[List[Fraction]]:
    f = (np.asarray(rows_u16, np.uint16).astype(np.uint32) << 16).view(np.float32)
    return [[Fraction(float(x)) for x in row] for row in f]


def _beats(a: Tuple[Fraction, int], b: Tuple[Fraction, int]) -> bool:
    return a[0] > b[0] or (a[0] == b[0] and a[1] < b[1])


def ranked_top(cands: Sequence[Tuple[Fraction, int]], n: int) -> List[int]:
    """Indices of the n best candidates in rank order, by counting (O(len^2))."""
    out = [-1] * n
    for c in cands:
        r = sum(1 for o in cands if _beats(o, c))
        if r < n:
            out[r] = c[1]
    return out


def pool(keys: List[List[Fraction]], length: int, B: int) -> List[List[Fraction]]:
    reps = []
    for b in range((length + B - 1) // B):
        rows = keys[b * B:min((b + 1) * B, length)]
        reps.append([sum(col, Fraction(0)) / len(rows) for col in zip(*rows)])
    return reps


def dot(a, b) -> Fraction:
    return sum((x * y for x, y in zip(a, b)), Fraction(0))


def blocks_for(qv, reps, pos: int, B: int, m: int) -> List[int]:
    own = pos // B
    if own + 1 <= m:
        return list(range(own + 1))
    forced = []
    for b in (own, own - 1, 0):
        if len(forced) < m and b not in forced:
            forced.append(b)
    rest = [(dot(qv, reps[b]), b) for b in range(own + 1) if b not in forced]
    chosen = [b for b in ranked_top(rest, m - len(forced)) if b >= 0]
    return sorted(forced + chosen)


def hisa_row(qrow_u16, keys_u16, pos: int, B: int, m: int, topk: int, length: int = None):
    """One query of one sequence: (top-k indices, selected blocks)."""
    length = pos + 1 if length is None else length
    keys = _vals(keys_u16[:length])
    qv = _vals(np.asarray(qrow_u16)[None])[0]
    reps = pool(keys, length, B)
    blocks = blocks_for(qv, reps, pos, B, m)
    cands = [(dot(qv, keys[j]), j) for b in blocks for j in range(b * B, min((b + 1) * B, pos + 1))]
    return ranked_top(cands, topk), blocks


def dsa_row(qrow_u16, keys_u16, pos: int, topk: int):
    keys = _vals(keys_u16[:pos + 1])
    qv = _vals(np.asarray(qrow_u16)[None])[0]
    cands = [(dot(qv, keys[j]), j) for j in range(pos + 1)]
    return ranked_top(cands, topk)


def attention(q_heads, keys, values, idx, scale):
    """Attention of one query row over its selected tokens, written independently of
    the C oracle: each weight is 1 / sum_t exp(s_t - s_j) (no running maximum), every
    sum is math.fsum.  q_heads: H lists of dv floats; keys / values: token -> dv
    floats; idx: token positions, -1 = none.  Returns (H lists of dv floats, H lse)."""
    import math
    sel = [j for j in idx if j >= 0]
    outs, lses = [], []
    for qh in q_heads:
        if not sel:
            outs.append([0.0] * len(qh))
            lses.append(-math.inf)
            continue
        s = [scale * math.fsum(a * b for a, b in zip(qh, keys[j])) for j in sel]
        w = [1.0 / math.fsum(math.exp(st - sj) for st in s) for sj in s]
        outs.append([math.fsum(w[t] * values[j][d] for t, j in enumerate(sel))
                     for d in range(len(qh))])
        top = max(s)
        lses.append(top + math.log(math.fsum(math.exp(st - top) for st in s)))
    return outs, lses
