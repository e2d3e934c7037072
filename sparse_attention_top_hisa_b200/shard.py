"""Partition of an indexer batch over ranks (one process per GPU), host side.

Queries are independent given their sequence's keys and representatives, so a
batch splits over GPUs with no exchange between them: every rank runs the
library's entry points on its own slice and writes its own output rows.

The global query rows [0, total_q) are cut into ``world`` contiguous ranges.  A
range may cover whole sequences (decode: one query per sequence; packed varlen)
and parts of sequences (one long prefill).  A query at position i reads only keys
j <= i, so the part [p0, p1) of a sequence's query positions is itself a valid
sequence of p1 live keys whose queries are its last p1 - p0 positions -- exactly
the layout the C ABI describes (cu_seqlens_q places the last q_len positions).
The block that holds key p1 - 1 is then partial in the shard; it is the own block
of the shard's last queries (always selected) and lies after every earlier query
of the shard, so its representative never decides a selection and the shard's
rows equal the unsharded rows exactly.

A shard keeps the key regions of its sequences; region starts stay multiples of
B after rebasing, and the representative rows move with them (rep row = key row
/ B).
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import numpy as np


@dataclass
class Shard:
    """One rank's slice of a batch (all arrays host-side, int32)."""

    rank: int
    world: int
    row0: int            # global query rows [row0, row1) of this shard = its output rows
    row1: int
    seq0: int            # global sequences [seq0, seq1) it touches
    seq1: int
    key0: int            # global key rows [key0, key1) of its regions
    key1: int
    cu_seqlens_q: np.ndarray  # [S'+1], rebased to 0
    cu_seqlens_k: np.ndarray  # [S'+1], rebased to 0 (region starts, multiples of B)
    seqlens_k: np.ndarray     # [S'] live keys the shard's queries can see
    max_seqlen_k: int

    @property
    def num_seqs(self) -> int:
        return self.seq1 - self.seq0

    @property
    def total_q(self) -> int:
        return self.row1 - self.row0

    @property
    def rep0(self) -> int:
        """First global representative row of the shard's regions."""
        return self.key0 // self.B

    B: int = 128


def _check(cu_q, cu_k, seqlens, B):
    cu_q = np.asarray(cu_q, np.int64)
    cu_k = np.asarray(cu_k, np.int64)
    S = cu_q.size - 1
    if S < 0 or cu_k.size != S + 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both hold num_seqs + 1 entries")
    lens = (cu_k[1:] - cu_k[:-1]) if seqlens is None else np.asarray(seqlens, np.int64)
    if lens.size != S:
        raise ValueError("seqlens_k must hold num_seqs entries")
    qlen = cu_q[1:] - cu_q[:-1]
    if np.any(qlen < 0) or np.any(cu_k[1:] < cu_k[:-1]):
        raise ValueError("cu_seqlens must be non-decreasing")
    if np.any(cu_k % B):
        raise ValueError("key region starts must be multiples of B")
    if np.any(qlen > lens) or np.any(lens > cu_k[1:] - cu_k[:-1]):
        raise ValueError("every sequence needs q_len <= len <= its region")
    return cu_q, cu_k, lens


def row_bounds(total_q: int, world: int, cost: Optional[np.ndarray] = None) -> List[int]:
    """Cut [0, total_q) into `world` contiguous ranges of about equal cost (one cost
    per query row; equal costs when None).  Returns world + 1 boundaries."""
    if world < 1:
        raise ValueError("world must be >= 1")
    if cost is None:
        return [(total_q * r) // world for r in range(world + 1)]
    c = np.concatenate([[0.0], np.cumsum(np.asarray(cost, np.float64))])
    tot = c[-1]
    out = [0]
    for r in range(1, world):
        out.append(int(np.searchsorted(c, tot * r / world, side="left")))
        out[-1] = min(max(out[-1], out[-2]), total_q)
    out.append(total_q)
    return out


def query_cost(cu_q, cu_k, seqlens, B: int, m: int) -> np.ndarray:
    """Work estimate per query row: the candidate tokens of stage 2 (min(m, own + 1)
    blocks of B) plus the block scores of stage 1 (own + 1)."""
    cu_q, cu_k, lens = _check(cu_q, cu_k, seqlens, B)
    out = np.empty(int(cu_q[-1]), np.float64)
    for s in range(cu_q.size - 1):
        a, b = int(cu_q[s]), int(cu_q[s + 1])
        pos = np.arange(int(lens[s]) - (b - a), int(lens[s]))
        own = pos // B
        out[a:b] = np.minimum(m, own + 1) * B + own + 1
    return out


def shard(cu_q, cu_k, seqlens, world: int, rank: int, B: int = 128,
          bounds: Optional[List[int]] = None) -> Shard:
    """Rank `rank`'s slice of the batch (cu_seqlens_q / cu_seqlens_k / seqlens_k as
    passed to the C ABI).  bounds: row_bounds(...) to use (default: equal query
    counts)."""
    if not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    cu_q, cu_k, lens = _check(cu_q, cu_k, seqlens, B)
    S = cu_q.size - 1
    total_q = int(cu_q[-1])
    if bounds is None:
        bounds = row_bounds(total_q, world)
    r0, r1 = int(bounds[rank]), int(bounds[rank + 1])
    if not 0 <= r0 <= r1 <= total_q:
        raise ValueError("bad row bounds")
    if r0 == r1:
        z = np.zeros(1, np.int32)
        return Shard(rank, world, r0, r1, 0, 0, 0, 0, z, z.copy(), np.zeros(0, np.int32), 0, B)
    # sequences holding rows r0 and r1 - 1 (sequences with no query rows are skipped)
    s0 = int(np.searchsorted(cu_q, r0, side="right") - 1)
    while cu_q[s0 + 1] <= r0:
        s0 += 1
    s1 = int(np.searchsorted(cu_q, r1 - 1, side="right") - 1)
    while cu_q[s1 + 1] <= r1 - 1:
        s1 += 1
    s1 += 1
    nq, nk, ln = [0], [0], []
    base_k = int(cu_k[s0])
    for s in range(s0, s1):
        a, b = max(int(cu_q[s]), r0), min(int(cu_q[s + 1]), r1)
        qlen = int(cu_q[s + 1] - cu_q[s])
        first_pos = int(lens[s]) - qlen
        p1 = first_pos + (b - int(cu_q[s]))
        nq.append(nq[-1] + max(b - a, 0))
        nk.append(int(cu_k[s + 1]) - base_k)
        ln.append(p1 if b > a else int(lens[s]))  # a sequence with no query rows keeps its keys
    return Shard(rank, world, r0, r1, s0, s1, base_k, int(cu_k[s1]),
                 np.asarray(nq, np.int32), np.asarray(nk, np.int32),
                 np.asarray(ln, np.int32), int(max(ln) if ln else 0), B)
