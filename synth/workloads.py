"""Seeded synthetic workloads (numpy PCG64), one per benchmark configuration.

Every generator returns plain numpy arrays:

* ``q``  uint16 [total_q, d]   bf16 bit patterns of the index queries,
* ``k``  uint16 [rows_k, d]    bf16 bit patterns of the index keys; sequence s owns
  the key region ``[cu_k[s], cu_k[s+1])``, whose start is a multiple of ``B``,
* ``cu_q`` int32 [S+1]        query offsets, ``cu_k`` int32 [S+1] key-region offsets,
* ``seqlens`` int32 [S]       live key count per sequence.

Queries of sequence s are the *last* ``cu_q[s+1]-cu_q[s]`` positions of that
sequence.  Key rows of a region that lie beyond the live length are filled
with a large poison value so that a reader that strays past ``seqlens`` is
noticed.  Nothing here pools, scores or selects: the generators only draw
numbers and lay them out.
"""

from __future__ import annotations

import dataclasses
from typing import List, Optional, Tuple

import numpy as np

D_IDX = 64          # index-head width used by the configurations
BLOCK = 128         # tokens per block used by the configurations
BF16_ONE = 0x3F80   # bf16 bit pattern of 1.0
POISON = 1.0e4      # value written into key rows past the live length


def bf16_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); return bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    h = np.ascontiguousarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass
class Workload:
    name: str
    q: np.ndarray
    k: np.ndarray
    cu_q: np.ndarray
    cu_k: np.ndarray
    seqlens: np.ndarray
    B: int
    m: int
    topk: int
    d: int = D_IDX
    exact: bool = False
    needles: List[Tuple[int, int]] = dataclasses.field(default_factory=list)

    @property
    def num_seqs(self) -> int:
        return int(self.seqlens.shape[0])

    @property
    def total_q(self) -> int:
        return int(self.q.shape[0])

    @property
    def max_seqlen_k(self) -> int:
        return int(self.seqlens.max()) if self.seqlens.size else 0

    @property
    def rep_rows(self) -> int:
        return int(self.k.shape[0]) // self.B


@dataclasses.dataclass
class DecodeWorkload:
    """Decode state: a key cache with spare capacity plus per-step new keys and queries."""
    name: str
    k_cache: np.ndarray      # uint16 [S*cap, d]
    cu_k: np.ndarray         # int32 [S+1] region starts (multiples of B)
    seqlens0: np.ndarray     # int32 [S] initial live lengths
    new_keys: np.ndarray     # uint16 [steps, S, n_new, d]
    queries: np.ndarray      # uint16 [steps, S, d]
    B: int
    m: int
    topk: int
    d: int = D_IDX

    @property
    def num_seqs(self) -> int:
        return int(self.seqlens0.shape[0])

    @property
    def steps(self) -> int:
        return int(self.queries.shape[0])

    @property
    def capacity(self) -> int:
        return int(self.cu_k[1] - self.cu_k[0])


def _round_up(x: int, b: int) -> int:
    return (x + b - 1) // b * b


def _layout(lengths: List[int], B: int, d: int, draw, rng) -> Tuple[np.ndarray, np.ndarray, np.ndarray, np.ndarray]:
    """Pack per-sequence keys/queries; region starts are multiples of B."""
    S = len(lengths)
    cu_q = np.zeros(S + 1, np.int32)
    cu_k = np.zeros(S + 1, np.int32)
    for s, L in enumerate(lengths):
        cu_q[s + 1] = cu_q[s] + L
        cu_k[s + 1] = cu_k[s] + _round_up(max(L, 1), B)
    q = np.empty((int(cu_q[-1]), d), np.uint16)
    k = np.full((int(cu_k[-1]), d), bf16_from_f32(np.array([POISON], np.float32))[0], np.uint16)
    for s, L in enumerate(lengths):
        qs = draw(rng, (L, d))
        ks = draw(rng, (L, d))
        q[cu_q[s]:cu_q[s] + L] = qs
        k[cu_k[s]:cu_k[s] + L] = ks
    return q, k, cu_q, cu_k


def _draw_int(rng, shape):
    # discrete uniform over {-4, ..., 4}; every value is exact in bf16
    return bf16_from_f32(rng.integers(-4, 5, size=shape).astype(np.float32))


def _draw_gauss(rng, shape):
    return bf16_from_f32(rng.standard_normal(size=shape, dtype=np.float32))


def integer_prefill(L: int, seed: int, B: int = BLOCK, m: int = 8, topk: int = 256,
                    d: int = D_IDX, lengths: Optional[List[int]] = None) -> Workload:
    """Integer-valued q/k (uniform over {-4..4}); every score and mean is exact in fp32."""
    rng = np.random.Generator(np.random.PCG64(seed))
    lens = list(lengths) if lengths is not None else [L]
    q, k, cu_q, cu_k = _layout(lens, B, d, _draw_int, rng)
    return Workload("integer_prefill", q, k, cu_q, cu_k, np.array(lens, np.int32), B, m, topk, d,
                    exact=True)


def gaussian_prefill(L: int, seed: int, B: int = BLOCK, m: int = 64, topk: int = 2048,
                     d: int = D_IDX, lengths: Optional[List[int]] = None) -> Workload:
    """q/k drawn i.i.d. from N(0,1), rounded to bf16."""
    rng = np.random.Generator(np.random.PCG64(seed))
    lens = list(lengths) if lengths is not None else [L]
    q, k, cu_q, cu_k = _layout(lens, B, d, _draw_gauss, rng)
    return Workload("gaussian_prefill", q, k, cu_q, cu_k, np.array(lens, np.int32), B, m, topk, d)


def needle_prefill(L: int, seed: int, n_needles: int = 16, B: int = BLOCK, m: int = 64,
                   topk: int = 2048, d: int = D_IDX) -> Workload:
    """Gaussian prefill with planted needles.

    For each needle a query position i and an earlier key position j are drawn
    with ``B <= j <= i - 3B`` (so the needle never sits in block 0, the query's
    own block or the block before it), and key j is replaced by
    ``4 * q_i / |q_i| + eps`` with ``eps ~ N(0, 0.25^2 I)``.
    """
    w = gaussian_prefill(L, seed, B, m, topk, d)
    rng = np.random.Generator(np.random.PCG64(seed + 7919))
    used_i, used_j = set(), set()
    needles = []
    qf = bf16_to_f32(w.q)
    while len(needles) < n_needles:
        i = int(rng.integers(4 * B, L))
        j = int(rng.integers(B, i - 3 * B + 1))
        if i in used_i or j in used_j:
            continue
        direction = qf[i].astype(np.float64)
        direction /= np.linalg.norm(direction)
        key = 4.0 * direction + 0.25 * rng.standard_normal(d)
        w.k[j] = bf16_from_f32(key.astype(np.float32))
        used_i.add(i)
        used_j.add(j)
        needles.append((i, j))
    w.name = "needle_prefill"
    w.needles = needles
    return w


def varlen_lengths(n: int, seed: int, lo: int = 4096, hi: int = 65536, B: int = BLOCK) -> List[int]:
    """Lengths uniform in [lo, hi], rounded to the nearest multiple of B, clamped to [lo, hi]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    raw = rng.integers(lo, hi + 1, size=n)
    out = []
    for x in raw:
        r = int(np.floor(x / B + 0.5)) * B
        out.append(min(max(r, lo), hi))
    return out


def varlen_prefill(lengths: List[int], seed: int, B: int = BLOCK, m: int = 64, topk: int = 2048,
                   d: int = D_IDX, integer: bool = False) -> Workload:
    """Packed varlen prefill: sequences concatenated, key regions aligned to B."""
    if integer:
        w = integer_prefill(0, seed, B, m, topk, d, lengths=lengths)
    else:
        w = gaussian_prefill(0, seed, B, m, topk, d, lengths=lengths)
    w.name = "varlen_prefill"
    return w


def decode_workload(num_seqs: int, len0: int, steps: int, seed: int, B: int = BLOCK,
                    m: int = 64, topk: int = 2048, d: int = D_IDX, n_new: int = 1,
                    integer: bool = False) -> DecodeWorkload:
    """Key caches of ``len0`` live rows with room for ``steps*n_new`` more rows."""
    rng = np.random.Generator(np.random.PCG64(seed))
    draw = _draw_int if integer else _draw_gauss
    cap = _round_up(len0 + steps * n_new, B)
    cu_k = (np.arange(num_seqs + 1, dtype=np.int64) * cap).astype(np.int32)
    poison = bf16_from_f32(np.array([POISON], np.float32))[0]
    k_cache = np.full((num_seqs * cap, d), poison, np.uint16)
    for s in range(num_seqs):
        k_cache[s * cap:s * cap + len0] = draw(rng, (len0, d))
    new_keys = draw(rng, (steps, num_seqs, n_new, d))
    queries = draw(rng, (steps, num_seqs, d))
    return DecodeWorkload("decode", k_cache, cu_k, np.full(num_seqs, len0, np.int32), new_keys,
                          queries, B, m, topk, d)


CONFIG_NAMES = {
    1: "tiny_prefill_int_L4096",
    2: "decode_16x32768_256steps",
    3: "prefill_L32768_needles",
    4: "prefill_L131072",
    5: "varlen_prefill_8seqs",
}


def config_workload(idx: int, steps: Optional[int] = None):
    """The five benchmark configurations (seed = 20260 + index)."""
    seed = 20260 + idx
    if idx == 1:
        return integer_prefill(4096, seed, m=8, topk=256)
    if idx == 2:
        return decode_workload(16, 32768, 256 if steps is None else steps, seed, m=64, topk=2048)
    if idx == 3:
        return needle_prefill(32768, seed, n_needles=16, m=64, topk=2048)
    if idx == 4:
        return gaussian_prefill(131072, seed, m=64, topk=2048)
    if idx == 5:
        return varlen_prefill(varlen_lengths(8, seed), seed + 1, m=64, topk=2048)
    raise ValueError(f"unknown configuration {idx}")
