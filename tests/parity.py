"""Parity helpers: move synthetic workloads to the GPU and compare the CUDA path's
rows with the CPU oracle's, exactly (integer inputs) or by the band rule
(Gaussian inputs).

Band rule (scores within 1e-3 relative; index sets may differ only at the k-th
score): with s_k the k-th best exact score of a row and tol = 1e-3 * max(|s_k|, 1),
  * the GPU's block set may differ from the oracle's only in blocks whose oracle
    score lies within tol of the lowest freely selected block's score;
  * the oracle's stage 2 is re-run on the GPU's block set; an index may be in
    exactly one of the two rows only if its exact score lies within tol of s_k;
  * the GPU row is non-increasing in exact score (within tol), its scores match
    the exact ones within tol, and the count of -1 entries is identical.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle
from synth import bf16_to_f32

REL_TOL = 1e-3


def dev_bf16(arr_u16: np.ndarray, device="cuda") -> torch.Tensor:
    a = np.ascontiguousarray(arr_u16, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)


def dev_i32(arr, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.int32)).to(device)


class OnDevice:
    """The tensors of a synth.Workload on the GPU."""

    def __init__(self, w, device="cuda"):
        self.w = w
        self.q = dev_bf16(w.q, device)
        self.k = dev_bf16(w.k, device)
        self.cu_q = dev_i32(w.cu_q, device)
        self.cu_k = dev_i32(w.cu_k, device)
        self.seqlens = dev_i32(w.seqlens, device)
        self.max_seqlen_k = w.max_seqlen_k


def exact_scores(w, rows: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """fp64 q.k for each (row, index) pair; NaN where idx == -1."""
    qf = bf16_to_f32(w.q[rows]).astype(np.float64)
    out = np.full(idx.shape, np.nan)
    for t, row in enumerate(rows):
        s = int(np.searchsorted(w.cu_q, row, side="right") - 1)
        while w.cu_q[s + 1] <= row:
            s += 1
        valid = idx[t] >= 0
        kv = bf16_to_f32(w.k[int(w.cu_k[s]) + idx[t][valid]]).astype(np.float64)
        out[t][valid] = kv @ qf[t]
    return out


def sample_rows(w, n: int, seed: int) -> np.ndarray:
    """Seeded rows plus the edges of every sequence and of a few blocks."""
    rng = np.random.Generator(np.random.PCG64(seed))
    rows = set(rng.integers(0, w.total_q, size=n).tolist())
    for s in range(w.num_seqs):
        a, b = int(w.cu_q[s]), int(w.cu_q[s + 1])
        for r in (a, a + 1, a + w.B - 1, a + w.B, a + 3 * w.B + 5, b - 1):
            if a <= r < b:
                rows.add(r)
    return np.array(sorted(rows), np.int32)


def _tol(x: float) -> float:
    return REL_TOL * max(abs(x), 1.0)


def check_token_band(w, rows, gpu_idx, gpu_scores, ref_idx, ref_scores, what="row"):
    """GPU rows against an exact reference computed on the same candidate sets."""
    ex = exact_scores(w, rows, gpu_idx)
    problems = []
    for t, row in enumerate(rows):
        g, r = gpu_idx[t], ref_idx[t]
        nv_g, nv_r = int((g >= 0).sum()), int((r >= 0).sum())
        if nv_g != nv_r or np.any(g[nv_g:] != -1):
            problems.append((row, "valid count", nv_g, nv_r))
            continue
        if nv_r == 0:
            continue
        sk = ref_scores[t][nv_r - 1]
        tol = _tol(sk)
        gs, rs = set(g[:nv_g].tolist()), set(r[:nv_r].tolist())
        if len(gs) != nv_g:
            problems.append((row, "duplicate index"))
            continue
        diff = gs ^ rs
        if diff:
            dj = np.array(sorted(diff), np.int32)
            ds = exact_scores(w, np.array([row]), dj[None])[0]
            if np.any(np.abs(ds - sk) > tol):
                problems.append((row, "set differs outside the band", sorted(diff)[:8]))
                continue
        e = ex[t][:nv_g]
        if np.any(np.diff(e) > tol):
            problems.append((row, "order"))
            continue
        if gpu_scores is not None:
            gsc = gpu_scores[t][:nv_g].astype(np.float64)
            if np.any(np.abs(gsc - e) > REL_TOL * np.maximum(np.abs(e), 1.0)):
                problems.append((row, "scores"))
                continue
    assert not problems, f"{what}: {len(problems)} rows fail the band rule, e.g. {problems[:5]}"


def check_block_band(w, rows, gpu_blocks, ora_blocks, ora_reps):
    """Block sets may differ only in blocks scoring within the band of the cut-off."""
    nblk = (w.max_seqlen_k + w.B - 1) // w.B
    bs = oracle.block_scores(w.q, ora_reps, w.cu_q, w.cu_k, w.seqlens, w.B, nblk, rows=rows)
    problems = []
    for t, row in enumerate(rows):
        g = [b for b in gpu_blocks[t] if b >= 0]
        o = [b for b in ora_blocks[t] if b >= 0]
        if g == o:
            continue
        if len(g) != len(o):
            problems.append((row, "count", len(g), len(o)))
            continue
        s = int(np.searchsorted(w.cu_q, row, side="right") - 1)
        while w.cu_q[s + 1] <= row:
            s += 1
        L = int(w.seqlens[s])
        pos = L - int(w.cu_q[s + 1] - w.cu_q[s]) + (row - int(w.cu_q[s]))
        own = pos // w.B
        forced = {own, own - 1, 0}
        free = [b for b in o if b not in forced]
        cut = min(bs[t][b] for b in free) if free else None
        for b in set(g) ^ set(o):
            if b in forced or cut is None or abs(bs[t][b] - cut) > _tol(cut):
                problems.append((row, "block", b))
                break
    assert not problems, f"block sets: {len(problems)} rows fail the band rule, e.g. {problems[:5]}"


def query_positions(w) -> np.ndarray:
    """Sequence-local position of every query row (the last q_len positions)."""
    out = np.empty(w.total_q, np.int64)
    for s in range(w.num_seqs):
        a, b = int(w.cu_q[s]), int(w.cu_q[s + 1])
        L = int(w.seqlens[s])
        out[a:b] = np.arange(L - (b - a), L)
    return out


def check_rows_structure(w, idx: np.ndarray, sc: np.ndarray, flat: bool, chunk: int = 16384):
    """Every row, checked on the device: -1 only as a suffix; 0 <= j <= i; no duplicate
    index; scores non-increasing with equal scores in ascending index; and exactly
    min(k, c_i) valid entries, c_i the candidate count (i + 1 for the flat scan;
    (min(m, own + 1) - 1) * B + i % B + 1 for HISA, whose own block is always selected
    and whose other selected blocks lie wholly before the query)."""
    pos_all = query_positions(w)
    own = pos_all // w.B
    cand = pos_all + 1 if flat else (np.minimum(w.m, own + 1) - 1) * w.B + pos_all % w.B + 1
    want = np.minimum(w.topk, cand)
    for r0 in range(0, idx.shape[0], chunk):
        r1 = min(idx.shape[0], r0 + chunk)
        I = torch.from_numpy(np.ascontiguousarray(idx[r0:r1])).cuda().long()
        S = torch.from_numpy(np.ascontiguousarray(sc[r0:r1])).cuda()
        pos = torch.from_numpy(pos_all[r0:r1]).cuda()
        valid = I >= 0
        assert not bool((I < -1).any()), "index below -1"
        assert not bool((valid[:, 1:] & ~valid[:, :-1]).any()), "-1 before a valid entry"
        assert not bool(((I > pos[:, None]) & valid).any()), "index after the query"
        nv = valid.sum(dim=1).cpu().numpy()
        assert np.array_equal(nv, want[r0:r1]), "valid count differs from min(k, candidates)"
        srt = torch.sort(I, dim=1).values
        assert not bool(((srt[:, 1:] == srt[:, :-1]) & (srt[:, 1:] >= 0)).any()), "duplicate"
        v2 = valid[:, 1:]
        assert not bool(((S[:, 1:] > S[:, :-1]) & v2).any()), "scores increase along a row"
        assert not bool(((S[:, 1:] == S[:, :-1]) & v2 & (I[:, 1:] < I[:, :-1])).any()), \
            "equal scores out of index order"
        del I, S, pos, valid, srt
    torch.cuda.empty_cache()
