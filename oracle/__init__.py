"""CPU oracle for the HISA indexer (test infrastructure only).

This package is the slow, plain reference the CUDA library is checked against.
Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import it.  The product package never imports it, and it never imports
the product package.  The arithmetic lives in ``hisa_oracle.c`` (fp64, plain
loops, one thread per query row); this module builds it with gcc and wraps it
with ctypes.  ``brute.py`` holds an independent pure-Python brute force for
tiny inputs.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hisa_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "liboracle.so")
_lib = None

ERRORS = {0: "ok", 1: "invalid argument", 2: "non-finite input", 3: "allocation failed"}


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, -O2, pthreads) into oracle/_build/liboracle.so."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-shared", "-fPIC", "-pthread",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_pool.argtypes = [P, P, P, I, I, I, P]
        lib.oracle_block_select.argtypes = [P, P, P, P, P, I, I, I, I, I, P, I, P, P, I]
        lib.oracle_block_scores.argtypes = [P, P, P, P, P, I, I, I, I, I, P, I, P, I]
        lib.oracle_token_select.argtypes = [P, P, P, I, P, P, P, I, I, I, I, I, P, I, P, P, I]
        lib.oracle_dsa.argtypes = [P, P, P, P, P, I, I, I, I, P, I, P, P, I]
        lib.oracle_hisa.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, I, P, P, P, P, I]
        lib.oracle_sparse_attention.argtypes = [P, P, P, P, P, P, I, I, I, I, I,
                                                ctypes.c_double, P, P, I]
        lib.oracle_set_mutation.argtypes = [I]
        lib.oracle_get_mutation.restype = I
        for f in ("oracle_sparse_attention", "oracle_pool", "oracle_block_select", "oracle_block_scores",
                  "oracle_token_select", "oracle_dsa", "oracle_hisa"):
            getattr(lib, f).restype = I
        _lib = lib
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def _check(code: int, what: str):
    if code != 0:
        raise OracleError(f"{what}: {ERRORS.get(code, code)}")


def set_mutation(code: int) -> None:
    """Test hook: plant one deliberate mistake (0 restores the oracle)."""
    _load().oracle_set_mutation(int(code))


def get_mutation() -> int:
    return int(_load().oracle_get_mutation())


def _layout(cu_q, cu_k, seqlens):
    return _c(cu_q, np.int32), _c(cu_k, np.int32), _c(seqlens, np.int32)


def pool(k, cu_k, seqlens, B: int) -> np.ndarray:
    """Mean-pooled representatives, fp64 [ceil(rows_k/B), d] (rows past the live blocks are 0)."""
    k = _c(k, np.uint16)
    cu_k = _c(cu_k, np.int32)
    seqlens = _c(seqlens, np.int32)
    S = cu_k.shape[0] - 1
    d = k.shape[1]
    reps = np.zeros(((int(cu_k[-1]) + B - 1) // B, d), np.float64)
    _check(_load().oracle_pool(_p(k), _p(cu_k), _p(seqlens), S, d, B, _p(reps)), "oracle_pool")
    return reps


def _rows(rows, total_q):
    if rows is None:
        return None, total_q
    r = _c(rows, np.int32)
    return r, int(r.shape[0])


def block_select(q, reps, cu_q, cu_k, seqlens, B: int, m: int, rows=None, nthreads: int = 0):
    """Stage 1: selected blocks per query row (ascending, -1 padded) and their fp64 scores."""
    q = _c(q, np.uint16)
    reps = _c(reps, np.float64)
    cu_q, cu_k, seqlens = _layout(cu_q, cu_k, seqlens)
    total_q, d = q.shape
    r, nr = _rows(rows, total_q)
    blocks = np.empty((nr, m), np.int32)
    scores = np.empty((nr, m), np.float64)
    _check(_load().oracle_block_select(_p(q), _p(reps), _p(cu_q), _p(cu_k), _p(seqlens),
                                       cu_q.shape[0] - 1, total_q, d, B, m, _p(r), nr,
                                       _p(blocks), _p(scores), nthreads), "oracle_block_select")
    return blocks, scores


def block_scores(q, reps, cu_q, cu_k, seqlens, B: int, max_blocks: int, rows=None,
                 nthreads: int = 0) -> np.ndarray:
    """Every block score per query row (NaN for blocks wholly after the query)."""
    q = _c(q, np.uint16)
    reps = _c(reps, np.float64)
    cu_q, cu_k, seqlens = _layout(cu_q, cu_k, seqlens)
    total_q, d = q.shape
    r, nr = _rows(rows, total_q)
    out = np.empty((nr, max_blocks), np.float64)
    _check(_load().oracle_block_scores(_p(q), _p(reps), _p(cu_q), _p(cu_k), _p(seqlens),
                                       cu_q.shape[0] - 1, total_q, d, B, max_blocks, _p(r), nr,
                                       _p(out), nthreads), "oracle_block_scores")
    return out


def token_select(q, k, blocks, cu_q, cu_k, seqlens, B: int, topk: int, rows=None,
                 nthreads: int = 0):
    """Stage 2: top-k token indices (and fp64 scores) over the given block sets."""
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    blocks = _c(blocks, np.int32)
    cu_q, cu_k, seqlens = _layout(cu_q, cu_k, seqlens)
    total_q, d = q.shape
    r, nr = _rows(rows, total_q)
    assert blocks.shape[0] == nr
    idx = np.empty((nr, topk), np.int32)
    sc = np.empty((nr, topk), np.float64)
    _check(_load().oracle_token_select(_p(q), _p(k), _p(blocks), blocks.shape[1], _p(cu_q),
                                       _p(cu_k), _p(seqlens), cu_q.shape[0] - 1, total_q, d, B,
                                       topk, _p(r), nr, _p(idx), _p(sc), nthreads),
           "oracle_token_select")
    return idx, sc


def dsa(q, k, cu_q, cu_k, seqlens, topk: int, rows=None, nthreads: int = 0):
    """Flat DSA: exact top-k over every causal key."""
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    cu_q, cu_k, seqlens = _layout(cu_q, cu_k, seqlens)
    total_q, d = q.shape
    r, nr = _rows(rows, total_q)
    idx = np.empty((nr, topk), np.int32)
    sc = np.empty((nr, topk), np.float64)
    _check(_load().oracle_dsa(_p(q), _p(k), _p(cu_q), _p(cu_k), _p(seqlens), cu_q.shape[0] - 1,
                              total_q, d, topk, _p(r), nr, _p(idx), _p(sc), nthreads),
           "oracle_dsa")
    return idx, sc


def hisa(q, k, cu_q, cu_k, seqlens, B: int, m: int, topk: int, rows=None, nthreads: int = 0):
    """Whole HISA indexer. Returns (idx, scores, blocks, reps)."""
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    cu_q, cu_k, seqlens = _layout(cu_q, cu_k, seqlens)
    total_q, d = q.shape
    r, nr = _rows(rows, total_q)
    idx = np.empty((nr, topk), np.int32)
    sc = np.empty((nr, topk), np.float64)
    blocks = np.empty((nr, m), np.int32)
    reps = np.zeros(((int(cu_k[-1]) + B - 1) // B, d), np.float64)
    _check(_load().oracle_hisa(_p(q), _p(k), _p(cu_q), _p(cu_k), _p(seqlens), cu_q.shape[0] - 1,
                               total_q, d, B, m, topk, _p(r), nr, _p(idx), _p(sc), _p(blocks),
                               _p(reps), nthreads), "oracle_hisa")
    return idx, sc, blocks, reps


def hisa_workload(w, rows=None, nthreads: int = 0):
    """oracle.hisa on a synth.Workload."""
    return hisa(w.q, w.k, w.cu_q, w.cu_k, w.seqlens, w.B, w.m, w.topk, rows, nthreads)


def dsa_workload(w, rows=None, nthreads: int = 0):
    """oracle.dsa on a synth.Workload."""
    return dsa(w.q, w.k, w.cu_q, w.cu_k, w.seqlens, w.topk, rows, nthreads)


def sparse_attention(q, k, v, idx, cu_q, cu_k, H: int, scale: float, nthreads: int = 0):
    """Attention over the selected tokens (see hisa_oracle.c, oracle_sparse_attention).

    q: bf16 bits [total_q, H, dv]; k, v: bf16 bits [rows_k, dv]; idx: int32
    [total_q, topk] sequence-local positions, -1 = none.  Returns (out f64
    [total_q, H, dv], lse f64 [total_q, H]).
    """
    L = _load()
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    idx = _c(idx, np.int32)
    cu_q = _c(cu_q, np.int32)
    cu_k = _c(cu_k, np.int32)
    total_q, topk = idx.shape
    dv = k.shape[1]
    assert q.shape == (total_q, H, dv) and v.shape == k.shape
    out = np.zeros((total_q, H, dv), np.float64)
    lse = np.zeros((total_q, H), np.float64)
    _check(L.oracle_sparse_attention(_p(q), _p(k), _p(v), _p(idx), _p(cu_q), _p(cu_k),
                                     len(cu_q) - 1, total_q, H, dv, topk, float(scale), _p(out),
                                     _p(lse), nthreads), "oracle_sparse_attention")
    return out, lse
