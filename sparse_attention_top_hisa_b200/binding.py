"""ctypes binding of libhisa.so (the C ABI declared in include/hisa.h).

The functions keep the C names and only marshal arguments: torch tensors are
checked for device, dtype and contiguity, their device pointers and the current
CUDA stream are passed through, and a non-zero status raises ``HisaError``.
Every step of the indexer runs in the library's CUDA kernels; there is no
fallback of any kind, and importing this module fails loudly when the library
has not been built.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhisa.so")

HISA_INDEX_DIM = 64
HISA_BLOCK = 128
HISA_MAX_M = 512
HISA_MAX_TOPK = 2048

STATUS = {
    0: "HISA_OK",
    1: "HISA_ERR_INVALID_ARG",
    2: "HISA_ERR_UNALIGNED",
    3: "HISA_ERR_WORKSPACE",
    4: "HISA_ERR_CUDA",
    5: "HISA_ERR_TIMEOUT",
    6: "HISA_ERR_NOT_IMPLEMENTED",
    7: "HISA_ERR_CAPACITY",
}

# every symbol include/hisa.h declares
EXPORTED = (
    "hisa_status_string",
    "hisa_version",
    "hisa_pool_blocks",
    "hisa_append_keys",
    "hisa_select",
    "hisa_select_workspace_size",
    "dsa_flat_select",
    "dsa_flat_workspace_size",
    "hisa_device_status",
    "hisa_sparse_attention",
    "hisa_timing_enable",
    "hisa_kernel_kinds",
    "hisa_kernel_name",
    "hisa_timing_collect",
    "hisa_select_noalloc",
    "hisa_select_varm",
    "hisa_fraction_blocks",
    "hisa_block_sparse_select",
    "hisa_block_sparse_workspace_size",
    "hisa_test_fault",
    "hisa_decode_step",
)


class HisaError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)} ({lib().hisa_status_string(code).decode()})")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libhisa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              f"`python -m sparse_attention_top_hisa_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.hisa_status_string.argtypes = [I]
        L.hisa_status_string.restype = ctypes.c_char_p
        L.hisa_version.restype = I
        L.hisa_pool_blocks.argtypes = [P, P, P, I, I, I, P, P]
        L.hisa_append_keys.argtypes = [P, P, P, P, P, I, I, I, P]
        L.hisa_select.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, P, P, P, P, Z, P]
        L.hisa_select_workspace_size.argtypes = [I, I, I, I, I, I]
        L.hisa_select_workspace_size.restype = Z
        L.dsa_flat_select.argtypes = [P, P, P, P, P, I, I, I, I, P, P, P, Z, P]
        L.dsa_flat_workspace_size.argtypes = [I, I, I, I]
        L.dsa_flat_workspace_size.restype = Z
        L.hisa_device_status.argtypes = [P, I, P]
        L.hisa_timing_enable.argtypes = [I]
        L.hisa_timing_enable.restype = I
        L.hisa_kernel_kinds.restype = I
        L.hisa_kernel_name.argtypes = [I]
        L.hisa_kernel_name.restype = ctypes.c_char_p
        L.hisa_timing_collect.argtypes = [P, P, P, I, I]
        L.hisa_timing_collect.restype = I
        L.hisa_sparse_attention.argtypes = [P, P, P, P, P, P, I, I, I, I, ctypes.c_float, P, P,
                                            P]
        L.hisa_select_varm.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, P, P, P, P, Z, P]
        L.hisa_fraction_blocks.argtypes = [P, P, I, I, ctypes.c_double, I, P, P]
        L.hisa_block_sparse_select.argtypes = [P, P, P, P, P, I, I, I, I, I, P, P, P, Z, P]
        L.hisa_block_sparse_workspace_size.argtypes = [I, I, I, I, I]
        L.hisa_block_sparse_workspace_size.restype = Z
        L.hisa_decode_step.argtypes = [P, P, P, P, P, P, I, I, I, I, I, P, P, P, P]
        L.hisa_decode_step.restype = I
        L.hisa_test_fault.argtypes = [I]
        L.hisa_test_fault.restype = I
        for f in ("hisa_pool_blocks", "hisa_append_keys", "hisa_select", "dsa_flat_select",
                  "hisa_device_status", "hisa_sparse_attention", "hisa_select_varm",
                  "hisa_fraction_blocks", "hisa_block_sparse_select"):
            getattr(L, f).restype = I
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(code: int, what: str):
    if code != 0:
        raise HisaError(code, what)


def _need(t: Optional[torch.Tensor], name: str, dtype, cols: Optional[int] = None,
          optional: bool = False):
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if cols is not None and (t.dim() != 2 or t.shape[1] != cols):
        raise ValueError(f"{name} must have shape [*, {cols}], got {tuple(t.shape)}")


def hisa_pool_blocks(k_idx: torch.Tensor, cu_seqlens_k: torch.Tensor,
                     seqlens_k: Optional[torch.Tensor], max_seqlen_k: int, B: int = HISA_BLOCK,
                     reps: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Mean-pool keys into per-block representatives; returns reps fp32 [rows_k/B, 64]."""
    _need(k_idx, "k_idx", torch.bfloat16, HISA_INDEX_DIM)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32)
    _need(seqlens_k, "seqlens_k", torch.int32, optional=True)
    nrep = (k_idx.shape[0] + B - 1) // B
    if reps is None:
        reps = torch.zeros(nrep, HISA_INDEX_DIM, dtype=torch.float32, device=k_idx.device)
    _need(reps, "reps", torch.float32, HISA_INDEX_DIM)
    _check(lib().hisa_pool_blocks(_ptr(k_idx), _ptr(cu_seqlens_k), _ptr(seqlens_k),
                                  cu_seqlens_k.numel() - 1, int(max_seqlen_k), B, _ptr(reps),
                                  _stream(stream)), "hisa_pool_blocks")
    return reps


def hisa_append_keys(k_cache: torch.Tensor, reps: torch.Tensor, cu_seqlens_k: torch.Tensor,
                     seqlens_k: torch.Tensor, new_keys: torch.Tensor, B: int = HISA_BLOCK,
                     stream=None) -> None:
    """Append new_keys [S, n_new, 64] to the cache and refresh the touched representatives."""
    _need(k_cache, "k_cache", torch.bfloat16, HISA_INDEX_DIM)
    _need(reps, "reps", torch.float32, HISA_INDEX_DIM)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32)
    _need(seqlens_k, "seqlens_k", torch.int32)
    _need(new_keys, "new_keys", torch.bfloat16)
    S = cu_seqlens_k.numel() - 1
    if new_keys.dim() != 3 or new_keys.shape[0] != S or new_keys.shape[2] != HISA_INDEX_DIM:
        raise ValueError(f"new_keys must be [S, n_new, 64], got {tuple(new_keys.shape)}")
    _check(lib().hisa_append_keys(_ptr(k_cache), _ptr(reps), _ptr(cu_seqlens_k), _ptr(seqlens_k),
                                  _ptr(new_keys), new_keys.shape[1], S, B, _stream(stream)),
           "hisa_append_keys")


def hisa_select_workspace_size(total_q: int, num_seqs: int, max_seqlen_k: int, m: int, k: int,
                               B: int = HISA_BLOCK) -> int:
    return int(lib().hisa_select_workspace_size(total_q, num_seqs, max_seqlen_k, B, m, k))


def dsa_flat_workspace_size(total_q: int, num_seqs: int, max_seqlen_k: int, k: int) -> int:
    return int(lib().dsa_flat_workspace_size(total_q, num_seqs, max_seqlen_k, k))


def _workspace(nbytes: int, device, ws: Optional[torch.Tensor]) -> torch.Tensor:
    if ws is not None:
        if ws.dtype != torch.uint8 or not ws.is_cuda or ws.numel() < nbytes:
            raise ValueError(f"workspace must be a CUDA uint8 tensor of >= {nbytes} bytes")
        return ws
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def hisa_select(q_idx: torch.Tensor, k_idx: torch.Tensor, reps: torch.Tensor,
                cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor,
                seqlens_k: Optional[torch.Tensor], max_seqlen_k: int, m: int, k: int,
                B: int = HISA_BLOCK, out_idx: Optional[torch.Tensor] = None,
                out_scores: Optional[torch.Tensor] = None,
                out_blocks: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """HISA top-k token selection; returns out_idx int32 [total_q, k]."""
    _need(q_idx, "q_idx", torch.bfloat16, HISA_INDEX_DIM)
    _need(k_idx, "k_idx", torch.bfloat16, HISA_INDEX_DIM)
    _need(reps, "reps", torch.float32, HISA_INDEX_DIM)
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32)
    _need(seqlens_k, "seqlens_k", torch.int32, optional=True)
    total_q, S = q_idx.shape[0], cu_seqlens_q.numel() - 1
    if out_idx is None:
        out_idx = torch.empty(total_q, k, dtype=torch.int32, device=q_idx.device)
    _need(out_idx, "out_idx", torch.int32, k)
    _need(out_scores, "out_scores", torch.float32, k, optional=True)
    _need(out_blocks, "out_blocks", torch.int32, m, optional=True)
    need = hisa_select_workspace_size(total_q, S, max_seqlen_k, m, k, B)
    ws = _workspace(need, q_idx.device, workspace)
    _check(lib().hisa_select(_ptr(q_idx), _ptr(k_idx), _ptr(reps), _ptr(cu_seqlens_q),
                             _ptr(cu_seqlens_k), _ptr(seqlens_k), S, total_q, int(max_seqlen_k),
                             B, m, k, _ptr(out_idx), _ptr(out_scores), _ptr(out_blocks), _ptr(ws),
                             ws.numel(), _stream(stream)), "hisa_select")
    return out_idx


def hisa_decode_step(k_cache: torch.Tensor, reps: torch.Tensor, cu_seqlens_k: torch.Tensor,
                     seqlens_k: torch.Tensor, new_keys: torch.Tensor, q_idx: torch.Tensor,
                     max_seqlen_k: int, m: int, k: int, B: int = HISA_BLOCK,
                     out_idx: Optional[torch.Tensor] = None,
                     out_scores: Optional[torch.Tensor] = None,
                     out_blocks: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One decode step in one launch: append new_keys [S, 64] (one per sequence) and select
    for q_idx [S, 64] at the new positions; returns out_idx int32 [S, k]."""
    _need(k_cache, "k_cache", torch.bfloat16, HISA_INDEX_DIM)
    _need(reps, "reps", torch.float32, HISA_INDEX_DIM)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32)
    _need(seqlens_k, "seqlens_k", torch.int32)
    _need(new_keys, "new_keys", torch.bfloat16)
    _need(q_idx, "q_idx", torch.bfloat16, HISA_INDEX_DIM)
    S = cu_seqlens_k.numel() - 1
    if new_keys.numel() != S * HISA_INDEX_DIM or q_idx.shape[0] != S:
        raise ValueError("new_keys and q_idx need one row per sequence")
    if out_idx is None:
        out_idx = torch.empty(S, k, dtype=torch.int32, device=q_idx.device)
    _need(out_idx, "out_idx", torch.int32, k)
    _need(out_scores, "out_scores", torch.float32, k, optional=True)
    _need(out_blocks, "out_blocks", torch.int32, m, optional=True)
    _check(lib().hisa_decode_step(_ptr(k_cache), _ptr(reps), _ptr(cu_seqlens_k), _ptr(seqlens_k),
                                  _ptr(new_keys), _ptr(q_idx), S, int(max_seqlen_k), B, m, k,
                                  _ptr(out_idx), _ptr(out_scores), _ptr(out_blocks),
                                  _stream(stream)), "hisa_decode_step")
    return out_idx


def hisa_select_varm(q_idx: torch.Tensor, k_idx: torch.Tensor, reps: torch.Tensor,
                     cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor,
                     seqlens_k: Optional[torch.Tensor], m_seq: torch.Tensor, max_seqlen_k: int,
                     m_max: int, k: int, B: int = HISA_BLOCK,
                     out_idx: Optional[torch.Tensor] = None,
                     out_scores: Optional[torch.Tensor] = None,
                     out_blocks: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """HISA selection with a block budget per sequence (m_seq int32 [num_seqs] on the
    device, each in [1, m_max]); returns out_idx int32 [total_q, k]."""
    _need(q_idx, "q_idx", torch.bfloat16, HISA_INDEX_DIM)
    _need(k_idx, "k_idx", torch.bfloat16, HISA_INDEX_DIM)
    _need(reps, "reps", torch.float32, HISA_INDEX_DIM)
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32)
    _need(seqlens_k, "seqlens_k", torch.int32, optional=True)
    _need(m_seq, "m_seq", torch.int32)
    total_q, S = q_idx.shape[0], cu_seqlens_q.numel() - 1
    if m_seq.numel() != S:
        raise ValueError("m_seq must hold one budget per sequence")
    if out_idx is None:
        out_idx = torch.empty(total_q, k, dtype=torch.int32, device=q_idx.device)
    _need(out_idx, "out_idx", torch.int32, k)
    _need(out_scores, "out_scores", torch.float32, k, optional=True)
    _need(out_blocks, "out_blocks", torch.int32, m_max, optional=True)
    need = hisa_select_workspace_size(total_q, S, max_seqlen_k, m_max, k, B)
    ws = _workspace(need, q_idx.device, workspace)
    _check(lib().hisa_select_varm(_ptr(q_idx), _ptr(k_idx), _ptr(reps), _ptr(cu_seqlens_q),
                                  _ptr(cu_seqlens_k), _ptr(seqlens_k), _ptr(m_seq), S, total_q,
                                  int(max_seqlen_k), B, m_max, k, _ptr(out_idx), _ptr(out_scores),
                                  _ptr(out_blocks), _ptr(ws), ws.numel(), _stream(stream)),
           "hisa_select_varm")
    return out_idx


def hisa_fraction_blocks(cu_seqlens_k: torch.Tensor, seqlens_k: Optional[torch.Tensor], f: float,
                         m_max: int = HISA_MAX_M, B: int = HISA_BLOCK,
                         m_seq: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Per-sequence block budgets m_s = min(m_max, ceil(f * ceil(len_s / B))), computed on
    the device; returns m_seq int32 [num_seqs]."""
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32)
    _need(seqlens_k, "seqlens_k", torch.int32, optional=True)
    S = cu_seqlens_k.numel() - 1
    if m_seq is None:
        m_seq = torch.empty(S, dtype=torch.int32, device=cu_seqlens_k.device)
    _need(m_seq, "m_seq", torch.int32)
    _check(lib().hisa_fraction_blocks(_ptr(cu_seqlens_k), _ptr(seqlens_k), S, B, float(f), m_max,
                                      _ptr(m_seq), _stream(stream)), "hisa_fraction_blocks")
    return m_seq


def hisa_block_sparse_workspace_size(total_q: int, num_seqs: int, max_seqlen_k: int, m: int,
                                     B: int = HISA_BLOCK) -> int:
    return int(lib().hisa_block_sparse_workspace_size(total_q, num_seqs, max_seqlen_k, B, m))


def hisa_block_sparse_select(q_idx: torch.Tensor, reps: torch.Tensor, cu_seqlens_q: torch.Tensor,
                             cu_seqlens_k: torch.Tensor, seqlens_k: Optional[torch.Tensor],
                             max_seqlen_k: int, m: int, B: int = HISA_BLOCK,
                             out_idx: Optional[torch.Tensor] = None,
                             out_blocks: Optional[torch.Tensor] = None,
                             workspace: Optional[torch.Tensor] = None,
                             stream=None) -> torch.Tensor:
    """Stage 1 alone: every causal token of the m selected blocks, ascending; returns
    out_idx int32 [total_q, m * B]."""
    _need(q_idx, "q_idx", torch.bfloat16, HISA_INDEX_DIM)
    _need(reps, "reps", torch.float32, HISA_INDEX_DIM)
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32)
    _need(seqlens_k, "seqlens_k", torch.int32, optional=True)
    total_q, S = q_idx.shape[0], cu_seqlens_q.numel() - 1
    if out_idx is None:
        out_idx = torch.empty(total_q, m * B, dtype=torch.int32, device=q_idx.device)
    _need(out_idx, "out_idx", torch.int32, m * B)
    _need(out_blocks, "out_blocks", torch.int32, m, optional=True)
    need = hisa_block_sparse_workspace_size(total_q, S, max_seqlen_k, m, B)
    ws = _workspace(need, q_idx.device, workspace)
    _check(lib().hisa_block_sparse_select(_ptr(q_idx), _ptr(reps), _ptr(cu_seqlens_q),
                                          _ptr(cu_seqlens_k), _ptr(seqlens_k), S, total_q,
                                          int(max_seqlen_k), B, m, _ptr(out_idx),
                                          _ptr(out_blocks), _ptr(ws), ws.numel(),
                                          _stream(stream)), "hisa_block_sparse_select")
    return out_idx


def dsa_flat_select(q_idx: torch.Tensor, k_idx: torch.Tensor, cu_seqlens_q: torch.Tensor,
                    cu_seqlens_k: torch.Tensor, seqlens_k: Optional[torch.Tensor],
                    max_seqlen_k: int, k: int, out_idx: Optional[torch.Tensor] = None,
                    out_scores: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Flat DSA top-k over every causal key; returns out_idx int32 [total_q, k]."""
    _need(q_idx, "q_idx", torch.bfloat16, HISA_INDEX_DIM)
    _need(k_idx, "k_idx", torch.bfloat16, HISA_INDEX_DIM)
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32)
    _need(seqlens_k, "seqlens_k", torch.int32, optional=True)
    total_q, S = q_idx.shape[0], cu_seqlens_q.numel() - 1
    if out_idx is None:
        out_idx = torch.empty(total_q, k, dtype=torch.int32, device=q_idx.device)
    _need(out_idx, "out_idx", torch.int32, k)
    _need(out_scores, "out_scores", torch.float32, k, optional=True)
    need = dsa_flat_workspace_size(total_q, S, max_seqlen_k, k)
    ws = _workspace(need, q_idx.device, workspace)
    _check(lib().dsa_flat_select(_ptr(q_idx), _ptr(k_idx), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
                                 _ptr(seqlens_k), S, total_q, int(max_seqlen_k), k, _ptr(out_idx),
                                 _ptr(out_scores), _ptr(ws), ws.numel(), _stream(stream)),
           "dsa_flat_select")
    return out_idx


def hisa_device_status(clear: bool = True, stream=None) -> int:
    """Synchronise the stream and return (optionally clear) the sticky device status bits."""
    v = ctypes.c_int32(0)
    _check(lib().hisa_device_status(ctypes.byref(v), 1 if clear else 0, _stream(stream)),
           "hisa_device_status")
    return int(v.value)


def hisa_test_fault(mode: int) -> None:
    """Tests of the timeout path only: mode 1 makes the tensor-core token-scoring launches
    issue no loads (their bounded waits run out); 0 restores normal operation."""
    _check(lib().hisa_test_fault(int(mode)), "hisa_test_fault")


def hisa_timing_enable(on: bool) -> None:
    """Bracket every library kernel launch with CUDA events on its stream (or stop)."""
    _check(lib().hisa_timing_enable(1 if on else 0), "hisa_timing_enable")


def hisa_timing_collect(reset: bool = True) -> dict:
    """Per kernel kind: {'ms': total event time, 'launches': count, 'timed': timed count}."""
    L = lib()
    n = L.hisa_kernel_kinds()
    ms = (ctypes.c_double * n)()
    launches = (ctypes.c_longlong * n)()
    timed = (ctypes.c_longlong * n)()
    _check(L.hisa_timing_collect(ms, launches, timed, n, 1 if reset else 0),
           "hisa_timing_collect")
    return {L.hisa_kernel_name(i).decode(): {"ms": ms[i], "launches": launches[i],
                                             "timed": timed[i]} for i in range(n)}


HISA_ATT_DIM = 128


def hisa_sparse_attention(q_att: torch.Tensor, k_att: torch.Tensor, v_att: torch.Tensor,
                          topk_idx: torch.Tensor, cu_seqlens_q: torch.Tensor,
                          cu_seqlens_k: torch.Tensor, scale: float,
                          out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                          stream=None) -> torch.Tensor:
    """Attention over each query's selected tokens; returns out fp32 [total_q, H, 128]."""
    _need(q_att, "q_att", torch.bfloat16)
    _need(k_att, "k_att", torch.bfloat16, HISA_ATT_DIM)
    _need(v_att, "v_att", torch.bfloat16, HISA_ATT_DIM)
    _need(topk_idx, "topk_idx", torch.int32)
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32)
    if q_att.dim() != 3 or q_att.shape[2] != HISA_ATT_DIM:
        raise ValueError(f"q_att must be [total_q, H, {HISA_ATT_DIM}], got {tuple(q_att.shape)}")
    total_q, H = q_att.shape[0], q_att.shape[1]
    if topk_idx.dim() != 2 or topk_idx.shape[0] != total_q:
        raise ValueError("topk_idx must be [total_q, k]")
    if out is None:
        out = torch.empty(total_q, H, HISA_ATT_DIM, dtype=torch.float32, device=q_att.device)
    _need(out, "out", torch.float32)
    _need(lse, "lse", torch.float32, optional=True)
    _check(lib().hisa_sparse_attention(_ptr(q_att), _ptr(k_att), _ptr(v_att), _ptr(topk_idx),
                                       _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
                                       cu_seqlens_q.numel() - 1, total_q, H, topk_idx.shape[1],
                                       float(scale), _ptr(out), _ptr(lse), _stream(stream)),
           "hisa_sparse_attention")
    return out
