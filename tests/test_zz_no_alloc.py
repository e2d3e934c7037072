"""hisa_select_noalloc against hisa_select, through the C ABI.

hisa_select_noalloc serves callers that cannot allocate device memory when they
need a selection (an engine plug-in with a fixed memory plan, a decode path that
must not synchronise on cudaMalloc): it takes no workspace and uses a fixed
scratch array inside the library.  Its rows must equal hisa_select's rows (the
same kernels run on the same inputs, so the comparison is exact), call after
call, because every call reuses the same array.  This file is collected last.
"""

import ctypes

import numpy as np
import pytest
import torch

from parity import OnDevice, dev_bf16, dev_i32
from synth import decode_workload, gaussian_prefill

pytestmark = pytest.mark.gpu


def _lib():
    import sparse_attention_top_hisa_b200 as H
    L = H.lib()
    P, I = ctypes.c_void_p, ctypes.c_int
    L.hisa_select_noalloc.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, P, P, P, P]
    L.hisa_select_noalloc.restype = I
    return H, L


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call_noalloc(L, q, k, reps, cu_q, cu_k, sl, S, total_q, maxlen, m, topk):
    idx = torch.full((total_q, topk), 7, dtype=torch.int32, device="cuda")
    sc = torch.full((total_q, topk), 7.0, dtype=torch.float32, device="cuda")
    bl = torch.full((total_q, m), 7, dtype=torch.int32, device="cuda")
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = L.hisa_select_noalloc(_p(q), _p(k), _p(reps), _p(cu_q), _p(cu_k), _p(sl), S, total_q,
                               maxlen, 128, m, topk, _p(idx), _p(sc), _p(bl), st)
    assert rc == 0, rc
    torch.cuda.synchronize()
    return idx, sc, bl


def _cases():
    # prefill (tensor-core path): scratch = block lists, inverted lists and score rows
    w = gaussian_prefill(3000, 31, m=8, topk=256)
    dw = OnDevice(w)
    yield "prefill", dw.q, dw.k, dw.cu_q, dw.cu_k, dw.seqlens, 1, w.total_q, w.max_seqlen_k, 8, 256
    # decode: 16 single-query sequences (the cluster kernel, which uses no scratch)
    d = decode_workload(16, 5000, 1, 32, m=16, topk=512)
    kc = dev_bf16(d.k_cache)
    cu_k = dev_i32(d.cu_k)
    sl = dev_i32(d.seqlens0)
    q = dev_bf16(d.queries[0])
    yield ("decode", q, kc, dev_i32(np.arange(17)), cu_k, sl, 16, 16, int(d.seqlens0.max()), 16,
           512)


def test_noalloc_matches_select_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    H, L = _lib()
    H.hisa_device_status(clear=True)
    for name, q, k, cu_q, cu_k, sl, S, total_q, maxlen, m, topk in _cases():
        reps = H.hisa_pool_blocks(k, cu_k, sl, maxlen)
        sc_ref = torch.empty(total_q, topk, dtype=torch.float32, device="cuda")
        bl_ref = torch.empty(total_q, m, dtype=torch.int32, device="cuda")
        ref = H.hisa_select(q, k, reps, cu_q, cu_k, sl, maxlen, m, topk, out_scores=sc_ref,
                            out_blocks=bl_ref)
        torch.cuda.synchronize()
        for call in range(2):
            idx, sc, bl = _call_noalloc(L, q, k, reps, cu_q, cu_k, sl, S, total_q, maxlen, m, topk)
            assert torch.equal(idx, ref), (name, call)
            assert torch.equal(sc, sc_ref), (name, call)
            assert torch.equal(bl, bl_ref), (name, call)
    assert H.hisa_device_status() == 0


def test_noalloc_rejects_oversized_requests():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    H, L = _lib()
    t = torch.zeros(256, 64, dtype=torch.bfloat16, device="cuda")
    r = torch.zeros(2, 64, dtype=torch.float32, device="cuda")
    cu = dev_i32([0, 256])
    out = torch.zeros(1, 16, dtype=torch.int32, device="cuda")
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # 100000 queries x m=128 needs ~51 MB of block lists: refused before any launch
    rc = L.hisa_select_noalloc(_p(t), _p(t), _p(r), _p(cu), _p(cu), None, 1, 100000, 256, 128,
                               128, 16, _p(out), None, None, st)
    assert rc == 3
