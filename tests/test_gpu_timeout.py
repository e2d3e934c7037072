"""The timeout path of a bounded device-side wait, on the GPU, without faulting it.

hisa_test_fault(1) makes the tensor-core token-scoring launches issue no loads, so the
MMA thread's first wait on a stage that is never filled runs out after about a second.
Nothing asynchronous is in flight at that point (no copy and no MMA was issued; the
host model of the protocol, test_score_protocol.py, checks the same give-up path).
The call must come back, the device status word must hold HISA_ERR_TIMEOUT, every row
of that call must be -1 (scores 0), and the next call, with the switch off, must be
correct again on the same context.
"""

import time

import numpy as np
import pytest
import torch

import oracle
from parity import OnDevice
from synth import varlen_prefill

pytestmark = pytest.mark.gpu

HISA_ERR_TIMEOUT = 5


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_attention_top_hisa_b200 as H
    H.hisa_device_status(clear=True)
    yield
    H.hisa_test_fault(0)


def test_scoring_wait_times_out_and_rows_are_padded():
    import sparse_attention_top_hisa_b200 as H
    w = varlen_prefill([1500, 700], 61, m=8, topk=256, integer=True)  # 2200 queries: many tiles
    dw = OnDevice(w)
    reps = H.hisa_pool_blocks(dw.k, dw.cu_k, dw.seqlens, w.max_seqlen_k)
    sc = torch.full((w.total_q, w.topk), 7.0, dtype=torch.float32, device="cuda")
    out = torch.full((w.total_q, w.topk), 12345, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    H.hisa_device_status(clear=True)
    H.hisa_test_fault(1)
    try:
        t0 = time.perf_counter()
        H.hisa_select(dw.q, dw.k, reps, dw.cu_q, dw.cu_k, dw.seqlens, w.max_seqlen_k, w.m, w.topk,
                      out_idx=out, out_scores=sc)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        H.hisa_test_fault(0)
    st = H.hisa_device_status(clear=True)
    assert st & (1 << HISA_ERR_TIMEOUT), f"status {st:#x} lacks the timeout bit"
    assert elapsed < 30.0
    assert bool((out == -1).all()), "rows of the timed-out call are not all -1"
    assert bool((sc == 0).all())
    # the context is still usable: the same call, switch off, is exact again
    idx = H.hisa_select(dw.q, dw.k, reps, dw.cu_q, dw.cu_k, dw.seqlens, w.max_seqlen_k, w.m,
                        w.topk)
    torch.cuda.synchronize()
    assert H.hisa_device_status(clear=True) == 0
    o_idx, _, _, _ = oracle.hisa_workload(w)
    assert np.array_equal(idx.cpu().numpy(), o_idx)
