"""Sequence- and row-sharded selection on one GPU: the shards of a batch, run one
after another through the C ABI, give exactly the rows of the unsharded call.

The multi-GPU path runs each shard on its own GPU with no exchange; here the
shards run in turn on one device (no shard waits on another), which checks the
split and the rebased layouts the ranks would use.  Integer inputs make every
score exact, so the rows must match bit for bit.
"""

import numpy as np
import pytest
import torch

from parity import OnDevice
from sparse_attention_top_hisa_b200.shard import query_cost, row_bounds, shard
from synth import Workload, decode_workload, integer_prefill, varlen_prefill

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_attention_top_hisa_b200 as H
    H.hisa_device_status(clear=True)
    yield


def H():
    import sparse_attention_top_hisa_b200 as mod
    return mod


def _i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def _run(q, k, cu_q, cu_k, lens, max_len, m, topk):
    h = H()
    reps = h.hisa_pool_blocks(k, cu_k, lens, max_len)
    total_q = q.shape[0]
    sc = torch.empty(total_q, topk, dtype=torch.float32, device="cuda")
    bl = torch.empty(total_q, m, dtype=torch.int32, device="cuda")
    idx = h.hisa_select(q, k, reps, cu_q, cu_k, lens, max_len, m, topk, out_scores=sc,
                        out_blocks=bl)
    return idx, sc, bl


def _check_shards(w, dw, world, balanced):
    full = [t.cpu().numpy() for t in _run(dw.q, dw.k, dw.cu_q, dw.cu_k, dw.seqlens,
                                          dw.max_seqlen_k, w.m, w.topk)]
    cost = query_cost(w.cu_q, w.cu_k, w.seqlens, w.B, w.m) if balanced else None
    bounds = row_bounds(w.total_q, world, cost)
    parts = [[], [], []]
    for r in range(world):
        sh = shard(w.cu_q, w.cu_k, w.seqlens, world, r, w.B, bounds)
        if sh.total_q == 0:
            continue
        got = _run(dw.q[sh.row0:sh.row1], dw.k[sh.key0:sh.key1], _i32(sh.cu_seqlens_q),
                   _i32(sh.cu_seqlens_k), _i32(sh.seqlens_k), sh.max_seqlen_k, w.m, w.topk)
        for p, t in zip(parts, got):
            p.append(t.cpu().numpy())
    torch.cuda.synchronize()
    assert H().hisa_device_status() == 0
    for p, f in zip(parts, full):
        assert np.array_equal(np.concatenate(p), f)


@pytest.mark.parametrize("world", [2, 3])
def test_row_shards_of_one_prefill(world):
    w = integer_prefill(5000, 41, m=8, topk=256)
    _check_shards(w, OnDevice(w), world, balanced=False)


@pytest.mark.parametrize("world", [2, 3, 4])
def test_shards_of_packed_varlen(world):
    w = varlen_prefill([1000, 129, 4096, 37, 2500, 640], 42, m=6, topk=300, integer=True)
    _check_shards(w, OnDevice(w), world, balanced=True)


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_shards_of_a_decode_batch(world):
    """16 decode sequences (one query each) split over ranks by whole sequences."""
    d = decode_workload(16, 3000, 1, 43, m=8, topk=512, integer=True)
    w = Workload("decode", d.queries[0], d.k_cache, np.arange(17, dtype=np.int32), d.cu_k,
                 d.seqlens0, d.B, d.m, d.topk, exact=True)
    _check_shards(w, OnDevice(w), world, balanced=False)
