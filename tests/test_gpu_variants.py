"""The selection variants against the oracle, through the C ABI: stage 1 on its own
(hisa_block_sparse_select), a block budget per sequence (hisa_select_varm with
hisa_fraction_blocks), and block budgets above 128 (the select that reads the score
rows from memory).  Integer inputs are compared bit for bit; the 32768-token needle
prefill follows the band rule of parity.py.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from parity import OnDevice, check_block_band, dev_bf16, dev_i32, sample_rows
from synth import config_workload, varlen_prefill

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


def _positions(w, rows):
    out = []
    for row in rows:
        s = int(np.searchsorted(w.cu_q, row, side="right") - 1)
        while w.cu_q[s + 1] <= row:
            s += 1
        L = int(w.seqlens[s])
        out.append(L - int(w.cu_q[s + 1] - w.cu_q[s]) + (int(row) - int(w.cu_q[s])))
    return np.array(out, np.int64)


def _expand(blocks, pos, B):
    """Every token j <= pos of the listed blocks (ascending), -1 padded to m * B."""
    m = blocks.shape[0]
    row = np.full(m * B, -1, np.int64)
    for s, b in enumerate(blocks):
        if b < 0:
            continue
        j = b * B + np.arange(B)
        row[s * B:(s + 1) * B] = np.where(j <= pos, j, -1)
    return row


# ---------------------------------------------------------------------------
# stage 1 alone

@pytest.mark.parametrize("lengths,m", [([4096], 8), ([129, 1000, 2500, 37], 4), ([3000], 1)])
def test_block_sparse_exact_integer(lengths, m):
    w = varlen_prefill(lengths, 300 + m, m=m, topk=m * 128, integer=True)
    dw = OnDevice(w)
    h = H()
    reps = h.hisa_pool_blocks(dw.k, dw.cu_k, dw.seqlens, w.max_seqlen_k)
    bl = torch.empty(w.total_q, m, dtype=torch.int32, device="cuda")
    idx = h.hisa_block_sparse_select(dw.q, reps, dw.cu_q, dw.cu_k, dw.seqlens, w.max_seqlen_k, m,
                                     out_blocks=bl)
    torch.cuda.synchronize()
    assert h.hisa_device_status() == 0
    o_reps = oracle.pool(w.k, w.cu_k, w.seqlens, w.B)
    o_bl, _ = oracle.block_select(w.q, o_reps, w.cu_q, w.cu_k, w.seqlens, w.B, m)
    assert np.array_equal(bl.cpu().numpy(), o_bl)
    pos = _positions(w, np.arange(w.total_q))
    ref = np.stack([_expand(o_bl[r], pos[r], w.B) for r in range(w.total_q)])
    assert np.array_equal(idx.cpu().numpy(), ref)
    # with m * B = k, HISA's stage 2 keeps every candidate: the same token sets
    o_idx, _, _, _ = oracle.hisa_workload(w)
    got = idx.cpu().numpy()
    for r in range(w.total_q):
        assert set(got[r][got[r] >= 0].tolist()) == set(o_idx[r][o_idx[r] >= 0].tolist())


def test_block_sparse_needles_m_times_B_equals_k():
    """The 32768-token needle prefill, m = k / B = 16: the block sets follow the band
    rule against the oracle, each row is exactly the tokens of its blocks, and hisa_select
    with the same m and k = m * B selects the same token sets."""
    w = config_workload(3)
    m, k = w.topk // w.B, w.topk
    dw = OnDevice(w)
    h = H()
    reps = h.hisa_pool_blocks(dw.k, dw.cu_k, dw.seqlens, w.max_seqlen_k)
    bl = torch.empty(w.total_q, m, dtype=torch.int32, device="cuda")
    idx = h.hisa_block_sparse_select(dw.q, reps, dw.cu_q, dw.cu_k, dw.seqlens, w.max_seqlen_k, m,
                                     out_blocks=bl)
    hidx = h.hisa_select(dw.q, dw.k, reps, dw.cu_q, dw.cu_k, dw.seqlens, w.max_seqlen_k, m, k)
    torch.cuda.synchronize()
    assert h.hisa_device_status() == 0
    got, blk, hs = idx.cpu().numpy(), bl.cpu().numpy(), hidx.cpu().numpy()
    rows = sample_rows(w, 300, 17)
    o_reps = oracle.pool(w.k, w.cu_k, w.seqlens, w.B)
    o_bl, _ = oracle.block_select(w.q, o_reps, w.cu_q, w.cu_k, w.seqlens, w.B, m, rows=rows)
    check_block_band(w, rows, blk[rows], o_bl, o_reps)
    pos = _positions(w, np.arange(w.total_q))
    for r in range(0, w.total_q, 61):
        assert np.array_equal(got[r], _expand(blk[r], pos[r], w.B))
    # the same blocks (same stage 1 kernels), every candidate kept: equal sets, all rows
    gs = np.sort(np.where(got >= 0, got, np.iinfo(np.int32).max), axis=1)
    hs_ = np.sort(np.where(hs >= 0, hs, np.iinfo(np.int32).max), axis=1)
    assert np.array_equal(gs[:, :k], hs_)


# ---------------------------------------------------------------------------
# block budget per sequence

def _fraction_budgets(lengths, f, m_max, B=128):
    return np.array([min(m_max, max(1, math.ceil(f * ((L + B - 1) // B)))) for L in lengths],
                    np.int32)


def test_fraction_blocks_on_the_device():
    h = H()
    lengths = [1, 127, 128, 129, 4096, 40000, 65536, 300]
    w = varlen_prefill(lengths, 3, m=8, topk=64, integer=True)
    for f, m_max in ((0.5, 512), (0.25, 64), (1.0, 512), (0.01, 7)):
        ms = h.hisa_fraction_blocks(dev_i32(w.cu_k), dev_i32(w.seqlens), f, m_max)
        torch.cuda.synchronize()
        assert np.array_equal(ms.cpu().numpy(), _fraction_budgets(lengths, f, m_max)), (f, m_max)
    assert h.hisa_device_status() == 0


@pytest.mark.parametrize("f", [0.5, 0.25])
def test_varm_equals_per_sequence_oracle(f):
    """Packed integer varlen with m_s = ceil(f * M_s): every sequence's rows equal the
    oracle run on that sequence alone with m = m_s (the long sequence, whose budget is
    above 128, on sampled rows)."""
    lengths = [3000, 129, 40000, 700, 9000]
    w = varlen_prefill(lengths, 77, m=512, topk=1024, integer=True)
    dw = OnDevice(w)
    h = H()
    m_max = 512
    ms = h.hisa_fraction_blocks(dw.cu_k, dw.seqlens, f, m_max)
    reps = h.hisa_pool_blocks(dw.k, dw.cu_k, dw.seqlens, w.max_seqlen_k)
    sc = torch.empty(w.total_q, w.topk, dtype=torch.float32, device="cuda")
    bl = torch.empty(w.total_q, m_max, dtype=torch.int32, device="cuda")
    idx = h.hisa_select_varm(dw.q, dw.k, reps, dw.cu_q, dw.cu_k, dw.seqlens, ms, w.max_seqlen_k,
                             m_max, w.topk, out_scores=sc, out_blocks=bl)
    torch.cuda.synchronize()
    assert h.hisa_device_status() == 0
    budgets = ms.cpu().numpy()
    assert np.array_equal(budgets, _fraction_budgets(lengths, f, m_max))
    got, gsc, gbl = idx.cpu().numpy(), sc.cpu().numpy(), bl.cpu().numpy()
    rng = np.random.Generator(np.random.PCG64(5))
    for s, L in enumerate(lengths):
        a, b = int(w.cu_q[s]), int(w.cu_q[s + 1])
        k0, k1 = int(w.cu_k[s]), int(w.cu_k[s + 1])
        local = np.arange(b - a, dtype=np.int32)
        if L > 5000:
            local = np.unique(np.r_[rng.choice(b - a, 48, replace=False), 0, 127, 128, b - a - 1])
            local = local.astype(np.int32)
        m_s = int(budgets[s])
        o_idx, o_sc, o_bl, _ = oracle.hisa(w.q[a:b], w.k[k0:k1], np.array([0, b - a], np.int32),
                                           np.array([0, k1 - k0], np.int32),
                                           np.array([L], np.int32), w.B, m_s, w.topk, rows=local)
        assert np.array_equal(got[a + local], o_idx), s
        valid = o_idx >= 0
        assert np.array_equal(gsc[a + local][valid].astype(np.float64), o_sc[valid]), s
        assert np.array_equal(gbl[a + local][:, :m_s], o_bl), s
        assert np.all(gbl[a + local][:, m_s:] == -1), s


def test_varm_with_equal_budgets_is_hisa_select():
    w = varlen_prefill([2000, 129, 5000], 78, m=24, topk=512)
    dw = OnDevice(w)
    h = H()
    reps = h.hisa_pool_blocks(dw.k, dw.cu_k, dw.seqlens, w.max_seqlen_k)
    ms = dev_i32(np.full(w.num_seqs, 24, np.int32))
    a = h.hisa_select_varm(dw.q, dw.k, reps, dw.cu_q, dw.cu_k, dw.seqlens, ms, w.max_seqlen_k, 24,
                           512)
    b = h.hisa_select(dw.q, dw.k, reps, dw.cu_q, dw.cu_k, dw.seqlens, w.max_seqlen_k, 24, 512)
    torch.cuda.synchronize()
    assert h.hisa_device_status() == 0
    assert torch.equal(a, b)


def test_varm_decode_budgets():
    """Few queries (the cluster path) with different budgets per sequence."""
    h = H()
    lengths = [5000, 9000, 3000, 12000]
    w = varlen_prefill(lengths, 79, m=64, topk=512, integer=True)
    rows = np.array([int(w.cu_q[s + 1]) - 1 for s in range(w.num_seqs)])
    q1 = w.q[rows]
    cu_q = np.arange(w.num_seqs + 1, dtype=np.int32)
    budgets = np.array([5, 64, 1, 17], np.int32)
    dk = dev_bf16(w.k)
    dcu_k, dsl = dev_i32(w.cu_k), dev_i32(w.seqlens)
    reps = h.hisa_pool_blocks(dk, dcu_k, dsl, w.max_seqlen_k)
    bl = torch.empty(w.num_seqs, 64, dtype=torch.int32, device="cuda")
    idx = h.hisa_select_varm(dev_bf16(q1), dk, reps, dev_i32(cu_q), dcu_k, dsl, dev_i32(budgets),
                             w.max_seqlen_k, 64, 512, out_blocks=bl)
    torch.cuda.synchronize()
    assert h.hisa_device_status() == 0
    for s in range(w.num_seqs):
        k0, k1 = int(w.cu_k[s]), int(w.cu_k[s + 1])
        o_idx, _, o_bl, _ = oracle.hisa(q1[s:s + 1], w.k[k0:k1], np.array([0, 1], np.int32),
                                        np.array([0, k1 - k0], np.int32),
                                        np.array([lengths[s]], np.int32), w.B, int(budgets[s]),
                                        512)
        assert np.array_equal(idx.cpu().numpy()[s], o_idx[0]), s
        assert np.array_equal(bl.cpu().numpy()[s][:budgets[s]], o_bl[0]), s


def test_varm_rejects_bad_budgets_on_the_device():
    h = H()
    w = varlen_prefill([1000, 2000], 80, m=8, topk=64, integer=True)
    dw = OnDevice(w)
    reps = h.hisa_pool_blocks(dw.k, dw.cu_k, dw.seqlens, w.max_seqlen_k)
    h.hisa_device_status(clear=True)
    h.hisa_select_varm(dw.q, dw.k, reps, dw.cu_q, dw.cu_k, dw.seqlens,
                       dev_i32(np.array([0, 9], np.int32)), w.max_seqlen_k, 8, 64)
    st = h.hisa_device_status(clear=True)
    assert st & (1 << 1)  # HISA_ERR_INVALID_ARG


@pytest.mark.parametrize("m", [200, 512])
def test_large_m_exact_integer(m):
    """Budgets above 128: list entries with 9 slot bits and the memory-read select."""
    w = varlen_prefill([70000, 3000], 81 + m, m=m, topk=2048, integer=True)
    dw = OnDevice(w)
    h = H()
    reps = h.hisa_pool_blocks(dw.k, dw.cu_k, dw.seqlens, w.max_seqlen_k)
    sc = torch.empty(w.total_q, w.topk, dtype=torch.float32, device="cuda")
    idx = h.hisa_select(dw.q, dw.k, reps, dw.cu_q, dw.cu_k, dw.seqlens, w.max_seqlen_k, m, w.topk,
                        out_scores=sc)
    torch.cuda.synchronize()
    assert h.hisa_device_status() == 0
    rows = sample_rows(w, 60, 3)
    o_idx, o_sc, _, _ = oracle.hisa_workload(w, rows=rows)
    assert np.array_equal(idx.cpu().numpy()[rows], o_idx)
    valid = o_idx >= 0
    assert np.array_equal(sc.cpu().numpy()[rows][valid].astype(np.float64), o_sc[valid])
