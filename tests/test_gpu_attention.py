"""The sparse attention step (hisa_sparse_attention) against the CPU oracle, through
the C ABI.

Inputs are bf16 (exact in both); the GPU accumulates in fp32 and uses the fast CUDA
exponential (__expf, a few ulp), the oracle works in fp64.  Tolerance, from the arithmetic: a score is an fp32 dot
product of 128 terms (relative error ~1e-5 of |q||k|, with scale 1/sqrt(128) at most
~1e-4 absolute), which moves a softmax weight by that much relative; the output is a
convex combination of value rows of magnitude <= ~5, accumulated over <= 2048 terms in
fp32.  So |out - ref| <= 1e-3 + 1e-3 |ref| and |lse - ref| <= 1e-4 + 1e-5 |ref|.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from parity import OnDevice, dev_bf16, dev_i32, sample_rows
from synth import bf16_from_f32, config_workload, decode_workload, gaussian_prefill

pytestmark = pytest.mark.gpu

ATT_D = 128


def H():
    import sparse_attention_top_hisa_b200 as mod
    return mod


def _att_inputs(rows_k, total_q, heads, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    q = bf16_from_f32(rng.standard_normal((total_q, heads, ATT_D), dtype=np.float32))
    k = bf16_from_f32(rng.standard_normal((rows_k, ATT_D), dtype=np.float32))
    v = bf16_from_f32(rng.standard_normal((rows_k, ATT_D), dtype=np.float32))
    return q, k, v


def _run(q, k, v, idx, cu_q, cu_k, heads, scale):
    h = H()
    out = torch.full((idx.shape[0], heads, ATT_D), 7.0, dtype=torch.float32, device="cuda")
    lse = torch.full((idx.shape[0], heads), 7.0, dtype=torch.float32, device="cuda")
    h.hisa_sparse_attention(dev_bf16(q).view(-1, heads, ATT_D), dev_bf16(k), dev_bf16(v),
                            dev_i32(idx), dev_i32(cu_q), dev_i32(cu_k), scale, out=out, lse=lse)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


def _check(out, lse, ref_out, ref_lse):
    assert np.all(np.abs(out - ref_out) <= 1e-3 + 1e-3 * np.abs(ref_out)), \
        float(np.max(np.abs(out - ref_out)))
    inf = np.isinf(ref_lse)
    assert np.all(np.isinf(lse[inf]) & (lse[inf] < 0))
    assert np.all(np.abs(lse[~inf] - ref_lse[~inf]) <= 1e-4 + 1e-5 * np.abs(ref_lse[~inf]))
    assert np.all(out[np.broadcast_to(inf[..., None], out.shape)] == 0)


def test_attention_decode_rows_from_hisa():
    """16 decode queries (8-CTA clusters), the indices hisa_select chose."""
    h = H()
    S, L, m, topk, heads = 16, 5000, 16, 512, 16
    d = decode_workload(S, L, 1, 31, m=m, topk=topk)
    kc, cu_k, lens = dev_bf16(d.k_cache), dev_i32(d.cu_k), dev_i32(d.seqlens0)
    reps = h.hisa_pool_blocks(kc, cu_k, lens, L)
    idx = h.hisa_select(dev_bf16(d.queries[0]), kc, reps, dev_i32(np.arange(S + 1)), cu_k, lens,
                        L, m, topk).cpu().numpy()
    q, k, v = _att_inputs(d.k_cache.shape[0], S, heads, 5)
    cu_q = np.arange(S + 1, dtype=np.int32)
    scale = 1.0 / math.sqrt(ATT_D)
    h.hisa_device_status(clear=True)
    out, lse = _run(q, k, v, idx, cu_q, d.cu_k, heads, scale)
    assert h.hisa_device_status() == 0
    ref_out, ref_lse = oracle.sparse_attention(q, k, v, idx, cu_q, d.cu_k, heads, scale)
    _check(out, lse, ref_out, ref_lse)


def test_attention_prefill_rows_from_hisa():
    """1200 prefill queries (one CTA each), early rows padded with -1."""
    h = H()
    w = gaussian_prefill(1200, 17, m=4, topk=256)
    dk, cu_q, cu_k, sl = dev_bf16(w.k), dev_i32(w.cu_q), dev_i32(w.cu_k), dev_i32(w.seqlens)
    reps = h.hisa_pool_blocks(dk, cu_k, sl, w.max_seqlen_k)
    idx = h.hisa_select(dev_bf16(w.q), dk, reps, cu_q, cu_k, sl, w.max_seqlen_k, w.m,
                        w.topk).cpu().numpy()
    heads = 4
    q, k, v = _att_inputs(w.k.shape[0], w.total_q, heads, 6)
    scale = 0.09
    out, lse = _run(q, k, v, idx, w.cu_q, w.cu_k, heads, scale)
    assert H().hisa_device_status() == 0
    ref_out, ref_lse = oracle.sparse_attention(q, k, v, idx, w.cu_q, w.cu_k, heads, scale)
    _check(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("heads,topk,nq", [(1, 100, 5), (32, 333, 3), (8, 64, 400)])
def test_attention_edges(heads, topk, nq):
    """Arbitrary index order with padding anywhere, rows with no index, k not a multiple
    of the tile, one and 32 heads, both cluster sizes."""
    rng = np.random.Generator(np.random.PCG64(heads * 1000 + topk))
    lengths = [600, 1500]
    cu_k = np.array([0, 640, 2176], np.int32)
    per = [nq, nq + 1]
    cu_q = np.array([0, per[0], per[0] + per[1]], np.int32)
    total_q = int(cu_q[-1])
    idx = np.full((total_q, topk), -1, np.int32)
    for s in range(2):
        for r in range(int(cu_q[s]), int(cu_q[s + 1])):
            if r % 4 == 3:
                continue  # a row with no index
            n = int(rng.integers(1, topk + 1))
            idx[r, rng.choice(topk, n, replace=False)] = rng.choice(lengths[s], n, replace=False)
    q, k, v = _att_inputs(int(cu_k[-1]), total_q, heads, 7)
    out, lse = _run(q, k, v, idx, cu_q, cu_k, heads, 0.1)
    assert H().hisa_device_status() == 0
    ref_out, ref_lse = oracle.sparse_attention(q, k, v, idx, cu_q, cu_k, heads, 0.1)
    _check(out, lse, ref_out, ref_lse)


def test_attention_out_of_region_index_is_reported():
    h = H()
    cu_k = np.array([0, 256], np.int32)
    cu_q = np.array([0, 2], np.int32)
    idx = np.array([[0, 5, 300, -1], [7, -1, -1, 1]], np.int32)  # 300 is outside the region
    q, k, v = _att_inputs(256, 2, 2, 8)
    h.hisa_device_status(clear=True)
    out, lse = _run(q, k, v, idx, cu_q, cu_k, 2, 0.1)
    assert h.hisa_device_status(clear=True) & (1 << 1)
    fixed = idx.copy()
    fixed[0, 2] = -1  # the reported entry is ignored
    ref_out, ref_lse = oracle.sparse_attention(q, k, v, fixed, cu_q, cu_k, 2, 0.1)
    _check(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("order", ["rising", "falling", "shuffled"])
@pytest.mark.parametrize("heads", [8, 20])
@pytest.mark.parametrize("nq", [1, 150])
def test_attention_score_ramp(order, heads, nq):
    """Scores that climb by about 12 nats per tile of 128 tokens (about 200 over the
    row): visited in rising order every tile raises the running maximum (the rescale
    of the output and the sum on each tile), falling order keeps the first maximum
    and lets later probabilities underflow, shuffled order mixes both.  One query
    per sequence runs on clusters, 150 per sequence on one CTA per query."""
    rng = np.random.Generator(np.random.PCG64(heads * 7 + nq + len(order)))
    S, L, topk = 2, 2048, 2048
    u = rng.standard_normal(ATT_D)
    u /= np.linalg.norm(u)
    slope = 200.0 / (L * 15.0 / math.sqrt(ATT_D))  # score ~ 200 * j / L at a head factor of 15
    k = np.concatenate([np.outer(np.arange(L) * slope, u) for _ in range(S)])
    k = bf16_from_f32((k + 0.05 * rng.standard_normal(k.shape)).astype(np.float32))
    v = bf16_from_f32(rng.standard_normal((S * L, ATT_D), dtype=np.float32))
    total_q = S * nq
    a = rng.uniform(10.0, 20.0, (total_q, heads))
    q = bf16_from_f32((a[..., None] * u).astype(np.float32))
    base = np.arange(L, dtype=np.int32)
    if order == "falling":
        base = base[::-1].copy()
    idx = np.empty((total_q, topk), np.int32)
    for r in range(total_q):
        idx[r] = rng.permutation(base) if order == "shuffled" else base
    cu_k = np.array([0, L, 2 * L], np.int32)
    cu_q = np.array([0, nq, 2 * nq], np.int32)
    scale = 1.0 / math.sqrt(ATT_D)
    H().hisa_device_status(clear=True)
    out, lse = _run(q, k, v, idx, cu_q, cu_k, heads, scale)
    assert H().hisa_device_status() == 0
    ref_out, ref_lse = oracle.sparse_attention(q, k, v, idx, cu_q, cu_k, heads, scale)
    assert float(ref_lse.max()) > 150.0  # the ramp is as steep as intended
    _check(out, lse, ref_out, ref_lse)


def test_attention_prefill_32k_full_size_sampled():
    """The 32K needle prefill at the size the bench times: 32768 queries x 2048 selected
    tokens (the indices hisa_select chose), 16 heads, one CTA per query; sampled rows
    (seeded, plus sequence and block edges) against the oracle."""
    h = H()
    w = config_workload(3)
    dw = OnDevice(w)
    reps = h.hisa_pool_blocks(dw.k, dw.cu_k, dw.seqlens, dw.max_seqlen_k)
    idx = h.hisa_select(dw.q, dw.k, reps, dw.cu_q, dw.cu_k, dw.seqlens, dw.max_seqlen_k, w.m,
                        w.topk).cpu().numpy()
    del dw, reps
    heads = 16
    q, k, v = _att_inputs(w.k.shape[0], w.total_q, heads, 11)
    scale = 1.0 / math.sqrt(ATT_D)
    h.hisa_device_status(clear=True)
    out, lse = _run(q, k, v, idx, w.cu_q, w.cu_k, heads, scale)
    assert h.hisa_device_status() == 0
    rows = sample_rows(w, 40, 12)
    ref_out, ref_lse = oracle.sparse_attention(q[rows], k, v, idx[rows],
                                               np.array([0, len(rows)], np.int32), w.cu_k,
                                               heads, scale)
    _check(out[rows], lse[rows], ref_out, ref_lse)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))


def test_attention_decode_full_size():
    """The decode batch at the size the bench times: 16 sequences x 32768 keys, k = 2048,
    16 heads (the split over a cluster per query); every row against the oracle."""
    h = H()
    d = config_workload(2, steps=1)
    S, cap = d.num_seqs, d.capacity
    kc, cu_k, lens = dev_bf16(d.k_cache), dev_i32(d.cu_k), dev_i32(d.seqlens0)
    reps = h.hisa_pool_blocks(kc, cu_k, lens, cap)
    idx = h.hisa_select(dev_bf16(d.queries[0]), kc, reps, dev_i32(np.arange(S + 1)), cu_k, lens,
                        cap, d.m, d.topk).cpu().numpy()
    heads = 16
    q, k, v = _att_inputs(d.k_cache.shape[0], S, heads, 13)
    cu_q = np.arange(S + 1, dtype=np.int32)
    scale = 1.0 / math.sqrt(ATT_D)
    h.hisa_device_status(clear=True)
    out, lse = _run(q, k, v, idx, cu_q, d.cu_k, heads, scale)
    assert h.hisa_device_status() == 0
    ref_out, ref_lse = oracle.sparse_attention(q, k, v, idx, cu_q, d.cu_k, heads, scale)
    _check(out, lse, ref_out, ref_lse)
