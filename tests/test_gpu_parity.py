"""CUDA path against the CPU oracle, through the C ABI.

Integer-valued inputs must match bit for bit (every fp32 score and mean is
exact there); Gaussian inputs follow the band rule of parity.py.  Sizes span
several blocks with ragged tails; the full benchmark shapes are checked on
sampled rows the oracle computes one by one.
"""

import numpy as np
import pytest
import torch

import oracle
from parity import (OnDevice, check_block_band, check_rows_structure, check_token_band, dev_bf16,
                    dev_i32, exact_scores, sample_rows)
from synth import (bf16_from_f32, config_workload, decode_workload, gaussian_prefill,
                   integer_prefill, varlen_prefill)

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


def fp32_reps_from_exact(w, o_reps):
    """Integer keys: the oracle's exact block sums divided by the key count in fp32 with
    one correctly rounded division, which is how the CUDA path forms a mean (full blocks
    divide by 128 and are exact either way)."""
    out = o_reps.astype(np.float32)
    for s in range(w.num_seqs):
        L = int(w.seqlens[s])
        for b in range((L + w.B - 1) // w.B):
            cnt = min(w.B, L - b * w.B)
            r = int(w.cu_k[s]) // w.B + b
            sums = np.round(o_reps[r] * cnt)
            out[r] = sums.astype(np.float32) / np.float32(cnt)
    return out


def run_hisa(dw, m, topk):
    h = H()
    reps = h.hisa_pool_blocks(dw.k, dw.cu_k, dw.seqlens, dw.max_seqlen_k)
    total_q = dw.q.shape[0]
    sc = torch.empty(total_q, topk, dtype=torch.float32, device="cuda")
    bl = torch.empty(total_q, m, dtype=torch.int32, device="cuda")
    idx = h.hisa_select(dw.q, dw.k, reps, dw.cu_q, dw.cu_k, dw.seqlens, dw.max_seqlen_k, m, topk,
                        out_scores=sc, out_blocks=bl)
    torch.cuda.synchronize()
    assert h.hisa_device_status() == 0
    return idx.cpu().numpy(), sc.cpu().numpy(), bl.cpu().numpy(), reps.cpu().numpy()


def run_dsa(dw, topk):
    h = H()
    total_q = dw.q.shape[0]
    sc = torch.empty(total_q, topk, dtype=torch.float32, device="cuda")
    idx = h.dsa_flat_select(dw.q, dw.k, dw.cu_q, dw.cu_k, dw.seqlens, dw.max_seqlen_k, topk,
                            out_scores=sc)
    torch.cuda.synchronize()
    assert h.hisa_device_status() == 0
    return idx.cpu().numpy(), sc.cpu().numpy()


# ---------------------------------------------------------------------------
# pooling

def test_pool_exact_integer():
    w = config_workload(1)
    dw = OnDevice(w)
    reps = H().hisa_pool_blocks(dw.k, dw.cu_k, dw.seqlens, dw.max_seqlen_k).cpu().numpy()
    ref = oracle.pool(w.k, w.cu_k, w.seqlens, w.B)
    assert np.array_equal(reps.astype(np.float64), ref)


def test_pool_gaussian_ragged():
    w = varlen_prefill([1000, 129, 37, 4096, 128], 7, m=8, topk=64)
    dw = OnDevice(w)
    reps = H().hisa_pool_blocks(dw.k, dw.cu_k, dw.seqlens, dw.max_seqlen_k).cpu().numpy()
    ref = oracle.pool(w.k, w.cu_k, w.seqlens, w.B)
    assert np.allclose(reps, ref, rtol=1e-5, atol=1e-6)


# ---------------------------------------------------------------------------
# HISA and DSA, exact mode

INTEGER_CASES = [
    # (lengths, m, k)
    ([4096], 8, 256),          # the tiny benchmark configuration
    ([1000], 8, 256),          # ragged tail block
    ([300], 3, 2048),          # k larger than every candidate set
    ([129, 1000, 4096, 37], 4, 100),  # packed varlen
    ([2000], 1, 64),           # m < 3: only the own block is forced
    ([2000], 2, 64),           # m < 3: own and previous
    ([640], 5, 128),           # m equal to the number of blocks
]


@pytest.mark.parametrize("lengths,m,k", INTEGER_CASES, ids=[str(c) for c in INTEGER_CASES])
def test_hisa_exact_integer(lengths, m, k):
    w = varlen_prefill(lengths, 100 + len(lengths) + m, m=m, topk=k, integer=True)
    dw = OnDevice(w)
    idx, sc, bl, reps = run_hisa(dw, m, k)
    o_idx, o_sc, o_bl, o_reps = oracle.hisa_workload(w)
    assert np.array_equal(reps, fp32_reps_from_exact(w, o_reps))
    assert np.array_equal(bl, o_bl)
    assert np.array_equal(idx, o_idx)
    valid = o_idx >= 0
    assert np.array_equal(sc[valid].astype(np.float64), o_sc[valid])
    assert np.all(sc[~valid] == 0)


@pytest.mark.parametrize("lengths,k", [([4096], 256), ([129, 1000, 2500], 300), ([77], 2048)])
def test_dsa_exact_integer(lengths, k):
    w = varlen_prefill(lengths, 200 + k, m=8, topk=k, integer=True)
    dw = OnDevice(w)
    idx, sc = run_dsa(dw, k)
    o_idx, o_sc = oracle.dsa_workload(w)
    assert np.array_equal(idx, o_idx)
    valid = o_idx >= 0
    assert np.array_equal(sc[valid].astype(np.float64), o_sc[valid])


# Few queries (fewer than two per SM) take the cluster path: decode-shaped states with
# long key caches, exact on integer inputs.
DECODE_INT_CASES = [
    # (num_seqs, live keys, m, k)
    (16, 5000, 16, 512),     # a decode batch; ties at the block and token boundaries
    (3, 40000, 64, 2048),    # long caches: 313 eligible blocks
    (5, 300, 8, 256),        # at most m blocks: every block is selected
    (4, 2000, 1, 64),        # m < 3: only the own block is forced
    (4, 2000, 2, 64),        # m < 3: own and previous
    (2, 9000, 128, 2048),    # the largest m
]


@pytest.mark.parametrize("S,L,m,k", DECODE_INT_CASES, ids=[str(c) for c in DECODE_INT_CASES])
def test_decode_exact_integer(S, L, m, k):
    h = H()
    d = decode_workload(S, L, 1, 700 + m, m=m, topk=k, integer=True)
    kc, cu_k, lens = dev_bf16(d.k_cache), dev_i32(d.cu_k), dev_i32(d.seqlens0)
    cu_q = dev_i32(np.arange(S + 1))
    q = dev_bf16(d.queries[0])
    reps = h.hisa_pool_blocks(kc, cu_k, lens, L)
    sc = torch.empty(S, k, dtype=torch.float32, device="cuda")
    bl = torch.empty(S, m, dtype=torch.int32, device="cuda")
    idx = h.hisa_select(q, kc, reps, cu_q, cu_k, lens, L, m, k, out_scores=sc, out_blocks=bl)
    torch.cuda.synchronize()
    assert h.hisa_device_status() == 0
    o_idx, o_sc, o_bl, _ = oracle.hisa(d.queries[0], d.k_cache, np.arange(S + 1, dtype=np.int32),
                                       d.cu_k, d.seqlens0, d.B, m, k)
    assert np.array_equal(bl.cpu().numpy(), o_bl)
    assert np.array_equal(idx.cpu().numpy(), o_idx)
    scn = sc.cpu().numpy()
    valid = o_idx >= 0
    assert np.array_equal(scn[valid].astype(np.float64), o_sc[valid])
    assert np.all(scn[~valid] == 0)


def test_few_queries_several_per_sequence_exact():
    """The cluster path with several query rows per sequence (the last 40 positions of
    each of two sequences), exact on integer inputs."""
    h = H()
    w = varlen_prefill([3000, 1500], 41, m=8, topk=256, integer=True)
    tail = 40
    rows = np.concatenate([np.arange(int(w.cu_q[s + 1]) - tail, int(w.cu_q[s + 1]))
                           for s in range(w.num_seqs)])
    qsel = w.q[rows]
    cu_q = np.arange(w.num_seqs + 1, dtype=np.int32) * tail
    dq, dk = dev_bf16(qsel), dev_bf16(w.k)
    dcu_q, dcu_k, dsl = dev_i32(cu_q), dev_i32(w.cu_k), dev_i32(w.seqlens)
    reps = h.hisa_pool_blocks(dk, dcu_k, dsl, w.max_seqlen_k)
    idx = h.hisa_select(dq, dk, reps, dcu_q, dcu_k, dsl, w.max_seqlen_k, 8, 256)
    torch.cuda.synchronize()
    assert h.hisa_device_status() == 0
    o_idx, _, _, _ = oracle.hisa(qsel, w.k, cu_q, w.cu_k, w.seqlens, w.B, 8, 256)
    assert np.array_equal(idx.cpu().numpy(), o_idx)


def test_few_queries_all_scores_equal():
    """Every score equal on the cluster path: the distributed select takes its radix
    route and every row is its lowest-index candidates."""
    h = H()
    S, L, m, k = 3, 3000, 8, 512
    d = decode_workload(S, L, 1, 9, m=m, topk=k, integer=True)
    ones = bf16_from_f32(np.ones((1, 64), np.float32))[0]
    d.k_cache[:] = ones
    d.queries[:] = ones
    kc, cu_k, lens = dev_bf16(d.k_cache), dev_i32(d.cu_k), dev_i32(d.seqlens0)
    reps = h.hisa_pool_blocks(kc, cu_k, lens, L)
    idx = h.hisa_select(dev_bf16(d.queries[0]), kc, reps, dev_i32(np.arange(S + 1)), cu_k, lens,
                        L, m, k)
    torch.cuda.synchronize()
    assert h.hisa_device_status() == 0
    o_idx, _, _, _ = oracle.hisa(d.queries[0], d.k_cache, np.arange(S + 1, dtype=np.int32),
                                 d.cu_k, d.seqlens0, d.B, m, k)
    assert np.array_equal(idx.cpu().numpy(), o_idx)


def test_equal_keys_degenerate():
    """Every score equal: rows are the lowest-index candidates; the flat scan's candidate
    lists overflow and take the exact fallback."""
    L, k = 3000, 256
    ones = bf16_from_f32(np.ones((L, 64), np.float32))
    cu = np.array([0, L + (-L) % 128], np.int32)
    kk = np.zeros((int(cu[1]), 64), np.uint16)
    kk[:L] = ones
    w = varlen_prefill([L], 1, m=8, topk=k, integer=True)
    w.q[:] = ones
    w.k[:] = kk
    dw = OnDevice(w)
    idx, _ = run_dsa(dw, k)
    o_idx, _ = oracle.dsa_workload(w)
    assert np.array_equal(idx, o_idx)
    h_idx, _, _, _ = run_hisa(dw, 8, k)
    o_h, _, _, _ = oracle.hisa_workload(w)
    assert np.array_equal(h_idx, o_h)


def test_dsa_sampled_threshold_too_high_takes_the_fallback():
    """Long tiles estimate their pass-2 threshold from every eighth key block.  Here those
    blocks hold keys aligned with the queries and every other block keys opposed to them,
    so the estimate lands far above the true k-th score, the candidate lists come out
    short, and the rows must go through the exact fallback.  Integer inputs: bit-exact."""
    L, k = 12000, 2048
    rng = np.random.default_rng(812)
    w = varlen_prefill([L], 3, m=8, topk=k, integer=True)
    u = rng.integers(-2, 3, size=64).astype(np.float32)
    u[u == 0] = 1.0
    q = u + rng.integers(-1, 2, size=(L, 64))
    blk = np.arange(L) // 128
    sign = np.where(blk % 8 == 0, 1.0, -1.0)[:, None]
    kk = sign * u + rng.integers(-1, 2, size=(L, 64))
    w.q[:] = bf16_from_f32(q.astype(np.float32))
    w.k[:L] = bf16_from_f32(kk.astype(np.float32))
    dw = OnDevice(w)
    idx, sc = run_dsa(dw, k)
    o_idx, o_sc = oracle.dsa_workload(w)
    assert np.array_equal(idx, o_idx)
    valid = o_idx >= 0
    assert np.array_equal(sc[valid].astype(np.float64), o_sc[valid])


def test_hisa_equals_dsa_when_every_block_is_selected():
    """m >= number of blocks: HISA is the flat scan, bit for bit, on Gaussian inputs too."""
    w = gaussian_prefill(4096 + 77, 5, m=64, topk=512)
    dw = OnDevice(w)
    idx, sc, _, _ = run_hisa(dw, 64, 512)
    didx, dsc = run_dsa(dw, 512)
    assert np.array_equal(idx, didx)
    assert np.array_equal(sc, dsc)


# ---------------------------------------------------------------------------
# Gaussian inputs, band rule

def _gauss_hisa_check(w, n_rows, seed):
    dw = OnDevice(w)
    idx, sc, bl, reps = run_hisa(dw, w.m, w.topk)
    rows = sample_rows(w, n_rows, seed)
    o_idx, o_sc, o_bl, o_reps = oracle.hisa_workload(w, rows=rows)
    assert np.allclose(reps[:o_reps.shape[0]], o_reps, rtol=1e-5, atol=1e-6)
    check_block_band(w, rows, bl[rows], o_bl, o_reps)
    # stage 2 re-run on the GPU's own block sets
    r_idx, r_sc = oracle.token_select(w.q, w.k, bl[rows], w.cu_q, w.cu_k, w.seqlens, w.B, w.topk,
                                      rows=rows)
    check_token_band(w, rows, idx[rows], sc[rows], r_idx, r_sc, "hisa")
    # every row, not just the sampled ones, is structurally valid
    check_rows_structure(w, idx, sc, flat=False)
    return idx, sc, bl


def _gauss_dsa_check(w, n_rows, seed):
    dw = OnDevice(w)
    idx, sc = run_dsa(dw, w.topk)
    rows = sample_rows(w, n_rows, seed)
    o_idx, o_sc = oracle.dsa_workload(w, rows=rows)
    check_token_band(w, rows, idx[rows], sc[rows], o_idx, o_sc, "dsa")
    check_rows_structure(w, idx, sc, flat=True)
    return idx


def test_gaussian_small_several_tiles():
    w = gaussian_prefill(3000, 9, m=8, topk=256)
    _gauss_hisa_check(w, 300, 1)
    _gauss_dsa_check(w, 300, 2)


def test_gaussian_varlen_small():
    w = varlen_prefill([1000, 4096, 129, 2000], 13, m=6, topk=300)
    _gauss_hisa_check(w, 300, 3)
    _gauss_dsa_check(w, 300, 4)


def test_config_prefill_32k_needles_sampled():
    w = config_workload(3)
    _gauss_hisa_check(w, 160, 5)
    _gauss_dsa_check(w, 96, 6)


def test_config_prefill_128k_sampled():
    w = config_workload(4)
    _gauss_hisa_check(w, 256, 7)
    _gauss_dsa_check(w, 256, 8)


def test_config_varlen_sampled():
    w = config_workload(5)
    _gauss_hisa_check(w, 256, 9)
    _gauss_dsa_check(w, 256, 10)


# ---------------------------------------------------------------------------
# decode: appends keep the representatives equal to a fresh pool, and each step's
# selection matches the oracle on the same state

def test_decode_steps():
    h = H()
    dwl = config_workload(2, steps=6)
    S, cap = dwl.num_seqs, dwl.capacity
    kc = dev_bf16(dwl.k_cache)
    cu_k = dev_i32(dwl.cu_k)
    lens = dev_i32(dwl.seqlens0)
    cu_q = dev_i32(np.arange(S + 1))
    reps = h.hisa_pool_blocks(kc, cu_k, lens, int(dwl.seqlens0.max()))
    host_k = dwl.k_cache.copy()
    host_len = dwl.seqlens0.copy()
    for step in range(dwl.steps):
        nk = dev_bf16(dwl.new_keys[step])
        h.hisa_append_keys(kc, reps, cu_k, lens, nk)
        for s in range(S):
            host_k[dwl.cu_k[s] + host_len[s]] = dwl.new_keys[step, s, 0]
        host_len = host_len + 1
        q = dev_bf16(dwl.queries[step])
        maxlen = int(host_len.max())
        sc = torch.empty(S, dwl.topk, dtype=torch.float32, device="cuda")
        bl = torch.empty(S, dwl.m, dtype=torch.int32, device="cuda")
        idx = h.hisa_select(q, kc, reps, cu_q, cu_k, lens, maxlen, dwl.m, dwl.topk, out_scores=sc,
                            out_blocks=bl)
        torch.cuda.synchronize()
        assert h.hisa_device_status() == 0
        assert np.array_equal(lens.cpu().numpy(), host_len)
        assert np.array_equal(kc.cpu().view(torch.int16).numpy().view(np.uint16), host_k)
        # representatives maintained by appends == a fresh pool, bit for bit
        fresh = h.hisa_pool_blocks(kc, cu_k, lens, maxlen)
        assert torch.equal(fresh, reps)

        class W:  # the decode state as a workload for the parity helpers
            pass
        w = W()
        w.q, w.k, w.cu_q, w.cu_k, w.seqlens = dwl.queries[step], host_k, np.arange(S + 1, dtype=np.int32), dwl.cu_k, host_len
        w.B, w.m, w.topk, w.total_q, w.num_seqs, w.max_seqlen_k = dwl.B, dwl.m, dwl.topk, S, S, maxlen
        rows = np.arange(S, dtype=np.int32)
        o_idx, o_sc, o_bl, o_reps = oracle.hisa(w.q, w.k, w.cu_q, w.cu_k, w.seqlens, w.B, w.m,
                                                w.topk)
        assert np.allclose(reps.cpu().numpy()[:o_reps.shape[0]], o_reps, rtol=1e-5, atol=1e-6)
        check_block_band(w, rows, bl.cpu().numpy(), o_bl, o_reps)
        r_idx, r_sc = oracle.token_select(w.q, w.k, bl.cpu().numpy(), w.cu_q, w.cu_k, w.seqlens,
                                          w.B, w.topk)
        check_token_band(w, rows, idx.cpu().numpy(), sc.cpu().numpy(), r_idx, r_sc, "decode")
        # the decode row equals the prefill row of the same position
        if step == dwl.steps - 1:
            s = 3
            L = int(host_len[s])
            kk = dev_bf16(host_k[dwl.cu_k[s]:dwl.cu_k[s] + L])
            one = dev_i32([0, L])
            qq = torch.zeros(L, 64, dtype=torch.bfloat16, device="cuda")
            qq[L - 1] = q[s]
            pre_reps = h.hisa_pool_blocks(kk, one, None, L)
            pre = h.hisa_select(qq[L - 1:].contiguous(), kk, pre_reps, dev_i32([0, 1]), one, None, L,
                                dwl.m, dwl.topk)
            assert torch.equal(pre[0], idx[s])


def test_decode_side_stream_and_graph_match_default_stream():
    """On a non-default stream the append and decode kernels are launched as
    programmatic dependents of the previous kernel; eager and graph-captured runs
    there must reproduce the default-stream rows bit for bit."""
    h = H()
    dwl = config_workload(2, steps=4)
    S, cap = dwl.num_seqs, dwl.capacity
    cu_k = dev_i32(dwl.cu_k)
    cu_q = dev_i32(np.arange(S + 1))
    newk = dev_bf16(dwl.new_keys)
    qs = dev_bf16(dwl.queries.reshape(-1, 64)).view(dwl.steps, S, 64)

    def fresh():
        kc = dev_bf16(dwl.k_cache)
        lens = dev_i32(dwl.seqlens0)
        reps = h.hisa_pool_blocks(kc, cu_k, lens, cap)
        outs = [torch.empty(S, dwl.topk, dtype=torch.int32, device="cuda") for _ in range(dwl.steps)]
        return kc, lens, reps, outs

    def run(state):
        kc, lens, reps, outs = state
        for i in range(dwl.steps):
            h.hisa_append_keys(kc, reps, cu_k, lens, newk[i])
            h.hisa_select(qs[i], kc, reps, cu_q, cu_k, lens, cap, dwl.m, dwl.topk, out_idx=outs[i])

    ref = fresh()
    run(ref)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    eager = fresh()
    torch.cuda.synchronize()
    with torch.cuda.stream(side):
        run(eager)
    side.synchronize()
    graphed = fresh()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            run(graphed)
    g.replay()
    torch.cuda.synchronize()
    assert h.hisa_device_status() == 0
    for st in (eager, graphed):
        assert torch.equal(st[0], ref[0]) and torch.equal(st[1], ref[1]) and torch.equal(st[2], ref[2])
        for a, b in zip(st[3], ref[3]):
            assert torch.equal(a, b)
    del g


# ---------------------------------------------------------------------------
# errors found on the device

def test_device_errors_are_reported():
    h = H()
    h.hisa_device_status(clear=True)
    w = integer_prefill(512, 3, m=4, topk=32)
    dw = OnDevice(w)
    bad_cu = dev_i32([64, 576])  # region start not a multiple of 128
    k2 = dev_bf16(np.concatenate([np.zeros((64, 64), np.uint16), w.k]))
    reps = torch.zeros(5, 64, dtype=torch.float32, device="cuda")
    h.hisa_pool_blocks(k2, bad_cu, None, 512, reps=reps)
    st = h.hisa_device_status(clear=True)
    assert st & (1 << 2)
    out = h.hisa_select(dw.q, k2, reps, dw.cu_q, bad_cu, None, 512, 4, 32)
    st = h.hisa_device_status(clear=True)
    assert st & (1 << 2)
    assert torch.all(out == -1)
    # an append past the region's capacity leaves the sequence unchanged
    kc = dev_bf16(np.zeros((128, 64), np.uint16))
    cu = dev_i32([0, 128])
    lens = dev_i32([128])
    reps = torch.zeros(1, 64, dtype=torch.float32, device="cuda")
    nk = dev_bf16(np.ones((1, 1, 64), np.uint16))
    h.hisa_append_keys(kc, reps, cu, lens, nk)
    st = h.hisa_device_status(clear=True)
    assert st & (1 << 7)
    assert int(lens.item()) == 128
    assert h.hisa_device_status() == 0
