"""The whole decode workload: 16 sequences of 32768 keys, 256 steps of (append one key,
select for one query), captured in one CUDA graph as the benchmark runs it.

One decode state takes all 256 steps, so its sequences cross the block boundary at
32896 keys (step 128 completes block 256, step 129 opens block 257).  Steps 1, 128,
129 and 256 are checked against the oracle on the host replay of the same appends
(band rule, Gaussian inputs); at the end the key cache equals the host copy and the
representatives maintained by 256 appends equal a fresh pool bit for bit.  The four
rotating states of the benchmark's graph are checked the same way at the end.
"""

import numpy as np
import pytest
import torch

import oracle
from parity import check_block_band, check_token_band, dev_bf16, dev_i32
from synth import config_workload

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


class _State:
    """A decode state on the device and its host replay."""

    def __init__(self, dwl):
        h = H()
        self.kc = dev_bf16(dwl.k_cache)
        self.lens = dev_i32(dwl.seqlens0)
        self.reps = h.hisa_pool_blocks(self.kc, dev_i32(dwl.cu_k), self.lens, dwl.capacity)
        self.host_k = dwl.k_cache.copy()
        self.host_len = dwl.seqlens0.copy().astype(np.int64)


def _oracle_check(dwl, host_k, host_len, q, idx, sc, bl, what):
    S = dwl.num_seqs

    class W:
        pass
    w = W()
    w.q, w.k, w.cu_q, w.cu_k = q, host_k, np.arange(S + 1, dtype=np.int32), dwl.cu_k
    w.seqlens = host_len.astype(np.int32)
    w.B, w.m, w.topk, w.total_q, w.num_seqs = dwl.B, dwl.m, dwl.topk, S, S
    w.max_seqlen_k = int(host_len.max())
    rows = np.arange(S, dtype=np.int32)
    o_idx, o_sc, o_bl, o_reps = oracle.hisa(w.q, w.k, w.cu_q, w.cu_k, w.seqlens, w.B, w.m, w.topk)
    check_block_band(w, rows, bl, o_bl, o_reps)
    r_idx, r_sc = oracle.token_select(w.q, w.k, bl, w.cu_q, w.cu_k, w.seqlens, w.B, w.topk)
    check_token_band(w, rows, idx, sc, r_idx, r_sc, what)


def _run_graph(dwl, states, steps, outs, scs, bls):
    """Capture the steps (step i on state i % len(states)) in one graph and replay it."""
    h = H()
    S, cap = dwl.num_seqs, dwl.capacity
    cu_k = dev_i32(dwl.cu_k)
    cu_q = dev_i32(np.arange(S + 1))
    newk = dev_bf16(dwl.new_keys)
    qs = dev_bf16(dwl.queries.reshape(-1, 64)).view(dwl.steps, S, 64)
    ws = torch.empty(h.hisa_select_workspace_size(S, S, cap, dwl.m, dwl.topk), dtype=torch.uint8,
                     device="cuda")

    def run():
        for i in range(steps):
            st = states[i % len(states)]
            h.hisa_append_keys(st.kc, st.reps, cu_k, st.lens, newk[i])
            h.hisa_select(qs[i], st.kc, st.reps, cu_q, cu_k, st.lens, cap, dwl.m, dwl.topk,
                          out_idx=outs[i], out_scores=scs[i], out_blocks=bls[i], workspace=ws)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            run()
    torch.cuda.current_stream().wait_stream(side)
    g.replay()
    torch.cuda.synchronize()
    assert h.hisa_device_status() == 0
    del g


def test_decode_256_steps_one_state_in_a_graph():
    h = H()
    dwl = config_workload(2)
    S, steps = dwl.num_seqs, dwl.steps
    assert steps == 256
    st = _State(dwl)
    check_at = {1, 128, 129, 256}
    outs = {i: torch.empty(S, dwl.topk, dtype=torch.int32, device="cuda") for i in range(steps)}
    scs = {i: torch.empty(S, dwl.topk, dtype=torch.float32, device="cuda") for i in range(steps)}
    bls = {i: torch.empty(S, dwl.m, dtype=torch.int32, device="cuda") for i in range(steps)}
    # the first call on the device happens before the capture (it looks up device symbols)
    h.hisa_select(dev_bf16(dwl.queries[0]), st.kc, st.reps, dev_i32(np.arange(S + 1)),
                  dev_i32(dwl.cu_k), st.lens, dwl.capacity, dwl.m, dwl.topk)
    _run_graph(dwl, [st], steps, outs, scs, bls)
    assert np.array_equal(st.lens.cpu().numpy(), dwl.seqlens0 + steps)
    host_k, host_len = st.host_k, st.host_len
    for i in range(steps):
        for s in range(S):
            host_k[dwl.cu_k[s] + host_len[s]] = dwl.new_keys[i, s, 0]
        host_len = host_len + 1
        if i + 1 in check_at:
            _oracle_check(dwl, host_k, host_len, dwl.queries[i], outs[i].cpu().numpy(),
                          scs[i].cpu().numpy(), bls[i].cpu().numpy(), f"decode step {i + 1}")
    assert int(host_len[0]) == 33024  # every slot of the capacity is used
    assert np.array_equal(st.kc.cpu().view(torch.int16).numpy().view(np.uint16), host_k)
    fresh = h.hisa_pool_blocks(st.kc, dev_i32(dwl.cu_k), st.lens, dwl.capacity)
    assert torch.equal(fresh, st.reps)


def test_decode_four_rotating_states_in_a_graph():
    """The benchmark's graph: 256 steps rotating over four independent states."""
    h = H()
    dwl = config_workload(2)
    S, steps = dwl.num_seqs, dwl.steps
    states = [_State(dwl) for _ in range(4)]
    outs = {i: torch.empty(S, dwl.topk, dtype=torch.int32, device="cuda") for i in range(steps)}
    scs = {i: torch.empty(S, dwl.topk, dtype=torch.float32, device="cuda") for i in range(steps)}
    bls = {i: torch.empty(S, dwl.m, dtype=torch.int32, device="cuda") for i in range(steps)}
    _run_graph(dwl, states, steps, outs, scs, bls)
    for r, st in enumerate(states):
        host_k, host_len = st.host_k, st.host_len
        last = None
        for i in range(r, steps, 4):
            for s in range(S):
                host_k[dwl.cu_k[s] + host_len[s]] = dwl.new_keys[i, s, 0]
            host_len = host_len + 1
            last = i
        assert np.array_equal(st.lens.cpu().numpy(), host_len)
        assert np.array_equal(st.kc.cpu().view(torch.int16).numpy().view(np.uint16), host_k)
        fresh = h.hisa_pool_blocks(st.kc, dev_i32(dwl.cu_k), st.lens, dwl.capacity)
        assert torch.equal(fresh, st.reps)
        _oracle_check(dwl, host_k, host_len, dwl.queries[last], outs[last].cpu().numpy(),
                      scs[last].cpu().numpy(), bls[last].cpu().numpy(), f"state {r} last step")


def test_fused_decode_step_equals_append_then_select():
    """hisa_decode_step (append and select in one launch) against hisa_append_keys followed
    by hisa_select, bit for bit, over 200 steps that cross a block boundary (32768 +
    128 keys), eagerly and captured in a graph; and the capacity error."""
    h = H()
    dwl = config_workload(2, steps=200)
    S, cap = dwl.num_seqs, dwl.capacity
    cu_k = dev_i32(dwl.cu_k)
    cu_q = dev_i32(np.arange(S + 1))
    a, b = _State(dwl), _State(dwl)
    newk = dev_bf16(dwl.new_keys.reshape(dwl.steps, S, 64))
    qs = dev_bf16(dwl.queries.reshape(-1, 64)).view(dwl.steps, S, 64)
    ws = torch.empty(h.hisa_select_workspace_size(S, S, cap, dwl.m, dwl.topk), dtype=torch.uint8,
                     device="cuda")
    outs = [torch.empty(S, dwl.topk, dtype=torch.int32, device="cuda") for _ in range(4)]
    scs = [torch.empty(S, dwl.topk, dtype=torch.float32, device="cuda") for _ in range(2)]
    bls = [torch.empty(S, dwl.m, dtype=torch.int32, device="cuda") for _ in range(2)]

    def separate(i):
        h.hisa_append_keys(a.kc, a.reps, cu_k, a.lens, newk[i].view(S, 1, 64))
        h.hisa_select(qs[i], a.kc, a.reps, cu_q, cu_k, a.lens, cap, dwl.m, dwl.topk,
                      out_idx=outs[0], out_scores=scs[0], out_blocks=bls[0], workspace=ws)

    def fused(i):
        h.hisa_decode_step(b.kc, b.reps, cu_k, b.lens, newk[i], qs[i], cap, dwl.m, dwl.topk,
                           out_idx=outs[1], out_scores=scs[1], out_blocks=bls[1])

    for i in range(150):
        separate(i)
        fused(i)
        if i % 10 == 9 or i in (127, 128, 129):
            torch.cuda.synchronize()
            assert torch.equal(outs[0], outs[1]), i
            assert torch.equal(scs[0], scs[1]), i
            assert torch.equal(bls[0], bls[1]), i
    torch.cuda.synchronize()
    assert h.hisa_device_status() == 0
    assert torch.equal(a.lens, b.lens) and torch.equal(a.kc, b.kc) and torch.equal(a.reps, b.reps)
    # the last 50 steps of the fused path captured in a graph on a side stream
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            for i in range(150, 200):
                h.hisa_decode_step(b.kc, b.reps, cu_k, b.lens, newk[i], qs[i], cap, dwl.m,
                                   dwl.topk, out_idx=outs[3])
    torch.cuda.current_stream().wait_stream(side)
    g.replay()
    for i in range(150, 200):
        separate(i)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[3])
    assert torch.equal(a.lens, b.lens) and torch.equal(a.kc, b.kc) and torch.equal(a.reps, b.reps)
    fresh = h.hisa_pool_blocks(b.kc, cu_k, b.lens, cap)
    assert torch.equal(fresh, b.reps)
    del g
    # a sequence whose region is full: left unchanged, row -1, HISA_ERR_CAPACITY
    full = dev_i32(np.full(S, cap, np.int32))
    before = b.kc.clone()
    out = h.hisa_decode_step(b.kc, b.reps, cu_k, full, newk[0], qs[0], cap, dwl.m, dwl.topk)
    st = h.hisa_device_status(clear=True)
    assert st & (1 << 7)
    assert bool((out == -1).all()) and torch.equal(b.kc, before)
    assert bool((full == cap).all())


def test_fused_decode_step_mixed_lengths():
    """hisa_decode_step on sequences of very different lengths, integer inputs: one
    sequence with a single block and two with at most m blocks (every block kept, the
    append after the selection), two selected by one warp, and one with more than 1024
    blocks (the CTA-wide top-m, the append after the selection); 40 steps, each
    sequence crossing a block boundary at its own step.  Bit for bit against
    hisa_append_keys followed by hisa_select, and the last step against the oracle."""
    from synth import decode_workload
    h = H()
    lens0 = np.array([100, 250, 1000, 5100, 70000, 140000], np.int32)
    S, steps, m, k = len(lens0), 40, 16, 512
    dwl = decode_workload(S, int(lens0.max()), steps, 4242, m=m, topk=k, integer=True)
    dwl.seqlens0 = lens0.copy()
    cap = dwl.capacity
    cu_k = dev_i32(dwl.cu_k)
    cu_q = dev_i32(np.arange(S + 1))
    a, b = _State(dwl), _State(dwl)
    newk = dev_bf16(dwl.new_keys.reshape(steps, S, 64))
    qs = dev_bf16(dwl.queries.reshape(-1, 64)).view(steps, S, 64)
    ws = torch.empty(h.hisa_select_workspace_size(S, S, cap, m, k), dtype=torch.uint8,
                     device="cuda")
    outs = [torch.empty(S, k, dtype=torch.int32, device="cuda") for _ in range(2)]
    scs = [torch.empty(S, k, dtype=torch.float32, device="cuda") for _ in range(2)]
    bls = [torch.empty(S, m, dtype=torch.int32, device="cuda") for _ in range(2)]
    for i in range(steps):
        h.hisa_append_keys(a.kc, a.reps, cu_k, a.lens, newk[i].view(S, 1, 64))
        h.hisa_select(qs[i], a.kc, a.reps, cu_q, cu_k, a.lens, cap, m, k, out_idx=outs[0],
                      out_scores=scs[0], out_blocks=bls[0], workspace=ws)
        h.hisa_decode_step(b.kc, b.reps, cu_k, b.lens, newk[i], qs[i], cap, m, k,
                           out_idx=outs[1], out_scores=scs[1], out_blocks=bls[1])
        torch.cuda.synchronize()
        assert torch.equal(outs[0], outs[1]), i
        assert torch.equal(scs[0], scs[1]), i
        assert torch.equal(bls[0], bls[1]), i
    assert h.hisa_device_status() == 0
    assert torch.equal(a.lens, b.lens) and torch.equal(a.kc, b.kc) and torch.equal(a.reps, b.reps)
    assert np.array_equal(b.lens.cpu().numpy(), lens0 + steps)
    fresh = h.hisa_pool_blocks(b.kc, cu_k, b.lens, cap)
    assert torch.equal(fresh, b.reps)
    # the last step against the oracle, on the host copy of the cache
    host_k = b.kc.cpu().view(torch.int16).numpy().view(np.uint16)
    o_idx, o_sc, o_bl, _ = oracle.hisa(dwl.queries[steps - 1], host_k, np.arange(S + 1, dtype=np.int32),
                                       dwl.cu_k, (lens0 + steps).astype(np.int32), dwl.B, m, k)
    assert np.array_equal(bls[1].cpu().numpy(), o_bl)
    assert np.array_equal(outs[1].cpu().numpy(), o_idx)
    valid = o_idx >= 0
    assert np.array_equal(scs[1].cpu().numpy()[valid].astype(np.float64), o_sc[valid])
