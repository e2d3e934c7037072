"""Pins that tie the CPU oracle to what the pages and the mathematics fix.

Each ``pin_*`` function raises ``AssertionError`` (or ``oracle.OracleError``)
when the oracle disagrees with an independent fact: a hand-worked example, the
pure-Python brute force, a closed form or an invariant of the method.  They are
collected as tests in ``test_oracle_pins.py`` and are also re-run there with a
deliberate mistake planted in the oracle, to show each mistake is caught.

Sources: aitrends.kr, "HISA: 세밀한 희소 어텐션을 위한 효율적인 계층적 인덱싱"
(paragraphs on pooling, stage 1, stage 2, KV-cache maintenance and varlen
packing); idea.jsleekr.com, section "DSA: 딥시크의 희소 어텐션"; the same
page's transcript section on the m = M pitfall (selecting every block makes
HISA identical to the flat scan).
"""

from __future__ import annotations

import json
import os
from fractions import Fraction

import numpy as np

import oracle
from oracle import brute
from synth import bf16_from_f32, bf16_to_f32, gaussian_prefill, integer_prefill, varlen_prefill

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _bf(x):
    return bf16_from_f32(np.asarray(x, np.float32))


def _single(keys, queries_by_pos, L, d):
    """A one-sequence prefill whose query rows are zero except at the given positions."""
    k = _bf(np.asarray(keys, np.float32).reshape(L, d))
    q = np.zeros((L, d), np.float32)
    for pos, qv in queries_by_pos.items():
        q[pos] = qv
    return _bf(q), k, np.array([0, L], np.int32), np.array([0, L], np.int32), np.array([L], np.int32)


# ---------------------------------------------------------------------------
# hand-worked examples (tests/golden)

def pin_golden_three_block():
    g = json.load(open(os.path.join(GOLDEN, "three_block_example.json")))
    L, d, B, K = len(g["keys"]), g["d"], g["B"], g["topk"]
    qs = {e["pos"]: e["q"] for e in g["queries"]}
    q, k, cu_q, cu_k, sl = _single(g["keys"], qs, L, d)
    reps = oracle.pool(k, cu_k, sl, B)
    assert np.array_equal(reps, np.asarray(g["reps"], np.float64)), reps
    for m in g["m"]:
        idx, sc, _, _ = oracle.hisa(q, k, cu_q, cu_k, sl, B, m, K)
        didx, dsc = oracle.dsa(q, k, cu_q, cu_k, sl, K)
        for e in g["queries"]:
            p = e["pos"]
            assert list(idx[p]) == e["idx"], (m, p, idx[p])
            assert list(didx[p]) == e["idx"], (m, p, didx[p])
            n = len(e["scores"])
            assert list(sc[p][:n]) == e["scores"], (m, p, sc[p])
            assert list(dsc[p][:n]) == e["scores"], (m, p, dsc[p])


def pin_golden_five_block():
    g = json.load(open(os.path.join(GOLDEN, "five_block_example.json")))
    B, d, K, L = g["B"], g["d"], g["topk"], 10
    for c in g["cases"]:
        keys = np.zeros((L, d), np.float32)
        for j, v in c["keys"].items():
            keys[int(j)] = v
        q, k, cu_q, cu_k, sl = _single(keys, {c["pos"]: c["q"]}, L, d)
        idx, sc, blocks, reps = oracle.hisa(q, k, cu_q, cu_k, sl, B, c["m"], K)
        if "reps" in c:
            assert np.array_equal(reps, np.asarray(c["reps"], np.float64)), (c["name"], reps)
        p = c["pos"]
        assert list(blocks[p]) == c["blocks"], (c["name"], blocks[p])
        assert list(idx[p]) == c["idx"], (c["name"], idx[p])
        assert list(sc[p]) == c["scores"], (c["name"], sc[p])
        didx, dsc = oracle.dsa(q, k, cu_q, cu_k, sl, K)
        assert list(didx[p]) == c["dsa_idx"], (c["name"], didx[p])
        assert list(dsc[p]) == c["dsa_scores"], (c["name"], dsc[p])


# ---------------------------------------------------------------------------
# brute force on tiny inputs

def _tiny_cases():
    """Small random problems covering partial blocks, several sequences, decode-style
    query tails, every m and several k.  Integer values make ties common."""
    rng = np.random.Generator(np.random.PCG64(1234))
    cases = []
    for t in range(14):
        B = int(rng.choice([2, 4]))
        d = int(rng.choice([2, 4]))
        S = int(rng.integers(1, 4))
        lens = [int(rng.integers(1, 41)) for _ in range(S)]
        qlens = [L if t % 2 == 0 else int(rng.integers(1, L + 1)) for L in lens]
        integer = t % 3 != 2
        cu_q = np.zeros(S + 1, np.int32)
        cu_k = np.zeros(S + 1, np.int32)
        for s in range(S):
            cu_q[s + 1] = cu_q[s] + qlens[s]
            cu_k[s + 1] = cu_k[s] + (lens[s] + B - 1) // B * B + B * int(rng.integers(0, 2))
        if integer:
            qf = rng.integers(-2, 3, size=(int(cu_q[-1]), d)).astype(np.float32)
            kf = rng.integers(-2, 3, size=(int(cu_k[-1]), d)).astype(np.float32)
        else:
            qf = rng.standard_normal((int(cu_q[-1]), d), dtype=np.float32)
            kf = rng.standard_normal((int(cu_k[-1]), d), dtype=np.float32)
        M = max((L + B - 1) // B for L in lens)
        m = int(rng.integers(1, M + 2))
        topk = int(rng.integers(1, max(lens) + 3))
        cases.append((_bf(qf), _bf(kf), cu_q, cu_k, np.array(lens, np.int32), B, m, topk))
    return cases


def pin_brute_force():
    for (q, k, cu_q, cu_k, sl, B, m, topk) in _tiny_cases():
        idx, _, blocks, reps = oracle.hisa(q, k, cu_q, cu_k, sl, B, m, topk)
        didx, _ = oracle.dsa(q, k, cu_q, cu_k, sl, topk)
        for s in range(len(sl)):
            L = int(sl[s])
            keys = k[cu_k[s]:cu_k[s] + L]
            # representatives, exactly
            kv = brute._vals(keys)
            exact = brute.pool(kv, L, B)
            for b, row in enumerate(exact):
                got = reps[cu_k[s] // B + b]
                assert all(Fraction(float(g)) == e for g, e in zip(got, row)) or \
                    np.allclose(got, [float(e) for e in row], rtol=1e-15, atol=0), (s, b)
            qlen = int(cu_q[s + 1] - cu_q[s])
            for r in range(qlen):
                row = int(cu_q[s]) + r
                pos = L - qlen + r
                want, want_blocks = brute.hisa_row(q[row], keys, pos, B, m, topk, L)
                assert list(idx[row]) == want, (B, m, topk, s, pos, list(idx[row]), want)
                assert [b for b in blocks[row] if b >= 0] == want_blocks, (s, pos)
                assert list(didx[row]) == brute.dsa_row(q[row], keys, pos, topk), (s, pos)


# ---------------------------------------------------------------------------
# invariants

def _medium(integer: bool, seed: int, L: int = 700, B: int = 16, d: int = 8, m: int = 6,
            topk: int = 40):
    if integer:
        return integer_prefill(L, seed, B=B, m=m, topk=topk, d=d)
    return gaussian_prefill(L, seed, B=B, m=m, topk=topk, d=d)


def pin_identity_m_equals_M():
    """Selecting every eligible block makes HISA the flat scan, row for row."""
    for integer in (True, False):
        w = _medium(integer, 11)
        M = (w.max_seqlen_k + w.B - 1) // w.B
        for m in (M, M + 3):
            idx, sc, _, _ = oracle.hisa(w.q, w.k, w.cu_q, w.cu_k, w.seqlens, w.B, m, w.topk)
            didx, dsc = oracle.dsa_workload(w)
            assert np.array_equal(idx, didx)
            assert np.array_equal(sc, dsc)


def _scores_of(w, row, pos, js):
    qv = bf16_to_f32(w.q[row]).astype(np.float64)
    kv = bf16_to_f32(w.k[np.asarray(js) + int(w.cu_k[0])]).astype(np.float64)
    return kv @ qv


def pin_invariants():
    """Output-structure invariants of both stages on medium random inputs."""
    for integer in (True, False):
        w = _medium(integer, 21)
        idx, sc, blocks, reps = oracle.hisa_workload(w)
        block_sc = oracle.block_scores(w.q, reps, w.cu_q, w.cu_k, w.seqlens, w.B,
                                       (w.max_seqlen_k + w.B - 1) // w.B)
        for pos in range(w.total_q):
            own = pos // w.B
            row = idx[pos]
            valid = row[row >= 0]
            # -1 only as a suffix; indices causal and distinct
            assert np.all(row[len(valid):] == -1)
            assert np.all(valid <= pos) and np.all(valid >= 0)
            assert len(set(valid.tolist())) == len(valid)
            sel = blocks[pos][blocks[pos] >= 0]
            # selected blocks contain the forced ones, have size min(m, own+1), ascending
            assert len(sel) == min(w.m, own + 1)
            assert np.all(np.diff(sel) > 0)
            forced = [own, own - 1, 0][:max(0, min(3, w.m))]
            assert all(b in sel for b in forced if b >= 0)
            # block stage: every unselected eligible block does not beat a selected free one
            free = [b for b in sel if b not in forced]
            if free:
                worst = min(free, key=lambda b: (block_sc[pos][b], -b))
                for b in range(own + 1):
                    if b in sel:
                        continue
                    assert (block_sc[pos][b], -b) < (block_sc[pos][worst], -worst)
            # candidate count (the O(mB) claim)
            ncand = sum(min((b + 1) * w.B, pos + 1) - b * w.B for b in sel)
            assert len(valid) == min(w.topk, ncand)
            # rows ordered by score descending, equal scores in increasing index
            s = _scores_of(w, pos, pos, valid)
            assert np.array_equal(s, sc[pos][:len(valid)])
            for a in range(len(valid) - 1):
                assert s[a] > s[a + 1] or (s[a] == s[a + 1] and valid[a] < valid[a + 1])
            # the row is the exact top-k of the union of the selected blocks
            cand = [j for b in sel for j in range(b * w.B, min((b + 1) * w.B, pos + 1))]
            cs = _scores_of(w, pos, pos, cand)
            order = sorted(range(len(cand)), key=lambda t: (-cs[t], cand[t]))
            assert [cand[t] for t in order[:w.topk]] == valid.tolist()


def pin_k_covers_all():
    """k at least the candidate count returns every candidate, sorted."""
    w = _medium(True, 31, L=300, topk=10_000)
    didx, dsc = oracle.dsa_workload(w)
    for pos in (0, 1, 17, 299):
        row = didx[pos]
        assert np.count_nonzero(row >= 0) == pos + 1
        assert sorted(row[row >= 0].tolist()) == list(range(pos + 1))


def pin_pool_closed_form():
    """Mean of an arithmetic progression is the mean of its ends; partial blocks divide by
    the count of keys present."""
    B, d, L = 8, 4, 29
    base = np.arange(L, dtype=np.float32)
    keys = np.stack([base, -2 * base, base * 0 + 3, base / 4], axis=1)
    k = _bf(keys)
    reps = oracle.pool(k, np.array([0, 32], np.int32), np.array([L], np.int32), B)
    for b in range((L + B - 1) // B):
        lo, hi = b * B, min((b + 1) * B, L) - 1
        mean = (lo + hi) / 2.0
        assert np.allclose(reps[b], [mean, -2 * mean, 3.0, mean / 4], rtol=0, atol=1e-12), (b, reps[b])


def pin_packing_invariance():
    """Packing sequences together changes nothing: varlen rows equal separate runs."""
    lens = [37, 128, 200, 5]
    w = varlen_prefill(lens, 41, B=16, m=4, topk=24, d=8, integer=True)
    idx, sc, _, _ = oracle.hisa_workload(w)
    didx, _ = oracle.dsa_workload(w)
    for s, L in enumerate(lens):
        k = w.k[w.cu_k[s]:w.cu_k[s + 1]]
        q = w.q[w.cu_q[s]:w.cu_q[s + 1]]
        one_q = np.array([0, L], np.int32)
        one_k = np.array([0, k.shape[0]], np.int32)
        sl = np.array([L], np.int32)
        i1, s1, _, _ = oracle.hisa(q, k, one_q, one_k, sl, w.B, w.m, w.topk)
        d1, _ = oracle.dsa(q, k, one_q, one_k, sl, w.topk)
        assert np.array_equal(i1, idx[w.cu_q[s]:w.cu_q[s + 1]])
        assert np.array_equal(d1, didx[w.cu_q[s]:w.cu_q[s + 1]])


def pin_decode_equals_prefill():
    """A single query at the end of a sequence truncated to pos+1 keys gives prefill row pos."""
    w = _medium(False, 51, L=400)
    idx, sc, _, _ = oracle.hisa_workload(w)
    didx, _ = oracle.dsa_workload(w)
    for pos in (0, 15, 16, 47, 100, 255, 399):
        L = pos + 1
        cap = (L + w.B - 1) // w.B * w.B
        k = w.k[:cap].copy()
        i1, _, _, _ = oracle.hisa(w.q[pos:pos + 1], k, np.array([0, 1], np.int32),
                                  np.array([0, cap], np.int32), np.array([L], np.int32),
                                  w.B, w.m, w.topk)
        d1, _ = oracle.dsa(w.q[pos:pos + 1], k, np.array([0, 1], np.int32),
                           np.array([0, cap], np.int32), np.array([L], np.int32), w.topk)
        assert np.array_equal(i1[0], idx[pos]), pos
        assert np.array_equal(d1[0], didx[pos]), pos


def pin_scaling_and_ties():
    """Scaling every query by 2 scales all scores exactly and leaves the indices alone;
    with all keys equal each row is its lowest-index candidates in order."""
    w = _medium(False, 61)
    idx, sc, _, _ = oracle.hisa_workload(w)
    q2 = _bf(bf16_to_f32(w.q) * 2.0)
    i2, s2, _, _ = oracle.hisa(q2, w.k, w.cu_q, w.cu_k, w.seqlens, w.B, w.m, w.topk)
    assert np.array_equal(idx, i2)
    assert np.array_equal(sc * 2.0, s2)
    L, B, m, topk, d = 300, 16, 5, 20, 8
    k = _bf(np.ones((L, d), np.float32))
    q = _bf(np.ones((L, d), np.float32))
    cu = np.array([0, L], np.int32)
    idx, _, blocks, _ = oracle.hisa(q, k, cu, cu, np.array([L], np.int32), B, m, topk)
    for pos in range(L):
        own = pos // B
        if own + 1 <= m:
            sel = list(range(own + 1))
        else:
            forced = {0, own - 1, own}
            free = [b for b in range(own + 1) if b not in forced][:m - 3]
            sel = sorted(forced | set(free))
        cand = [j for b in sel for j in range(b * B, min((b + 1) * B, pos + 1))]
        want = cand[:topk] + [-1] * max(0, topk - len(cand))
        assert list(idx[pos]) == want, pos


# ---------------------------------------------------------------------------
# the sparse attention step over the selected tokens

def _att_case(rng, S, H, dv, topk, lengths):
    """Random tiny attention problem: small-integer bf16 q/k/v, index rows with
    padding and arbitrary order."""
    cu_k = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    rows_k = int(cu_k[-1])
    k = _bf(rng.integers(-3, 4, size=(rows_k, dv)).astype(np.float32))
    v = _bf(rng.integers(-5, 6, size=(rows_k, dv)).astype(np.float32))
    nq = [int(rng.integers(1, 4)) for _ in range(S)]
    cu_q = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    total_q = int(cu_q[-1])
    q = _bf(rng.integers(-2, 3, size=(total_q, H, dv)).astype(np.float32))
    idx = np.full((total_q, topk), -1, np.int32)
    for s_ in range(S):
        for r in range(int(cu_q[s_]), int(cu_q[s_ + 1])):
            n = int(rng.integers(0, min(topk, lengths[s_]) + 1))
            sel = rng.choice(lengths[s_], size=n, replace=False)
            slots = rng.choice(topk, size=n, replace=False)
            idx[r, slots] = sel
    return q, k, v, idx, cu_q, cu_k


def _att_brute_row(q, k, v, idx, cu_q, cu_k, row, scale):
    s_ = int(np.searchsorted(cu_q, row, side="right") - 1)
    base = int(cu_k[s_])
    kf, vf, qf = bf16_to_f32(k).astype(float), bf16_to_f32(v).astype(float), bf16_to_f32(q[row]).astype(float)
    n = int(cu_k[s_ + 1]) - base
    keys = {j: list(kf[base + j]) for j in range(n)}
    vals = {j: list(vf[base + j]) for j in range(n)}
    return brute.attention([list(x) for x in qf], keys, vals, list(idx[row]), scale)


def pin_attention_brute():
    rng = np.random.Generator(np.random.PCG64(77))
    for case in range(8):
        H, dv, topk = [(1, 2, 3), (3, 5, 4), (2, 4, 6), (1, 7, 5)][case % 4]
        lengths = [int(x) for x in rng.integers(2, 9, size=int(rng.integers(1, 4)))]
        q, k, v, idx, cu_q, cu_k = _att_case(rng, len(lengths), H, dv, topk, lengths)
        scale = float(rng.uniform(0.1, 0.9))
        out, lse = oracle.sparse_attention(q, k, v, idx, cu_q, cu_k, H, scale, nthreads=2)
        for row in range(idx.shape[0]):
            bo, bl = _att_brute_row(q, k, v, idx, cu_q, cu_k, row, scale)
            assert np.allclose(out[row], np.array(bo), rtol=1e-12, atol=1e-12), (case, row)
            for h in range(H):
                if np.isinf(bl[h]):
                    assert np.isinf(lse[row, h]) and lse[row, h] < 0
                else:
                    assert abs(lse[row, h] - bl[h]) <= 1e-12 * max(1.0, abs(bl[h])), (case, row)


def pin_attention_golden():
    g = json.load(open(os.path.join(GOLDEN, "attention_example.json")))
    k = _bf(np.asarray(g["keys"], np.float32))
    v = _bf(np.asarray(g["values"], np.float32))
    q = _bf(np.asarray(g["q"], np.float32).reshape(1, 1, -1))
    idx = np.asarray([g["idx"]], np.int32)
    cu_q, cu_k = np.array([0, 1], np.int32), np.array([0, 2], np.int32)
    out, lse = oracle.sparse_attention(q, k, v, idx, cu_q, cu_k, 1, np.log(3.0))
    assert np.allclose(out[0, 0], g["out"], rtol=0, atol=1e-14), out
    assert abs(lse[0, 0] - np.log(4.0)) < 1e-14, lse
    out2, _ = oracle.sparse_attention(q, k, v, idx[:, ::-1].copy(), cu_q, cu_k, 1, np.log(3.0))
    assert np.allclose(out2, out, rtol=0, atol=1e-14)


def pin_attention_single_index():
    """One selected token: its weight is 1, the output is its value row, lse its score."""
    rng = np.random.Generator(np.random.PCG64(78))
    q, k, v, idx, cu_q, cu_k = _att_case(rng, 2, 2, 6, 5, [7, 5])
    idx[:] = -1
    for row in range(idx.shape[0]):
        s_ = int(np.searchsorted(cu_q, row, side="right") - 1)
        idx[row, row % 5] = row % (int(cu_k[s_ + 1]) - int(cu_k[s_]))
    out, lse = oracle.sparse_attention(q, k, v, idx, cu_q, cu_k, 2, 0.5)
    vf, kf, qf = bf16_to_f32(v).astype(float), bf16_to_f32(k).astype(float), bf16_to_f32(q).astype(float)
    for row in range(idx.shape[0]):
        s_ = int(np.searchsorted(cu_q, row, side="right") - 1)
        j = int(cu_k[s_]) + int(idx[row].max())
        for h in range(2):
            assert np.array_equal(out[row, h], vf[j]), (row, h)
            assert lse[row, h] == 0.5 * float(np.dot(qf[row, h], kf[j]))


def pin_attention_uniform():
    """A zero query scores every token 0: the output is the mean of the selected values."""
    rng = np.random.Generator(np.random.PCG64(79))
    q, k, v, idx, cu_q, cu_k = _att_case(rng, 2, 3, 4, 6, [8, 6])
    q[:] = 0
    out, lse = oracle.sparse_attention(q, k, v, idx, cu_q, cu_k, 3, 0.7)
    vf = bf16_to_f32(v).astype(float)
    for row in range(idx.shape[0]):
        s_ = int(np.searchsorted(cu_q, row, side="right") - 1)
        sel = [int(cu_k[s_]) + int(j) for j in idx[row] if j >= 0]
        for h in range(3):
            if not sel:
                assert np.all(out[row, h] == 0)
                continue
            exact = [float(sum(Fraction(vf[j][d]) for j in sel) / len(sel)) for d in range(4)]
            assert np.allclose(out[row, h], exact, rtol=1e-14, atol=1e-14), (row, h)
            assert abs(lse[row, h] - np.log(len(sel))) < 1e-13


def pin_attention_order_invariant():
    """The output does not depend on where the selected tokens sit in the index row."""
    rng = np.random.Generator(np.random.PCG64(80))
    q, k, v, idx, cu_q, cu_k = _att_case(rng, 3, 2, 5, 6, [9, 4, 7])
    out, lse = oracle.sparse_attention(q, k, v, idx, cu_q, cu_k, 2, 0.3)
    perm = np.stack([rng.permutation(row) for row in idx])
    out2, lse2 = oracle.sparse_attention(q, k, v, perm, cu_q, cu_k, 2, 0.3)
    assert np.allclose(out, out2, rtol=1e-13, atol=1e-13)
    assert np.allclose(lse, lse2, rtol=1e-13, atol=1e-13)


ALL_PINS = [
    pin_attention_brute, pin_attention_golden, pin_attention_single_index,
    pin_attention_uniform, pin_attention_order_invariant,
    pin_golden_three_block,
    pin_golden_five_block,
    pin_brute_force,
    pin_identity_m_equals_M,
    pin_invariants,
    pin_k_covers_all,
    pin_pool_closed_form,
    pin_packing_invariance,
    pin_decode_equals_prefill,
    pin_scaling_and_ties,
]
