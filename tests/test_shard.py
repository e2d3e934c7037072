"""Partition of a batch over ranks (sparse_attention_top_hisa_b200.shard), on CPU.

The multi-GPU path splits the query rows of a batch into contiguous ranges, one per
rank, with no exchange between ranks.  These tests check the arithmetic of the
split (every row exactly once, valid rebased layouts) on random batches, and that
the oracle run on every shard reproduces the unsharded oracle rows exactly -- the
second as real gloo ranks (world sizes 2 and 3, uneven counts), each rank computing
its own shard and rank 0 comparing the gathered rows.
"""

import json
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from sparse_attention_top_hisa_b200.shard import query_cost, row_bounds, shard  # noqa: E402
from test_multirank import _launch  # noqa: E402

B = 128


def _random_batch(rng, decode: bool):
    S = int(rng.integers(1, 9))
    lens = rng.integers(1, 5 * B, size=S)
    regions = [((int(L) + int(rng.integers(0, 3)) * B + B - 1) // B) * B for L in lens]
    cu_k = np.concatenate([[0], np.cumsum(regions)]).astype(np.int64)
    qlen = np.ones(S, np.int64) if decode else np.array([int(rng.integers(0, L + 1)) for L in lens])
    cu_q = np.concatenate([[0], np.cumsum(qlen)]).astype(np.int64)
    return cu_q, cu_k, lens.astype(np.int64)


@pytest.mark.parametrize("decode", [False, True])
def test_every_row_once_and_layouts_valid(decode):
    rng = np.random.Generator(np.random.PCG64(5))
    for _ in range(200):
        cu_q, cu_k, lens = _random_batch(rng, decode)
        total = int(cu_q[-1])
        for world in (1, 2, 3, 5):
            cost = query_cost(cu_q, cu_k, lens, B, 4) if world == 3 else None
            bounds = row_bounds(total, world, cost)
            assert bounds[0] == 0 and bounds[-1] == total and bounds == sorted(bounds)
            covered = []
            for r in range(world):
                sh = shard(cu_q, cu_k, lens, world, r, B, bounds)
                assert (sh.row0, sh.row1) == (bounds[r], bounds[r + 1])
                covered.extend(range(sh.row0, sh.row1))
                if sh.total_q == 0:
                    continue
                assert sh.cu_seqlens_q[0] == 0 and sh.cu_seqlens_q[-1] == sh.total_q
                assert np.all(sh.cu_seqlens_k % B == 0) and sh.cu_seqlens_k[0] == 0
                assert sh.key0 == cu_k[sh.seq0] and sh.key1 == cu_k[sh.seq1]
                assert sh.cu_seqlens_k[-1] == sh.key1 - sh.key0
                qlen = np.diff(sh.cu_seqlens_q)
                region = np.diff(sh.cu_seqlens_k)
                assert np.all(qlen <= sh.seqlens_k) and np.all(sh.seqlens_k <= region)
                assert sh.max_seqlen_k == int(sh.seqlens_k.max())
                # every shard query row keeps its global position
                for t in range(sh.num_seqs):
                    s = sh.seq0 + t
                    a, b = int(sh.cu_seqlens_q[t]), int(sh.cu_seqlens_q[t + 1])
                    for u in range(a, b):
                        g = sh.row0 + u
                        pos_shard = int(sh.seqlens_k[t]) - (b - a) + (u - a)
                        pos_glob = int(lens[s]) - int(cu_q[s + 1] - cu_q[s]) + (g - int(cu_q[s]))
                        assert pos_shard == pos_glob
            assert covered == list(range(total))


def test_cost_balanced_bounds():
    cost = np.r_[np.ones(100), 10 * np.ones(100)]
    b = row_bounds(200, 2, cost)
    assert b == [0, 155] or abs(cost[: b[1]].sum() - cost[b[1]:].sum()) <= 10


def test_bad_layouts_are_refused():
    with pytest.raises(ValueError):
        shard([0, 3], [0, 100], [50], 2, 0)          # region start not a multiple of B
    with pytest.raises(ValueError):
        shard([0, 60], [0, 128], [50], 2, 0)         # more queries than live keys
    with pytest.raises(ValueError):
        shard([0, 1], [0, 128], [1], 2, 2)           # rank outside the world


RANK_SCRIPT = r"""
import json, sys
sys.path.insert(0, {root!r})
sys.path.insert(0, {tests!r})
import numpy as np
import torch.distributed as dist
import bench
import oracle
from synth import varlen_prefill, integer_prefill
from sparse_attention_top_hisa_b200.shard import shard, row_bounds, query_cost
world, rank, _ = bench.dist_setup(None)
res = {{}}
for name, w in (("varlen", varlen_prefill([300, 129, 700, 40, 1000], 11, m=4, topk=64, integer=True)),
                ("single", integer_prefill(1500, 12, m=3, topk=100))):
    bounds = row_bounds(w.total_q, world, query_cost(w.cu_q, w.cu_k, w.seqlens, w.B, w.m))
    sh = shard(w.cu_q, w.cu_k, w.seqlens, world, rank, w.B, bounds)
    rows = None
    if sh.total_q:
        idx, sc, bl, _ = oracle.hisa(w.q[sh.row0:sh.row1], w.k[sh.key0:sh.key1], sh.cu_seqlens_q,
                                     sh.cu_seqlens_k, sh.seqlens_k, w.B, w.m, w.topk)
        rows = [sh.row0, sh.row1, idx.tolist(), sc.tolist(), bl.tolist()]
    got = [None] * world
    dist.all_gather_object(got, rows)
    if rank == 0:
        ref_idx, ref_sc, ref_bl, _ = oracle.hisa_workload(w)
        seen = 0
        ok = True
        for part in got:
            if part is None:
                continue
            r0, r1, idx, sc, bl = part
            ok &= r0 == seen
            ok &= np.array_equal(np.array(idx), ref_idx[r0:r1])
            ok &= np.array_equal(np.array(sc), ref_sc[r0:r1])
            ok &= np.array_equal(np.array(bl), ref_bl[r0:r1])
            seen = r1
        res[name] = bool(ok and seen == w.total_q)
dist.barrier()
dist.destroy_process_group()
print(json.dumps({{"rank": rank, "res": res}}))
"""


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_oracle_rows_equal_unsharded(world):
    script = RANK_SCRIPT.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    outs = _launch(world, script)
    got = [json.loads(o.strip().splitlines()[-1]) for o in outs]
    res = [g for g in got if g["rank"] == 0][0]["res"]
    assert res == {"varlen": True, "single": True}
