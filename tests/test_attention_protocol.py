"""The barrier protocol of the sparse-attention kernel, checked on the host.

A model of sparse_attn_tc_kernel's synchronisation (csrc/attention.cu): the loader
warps (one agent: they move together through their named barrier), thread 0 of the
compute warps (it issues the MMAs), the other compute threads, the tensor pipe (it
completes issued MMA groups in order, arriving on their mbarriers) and the loaders'
copy groups (they complete in order).  Random interleavings of these agents must never
deadlock, and every parity wait must find its mbarrier at most one phase ahead of the
phase it waits for: two phases ahead, the parity test would read the later phase as
not yet complete and the wait would never end on the GPU.

Each step follows the kernel: a three-stage ring (full / empty per stage), one
mbarrier per TMEM score buffer (tiles t and t + 2 share one), one for the output tile;
thread 0 issues tile t + 1's score product at the top of tile t when its stage is
already filled (else after the vote), the output product after the second compute
barrier, and releases the stage with it.
"""

import random

STAGES = 3


class Bar:
    def __init__(self, name):
        self.name, self.done = name, 0


def _ready(bar, fill):
    """The wait for completion number fill + 1 of `bar` (parity fill & 1)."""
    assert bar.done <= fill + 1, f"{bar.name} is two phases ahead of a waiter (fill {fill})"
    return bar.done >= fill + 1


def simulate(ntiles, seed, score_bars=2):
    rnd = random.Random(seed)
    full = [Bar(f"full{i}") for i in range(STAGES)]
    empty = [Bar(f"empty{i}") for i in range(STAGES)]
    one = Bar("s")
    bar_s = [Bar("s0"), Bar("s1")] if score_bars == 2 else [one, one]
    bar_o = Bar("o")
    pipe, groups, named, st = [], {}, {}, {"issued": 0}

    def s_fill(t):  # which completion of its score barrier tile t is
        return t >> 1 if score_bars == 2 else t

    def loader():
        for t in range(ntiles):
            if t >= STAGES:
                while not _ready(empty[t % STAGES], t // STAGES - 1):
                    yield
            groups[t] = False
            yield
            if t > 0:  # signal the previous tile once its copies are done
                while not groups[t - 1]:
                    yield
                full[(t - 1) % STAGES].done += 1
        if ntiles:
            while not groups[ntiles - 1]:
                yield
            full[(ntiles - 1) % STAGES].done += 1

    def issue_scores(t):
        pipe.append([bar_s[t & 1]])

    def compute(thread0):
        if thread0 and ntiles:
            while not _ready(full[0], 0):
                yield
            issue_scores(0)
            st["issued"] = 1
        for t in range(ntiles):
            if thread0 and st["issued"] == t + 1 and t + 1 < ntiles:
                if _ready(full[(t + 1) % STAGES], (t + 1) // STAGES):  # try, do not block
                    issue_scores(t + 1)
                    st["issued"] += 1
            while not _ready(full[t % STAGES], t // STAGES):
                yield
            while not _ready(bar_s[t & 1], s_fill(t)):
                yield
            key = ("vote", t)
            named.setdefault(key, set()).add(thread0)
            while len(named[key]) < 2:
                yield
            if thread0 and st["issued"] == t + 1 and t + 1 < ntiles:
                while not _ready(full[(t + 1) % STAGES], (t + 1) // STAGES):
                    yield
                issue_scores(t + 1)
                st["issued"] += 1
            key = ("sync2", t)
            named.setdefault(key, set()).add(thread0)
            while len(named[key]) < 2:
                yield
            if thread0:
                job = [bar_o]
                if t + STAGES < ntiles:
                    job.append(empty[t % STAGES])
                pipe.append(job)
            while not _ready(bar_o, t):
                yield

    def tensor_pipe():
        while True:
            if pipe and rnd.random() < 0.5:
                for b in pipe.pop(0):
                    b.done += 1
            yield

    def copies():
        while True:
            pending = [t for t, d in groups.items() if not d]
            if pending and rnd.random() < 0.5:
                groups[min(pending)] = True
            yield

    agents = {"loader": loader(), "thread0": compute(True), "others": compute(False)}
    background = [tensor_pipe(), copies()]
    for _ in range(200000):
        if not agents:
            return
        name = rnd.choice(list(agents))
        try:
            next(agents[name])
        except StopIteration:
            del agents[name]
        for g in background:
            next(g)
    raise AssertionError(f"no progress: ntiles={ntiles} seed={seed} waiting={list(agents)}")


def test_protocol_never_deadlocks_nor_aliases_a_phase():
    for ntiles in range(0, 18):
        for seed in range(200):
            simulate(ntiles, seed)


def test_one_shared_score_barrier_would_alias():
    """The protocol with both score buffers on one mbarrier (the hang met while building
    the kernel): an early score product can complete a second phase before the first
    waiter arrives."""
    failures = 0
    for seed in range(60):
        try:
            simulate(2, seed, score_bars=1)
        except AssertionError:
            failures += 1
    assert failures > 0
