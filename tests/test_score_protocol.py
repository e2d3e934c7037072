"""The barrier protocol of the tensor-core token-scoring kernel, and its timeout path,
checked on the host.

A model of token_score_tc_kernel's synchronisation (csrc/token_tc.cu): the loader
warps (one agent), the MMA thread, the epilogue warps (one agent), the tensor pipe (it
completes issued MMA groups in order, arriving on their mbarriers) and the copy engine
(TMA loads and cp.async groups, completing in issue order).  A three-stage shared-memory
ring (full / empty per stage) and two TMEM accumulators (acc_full / acc_empty each).

Every wait is bounded: it gives up after a budget of steps, raises the timeout and sets
the CTA's abort flag; waits that watch the flag give up as soon as it is set.  The MMA
thread, once it stops, waits for the completion of the last MMA group it issued before
the CTA ends (the accumulators then hold no product in flight when TMEM is freed).

Checked: random interleavings never deadlock and never alias a barrier phase; with a
generous budget nothing times out; with the loaders suppressed (the test mode of the
kernel, hisa_test_fault) the MMA thread's first wait runs out, every agent ends, nothing
was issued, and no copy or MMA is outstanding when the CTA ends.
"""

import random

STAGES = 3


class Bar:
    def __init__(self, name):
        self.name, self.done = name, 0


def _ready(bar, fill):
    assert bar.done <= fill + 1, f"{bar.name} is two phases ahead of a waiter (fill {fill})"
    return bar.done >= fill + 1


def simulate(ntiles, seed, budget=10 ** 6, no_loads=False):
    rnd = random.Random(seed)
    full = [Bar(f"full{i}") for i in range(STAGES)]
    empty = [Bar(f"empty{i}") for i in range(STAGES)]
    acc_full = [Bar("acc_full0"), Bar("acc_full1")]
    acc_empty = [Bar("acc_empty0"), Bar("acc_empty1")]
    pipe, copies = [], []
    st = {"abort": False, "timeouts": 0, "mma_issued": 0, "loads_issued": 0}

    def wait(bar, fill, watch_abort):
        """Bounded wait; returns False when it gave up (timeout or abort)."""
        n = 0
        while not _ready(bar, fill):
            if watch_abort and st["abort"]:
                return False
            n += 1
            if n > budget:
                st["timeouts"] += 1
                st["abort"] = True
                return False
            yield
        return True

    def loader():
        my_groups = []
        i = 0
        for t in ([] if no_loads else range(ntiles)):
            s = i % STAGES
            if i >= STAGES:
                ok = yield from wait(empty[s], i // STAGES - 1, True)
                if not ok:
                    break
            if st["abort"]:
                break
            g = {"done": False, "tile": i}
            copies.append(g)  # the key block (TMA) and the query gathers (cp.async)
            my_groups.append(g)
            st["loads_issued"] += 1
            yield
            if i > 0:  # two tiles in flight: the previous tile's copies, then its stage
                while not my_groups[-2]["done"]:
                    yield
                full[(i - 1) % STAGES].done += 1
            i += 1
        if i > 0:  # every copy this agent issued has landed before it ends
            while not all(g["done"] for g in my_groups):
                yield
            if not st["abort"]:
                full[(i - 1) % STAGES].done += 1

    def mma():
        issued = 0
        for i in range(ntiles):
            s, a = i % STAGES, i & 1
            ok = yield from wait(full[s], i // STAGES, False)
            if ok and i >= 2:
                ok = yield from wait(acc_empty[a], (i >> 1) - 1, False)
            if not ok or st["abort"]:
                break
            pipe.append([empty[s], acc_full[a]])
            issued += 1
            st["mma_issued"] += 1
            yield
        if issued:  # drain: the last group's accumulator barrier completes
            last = issued - 1
            while not acc_full[last & 1].done >= (last >> 1) + 1:
                yield

    def epilogue():
        for i in range(ntiles):
            a = i & 1
            ok = yield from wait(acc_full[a], i >> 1, True)
            if not ok:
                break
            yield  # TMEM loads and the score stores
            acc_empty[a].done += 1

    def tensor_pipe():
        while True:
            if pipe and rnd.random() < 0.5:
                for b in pipe.pop(0):
                    b.done += 1
            yield

    def copy_engine():
        while True:
            pending = [g for g in copies if not g["done"]]
            if pending and rnd.random() < 0.5:
                pending[0]["done"] = True
            yield

    agents = {"loader": loader(), "mma": mma(), "epilogue": epilogue()}
    background = [tensor_pipe(), copy_engine()]
    for _ in range(4 * 10 ** 6):
        if not agents:
            break
        name = rnd.choice(list(agents))
        try:
            next(agents[name])
        except StopIteration:
            del agents[name]
        for g in background:
            next(g)
    else:
        raise AssertionError(f"no progress: ntiles={ntiles} seed={seed} waiting={list(agents)}")
    # the CTA ends here: no copy and no MMA may still be in flight
    assert not pipe, "an MMA group is still in flight when the CTA ends"
    assert all(g["done"] for g in copies), "a copy is still in flight when the CTA ends"
    return st


def test_protocol_never_deadlocks_nor_times_out():
    for ntiles in range(0, 14):
        for seed in range(150):
            st = simulate(ntiles, seed)
            assert st["timeouts"] == 0 and st["mma_issued"] == ntiles


def test_suppressed_loads_give_up_with_nothing_in_flight():
    for ntiles in range(1, 10):
        for seed in range(50):
            st = simulate(ntiles, seed, budget=200, no_loads=True)
            assert st["timeouts"] >= 1 and st["abort"]
            assert st["loads_issued"] == 0 and st["mma_issued"] == 0


def test_random_give_ups_leave_nothing_in_flight():
    """Tight budgets make waits run out at random points of a normal run: the ends of
    the agents (copies drained by the loader, the last MMA group by the MMA thread)
    still leave nothing outstanding."""
    gave_up = 0
    for ntiles in range(1, 12):
        for seed in range(80):
            st = simulate(ntiles, seed, budget=3)
            gave_up += st["timeouts"] > 0
    assert gave_up > 0
