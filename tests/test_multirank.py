"""The host side of the multi-GPU path, as two gloo ranks on CPU.

The path shards without an exchange (every rank runs its own replica of the
workload), so the only multi-rank logic is bench.py's plumbing: the process group,
the barrier around the timed region, the max-over-ranks time, the whole-job
throughput computed from it, and the reference arm's rule that rank 0 alone works and
prints.  Each rank is a separate Python process (as under torchrun), rendezvous on
127.0.0.1.
"""

import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

RANK_SCRIPT = r"""
import json, sys
sys.path.insert(0, {root!r})
import bench
world, rank, local = bench.dist_setup(None)
bench.barrier(world)
t = bench.max_over_ranks(1.5 + rank, world)       # rank 1 is the slower one
v = bench.job_throughput(world, 1000, t)
import torch.distributed as dist
dist.barrier()
dist.destroy_process_group()
print(json.dumps({{"rank": rank, "world": world, "local": local, "t": t, "v": v}}))
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _launch(world, script, extra_env=None):
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(r),
                   LOCAL_RANK=str(r), WORLD_SIZE=str(world), CUDA_VISIBLE_DEVICES="")
        env.update(extra_env or {})
        procs.append(subprocess.Popen([sys.executable, "-c", script], env=env, cwd=ROOT,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            out, err = p.communicate(timeout=180)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            raise
        assert p.returncode == 0, err[-2000:]
        outs.append(out)
    return outs


def test_two_gloo_ranks_take_the_slowest_time():
    outs = _launch(2, RANK_SCRIPT.format(root=ROOT))
    got = sorted((json.loads(o.strip().splitlines()[-1]) for o in outs), key=lambda d: d["rank"])
    assert [d["rank"] for d in got] == [0, 1]
    for d in got:
        assert d["world"] == 2 and d["local"] == d["rank"]
        assert d["t"] == 2.5                          # the max over ranks, on every rank
        assert abs(d["v"] - 2 * 1000 / 2.5e-3) < 1e-6  # both ranks' units over that time


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25
    assert bench.job_throughput(1, 131072, 5.0) == 131072 / 5e-3


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun the reference arm's other ranks exit 0 at once, printing nothing."""
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2", CUDA_VISIBLE_DEVICES="")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, cwd=ROOT,
                       capture_output=True, text=True, timeout=120)
    assert p.returncode == 0, p.stderr[-2000:]
    assert p.stdout.strip() == ""
