#!/usr/bin/env python
"""Benchmark of the HISA token-selection indexer on one node.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one HISA selection over the 131072-token prefill (1 sequence, q/k
bf16 ~ N(0,1), d = 64, B = 128, m = 64, k = 2048): block pooling, stage 1
(block scores, top-m) and stage 2 (gather-score, top-k), all through the
library's C ABI.  Inputs live in HBM before the timed region; L2 is flushed
(a 256 MiB write) before every timed step, outside the step's CUDA events.
The same run measures, and reports under "details": the flat DSA scan on the
same input (the HISA/DSA speedup), the 32768-token needle prefill (speedup,
IoU, needle recall, stage 1 alone and a per-sequence block budget of half the
blocks), the 4096-token integer prefill and the packed varlen prefill (times,
agreement with the oracle, IoU), decode (16 sequences x 32768 keys, one
append and one selection per step, 256 steps in a CUDA graph over four
independent decode states so that the key caches cannot stay in L2), the
sparse attention step (16 heads x 128, bf16 K/V rows) over the decode batch's
and the 32K prefill's selections, and the CPU oracle timed on every
configuration.

Under torchrun (N > 1) the ranks share the one workload: each takes a
contiguous run of query rows balanced by estimated work, with its sequence's
keys, and writes its own output rows -- no collective on the data path
(strong scaling; times are the maximum over ranks).  ``--impl reference``
times the CPU oracle instead (the only other place this script runs the
oracle) on seeded samples of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "HISA top-k selection queries/s & ms at 32K/128K; HBM GB/s vs peak"
UNIT = "queries/s"
WORKLOAD = "prefill_L131072 (1 seq, q/k bf16 N(0,1), d=64, B=128, m=64, k=2048)"
# the other prefill workloads --config can time (profiling runs, not bench lines)
CONFIG_WORKLOADS = {
    1: "prefill_L4096 integer (1 seq, q/k bf16 integers in [-4, 4], d=64, B=128, m=8, k=256)",
    3: "prefill_L32768 needles (1 seq, q/k bf16 N(0,1) + 16 needles, d=64, B=128, m=64, k=2048)",
    4: WORKLOAD,
    5: "prefill varlen (8 seqs, q/k bf16 N(0,1), d=64, B=128, m=64, k=2048)",
}
L2_FLUSH_BYTES = 256 << 20
# row ranges of the end-to-end step (their index copies overlap the next range's select)
E2E_CHUNKS = 8

# DRAM bytes per step (dram__bytes_read.sum + dram__bytes_write.sum summed over the
# kernel's launches) on the 131072-token prefill, from an ncu capture of that kernel on
# the 32768-token prefill scaled by the selected (query, block) pairs of the two, with
# the sha256 prefix of the kernel's sources at capture time (a changed source voids it);
# the bench line divides it by the launches per step.
TRAFFIC = {
    # 32K: 957.4 MB read + 252.4 MB written, 1839104 pairs; 128K: 8130560 pairs
    "token_select_scratch": (5348619405, "45365b5016604859", ("token_select.cu", "select.cuh")),
    # 32K: 21.2 MB read + 878.1 MB written
    "token_score_tc": (3975557505, "8ed7b49db83627bf", ("token_tc.cu",)),
}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true", help="skip the details measurements")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline")
    ap.add_argument("--config", type=int, default=4, choices=[1, 3, 4, 5],
                    help="prefill workload of the timed step (profiling runs; default 4 = 128K)")
    ap.add_argument("--dsa-steps", type=int, default=0,
                    help="profiling runs: flat-scan calls on the same workload after the timed steps")
    ap.add_argument("--decode-profile", type=int, default=0, metavar="N",
                    help="profiling runs: only N eager decode steps (16 x 32768 keys, append + "
                         "selection on the default stream) and two attention calls over the "
                         "last selection, then exit")
    return ap.parse_args()


def cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------------------
# clocks during the measured region

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap,pci.bus_id")

    def __init__(self, bus_id: str):
        self.bus_id = bus_id.lower()
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        threading.Thread(target=self._read, daemon=True).start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in list(self.lines):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            bus = parts[7].lower()
            if self.bus_id and not (bus.endswith(self.bus_id) or self.bus_id.endswith(bus)):
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# helpers

PG_TIMEOUT_S = 120  # ranks that wait for one another end with an error, not a hang


def dist_setup(args):
    """One process per GPU (torchrun's RANK / LOCAL_RANK / WORLD_SIZE): NCCL on the
    GPUs; gloo on CPU, where only the host-side plumbing runs (tests)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=PG_TIMEOUT_S))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def _reduce_device():
    import torch.distributed as dist
    return "cuda" if dist.get_backend() == "nccl" else "cpu"


def barrier(world):
    """Every rank reaches this point, then the device is idle on this rank."""
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def max_over_ranks(x: float, world: int) -> float:
    """The largest of the ranks' values (every multi-GPU time is the slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=_reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, units_per_rank: int, ms: float) -> float:
    """Whole-job throughput under weak scaling: every rank processes units_per_rank in
    the max-over-ranks time ms."""
    return world * units_per_rank / (ms / 1e3)


def local_workload(w, world: int, rank: int):
    """This rank's shard of a workload: a contiguous run of query rows, cut so that the
    ranks' estimated work is balanced, with its sequences' key regions (no exchange
    between ranks; every rank writes its own output rows).  Returns the shard as a
    workload of its own and its global rows [row0, row1)."""
    if world == 1:
        return w, 0, w.total_q
    from synth import Workload
    from sparse_attention_top_hisa_b200.shard import query_cost, row_bounds, shard
    bounds = row_bounds(w.total_q, world, query_cost(w.cu_q, w.cu_k, w.seqlens, w.B, w.m))
    sh = shard(w.cu_q, w.cu_k, w.seqlens, world, rank, w.B, bounds)
    lw = Workload(f"{w.name}_shard{rank}of{world}", w.q[sh.row0:sh.row1], w.k[sh.key0:sh.key1],
                  sh.cu_seqlens_q, sh.cu_seqlens_k, sh.seqlens_k, w.B, w.m, w.topk, w.d, w.exact)
    return lw, sh.row0, sh.row1


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=_reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def to_dev_bf16(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def to_dev_i32(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def query_positions(w) -> np.ndarray:
    """Sequence-local position of every query row (the last q_len positions)."""
    out = np.empty(w.total_q, np.int64)
    for s in range(w.num_seqs):
        a, b = int(w.cu_q[s]), int(w.cu_q[s + 1])
        L = int(w.seqlens[s])
        out[a:b] = np.arange(L - (b - a), L)
    return out


def candidate_counts(w) -> np.ndarray:
    """c_i of every query: the tokens j <= i of its selected blocks.  Every selected
    block other than the query's own lies wholly before it; the own block (always
    selected) contributes i % B + 1."""
    pos = query_positions(w)
    own = pos // w.B
    nsel = np.minimum(w.m, own + 1)
    return (nsel - 1) * w.B + pos % w.B + 1


def algorithmic(w) -> dict:
    """The method's own work per step of every kernel on the prefill path, as the
    per-unit figures of the measurement plan fix it: bytes that must move (bound
    "hbm") or flops that must be done (bound "tensor").  Intermediates this design
    chooses to write and read back (block-score keys, (query, slot) lists, score rows)
    are not counted; the ncu traffic of a kernel against these figures shows them."""
    B, m, K, d = w.B, w.m, w.topk, 64
    pos = query_positions(w)
    own = pos // B
    nsel = np.minimum(m, own + 1)
    pairs = float(nsel.sum())
    eligible = float(np.where(own + 1 > m, own + 1, 0).sum())  # blocks scored in stage 1
    cands = float(candidate_counts(w).sum())
    live_rows = float(w.seqlens.sum())
    nblocks = float(((w.seqlens + B - 1) // B).sum())
    nq = float(w.total_q)
    return {
        "pool_blocks": {"bound": "hbm", "per_step": live_rows * 2 * d + nblocks * 4 * d,
                        "what": "128 B of key read per live token + 256 B of fp32 representative "
                                "written per block"},
        "block_score_tc": {"bound": "tensor", "per_step": eligible * 2 * d,
                           "what": "2*64 flop per eligible (query, block) pair of the queries that "
                                   "see more than m blocks"},
        "block_select": {"bound": "hbm", "per_step": nq * m * 4,
                         "what": "4 B per selected block written (the block lists)"},
        "inv_lists": {"bound": "hbm", "per_step": pairs * 4,
                      "what": "4 B per selected block read (the block lists)"},
        "token_score_tc": {"bound": "tensor", "per_step": cands * 2 * d,
                           "what": "2*64 flop per candidate token (j <= i in a selected block)"},
        "token_select_scratch": {"bound": "hbm", "per_step": nq * K * 4 + pairs * 4,
                                 "what": "k int32 indices written per query + its block list read"},
        "step": {"bound": "hbm",
                 "per_step": nq * 2 * d + live_rows * 2 * d + nblocks * 4 * d * 2 + nq * K * 4,
                 "what": "q and k read, representatives written and read, k int32 indices "
                         "written per query"},
    }


def roofline_entry(a: dict, amount: float, launch_ms: float, hbm_peak: float,
                   tc_peak: float) -> dict:
    """achieved = algorithmic amount per launch / launch time, against the measured peak
    of its bound (HBM copy bandwidth, or the bf16 tensor-core GEMM rate)."""
    if a["bound"] == "hbm":
        ach, peak, unit = amount / (launch_ms / 1e3) / 1e9, hbm_peak, "GB/s"
    else:
        ach, peak, unit = amount / (launch_ms / 1e3) / 1e12, tc_peak, "TFLOP/s"
    return {"bound": a["bound"], "achieved": round(ach, 3), "peak": peak, "unit": unit,
            "frac": round(ach / peak, 4), "launch_ms": round(launch_ms, 4),
            "algorithmic": a["what"], "algorithmic_per_launch": amount}


def iou_rows(a: np.ndarray, b: np.ndarray) -> float:
    vals = []
    for x, y in zip(a, b):
        x = x[x >= 0]
        y = y[y >= 0]
        u = np.union1d(x, y).size
        vals.append(np.intersect1d(x, y).size / u if u else 1.0)
    return float(np.mean(vals))


def source_sha(names) -> str:
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "sparse_attention_top_hisa_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# ---------------------------------------------------------------------------
# our arm

def run_ours(args, world, rank):
    import torch
    import sparse_attention_top_hisa_b200 as H
    from synth import config_workload

    hbm_peak, tc_peak, peak_src = peaks()
    dev = torch.cuda.current_device()
    props = torch.cuda.get_device_properties(dev)
    bus = ""
    try:
        bus = "%04x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
    except AttributeError:
        pass
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    w_full = config_workload(args.config)
    w, row0, row1 = local_workload(w_full, world, rank)
    B, m, K = w.B, w.m, w.topk
    nq = w.total_q
    nq_job = w_full.total_q
    q, k = to_dev_bf16(w.q), to_dev_bf16(w.k)
    cu_q, cu_k, sl = to_dev_i32(w.cu_q), to_dev_i32(w.cu_k), to_dev_i32(w.seqlens)
    out = torch.empty(nq, K, dtype=torch.int32, device="cuda")
    reps = torch.zeros(w.rep_rows, 64, dtype=torch.float32, device="cuda")
    ws = torch.empty(max(H.hisa_select_workspace_size(nq, w.num_seqs, w.max_seqlen_k, m, K), 256),
                     dtype=torch.uint8, device="cuda")

    def step():
        H.hisa_pool_blocks(k, cu_k, sl, w.max_seqlen_k, reps=reps)
        H.hisa_select(q, k, reps, cu_q, cu_k, sl, w.max_seqlen_k, m, K, out_idx=out, workspace=ws)

    H.hisa_device_status(clear=True)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert H.hisa_device_status() == 0, "device-side error during warm-up"

    sampler = ClockSampler(bus) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)

    # ---- timed region ----------------------------------------------------------
    H.hisa_timing_collect(reset=True)
    H.hisa_timing_enable(True)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier(world)
    t_wall = time.perf_counter()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    barrier(world)
    t_wall = time.perf_counter() - t_wall
    H.hisa_timing_enable(False)
    kt = H.hisa_timing_collect(reset=True)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    ms = max_over_ranks(sum(step_ms) / len(step_ms), world)
    launches = int(sum(v["launches"] for v in kt.values()))
    value = nq_job / (ms / 1e3)  # strong scaling: the ranks share one fixed workload

    # ---- end to end: host buffers through the public API --------------------------
    # Every step copies the inputs in from pinned host memory, pools, selects and copies
    # the indices back.  The rows are selected in E2E_CHUNKS contiguous ranges, each a
    # batch of its own (the shard layouts of sparse_attention_top_hisa_b200.shard, which
    # reproduce the unsharded rows exactly), and each range's indices go back to the host
    # on a copy stream while the next range is selected; "one_call" is the same with a
    # single hisa_select and the copy after it.
    from sparse_attention_top_hisa_b200.shard import query_cost, row_bounds, shard
    hq = torch.from_numpy(np.ascontiguousarray(w.q).view(np.int16)).view(torch.bfloat16).pin_memory()
    hk = torch.from_numpy(np.ascontiguousarray(w.k).view(np.int16)).view(torch.bfloat16).pin_memory()
    hcq = torch.from_numpy(w.cu_q.astype(np.int32)).pin_memory()
    hck = torch.from_numpy(w.cu_k.astype(np.int32)).pin_memory()
    hsl = torch.from_numpy(w.seqlens.astype(np.int32)).pin_memory()
    hout = torch.empty(nq, K, dtype=torch.int32).pin_memory()
    nch = E2E_CHUNKS if nq >= E2E_CHUNKS * 4096 else 1
    copy_stream = torch.cuda.Stream()
    # per-range layout arrays: pinned host staging and device copies, filled every step
    hdesc = [torch.empty(3 * (w.num_seqs + 1), dtype=torch.int32).pin_memory() for _ in range(nch)]
    ddesc = [torch.empty(3 * (w.num_seqs + 1), dtype=torch.int32, device="cuda")
             for _ in range(nch)]

    def e2e_step(chunked):
        q.copy_(hq, non_blocking=True)
        k.copy_(hk, non_blocking=True)
        cu_q.copy_(hcq, non_blocking=True)
        cu_k.copy_(hck, non_blocking=True)
        sl.copy_(hsl, non_blocking=True)
        if not chunked:
            step()
            hout.copy_(out, non_blocking=True)
            return 0
        H.hisa_pool_blocks(k, cu_k, sl, w.max_seqlen_k, reps=reps)
        lay = (hcq.numpy(), hck.numpy(), hsl.numpy())
        bounds = row_bounds(nq, nch, query_cost(*lay, B, m))
        extra = 0
        for c in range(nch):
            sh = shard(*lay, nch, c, B, bounds)
            ns = sh.num_seqs
            hd = hdesc[c]
            hd[:ns + 1] = torch.from_numpy(sh.cu_seqlens_q)
            hd[ns + 1:2 * ns + 2] = torch.from_numpy(sh.cu_seqlens_k)
            hd[2 * ns + 2:3 * ns + 2] = torch.from_numpy(sh.seqlens_k)
            dd = ddesc[c]
            dd[:3 * ns + 2].copy_(hd[:3 * ns + 2], non_blocking=True)
            extra += (3 * ns + 2) * 4
            H.hisa_select(q[sh.row0:sh.row1], k[sh.key0:sh.key1], reps[sh.rep0:], dd[:ns + 1],
                          dd[ns + 1:2 * ns + 2], dd[2 * ns + 2:3 * ns + 2], sh.max_seqlen_k, m, K,
                          out_idx=out[sh.row0:sh.row1], workspace=ws)
            done = torch.cuda.Event()
            done.record(stream)
            copy_stream.wait_event(done)
            with torch.cuda.stream(copy_stream):
                hout[sh.row0:sh.row1].copy_(out[sh.row0:sh.row1], non_blocking=True)
        stream.wait_stream(copy_stream)
        return extra

    def time_e2e(chunked):
        times, extra = [], 0
        for i in range(e2e_steps + 1):
            flush.fill_(i & 0xFF)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            extra = e2e_step(chunked)
            b.record(stream)
            b.synchronize()
            if i > 0:
                times.append(a.elapsed_time(b))
        return max_over_ranks(sum(times) / len(times), world), extra

    e2e_steps = max(2, min(args.steps, 5))
    e2e_one, _ = time_e2e(False)
    if nch > 1:
        ref = hout.clone()
        e2e, desc_bytes = time_e2e(True)
        assert torch.equal(hout, ref), "row ranges differ from the single call"
        del ref
    else:
        e2e, desc_bytes = e2e_one, 0
    assert H.hisa_device_status() == 0, "device-side error in the end-to-end steps"
    h2d = sum_over_ranks(sum(t.numel() * t.element_size() for t in (hq, hk, hcq, hck, hsl))
                         + desc_bytes, world)
    d2h = sum_over_ranks(hout.numel() * hout.element_size(), world)

    # ---- roofline of the dominant kernel -------------------------------------------
    alg = algorithmic(w)
    per_kernel = {}
    for name, v in kt.items():
        if not v["timed"] or name not in alg:
            continue
        a = alg[name]
        launch_ms = v["ms"] / v["timed"]
        launches_per_step = v["timed"] / args.steps
        amount = a["per_step"] / launches_per_step  # per launch
        per_kernel[name] = roofline_entry(a, amount, launch_ms, hbm_peak, tc_peak)
        per_kernel[name]["launches_per_step"] = launches_per_step
    for name, e in per_kernel.items():
        t = TRAFFIC.get(name)
        # stored counters hold for the 128K launch of the kernel source they were taken on
        e["traffic"] = (int(round(t[0] / e["launches_per_step"]))
                        if t and t[1] == source_sha(t[2]) and args.config == 4 and world == 1
                        else None)
        if e["traffic"]:
            e["traffic_GBs"] = round(e["traffic"] / (e["launch_ms"] * 1e6), 1)
            if alg[name]["bound"] == "hbm":
                e["traffic_over_algorithmic"] = round(e["traffic"] / e["algorithmic_per_launch"], 3)
    dname = max((n for n in per_kernel), key=lambda n: kt[n]["ms"])
    roof = dict(per_kernel[dname])
    roof["kernel"] = dname
    roof["peak_source"] = f"MEASURED_PEAKS.json ({peak_src})"
    step_alg = alg["step"]
    step_roof = roofline_entry(step_alg, step_alg["per_step"], ms, hbm_peak, tc_peak)

    if args.dsa_steps > 0:  # profiling aid: the flat scan on the same inputs
        dout = torch.empty(nq, K, dtype=torch.int32, device="cuda")
        dws = torch.empty(H.dsa_flat_workspace_size(nq, w.num_seqs, w.max_seqlen_k, K),
                          dtype=torch.uint8, device="cuda")
        for _ in range(args.dsa_steps):
            H.dsa_flat_select(q, k, cu_q, cu_k, sl, w.max_seqlen_k, K, out_idx=dout, workspace=dws)
        torch.cuda.synchronize()
        del dout, dws

    details = {"hisa_step": {"ms": round(ms, 4), "queries_per_s": round(nq_job / (ms / 1e3), 1),
                             "median_ms": round(float(np.median(step_ms)), 4),
                             "min_ms": round(float(min(step_ms)), 4),
                             "rank_rows": [int(row0), int(row1)],
                             "kernels": {n: {"ms_per_step": round(v["ms"] / args.steps, 4),
                                             "launches": v["launches"]}
                                         for n, v in kt.items() if v["launches"]},
                             "roofline_per_kernel": per_kernel,
                             "roofline_step": step_roof}}
    if rank == 0 and not args.no_extras:
        details.update(extras(args, w, q, k, cu_q, cu_k, sl, out, flush, stream, hbm_peak, tc_peak))

    clocks = sampler.stop() if sampler else None
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": CONFIG_WORKLOADS[args.config], "seq_len": int(w.max_seqlen_k),
                   "queries_per_step": nq_job,
                   "d": 64, "B": B, "m": m, "k": K, "inputs": f"bf16 q/k, PCG64 seed {20260 + args.config}",
                   "l2": "256 MiB flush before every timed step (outside the step events)",
                   "parallelism": (f"{world} ranks, contiguous query-row shards balanced by "
                                   "work, no collective on the data path" if world > 1
                                   else "single GPU")},
        "e2e": {"value": round(nq_job / (e2e / 1e3), 1), "unit": UNIT,
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "ms_per_step": round(e2e, 3), "row_ranges": nch,
                "one_call": {"value": round(nq_job / (e2e_one / 1e3), 1),
                             "ms_per_step": round(e2e_one, 3)}},
        "gpu_launches": launches,
        "roofline": roof,
        "clocks": clocks,
        "wall_s_timed_region": round(t_wall, 3),
        "details": details,
    }
    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(w)
    return line


def time_events(fn, reps, flush, stream):
    import torch
    out = []
    for i in range(reps):
        flush.fill_(i & 0xFF)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        out.append(a.elapsed_time(b))
    return out


def extras(args, w4, q4, k4, cu_q4, cu_k4, sl4, out4, flush, stream, hbm_peak, tc_peak):
    """Flat DSA at 128K, the 32K needle prefill, decode, IoU."""
    import torch
    import sparse_attention_top_hisa_b200 as H
    from synth import config_workload
    det = {}
    nq, K = w4.total_q, w4.topk
    # flat DSA at 128K
    dout = torch.empty(nq, K, dtype=torch.int32, device="cuda")
    dws = torch.empty(H.dsa_flat_workspace_size(nq, 1, w4.max_seqlen_k, K), dtype=torch.uint8,
                      device="cuda")
    dsa = lambda: H.dsa_flat_select(q4, k4, cu_q4, cu_k4, sl4, w4.max_seqlen_k, K, out_idx=dout,
                                    workspace=dws)
    dsa()
    H.hisa_timing_collect(reset=True)
    H.hisa_timing_enable(True)
    dms = time_events(dsa, 2, flush, stream)
    H.hisa_timing_enable(False)
    dkt = H.hisa_timing_collect(reset=True)
    hms = None
    rows = np.random.Generator(np.random.PCG64(1)).choice(nq, 2048, replace=False)
    iou = iou_rows(out4.cpu().numpy()[rows], dout.cpu().numpy()[rows])
    det["dsa_128k"] = {"ms": round(min(dms), 3), "iou_hisa_vs_dsa_2048_rows": round(iou, 4),
                       "kernels": {n: {"ms_per_call": round(v["ms"] / 2, 3), "launches": v["launches"]}
                                   for n, v in dkt.items() if v["launches"]}}
    del dout, dws
    torch.cuda.empty_cache()

    # 32K needle prefill
    w3 = config_workload(3)
    q3, k3 = to_dev_bf16(w3.q), to_dev_bf16(w3.k)
    cq3, ck3, sl3 = to_dev_i32(w3.cu_q), to_dev_i32(w3.cu_k), to_dev_i32(w3.seqlens)
    reps3 = torch.zeros(w3.rep_rows, 64, dtype=torch.float32, device="cuda")
    o3 = torch.empty(w3.total_q, w3.topk, dtype=torch.int32, device="cuda")
    d3 = torch.empty_like(o3)
    ws3 = torch.empty(H.hisa_select_workspace_size(w3.total_q, 1, w3.max_seqlen_k, w3.m, w3.topk),
                      dtype=torch.uint8, device="cuda")
    dws3 = torch.empty(H.dsa_flat_workspace_size(w3.total_q, 1, w3.max_seqlen_k, w3.topk),
                       dtype=torch.uint8, device="cuda")

    def h3():
        H.hisa_pool_blocks(k3, ck3, sl3, w3.max_seqlen_k, reps=reps3)
        H.hisa_select(q3, k3, reps3, cq3, ck3, sl3, w3.max_seqlen_k, w3.m, w3.topk, out_idx=o3,
                      workspace=ws3)

    def f3():
        H.dsa_flat_select(q3, k3, cq3, ck3, sl3, w3.max_seqlen_k, w3.topk, out_idx=d3,
                          workspace=dws3)
    h3()
    f3()
    hm3 = statistics.median(time_events(h3, 5, flush, stream))
    dm3 = statistics.median(time_events(f3, 3, flush, stream))
    a3, b3 = o3.cpu().numpy(), d3.cpu().numpy()
    rec_h = np.mean([j in a3[i] for i, j in w3.needles])
    rec_d = np.mean([j in b3[i] for i, j in w3.needles])
    rows3 = np.random.Generator(np.random.PCG64(2)).choice(w3.total_q, 4096, replace=False)
    det["prefill_32k"] = {"hisa_ms": round(hm3, 3), "dsa_ms": round(dm3, 3),
                          "hisa_speedup_over_dsa": round(dm3 / hm3, 2),
                          "hisa_queries_per_s": round(w3.total_q / (hm3 / 1e3), 1),
                          "iou_hisa_vs_dsa_4096_rows": round(iou_rows(a3[rows3], b3[rows3]), 4),
                          "needle_recall_hisa": float(rec_h), "needle_recall_dsa": float(rec_d)}
    # variants on the same inputs: stage 1 alone (every token of the best k/B blocks, no
    # token refinement: hisa_block_sparse_select) and a block budget of half of the
    # sequence's blocks (m_s = ceil(0.5 * M_s): hisa_fraction_blocks + hisa_select_varm)
    variants = {}
    mb = w3.topk // w3.B
    ob = torch.empty(w3.total_q, mb * w3.B, dtype=torch.int32, device="cuda")
    wsb = torch.empty(H.hisa_block_sparse_workspace_size(w3.total_q, 1, w3.max_seqlen_k, mb),
                      dtype=torch.uint8, device="cuda")

    def hb():
        H.hisa_pool_blocks(k3, ck3, sl3, w3.max_seqlen_k, reps=reps3)
        H.hisa_block_sparse_select(q3, reps3, cq3, ck3, sl3, w3.max_seqlen_k, mb, out_idx=ob,
                                   workspace=wsb)
    hb()
    msb = statistics.median(time_events(hb, 3, flush, stream))
    av = ob.cpu().numpy()
    variants[f"block_sparse_only_m{mb}"] = {
        "entry_point": "hisa_block_sparse_select", "m": mb, "ms": round(msb, 3),
        "iou_vs_dsa_4096_rows": round(iou_rows(av[rows3], b3[rows3]), 4),
        "needle_recall": float(np.mean([j in av[i] for i, j in w3.needles]))}
    del ob, wsb
    m_max = H.HISA_MAX_M
    ov = torch.empty_like(o3)
    wsv = torch.empty(H.hisa_select_workspace_size(w3.total_q, 1, w3.max_seqlen_k, m_max, w3.topk),
                      dtype=torch.uint8, device="cuda")
    msq = torch.empty(1, dtype=torch.int32, device="cuda")

    def hv():
        H.hisa_pool_blocks(k3, ck3, sl3, w3.max_seqlen_k, reps=reps3)
        H.hisa_fraction_blocks(ck3, sl3, 0.5, m_max, m_seq=msq)
        H.hisa_select_varm(q3, k3, reps3, cq3, ck3, sl3, msq, w3.max_seqlen_k, m_max, w3.topk,
                           out_idx=ov, workspace=wsv)
    hv()
    msv = statistics.median(time_events(hv, 3, flush, stream))
    av = ov.cpu().numpy()
    variants["hisa_half_blocks"] = {
        "entry_point": "hisa_fraction_blocks(f=0.5) + hisa_select_varm", "m": int(msq.item()),
        "ms": round(msv, 3), "iou_vs_dsa_4096_rows": round(iou_rows(av[rows3], b3[rows3]), 4),
        "needle_recall": float(np.mean([j in av[i] for i, j in w3.needles]))}
    del ov, wsv
    det["prefill_32k"]["variants"] = variants
    det["dsa_128k"]["hisa_speedup_over_dsa"] = None  # filled by the caller
    det["attention"] = attention_bench(w3, o3, flush, stream, hbm_peak, tc_peak)
    del q3, k3, o3, d3, ws3, dws3
    torch.cuda.empty_cache()
    det["decode"] = decode_bench(flush, stream, hbm_peak)
    det["prefill_4096_integer"] = prefill_bench(1, flush, stream)
    det["prefill_varlen_8seqs"] = prefill_bench(5, flush, stream)
    det["hbm_stream_ceilings"] = stream_ceilings(stream)
    return det


def prefill_bench(cfg, flush, stream, reps=5):
    """A prefill configuration: HISA (pool + select) and the flat scan on the same
    inputs, their times, and HISA-vs-DSA IoU (every row, or 4096 seeded rows)."""
    import torch
    import sparse_attention_top_hisa_b200 as H
    from synth import config_workload
    w = config_workload(cfg)
    q, k = to_dev_bf16(w.q), to_dev_bf16(w.k)
    cq, ck, sl = to_dev_i32(w.cu_q), to_dev_i32(w.cu_k), to_dev_i32(w.seqlens)
    reps_ = torch.zeros(w.rep_rows, 64, dtype=torch.float32, device="cuda")
    o = torch.empty(w.total_q, w.topk, dtype=torch.int32, device="cuda")
    d = torch.empty_like(o)
    ws = torch.empty(H.hisa_select_workspace_size(w.total_q, w.num_seqs, w.max_seqlen_k, w.m,
                                                  w.topk), dtype=torch.uint8, device="cuda")
    dws = torch.empty(H.dsa_flat_workspace_size(w.total_q, w.num_seqs, w.max_seqlen_k, w.topk),
                      dtype=torch.uint8, device="cuda")

    def hisa():
        H.hisa_pool_blocks(k, ck, sl, w.max_seqlen_k, reps=reps_)
        H.hisa_select(q, k, reps_, cq, ck, sl, w.max_seqlen_k, w.m, w.topk, out_idx=o,
                      workspace=ws)

    def dsa():
        H.dsa_flat_select(q, k, cq, ck, sl, w.max_seqlen_k, w.topk, out_idx=d, workspace=dws)
    hisa()
    dsa()
    hm = statistics.median(time_events(hisa, reps, flush, stream))
    dm = statistics.median(time_events(dsa, 3, flush, stream))
    a, b = o.cpu().numpy(), d.cpu().numpy()
    rows = (np.arange(w.total_q) if w.total_q <= 4096 else
            np.random.Generator(np.random.PCG64(3)).choice(w.total_q, 4096, replace=False))
    assert H.hisa_device_status() == 0
    res = {"queries": int(w.total_q), "sequences": int(w.num_seqs),
           "lengths": [int(x) for x in w.seqlens], "m": int(w.m), "k": int(w.topk),
           "hisa_ms": round(hm, 4), "hisa_queries_per_s": round(w.total_q / (hm / 1e3), 1),
           "dsa_ms": round(dm, 4), "hisa_speedup_over_dsa": round(dm / hm, 2),
           "iou_hisa_vs_dsa": round(iou_rows(a[rows], b[rows]), 4),
           "iou_rows": int(len(rows))}
    del q, k, o, d, ws, dws
    torch.cuda.empty_cache()
    return res


def stream_ceilings(stream, nbytes=4 << 30, reps=5):
    """Plain torch fill (write only) and copy (read + write) of 4 GiB: the ceilings the
    write-bound scoring kernel and the HBM peak are compared against."""
    import torch
    x = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    y = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    res = {}
    for name, fn, moved in (("write_only_fill_GBs", lambda: x.fill_(3), nbytes),
                            ("copy_read_plus_write_GBs", lambda: y.copy_(x), 2 * nbytes)):
        fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        b.synchronize()
        res[name] = round(moved / (a.elapsed_time(b) / reps / 1e3) / 1e9, 1)
    del x, y
    torch.cuda.empty_cache()
    return res


def decode_bench(flush, stream, hbm_peak, n_states=4, steps=256):
    """16 sequences x 32768 keys; each step appends one key per sequence and selects
    for one query per sequence (hisa_decode_step: one launch per step). Steps rotate
    over n_states independent decode states (4 x 67.6 MB of key cache > L2) and the 256
    steps run as one CUDA graph."""
    import torch
    import sparse_attention_top_hisa_b200 as H
    from synth import config_workload
    dw = config_workload(2, steps=steps)
    S, cap, m, K = dw.num_seqs, dw.capacity, dw.m, dw.topk
    cu_k = to_dev_i32(dw.cu_k)
    cu_q = to_dev_i32(np.arange(S + 1))
    states = []
    for r in range(n_states):
        kc = to_dev_bf16(dw.k_cache)
        lens = to_dev_i32(dw.seqlens0)
        reps = H.hisa_pool_blocks(kc, cu_k, lens, cap)
        out = torch.empty(S, K, dtype=torch.int32, device="cuda")
        states.append((kc, lens, reps, out))
    lens0 = to_dev_i32(dw.seqlens0)
    newk = to_dev_bf16(dw.new_keys)  # [steps, S, 1, 64]
    qs = to_dev_bf16(dw.queries.reshape(steps * S, 64)).view(steps, S, 64)
    ws = torch.empty(H.hisa_select_workspace_size(S, S, cap, m, K), dtype=torch.uint8, device="cuda")

    def run_steps():  # one launch per step: append and select fused (hisa_decode_step)
        for i in range(steps):
            kc, lens, reps, out = states[i % n_states]
            H.hisa_decode_step(kc, reps, cu_k, lens, newk[i].view(S, 64), qs[i], cap, m, K,
                               out_idx=out)

    def reset():
        for kc, lens, reps, out in states:
            lens.copy_(lens0)

    # warm-up (sets kernel attributes), then a timed pass for the per-kernel breakdown,
    # then capture
    run_steps()
    torch.cuda.synchronize()
    reset()
    H.hisa_timing_collect(reset=True)
    H.hisa_timing_enable(True)
    run_steps()
    H.hisa_timing_enable(False)
    breakdown = {n: round(v["ms"] / steps * 1e3, 2)
                 for n, v in H.hisa_timing_collect(reset=True).items() if v["timed"]}
    reset()
    H.hisa_timing_collect(reset=True)
    g = torch.cuda.CUDAGraph()
    s2 = torch.cuda.Stream()
    s2.wait_stream(stream)
    with torch.cuda.stream(s2):
        with torch.cuda.graph(g, stream=s2):
            run_steps()
    torch.cuda.current_stream().wait_stream(s2)
    launches_per_graph = int(sum(v["launches"] for v in H.hisa_timing_collect(reset=True).values()))
    times = []
    for i in range(3):
        reset()
        flush.fill_(i)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        b.synchronize()
        times.append(a.elapsed_time(b))
    assert H.hisa_device_status() == 0
    per_step_us = min(times) / steps * 1e3
    # algorithmic bytes per sequence-step: reps of the eligible blocks, the m*B gathered
    # keys, the query, the k output indices, and the append (last block re-read + one row
    # + one representative written)
    eligible = (int(dw.seqlens0[0]) + steps // 2) // 128 + 1
    per_seq = eligible * 256 + m * 128 * 128 + 128 + K * 4 + (128 * 128 + 128 + 256)
    gbs = per_seq * S / (per_step_us * 1e-6) / 1e9
    del g
    return {"us_per_step": round(per_step_us, 2), "steps_per_graph": steps,
            "launches_per_step": launches_per_graph / steps,
            "algorithmic_MB_per_step": round(per_seq * S / 1e6, 2),
            "GBs": round(gbs, 1), "frac_of_hbm_peak": round(gbs / hbm_peak, 4),
            "states": n_states, "kernel_us_per_step_eager": breakdown}


def attention_bench(w3, o3, flush, stream, hbm_peak, tc_peak, heads=16):
    """The sparse attention step over the selected tokens (synthetic q/k/v of width
    128, N(0,1) bf16, 16 heads sharing one key and one value row per token): decode
    (16 queries, the indices HISA selects on the decode workload) and the 32K needle
    prefill (the indices of its HISA run)."""
    import torch
    import sparse_attention_top_hisa_b200 as H
    from synth import config_workload
    res = {}
    rng = np.random.Generator(np.random.PCG64(31))
    D = 128
    scale = 1.0 / np.sqrt(D)

    def rnd(shape):
        return to_dev_bf16(bf16_rows(rng, shape))

    # decode: 16 sequences x 32768 keys, k = 2048
    dw = config_workload(2, steps=1)
    S, cap, m, K = dw.num_seqs, dw.capacity, dw.m, dw.topk
    cu_k, cu_q = to_dev_i32(dw.cu_k), to_dev_i32(np.arange(S + 1))
    kc, lens = to_dev_bf16(dw.k_cache), to_dev_i32(dw.seqlens0)
    reps = H.hisa_pool_blocks(kc, cu_k, lens, cap)
    idx = H.hisa_select(to_dev_bf16(dw.queries[0]), kc, reps, cu_q, cu_k, lens, cap, m, K)
    ka, va = rnd((S * cap, D)), rnd((S * cap, D))
    qa = rnd((S * heads, D)).view(S, heads, D)
    out = torch.empty(S, heads, D, dtype=torch.float32, device="cuda")
    fn = lambda: H.hisa_sparse_attention(qa, ka, va, idx, cu_q, cu_k, scale, out=out)
    fn()
    us = statistics.median(time_events(fn, 5, flush, stream)) * 1e3
    nbytes = S * (K * 2 * D * 2 + heads * D * 2 + heads * D * 4)
    res["decode_16q"] = {"heads": heads, "k": K, "us": round(us, 2),
                         "algorithmic_MB": round(nbytes / 1e6, 2),
                         "GBs": round(nbytes / (us * 1e-6) / 1e9, 1),
                         "frac_of_hbm_peak": round(nbytes / (us * 1e-6) / 1e9 / hbm_peak, 4)}
    del kc, reps, ka, va, qa, out
    # prefill: the 32K needle prefill's HISA indices
    nq = w3.total_q
    ka, va = rnd((w3.k.shape[0], D)), rnd((w3.k.shape[0], D))
    qa = rnd((nq * heads, D)).view(nq, heads, D)
    out = torch.empty(nq, heads, D, dtype=torch.float32, device="cuda")
    cq, ck = to_dev_i32(w3.cu_q), to_dev_i32(w3.cu_k)
    fn = lambda: H.hisa_sparse_attention(qa, ka, va, o3, cq, ck, scale, out=out)
    fn()
    ms = statistics.median(time_events(fn, 3, flush, stream))
    valid = int((o3 >= 0).sum().item())
    flop = 2.0 * 2.0 * heads * D * valid
    res["prefill_32k"] = {"heads": heads, "k": w3.topk, "ms": round(ms, 3),
                          "queries_per_s": round(nq / (ms / 1e3), 1),
                          "TFLOPs": round(flop / (ms / 1e3) / 1e12, 2),
                          "flop": "2*2*heads*128 per valid selected token (q.k and p.v)",
                          "frac_of_bf16_tensor_peak": round(flop / (ms / 1e3) / 1e12 / tc_peak, 4)}
    del ka, va, qa, out
    torch.cuda.empty_cache()
    return res


def bf16_rows(rng, shape):
    from synth import bf16_from_f32
    return bf16_from_f32(rng.standard_normal(shape, dtype=np.float32))


def _time_oracle(fn):
    t0 = time.perf_counter()
    fn()
    return time.perf_counter() - t0


def cpu_baseline(w, budget_s: float = 15.0):
    """The oracle (unchanged) on the host cores: a seeded sample of query rows of the
    benchmark workload (the line's value), the HISA oracle timed in full on every
    configuration, and the flat-DSA oracle in full on the 4K and 32K prefills and on 4096
    seeded rows of the 128K and varlen ones (its cost grows with the square of the
    length)."""
    import oracle
    from synth import config_workload
    n = cores()
    rng = np.random.Generator(np.random.PCG64(99))
    rows = np.sort(rng.choice(w.total_q, 512, replace=False)).astype(np.int32)
    t1 = _time_oracle(lambda: oracle.hisa_workload(w, rows=rows, nthreads=n))
    target = int(min(w.total_q, max(512, 512 * budget_s / max(t1, 1e-3))))
    rows = np.sort(rng.choice(w.total_q, target, replace=False)).astype(np.int32)
    t1 = _time_oracle(lambda: oracle.hisa_workload(w, rows=rows, nthreads=n))
    per = {}

    def entry(nrows, secs, full):
        return {"rows": int(nrows), "seconds": round(secs, 3),
                "queries_per_s": round(nrows / secs, 1), "sample": "all rows" if full else
                "4096 seeded rows"}
    for cfg in (1, 3, 4, 5):
        wc = w if cfg == 4 else config_workload(cfg)
        full = wc.total_q <= 32768
        r = None if full else np.sort(np.random.Generator(np.random.PCG64(cfg)).choice(
            wc.total_q, 4096, replace=False)).astype(np.int32)
        nr = wc.total_q if full else 4096
        per[str(cfg)] = {
            "hisa": entry(wc.total_q,
                          _time_oracle(lambda: oracle.hisa_workload(wc, nthreads=n)), True),
            "dsa": entry(nr, _time_oracle(lambda: oracle.dsa_workload(wc, rows=r, nthreads=n)),
                         full)}
    # decode: one step (append then select) of the 16 sequences, through the oracle's
    # pooling of the whole caches
    dw = config_workload(2, steps=1)
    S = dw.num_seqs
    kc = dw.k_cache.copy()
    lens = dw.seqlens0.copy()
    for s in range(S):
        kc[int(dw.cu_k[s]) + int(lens[s])] = dw.new_keys[0, s, 0]
    lens = lens + 1
    cu_q = np.arange(S + 1, dtype=np.int32)
    per["2"] = {
        "hisa": entry(S, _time_oracle(lambda: oracle.hisa(dw.queries[0], kc, cu_q, dw.cu_k, lens,
                                                          dw.B, dw.m, dw.topk, nthreads=n)),
                      True),
        "dsa": entry(S, _time_oracle(lambda: oracle.dsa(dw.queries[0], kc, cu_q, dw.cu_k, lens,
                                                        dw.topk, nthreads=n)), True)}
    return {"value": round(target / t1, 2), "unit": UNIT, "cores": n, "kind": "oracle",
            "sample": f"{target} seeded query rows of the {w.total_q} (pooling over all keys each "
                      "call)", "seconds": round(t1, 2), "per_config": per}


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle

def run_reference(args, world, rank):
    if rank != 0:
        return None
    import oracle
    from synth import config_workload
    w = config_workload(4)
    n = cores()
    rng = np.random.Generator(np.random.PCG64(7))
    sample = 4096
    times = []
    for i in range(args.warmup + args.steps):
        rows = np.sort(rng.choice(w.total_q, sample, replace=False)).astype(np.int32)
        t0 = time.perf_counter()
        oracle.hisa_workload(w, rows=rows, nthreads=n)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    v = sample / (ms / 1e3)
    return {"impl": "reference", "metric": METRIC, "value": round(v, 2), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "seq_len": 131072, "d": 64, "B": 128, "m": 64,
                       "k": 2048, "sample_rows_per_step": sample},
            "cpu_baseline": {"value": round(v, 2), "unit": UNIT, "cores": n, "kind": "oracle",
                             "sample": f"{sample} seeded query rows of the 131072 per step"},
            "e2e": {"value": round(v, 2), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def decode_profile(steps):
    """Eager decode steps for a profiler: the decode workload of decode_bench, one state."""
    import torch
    import sparse_attention_top_hisa_b200 as H
    from synth import config_workload
    dw = config_workload(2, steps=steps)
    S, cap, m, K = dw.num_seqs, dw.capacity, dw.m, dw.topk
    cu_k, cu_q = to_dev_i32(dw.cu_k), to_dev_i32(np.arange(S + 1))
    kc, lens = to_dev_bf16(dw.k_cache), to_dev_i32(dw.seqlens0)
    reps = H.hisa_pool_blocks(kc, cu_k, lens, cap)
    out = torch.empty(S, K, dtype=torch.int32, device="cuda")
    newk = to_dev_bf16(dw.new_keys)
    qs = to_dev_bf16(dw.queries.reshape(steps * S, 64)).view(steps, S, 64)
    for i in range(steps):  # the fused step the decode benchmark times
        H.hisa_decode_step(kc, reps, cu_k, lens, newk[i].reshape(S, 64), qs[i], cap, m, K,
                           out_idx=out)
    # then the attention step over the last selection (16 heads, width 128)
    rng = np.random.Generator(np.random.PCG64(31))
    ka = to_dev_bf16(bf16_rows(rng, (S * cap, 128)))
    va = to_dev_bf16(bf16_rows(rng, (S * cap, 128)))
    qa = to_dev_bf16(bf16_rows(rng, (S * 16, 128))).view(S, 16, 128)
    for _ in range(2):
        H.hisa_sparse_attention(qa, ka, va, out, cu_q, cu_k, 1.0 / np.sqrt(128))
    torch.cuda.synchronize()
    assert H.hisa_device_status() == 0


def main():
    args = parse_args()
    if args.decode_profile > 0:
        dist_setup(args)
        decode_profile(args.decode_profile)
        return
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    world, rank, _ = dist_setup(args)
    line = run_ours(args, world, rank)
    if rank == 0:
        d = line["details"]
        if "dsa_128k" in d:
            d["dsa_128k"]["hisa_speedup_over_dsa"] = round(d["dsa_128k"]["ms"] / line["ms_per_step"], 2)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
