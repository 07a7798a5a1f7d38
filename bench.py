#!/usr/bin/env python
"""Benchmark of content-routed block-sparse attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ssa|reference]

A step is one pass of the whole path (K/Q block summaries, routing, fused
attend) over one batch of the synthetic workload, inputs resident in HBM.
Default workload: the long GQA clustered-key prefill (1 x 14/2 heads,
N = 1,048,576, D = 64, Bk = Bq = 64, top-k 16, W = 1024), the largest
workload that fits one GPU; --config 2 is the 32K-token prefill.  Prints one
JSON line on rank 0.

* value     whole-job prefill tokens/s (device time, CUDA events per step,
            L2 flushed between steps by a 256 MiB write outside the events)
* e2e       the same metric through the public host-memory call
            (ssa.forward_host: pinned Q, K, V streamed to the device per KV
            group and query head on two copy streams, one ssa_forward per
            query head, O streamed back; all copies inside the timed region)
* roofline  the attend kernel: algorithmic gathered bytes (distinct routed +
            window key blocks of every query block, K and V, plus the Q read
            and O / LSE writes) per launch / its event-timed duration, against
            the measured HBM copy bandwidth
* ceilings  secondary ceilings of the attend kernel: the measured
            ex2.approx rate (exponentials of the softmax), the compulsory bytes
            (Q, K, V read once, O and LSE written once), the bf16 tensor peak
* warm_l2   the same step without the L2 flush between steps
* cpu_baseline  the float64 oracle on the host cores over a bounded sample

With --gpus N > 1 (torchrun) every rank runs an independent replica of the
workload (the path shards into independent problems; there is no exchange
step), the per-step time is the max over ranks, and value sums all ranks.
--impl reference times the oracle instead (host cores, bounded samples).
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse-attn prefill tokens/s; selected-key TFLOP/s as % of B200 roofline"
UNIT = "tokens/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attend_traffic.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=5, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--impl", default="ssa", choices=["ssa", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--seq-len", type=int, default=0,
                    help="run the chosen workload's recipe at another sequence length "
                         "(e.g. a smaller copy of the million-token workload for profiling)")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward of the read (lists held fixed) instead of the forward")
    ap.add_argument("--decode", action="store_true",
                    help="time one decode step (a query per head at the last position of the "
                         "workload's full K/V cache) instead of the prefill")
    ap.add_argument("--beta", type=float, default=0.0,
                    help="weight of the second-cumulant routing term (0: mean summaries only)")
    ap.add_argument("--tree-fanout", type=int, default=0,
                    help="two-level (fixed-beam tree) routing: key blocks per super-block")
    ap.add_argument("--tree-beam", type=int, default=0,
                    help="two-level routing: super-blocks kept per query block (default top_k)")
    ap.add_argument("--consensus", action="store_true",
                    help="GQA-shared consensus routing: the query heads of a KV group vote "
                         "and share one list per query block")
    return ap.parse_args(argv)


def load_peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    """Hash of the attend kernel's sources with comments and blank space
    removed: the stored DRAM counters stay valid while only comments change."""
    h = hashlib.sha256()
    for f in ("attend.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "content_routed_block_b200", "csrc", f)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        src = "\n".join(line.strip() for line in src.splitlines() if line.strip())
        h.update(src.encode())
    return h.hexdigest()[:16]


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.samples = []
        self.proc = None
        self.thread = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", self.gpu_id, "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def mark(self, which):
        if which == "start":
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        for t, line in self.samples:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) != 7:
                continue
            rows.append((t, parts))
        inside = [r for r in rows if self.t0 is not None and self.t0 <= r[0] <= (self.t1 or 1e30)]
        use = inside if inside else rows
        sm = [float(p[0]) for _, p in use if p[0].replace(".", "").isdigit()]
        smax = [float(p[1]) for _, p in use if p[1].replace(".", "").isdigit()]
        reasons = sorted({self.NAMES[i] for _, p in use for i in range(4) if p[3 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(use), "in_timed_region": bool(inside)}


# ----------------------------------------------------------------------------
# algorithmic work of one forward (from the routed lists)
# ----------------------------------------------------------------------------
# ----------------------------------------------------------------------------
# replicas over ranks: every rank runs the whole workload on its own GPU
# ----------------------------------------------------------------------------
def max_over_ranks(x: float, world: int, dev) -> float:
    """The largest of every rank's ``x`` (a per-step time): the job is as
    slow as its slowest replica.  ``dev`` is the device of the process
    group's backend (a CUDA device under NCCL, the CPU under gloo)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(tokens_per_rank: int, world: int, ms: float):
    """Whole-job tokens per step and tokens/s when each of ``world`` ranks
    processes ``tokens_per_rank`` tokens per step and the step takes ``ms``
    (the max over ranks): weak scaling, no exchange between replicas."""
    tokens = tokens_per_rank * world
    return tokens, tokens / (ms * 1e-3)


def algorithmic_work(w, idx, cnt):
    """Mean distinct keys per query (|S_i|), selected-key flops, and the attend
    kernel's algorithmic bytes: per routed list (a query block of a query head;
    of a KV group with consensus routing, where the group's heads share the
    keys), the distinct key blocks it needs (routed U window) x Bk rows x K and
    V, plus the Q read and the O and LSE writes."""
    import numpy as np
    B, Hq, N, D, Bk, Bq, W = w.B, w.Hq, w.N, w.D, w.block_k, w.block_q, w.window
    g = w.Hq // w.Hkv
    cons = bool(getattr(w, "consensus", False))
    nqb = N // Bq
    qb = np.arange(nqb)
    k = w.top_k
    keys_total = 0.0
    blocks_total = 0
    for b in range(B):
        for h in range(Hq):
            lh = h // g if cons else h             # the list this head reads
            count_blocks = (not cons) or h % g == 0
            sel = idx[b, lh] if k > 0 else np.zeros((nqb, 0), np.int64)
            valid = (np.arange(k)[None, :] < cnt[b, lh][:, None]) if k > 0 else sel.astype(bool)
            if not w.causal:
                keys_total += float(cnt[b, lh].sum()) * Bk * Bq
                blocks_total += int(cnt[b, lh].sum()) if count_blocks else 0
                continue
            # rows i of block qb: i = qb*Bq + r
            r = np.arange(Bq)
            i = qb[:, None] * Bq + r[None, :]                           # [nqb, Bq]
            win = np.minimum(W, i + 1)                                 # window keys
            lo = np.maximum(0, i - W + 1)                              # first window key
            c0 = sel.astype(np.int64) * Bk                             # [nqb, k]
            c1 = c0 + Bk - 1
            # overlap of routed block [c0, c1] with window [lo, i] (routed blocks end before i)
            ov = np.clip(c1[:, None, :] - np.maximum(c0[:, None, :], lo[:, :, None]) + 1, 0, Bk)
            ov = np.where(valid[:, None, :], ov, 0)
            routed = np.where(valid, Bk, 0).sum(axis=1)[:, None]        # [nqb, 1]
            keys_total += float((win + routed - ov.sum(axis=2)).sum())
            # distinct key blocks per query block: routed U window blocks
            wlo = np.maximum(0, qb * Bq - W + 1) // Bk
            whi = (qb * Bq + Bq - 1) // Bk
            in_win = (sel >= wlo[:, None]) & (sel <= whi[:, None]) & valid
            if count_blocks:
                blocks_total += int(((whi - wlo + 1) + valid.sum(axis=1) - in_win.sum(axis=1)).sum())
    kpq = keys_total / (B * Hq * N)
    flops = 4.0 * B * Hq * N * kpq * D
    gathered = blocks_total * Bk * 2 * D * 2
    io = B * Hq * N * D * 2 * 2 + B * Hq * N * 4
    return {"keys_per_query": kpq, "flops": flops, "gathered_bytes": gathered,
            "attend_bytes": gathered + io, "nominal_keys_per_query": k * Bk + W}


# ----------------------------------------------------------------------------
# oracle on the host cores (cpu_baseline and the reference arm)
# ----------------------------------------------------------------------------
def _cpu_worker(args):
    os.environ.setdefault("OMP_NUM_THREADS", "1")
    import numpy as np
    sys.path.insert(0, ROOT)
    import oracle as O
    from content_routed_block_b200.workloads import CONFIGS, make_inputs
    cfg, seq_len, consensus, beta, tree, b, h, blocks, seconds = args
    w = CONFIGS[cfg]
    if seq_len:
        w = w.with_(N=seq_len)
    g = w.Hq // w.Hkv
    # the unit of work: one query block of one query head, or (consensus) of
    # every head of the KV group, which vote on one shared list
    heads = list(range((h // g) * g, (h // g + 1) * g)) if consensus else [h]
    x = make_inputs(w, q_heads=heads, kv_heads=[h // g])
    sub = w.with_(Hq=len(heads), Hkv=1, B=1, consensus=consensus, beta=beta,
                  tree_fanout=tree[0], tree_beam=tree[1])
    p = O.Params.of(sub)
    q = O.upcast_bf16(x["q"][b:b + 1])           # the requested heads, in order
    k = O.upcast_bf16(x["k"][b:b + 1])
    v = O.upcast_bf16(x["v"][b:b + 1])
    # masked-dense read up to 32K tokens; beyond, the block-gathered form of
    # the same read (its [Bq, N] slab would be 512 MB per block at 1M tokens)
    attend = O.attend_masked_dense if w.N <= 32768 else O.attend_gathered_blocks
    t0 = time.perf_counter()
    ksum = O.block_summary(k, p.block_k)
    kcov = O.block_covariance(k[0, 0], p.block_k) if p.beta else None
    ksum2 = O.tree_summary(k, p.block_k, p.tree_fanout) if p.tree_fanout else None
    done = 0
    nh = len(heads)
    idx = np.full((1, nh, p.n_qblocks, p.top_k), -1, np.int32)
    cnt = np.zeros((1, nh, p.n_qblocks), np.int32)
    for qb in blocks:
        for j in range(nh):
            rows = q[:, j:j + 1, qb * p.block_q:(qb + 1) * p.block_q]
            qbar = O.block_summary(rows, p.block_q)[0, 0, 0]
            extra = {}
            if p.beta:
                extra = dict(beta=p.beta, q2=O.block_second_moment(rows, p.block_q)[0, 0, 0],
                             sigma=kcov)
            if p.tree_fanout:
                _, sel, _, _ = O.route_tree_row(qbar, ksum[0, 0], ksum2[0, 0],
                                                len(O.admissible_blocks(qb, p)), p)
            else:
                sel, _, _ = O.route_row(qbar, ksum[0, 0], O.admissible_blocks(qb, p), p.top_k,
                                        **extra)
            idx[0, j, qb, :len(sel)] = sel
            cnt[0, j, qb] = len(sel)
        if consensus:
            shared = O.consensus_row([idx[0, j, qb, :cnt[0, j, qb]] for j in range(nh)], p.top_k)
            idx[0, :, qb] = -1
            idx[0, :, qb, :len(shared)] = shared
            cnt[0, :, qb] = len(shared)
        attend(q, k, v, idx, cnt, p, blocks=[(0, j, qb) for j in range(nh)])
        done += nh
        if time.perf_counter() - t0 > seconds:
            break
    return done, time.perf_counter() - t0


class OraclePool:
    def __init__(self, cfg: int, seq_len: int = 0, consensus: bool = False, beta: float = 0.0,
                 tree=(0, 0)):
        import multiprocessing as mp
        self.cfg = cfg
        self.seq_len = seq_len
        self.consensus = consensus
        self.beta = beta
        self.tree = tuple(tree)
        self.cores = max(1, min(len(os.sched_getaffinity(0)), 64))
        old = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
        for k in old:
            os.environ[k] = "1"
        self.pool = mp.get_context("spawn").Pool(self.cores)
        for k, v in old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
        self.step = 0

    def run(self, seconds: float):
        """Each worker runs the oracle's whole path for seconds on its own
        (b, head) and a spread of query blocks; returns (tokens/s, (head,
        query block) units done, wall seconds).  One unit is 1/Hq of the work
        of Bq tokens (tokens/s counts positions over all heads), so
        tokens/s = units * Bq / Hq / wall."""
        import numpy as np
        from content_routed_block_b200.workloads import CONFIGS
        w = CONFIGS[self.cfg]
        if self.seq_len:
            w = w.with_(N=self.seq_len)
        nqb = w.N // w.block_q
        tasks = []
        rng = np.random.default_rng(self.step)
        self.step += 1
        for c in range(self.cores):
            b = c % w.B
            h = (c // w.B) % w.Hq
            blocks = rng.permutation(nqb).tolist()
            tasks.append((self.cfg, self.seq_len, self.consensus, self.beta, self.tree, b, h,
                          blocks, seconds))
        res = self.pool.map(_cpu_worker, tasks)
        blocks = sum(r[0] for r in res)
        wall = max(r[1] for r in res)
        return blocks * w.block_q / w.Hq / wall, blocks, wall

    def close(self):
        self.pool.terminate()


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = workload_of(args)
    per_step = max(0.5, min(5.0, 150.0 / max(1, args.steps + args.warmup)))
    pool = OraclePool(args.config, args.seq_len, args.consensus, args.beta, tree_of(w))
    try:
        for _ in range(args.warmup):
            pool.run(per_step)
        vals, blocks = [], 0
        t0 = time.time()
        for _ in range(args.steps):
            v, nb, _ = pool.run(per_step)
            vals.append(v)
            blocks += nb
        wall = time.time() - t0
    finally:
        pool.close()
    value = statistics.mean(vals)
    sample = (f"{blocks} (query head, query block) units of this workload over {args.steps} "
              f"steps, ~{per_step:.1f} s of oracle work per core per step; one unit is 1/Hq of "
              f"the work of {w.block_q} tokens")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * wall / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": pool.cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_of(args):
    from content_routed_block_b200.workloads import CONFIGS
    w = CONFIGS[args.config]
    if args.seq_len:
        w = w.with_(N=args.seq_len, name=f"{w.name}@{args.seq_len}")
    if getattr(args, "consensus", False):
        w = w.with_(consensus=True, name=f"{w.name}+consensus")
    if getattr(args, "beta", 0.0):
        w = w.with_(beta=float(args.beta), name=f"{w.name}+beta{args.beta:g}")
    if getattr(args, "tree_fanout", 0):
        beam = args.tree_beam or w.top_k
        w = w.with_(tree_fanout=args.tree_fanout, tree_beam=beam,
                    name=f"{w.name}+tree{args.tree_fanout}x{beam}")
    return w


def tree_of(w):
    return (int(getattr(w, "tree_fanout", 0)), int(getattr(w, "tree_beam", 0)))


def workload_config(w, args):
    return {"workload": f"{w.name}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} N={w.N} D={w.D} "
                        f"Bk={w.block_k} Bq={w.block_q} top_k={w.top_k} W={w.window} "
                        f"{'causal' if w.causal else 'non-causal'} {w.kind}"
                        f"{' consensus-routed' if w.consensus else ''}"
                        f"{f' second-cumulant beta={w.beta:g}' if w.beta else ''}"
                        f"{f' two-level routing fanout={w.tree_fanout} beam={w.tree_beam}' if w.tree_fanout else ''}",
            "global_batch": w.B * args.gpus, "seq_len": w.N, "parallelism": f"replicas{args.gpus}",
            "l2": "flushed between timed steps (256 MiB write)"}


# ----------------------------------------------------------------------------
# the CUDA path
# ----------------------------------------------------------------------------
def run_ssa(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    from content_routed_block_b200 import build, ssa
    from content_routed_block_b200.workloads import CONFIGS, make_inputs

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    ssa.lib()

    w = workload_of(args)
    p = ssa.params_of(w)
    x = make_inputs(w)
    host = {n: torch.from_numpy(x[n].view(np.int16)).view(torch.bfloat16) for n in "qkv"}
    qd, kd, vd = (host[n].to(dev) for n in "qkv")
    ws = torch.empty(ssa.workspace_size(p), dtype=torch.uint8, device=dev)
    o = torch.empty_like(qd)
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
    LH = w.Hkv if w.consensus else w.Hq          # heads the attended lists span
    idx = torch.empty((w.B, LH, w.N // w.block_q, w.top_k), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.B, LH, w.N // w.block_q), dtype=torch.int32, device=dev)
    idx_h = torch.empty((w.B, w.Hq, w.N // w.block_q, w.top_k), dtype=torch.int32, device=dev)
    cnt_h = torch.empty((w.B, w.Hq, w.N // w.block_q), dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        ssa.forward(qd, kd, vd, p, workspace=ws, out=o, lse_out=lse, idx_out=idx, cnt_out=cnt)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    ssa.check_error()

    props = torch.cuda.get_device_properties(dev)
    gpu_id = str(getattr(props, "uuid", "")) or str(local)
    if gpu_id and not gpu_id.startswith("GPU-") and len(gpu_id) > 8:
        gpu_id = "GPU-" + gpu_id
    sampler = ClockSampler(gpu_id)
    sampler.start()
    time.sleep(0.3)

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.mark("start")
    for s in range(args.steps):
        flush.zero_()
        starts[s].record()
        step()
        ends[s].record()
    torch.cuda.synchronize()
    sampler.mark("end")
    if world > 1:
        dist.barrier()
    sampler.stop()
    ssa.check_error()
    times = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    ms = max_over_ranks(statistics.mean(times), world, dev)
    tokens, value = replica_throughput(w.B * w.N, world, ms)

    # per-kernel split: the same path as separate calls with events between them
    n_split = min(args.steps, 200)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(n_split)]
    F = w.D + w.D * (w.D + 1) // 2 if w.beta else w.D      # summary / feature length
    ks = torch.empty((w.B, w.Hkv, w.N // w.block_k, F), dtype=torch.float32, device=dev)
    qs = torch.empty((w.B, w.Hq, w.N // w.block_q, F), dtype=torch.float32, device=dev)
    sc = (torch.empty((w.B, w.Hq, w.N // w.block_q, w.N // w.block_k), dtype=torch.float32,
                      device=dev) if w.beta else None)
    tree = w.tree_fanout > 0
    if tree:
        ks2 = torch.empty((w.B, w.Hkv, (w.N // w.block_k) // w.tree_fanout, w.D),
                          dtype=torch.float32, device=dev)
        sup = torch.empty((w.B, w.Hq, w.N // w.block_q, w.tree_beam), dtype=torch.int32,
                          device=dev)
        supc = torch.empty((w.B, w.Hq, w.N // w.block_q), dtype=torch.int32, device=dev)
    L = ssa.lib()
    import ctypes
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    pp = ctypes.byref(p)
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    rws_n = int(L.ssa_route_workspace_size(pp))         # the router's pre-split key image
    rws = torch.empty(max(rws_n, 256), dtype=torch.uint8, device=dev)
    for s in range(n_split):
        flush.zero_()
        e = ev[s]
        e[0].record()
        if w.beta:
            assert L.ssa_route_features(pp, P(kd), w.Hkv, w.block_k, 0, P(ks), st) == 0
            e[1].record()
            assert L.ssa_route_features(pp, P(qd), w.Hq, w.block_q, 1, P(qs), st) == 0
        else:
            assert L.ssa_block_summary(pp, P(kd), w.Hkv, w.block_k, P(ks), st) == 0
            e[1].record()
            assert L.ssa_block_summary(pp, P(qd), w.Hq, w.block_q, P(qs), st) == 0
        e[2].record()
        if tree:
            assert L.ssa_tree_summary(pp, P(ks), P(ks2), st) == 0
        e[3].record()
        ri, rc = (idx_h, cnt_h) if w.consensus else (idx, cnt)
        if w.beta:
            assert L.ssa_route_cumulant(pp, P(qs), P(ks), P(sc), P(ri) if w.top_k else None,
                                        P(rc), st) == 0
        elif tree:
            assert L.ssa_route_tree(pp, P(qs), P(ks), P(ks2), P(sup), P(supc),
                                    P(ri) if w.top_k else None, P(rc), st) == 0
        else:
            assert L.ssa_route_with_workspace(pp, P(qs), P(ks), P(ri) if w.top_k else None, P(rc),
                                              P(rws), rws_n, st) == 0
        e[4].record()
        if w.consensus:
            assert L.ssa_route_consensus(pp, P(idx_h) if w.top_k else None, P(cnt_h),
                                         P(idx) if w.top_k else None, P(cnt), st) == 0
        e[5].record()
        assert L.ssa_attend(pp, P(qd), P(kd), P(vd), P(idx) if w.top_k else None, P(cnt),
                            P(o), P(lse), st) == 0
        e[6].record()
    torch.cuda.synchronize()
    ssa.check_error()
    seg = lambda i: statistics.mean(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(n_split))  # noqa: E731
    pool_k_ms, pool_q_ms, tree_pool_ms = seg(0), seg(1), seg(2)
    route_ms, cons_ms, attend_ms = seg(3), seg(4), seg(5)

    # the same step without the L2 flush (inputs and lists may stay in L2)
    n_warm = min(args.steps, 100)
    wev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n_warm)]
    for _ in range(3):
        step()
    for a, z in wev:
        a.record()
        step()
        z.record()
    torch.cuda.synchronize()
    warm_ms = max_over_ranks(statistics.mean(a.elapsed_time(z) for a, z in wev), world, dev)
    ssa.check_error()

    # exponential rate of the softmax's ex2.approx on this GPU (a ceiling of
    # the attend kernel): 8 CTAs of 256 threads per SM, 8 chains per thread
    sink = torch.zeros(1, dtype=torch.float32, device=dev)
    n_sm = props.multi_processor_count
    ex2_ctas, ex2_iters = 8 * n_sm, 4096
    for _ in range(2):
        ssa.probe_ex2_rate(ex2_ctas, ex2_iters, sink)
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record()
    for _ in range(5):
        ssa.probe_ex2_rate(ex2_ctas, ex2_iters, sink)
    x1.record()
    torch.cuda.synchronize()
    ssa.check_error()
    ex2_rate = 5 * ex2_ctas * 256 * ex2_iters * 8 / (x0.elapsed_time(x1) * 1e-3)
    # two-level routing: share of the flat route's per-head selections that
    # the tree route also selects, on the same summaries (outside the timing)
    tree_recall = None
    if tree and w.top_k:
        flat_p = ssa.params_of(w, tree_fanout=0, tree_beam=0, consensus=False)
        fi, fc = ssa.route(qs, ks, flat_p)
        ti = (idx_h if w.consensus else idx).cpu().numpy().reshape(-1, w.top_k)
        fi = fi.cpu().numpy().reshape(-1, w.top_k)
        hit = ((fi[:, :, None] == ti[:, None, :]) & (fi[:, :, None] >= 0)).any(axis=2)
        tree_recall = float(hit.sum() / max(1, int(fc.sum().item())))

    work = algorithmic_work(w, idx.cpu().numpy(), cnt.cpu().numpy())
    peaks, peak_kind = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    tensor = float(peaks["bf16_tflops"])
    tflops = work["flops"] / (ms * 1e-3) / 1e12
    attend_tflops = work["flops"] / (attend_ms * 1e-3) / 1e12
    t_hbm = work["attend_bytes"] / (hbm * 1e9)
    t_tensor = work["flops"] / (tensor * 1e12)
    t_roof = max(t_hbm, t_tensor)
    # the attend kernel's binding roof: gathered bytes over HBM (per-head
    # lists, ~64 flop/B), or bf16 flops over the tensor peak (consensus lists
    # shared by g heads raise the intensity g-fold, past the B200 ridge)
    if t_hbm >= t_tensor:
        roof = {"bound": "hbm", "achieved": work["attend_bytes"] / (attend_ms * 1e-3) / 1e9,
                "peak": hbm, "unit": "GB/s", "peak_source": f"{peak_kind} hbm_gbs"}
    else:
        roof = {"bound": "tensor", "achieved": attend_tflops, "peak": tensor, "unit": "TFLOP/s",
                "peak_source": f"{peak_kind} bf16_tflops (burst)"}
    traffic, ncu = None, None
    if os.path.exists(TRAFFIC_FILE):
        with open(TRAFFIC_FILE) as f:
            tr = json.load(f)
        if tr.get("kernel_hash") == kernel_source_hash():
            key = (f"{args.config}{'c' if w.consensus else ''}{'t' if tree else ''}"
                   + (f"@{args.seq_len}" if args.seq_len else ""))
            traffic = tr.get("bytes_per_launch", {}).get(key)
            ncu = tr.get("pipes", {}).get(key)
    # secondary ceilings of the attend kernel: exponentials (one per key a
    # query reads) at the measured ex2 rate, the compulsory bytes (Q, K, V
    # read once; O and LSE written once) over HBM, and the bf16 tensor peak
    exps = w.B * w.Hq * w.N * work["keys_per_query"]
    compulsory = (w.B * w.Hq * w.N * w.D * 2 * 2 + 2 * w.B * w.Hkv * w.N * w.D * 2
                  + w.B * w.Hq * w.N * 4)
    ceilings = {
        "exp": {"exps_per_launch": exps, "measured_ex2_per_s": ex2_rate,
                "ms": exps / ex2_rate * 1e3, "frac": exps / ex2_rate * 1e3 / attend_ms},
        "compulsory_bytes": {"bytes_per_launch": compulsory, "ms": compulsory / (hbm * 1e9) * 1e3,
                             "frac": compulsory / (hbm * 1e9) * 1e3 / attend_ms},
        "tensor": {"flops_per_launch": work["flops"], "ms": t_tensor * 1e3,
                   "frac": t_tensor * 1e3 / attend_ms},
        "gathered_bytes": {"bytes_per_launch": work["attend_bytes"], "ms": t_hbm * 1e3,
                           "frac": t_hbm * 1e3 / attend_ms},
    }

    # end to end through the public call, from pinned host memory
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = (host[n].pin_memory() for n in "qkv")
        oh = torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory()
        bufs = {"q": qd, "k": kd, "v": vd, "o": o}
        n_e2e = min(args.steps, 100)
        for _ in range(3):
            ssa.forward_host(qh, kh, vh, p, oh, device=dev, dev_bufs=bufs)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n_e2e):
            ssa.forward_host(qh, kh, vh, p, oh, device=dev, dev_bufs=bufs)
        e1.record()
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, world, dev)
        h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
        e2e = {"value": tokens / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": oh.numel() * oh.element_size(), "ms_per_step": e2e_ms,
               "call": "ssa.forward_host: per-head streamed call (each KV group's K, V and "
                       "each query head's Q copied from pinned host memory on a copy stream, "
                       "one ssa_forward per query head as its inputs land, O copied back on a "
                       "second copy stream)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        pool = OraclePool(args.config, args.seq_len, args.consensus, args.beta, tree_of(w))
        try:
            v, nb, wall = pool.run(args.cpu_seconds)
        finally:
            pool.close()
        cpu = {"value": v, "unit": UNIT, "cores": pool.cores, "kind": "oracle",
               "sample": f"{nb} (query head, query block) units of this workload (each 1/Hq of "
                         f"the work of {w.block_q} tokens), whole path (summaries, routing"
                         f"{', consensus' if w.consensus else ''}"
                         f"{', second-cumulant scores' if w.beta else ''}, "
                         f"{'masked-dense' if w.N <= 32768 else 'block-gathered'} attend) in "
                         f"float64, {pool.cores} processes x ~{args.cpu_seconds:.0f} s"}

    clocks = sampler.summary()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "impl": "ssa",
        "config": workload_config(w, args),
        "selected_tflops": tflops,
        "keys_per_query": work["keys_per_query"],
        "nominal_keys_per_query": work["nominal_keys_per_query"],
        "kernels_ms": {("features_k" if w.beta else "pool_k"): pool_k_ms,
                       ("features_q" if w.beta else "pool_q"): pool_q_ms,
                       **({"tree_pool": tree_pool_ms} if tree else {}), "route": route_ms,
                       **({"consensus": cons_ms} if w.consensus else {}), "attend": attend_ms},
        **({"tree_recall_of_flat_route": tree_recall} if tree else {}),
        "roofline": {"bound": roof["bound"], "kernel": "attend_kernel",
                     "achieved": roof["achieved"], "peak": roof["peak"], "unit": roof["unit"],
                     "frac": roof["achieved"] / roof["peak"], "traffic": traffic,
                     "peak_source": roof["peak_source"],
                     "frac_basis": ("algorithmic gathered bytes (distinct routed and window key "
                                    "blocks of every routed list x Bk rows x K and V, plus the "
                                    "Q read and O/LSE writes) over the attend kernel's event "
                                    "time, against the measured HBM copy bandwidth; most of "
                                    "these bytes are served from L2, see dram_frac"
                                    if roof["bound"] == "hbm" else
                                    "selected-key bf16 flops over the attend kernel's event "
                                    "time, against the measured bf16 burst peak"),
                     "dram_frac": (traffic / (attend_ms * 1e-3) / 1e9 / hbm
                                   if traffic else None),
                     "ncu_pipes": ncu,
                     "bytes_per_launch": work["attend_bytes"],
                     "hbm_frac": work["attend_bytes"] / (attend_ms * 1e-3) / 1e9 / hbm,
                     "attend_tflops": attend_tflops,
                     "attend_tensor_frac": attend_tflops / float(peaks["bf16_tflops"]),
                     "path_frac_of_roofline": t_roof / (ms * 1e-3)},
        "ceilings": ceilings,
        "warm_l2": {"ms_per_step": warm_ms, "value": tokens / (warm_ms * 1e-3),
                    "note": "same step, no L2 flush between steps"},
        "cpu_baseline": cpu,
        "e2e": e2e,
        # per forward: pool (K and Q in one launch) + route + attend; with
        # beta: two feature launches + scores + select + attend; two-level:
        # pool + super-block pool + upper route + select + attend; +1 consensus
        "gpu_launches": ((5 if (w.beta or tree) else 3) + (1 if w.consensus else 0)
                         + (1 if (rws_n and not tree and not w.beta) else 0)) * args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# decode: one query per head at the end of the cache
# ----------------------------------------------------------------------------
def decode_work(w, cnt_sel, idx_sel):
    """Algorithmic bytes of one decode step: the block means the router reads
    (B * Hkv * nb * D * 4) and, per query head, the distinct keys it reads
    (routed blocks' keys below the window plus the window) as K and V rows,
    plus q, o and lse.  Also the mean keys per query."""
    i = w.N - 1
    nb = i // w.block_k
    lo = max(0, i - w.window + 1)
    keys = 0
    for b in range(w.B):
        for h in range(w.Hq):
            n = int(cnt_sel[b, h])
            far = 0
            for c in idx_sel[b, h, :n].tolist():
                start = c * w.block_k
                far += max(0, min(start + w.block_k, lo) - start)
            keys += far + (i - lo + 1)
    summaries = w.B * w.Hkv * nb * w.D * 4
    kv = keys * w.D * 2 * 2
    io = w.B * w.Hq * (w.D * 2 * 2 + 4)
    return {"bytes": summaries + kv + io, "keys_per_query": keys / (w.B * w.Hq),
            "summary_bytes": summaries, "kv_bytes": kv}


def run_decode(args):
    import numpy as np
    import torch

    from content_routed_block_b200 import build, ssa
    from content_routed_block_b200.workloads import make_inputs

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    w = workload_of(args)
    p = ssa.params_of(w)
    x = make_inputs(w)
    n_ctx = w.N
    qh = torch.from_numpy(np.ascontiguousarray(x["q"][:, :, n_ctx - 1]).view(np.int16)).view(torch.bfloat16)
    kd, vd = (torch.from_numpy(x[n].view(np.int16)).view(torch.bfloat16).to(dev) for n in "kv")
    qd = qh.to(dev)
    ksum0 = ssa.block_summary(kd, w.block_k, p)
    ksum = ksum0.clone()
    ws = torch.empty(ssa.decode_workspace_size(p), dtype=torch.uint8, device=dev)
    o = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        return ssa.decode(qd, kd, vd, n_ctx, ksum, p, workspace=ws, out=o)

    for _ in range(max(3, args.warmup)):
        _, _, idx, cnt = step()
    torch.cuda.synchronize()
    ssa.check_error()
    # A decode step is a few tens of microseconds of GPU work, less than the
    # host needs to issue it through Python; the timed steps replay the step
    # captured as a CUDA graph (one host call each), so the events see the
    # GPU's time.  The e2e line below keeps the host-side call.
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(cap):
        step()
    torch.cuda.current_stream(dev).wait_stream(cap)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph, stream=cap):
        step()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    ssa.check_error()
    props = torch.cuda.get_device_properties(dev)
    gpu_id = str(getattr(props, "uuid", "")) or str(local)
    if gpu_id and not gpu_id.startswith("GPU-") and len(gpu_id) > 8:
        gpu_id = "GPU-" + gpu_id
    sampler = ClockSampler(gpu_id)
    sampler.start()
    time.sleep(0.3)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.mark("start")
    for s_ in range(args.steps):
        flush.zero_()
        starts[s_].record()
        graph.replay()
        ends[s_].record()
    torch.cuda.synchronize()
    sampler.mark("end")
    if world > 1:
        dist.barrier()
    sampler.stop()
    ssa.check_error()
    ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in zip(starts, ends)), world, dev)
    tokens, value = replica_throughput(w.B, world, ms)
    work = decode_work(w, cnt.cpu().numpy(), idx.cpu().numpy())
    peaks, peak_kind = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    achieved = work["bytes"] / (ms * 1e-3) / 1e9

    # end to end: the query from pinned host memory in, O back to pinned host memory
    e2e = None
    if not args.no_e2e:
        qp = qh.pin_memory()
        oh = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16).pin_memory()
        for _ in range(3):
            qd.copy_(qp, non_blocking=True)
            step()
            oh.copy_(o, non_blocking=True)
        torch.cuda.synchronize()
        n_e2e = min(args.steps, 200)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n_e2e):
            qd.copy_(qp, non_blocking=True)
            step()
            oh.copy_(o, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1) / n_e2e
        e2e = {"value": tokens / (e2e_ms * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": qp.numel() * 2, "d2h_bytes_per_step": oh.numel() * 2,
               "ms_per_step": e2e_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle as O
        op = O.Params.of(w)
        q64 = O.upcast_bf16(x["q"][:, :, n_ctx - 1])
        k64, v64 = O.upcast_bf16(x["k"]), O.upcast_bf16(x["v"])
        t0 = time.perf_counter()
        reps = 0
        while True:
            O.decode_step(q64, k64, v64, n_ctx, op)
            reps += 1
            if time.perf_counter() - t0 > args.cpu_seconds:
                break
        wall = time.perf_counter() - t0
        cpu = {"value": reps * w.B / wall, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"{reps} whole decode steps of this workload (block means of the cache, "
                         f"routing and the read of every head) in float64 in one process"}
    clocks = sampler.summary()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    cfg = workload_config(w, args)
    cfg["workload"] = f"decode at n_ctx={n_ctx}: " + cfg["workload"]
    cfg["global_batch"] = w.B * world
    cfg["timing"] = "each timed step is one replay of the step captured as a CUDA graph"
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "impl": "ssa", "config": cfg,
        "keys_per_query": work["keys_per_query"],
        "roofline": {"bound": "hbm", "kernel": "decode (route + attend, merged by the last split)",
                     "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": None, "peak_source": f"{peak_kind} hbm_gbs",
                     "bytes_per_launch": work["bytes"], "summary_bytes": work["summary_bytes"],
                     "kv_bytes": work["kv_bytes"]},
        # per step: routing splits, attend splits (the last split per head merges)
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": 2 * args.steps, "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def run_backward(args):
    """The backward of the read (lists held fixed) after one forward: a step
    is one ssa_attend_backward over the whole workload."""
    import numpy as np
    import torch

    from content_routed_block_b200 import build, ssa
    from content_routed_block_b200.workloads import make_inputs, to_bf16_bits

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    w = workload_of(args)
    p = ssa.params_of(w)
    x = make_inputs(w)
    qd, kd, vd = (torch.from_numpy(x[n].view(np.int16)).view(torch.bfloat16).to(dev) for n in "qkv")
    g16 = to_bf16_bits(np.random.default_rng(w.seed + 1000).standard_normal(
        (w.B, w.Hq, w.N, w.D)).astype(np.float32))
    gh = torch.from_numpy(g16.view(np.int16)).view(torch.bfloat16)
    gd = gh.to(dev)
    o, lse, idx, cnt = ssa.forward(qd, kd, vd, p)
    outs = (torch.empty((w.B, w.Hq, w.N, w.D), dtype=torch.float32, device=dev),
            torch.empty((w.B, w.Hkv, w.N, w.D), dtype=torch.float32, device=dev),
            torch.empty((w.B, w.Hkv, w.N, w.D), dtype=torch.float32, device=dev))
    ws = torch.empty(max(ssa.lib().ssa_backward_workspace_size(__import__("ctypes").byref(p)), 1),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        ssa.backward(qd, kd, vd, o, lse, gd, idx, cnt, p, workspace=ws, out=outs)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    ssa.check_error()
    props = torch.cuda.get_device_properties(dev)
    gpu_id = str(getattr(props, "uuid", "")) or str(local)
    if gpu_id and not gpu_id.startswith("GPU-") and len(gpu_id) > 8:
        gpu_id = "GPU-" + gpu_id
    sampler = ClockSampler(gpu_id)
    sampler.start()
    time.sleep(0.3)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.mark("start")
    for s_ in range(args.steps):
        flush.zero_()
        starts[s_].record()
        step()
        ends[s_].record()
    torch.cuda.synchronize()
    sampler.mark("end")
    if world > 1:
        dist.barrier()
    sampler.stop()
    ssa.check_error()
    ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in zip(starts, ends)), world, dev)
    tokens, value = replica_throughput(w.B * w.N, world, ms)
    work = algorithmic_work(w, idx.cpu().numpy(), cnt.cpu().numpy())
    pairs = work["keys_per_query"] * w.B * w.Hq * w.N
    flops = 10.0 * w.D * pairs            # S, dP, dq, dk, dv: 2 D flops each per (query, key) pair
    achieved = flops / (ms * 1e-3) / 1e12
    simt = os.environ.get("SSA_BWD") == "simt"
    peaks, peak_kind = load_peaks()
    if simt:
        roof = {"bound": "alu", "kernel": "bwd_kernel (CUDA-core fp32 FMA)",
                "peak": 148 * 128 * 2 * 1.965e9 / 1e12,
                "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 flop x 1965 MHz"}
    else:
        roof = {"bound": "tensor", "kernel": "bwd_dq_kernel + bwd_dkdv_kernel (tcgen05)",
                "peak": float(peaks["bf16_tflops"]),
                "peak_source": f"{peak_kind} bf16_tflops (burst)"}

    e2e = None
    if not args.no_e2e:
        gp = gh.pin_memory()
        host_out = [torch.empty(t.shape, dtype=torch.float32).pin_memory() for t in outs]
        for _ in range(3):
            gd.copy_(gp, non_blocking=True)
            step()
            for hh, dd in zip(host_out, outs):
                hh.copy_(dd, non_blocking=True)
        torch.cuda.synchronize()
        n_e2e = min(args.steps, 20)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n_e2e):
            gd.copy_(gp, non_blocking=True)
            step()
            for hh, dd in zip(host_out, outs):
                hh.copy_(dd, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, world, dev)
        e2e = {"value": tokens / (e2e_ms * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": gp.numel() * 2,
               "d2h_bytes_per_step": sum(t.numel() * 4 for t in host_out), "ms_per_step": e2e_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle as O
        op = O.Params.of(w)
        q64, k64, v64 = (O.upcast_bf16(x[n]) for n in "qkv")
        g64 = O.upcast_bf16(g16)
        r = O.route(O.block_summary(q64, w.block_q), O.block_summary(k64, w.block_k), op,
                    rows=[(0, 0, qb) for qb in range(op.n_qblocks)])
        rng = np.random.default_rng(0)
        t0 = time.perf_counter()
        units = 0
        while time.perf_counter() - t0 < args.cpu_seconds:
            qb = int(rng.integers(op.n_qblocks))
            O.attend_backward(q64, k64, v64, g64, r.idx, r.cnt, op, blocks=[(0, 0, qb)])
            units += 1
        wall = time.perf_counter() - t0
        cpu = {"value": units * w.block_q / w.Hq / wall, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"{units} (query head, query block) units of this workload's backward "
                         f"(the oracle's fp64 masked-dense gradients; one unit is 1/Hq of the "
                         f"work of {w.block_q} tokens) in one process, ~{args.cpu_seconds:.0f} s"}
    clocks = sampler.summary()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    cfg = workload_config(w, args)
    cfg["workload"] = "backward (lists held fixed): " + cfg["workload"]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "impl": "ssa", "config": cfg,
        "keys_per_query": work["keys_per_query"],
        "roofline": {"bound": roof["bound"], "kernel": roof["kernel"],
                     "achieved": achieved, "peak": roof["peak"], "unit": "TFLOP/s",
                     "frac": achieved / roof["peak"], "traffic": None,
                     "peak_source": roof["peak_source"],
                     "frac_basis": "algorithmic flops (10 D per (query, key) pair: S, dP, dq, dk, "
                                   "dv) over the whole backward step",
                     "flops_per_launch": flops},
        "cpu_baseline": cpu, "e2e": e2e,
        # per step: CUDA-core form -- two memsets (dk, dv), the delta kernel
        # and the gradient kernel; tensor-core form -- delta, the list
        # transpose, dq, dk / dv and (GQA) the group sum kernels (the
        # transpose's memset is not a kernel of ours)
        "gpu_launches": (2 if simt else (4 if w.top_k else 3) + (1 if w.Hq > w.Hkv else 0))
                        * args.steps, "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def run_reference_decode(args):
    """The oracle's decode step, timed per step on one host core."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    import oracle as O
    from content_routed_block_b200.workloads import make_inputs
    w = workload_of(args)
    x = make_inputs(w)
    op = O.Params.of(w)
    n_ctx = w.N
    q64 = O.upcast_bf16(x["q"][:, :, n_ctx - 1])
    k64, v64 = O.upcast_bf16(x["k"]), O.upcast_bf16(x["v"])
    for _ in range(args.warmup):
        O.decode_step(q64, k64, v64, n_ctx, op)
    ts = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        O.decode_step(q64, k64, v64, n_ctx, op)
        ts.append(time.perf_counter() - t0)
    sec = statistics.mean(ts)
    value = w.B / sec
    cfg = workload_config(w, args)
    cfg["workload"] = f"decode at n_ctx={n_ctx}: " + cfg["workload"]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * sec, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"{args.steps} whole decode steps in float64, one process"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_reference_backward(args):
    """The oracle's backward, a bounded sample per step on one host core."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    import numpy as np
    import oracle as O
    from content_routed_block_b200.workloads import make_inputs, to_bf16_bits
    w = workload_of(args)
    op = O.Params.of(w)
    x = make_inputs(w, q_heads=[0], kv_heads=[0])
    q64, k64, v64 = (O.upcast_bf16(x[n]) for n in "qkv")
    g64 = O.upcast_bf16(to_bf16_bits(np.random.default_rng(w.seed + 1000).standard_normal(
        (1, 1, w.N, w.D)).astype(np.float32)))
    sub = O.Params.of(w.with_(B=1, Hq=1, Hkv=1))
    r = O.route(O.block_summary(q64[:1], w.block_q), O.block_summary(k64[:1], w.block_k), sub)
    per_step = max(0.5, min(5.0, 150.0 / max(1, args.steps + args.warmup)))
    rng = np.random.default_rng(0)
    vals, units_all = [], 0
    t_all = time.time()
    for s_ in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        units = 0
        while time.perf_counter() - t0 < per_step:
            O.attend_backward(q64[:1], k64[:1], v64[:1], g64, r.idx, r.cnt, sub,
                              blocks=[(0, 0, int(rng.integers(sub.n_qblocks)))])
            units += 1
        if s_ >= args.warmup:
            vals.append(units * w.block_q / w.Hq / (time.perf_counter() - t0))
            units_all += units
    wall = time.time() - t_all
    value = statistics.mean(vals)
    sample = (f"{units_all} (query head, query block) units of this workload's backward over "
              f"{args.steps} steps, ~{per_step:.1f} s each, one process; one unit is 1/Hq of the "
              f"work of {w.block_q} tokens")
    cfg = workload_config(w, args)
    cfg["workload"] = "backward (lists held fixed): " + cfg["workload"]
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * wall / max(1, args.steps + args.warmup), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": cfg,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.decode:
        (run_reference_decode if args.impl == "reference" else run_decode)(args)
        return
    if args.backward:
        (run_reference_backward if args.impl == "reference" else run_backward)(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ssa(args)


if __name__ == "__main__":
    main()
