#!/usr/bin/env python
"""Benchmark of the B200 lightning indexer (score + top-k) on synthetic inputs.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one pass of the indexer hot path over one batch of resident inputs:
for the default workload (the DeepSeek-V3.2-shaped prefill chunk: T=4096
queries at the end of a 32768-token prefix, H_I=64, d=128, top-k=2048) that is
tcgen05 scoring of every visible (query, key) pair followed by the per-query
radix top-k, both through the C-ABI entry point indexer_score_topk.
Other workloads: tiny, decode (FP8), misa (MISA-dagger), hisa.

The metric is scored query-key pairs per second (visible pairs of the dense
problem, so routed / filtered variants show their speed-up in the same unit).
Timing: W warm-up steps, then K steps, each preceded by a 256 MiB L2 flush
and timed with CUDA events on the launching stream; a barrier + synchronize
bracket the timed region; the max over ranks is reported. With N > 1 every
rank runs an independent replica on its own GPU (the path has no exchange
step), so the aggregate is weak scaling.

Extra keys: roofline of the dominant kernel (every kernel of the step timed
alone on the inputs the step gives it; the slowest is the roofline's, all are
listed under "kernels"),
cpu_baseline (the fp64 oracle on a bounded sample, host cores), e2e (host
buffers: every step copies its inputs in and its indices out inside the timed
region, double-buffered so copies overlap the previous step's call), clocks
sampled during the timed region, gpu_launches.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DSA indexer score+top-k: Gpairs/s and % roofline (prefill TC, decode HBM)"
UNIT = "Gpairs/s"
FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ workloads
def workload_desc(name, queries=None, batch=None):
    from sparse_attention_token_score_b200 import workloads as wl
    c = dict(wl.CONFIGS[name])
    if queries:  # a smaller chunk at the end of the same prefix (profiling cases)
        c["T"] = int(queries)
        if "q_offset" in c:
            c["q_offset"] = c["L"] - c["T"]
    if batch and "batch" in c:  # fewer sequences (profiling cases)
        c["batch"] = int(batch)
    batch = c.get("batch", 1)
    off = c.get("q_offset", c["L"] - 1)
    pairs = wl.visible_pairs(c["T"], c["L"], off, batch)
    tag = {"tiny": "tiny_prefill", "dsa": "dsa_chunk", "decode": "decode_fp8",
           "misa": "misa_dagger", "hisa": "hisa"}[name]
    label = f"{tag}_B{batch}_T{c['T']}_L{c['L']}_H{c['H']}_d{c['d']}_k{c['topk']}"
    if name == "misa":
        label += f"_blk{c['block']}_h{c['h']}_kp{c['kprime']}"
    if name == "hisa":
        label += f"_blk{c['block']}_m{c['m']}"
    return c, batch, off, pairs, label


class Runner:
    """Device-resident inputs + the C-ABI call of one workload."""

    def __init__(self, name, inp, torch, queries=None, batch=None):
        from sparse_attention_token_score_b200 import binding as B
        self.B, self.torch, self.name = B, torch, name
        self.c, self.batch, self.off, self.pairs, self.label = workload_desc(name, queries, batch)
        self.inp = inp
        q, k, w, qs, ks = B.to_device(inp)
        self.dev = (q, k, w, qs, ks)
        self.ix = B.Indexer(q, k, w, inp.q_offset, qs, ks)
        c = self.c
        self.topk = c["topk"]
        self.idx = torch.empty((self.batch, c["T"], self.topk), dtype=torch.int32, device="cuda")
        a = self.ix.args
        if name in ("tiny", "dsa", "decode"):
            self.ws = B.alloc_workspace(B.indexer_workspace_size(a, self.topk))
            self.launches = 2
        elif name == "misa":
            self.ws = B.alloc_workspace(B.misa_workspace_size(a, c["block"], c["h"], self.topk, c["kprime"]))
            self.launches = 7  # meanpool, router, select_heads, routed score, top-k', gather score, top-k
        else:
            self.ws = B.alloc_workspace(B.hisa_workspace_size(a, c["block"], c["m"], self.topk))
            self.launches = 5  # meanpool, block score, top-m, gather score, top-k
        self.dtype = "e4m3" if inp.dtype != "bf16" else "bf16"

    def step(self, args=None, out=None):
        B, c = self.B, self.c
        a = self.ix.args if args is None else args
        o = self.idx if out is None else out
        if self.name in ("tiny", "dsa", "decode"):
            B.indexer_score_topk(a, self.topk, o, None, self.ws)
        elif self.name == "misa":
            B.misa_route_score_topk(a, c["block"], c["h"], self.topk, c["kprime"], o, None, None,
                                    None, self.ws)
        else:
            B.hisa_block_filter_topk(a, c["block"], c["m"], self.topk, o, None, None, self.ws)

    # ---- the step's kernels, each launched alone through the C-ABI on the
    # inputs the step gives it (roofline and per-kernel shares)
    def kernels(self):
        """List of (name, callable, algorithmic units per launch, bound), in
        the step's order. Units: FLOPs for tensor-bound kernels (2 * d per
        head per scored pair), bytes for HBM-bound ones."""
        B, torch, c = self.B, self.torch, self.c
        T, L, H, d, k = c["T"], c["L"], c["H"], c["d"], self.topk
        rows = self.batch * T
        ws = B.alloc_workspace(256)
        keep = [ws]
        out = []
        if self.name in ("tiny", "dsa", "decode"):
            sc = torch.empty((self.batch, T, L), dtype=torch.float32, device="cuda")
            idx = torch.empty((self.batch, T, k), dtype=torch.int32, device="cuda")
            keep += [sc, idx]
            f_score = lambda: B.indexer_scores(self.ix.args, sc, L, ws)
            f_score()
            if self.name == "decode":
                # one FP8 key row + its fp32 scale per visible pair
                out.append(("score_tc<fp8>", f_score, self.pairs * (d + 4), "hbm"))
            else:
                out.append(("score_tc<bf16>", f_score, self.pairs * 2.0 * d * H, "tensor"))
            # every visible score read once, k indices written per row
            out.append(("topk_rows", lambda: B.indexer_topk_rows(sc, rows, L, T, self.inp.q_offset, 1, L, k,
                                                                 None, 0, 1, idx, None, ws),
                        self.pairs * 4 + rows * k * 4, "hbm"))
        elif self.name == "misa":
            h, kp = c["h"], c["kprime"]
            q, kk, w, _, _ = self.dev
            # the routed pass scores with h heads per query: the same kernel on a
            # query tensor of h heads (head choice does not change its cost)
            qh, wh = q[:, :, :h].contiguous(), w[:, :, :h].contiguous()
            ah = B.make_args(qh, kk, wh, self.inp.q_offset)
            routed = torch.empty((self.batch, T, L), dtype=torch.float32, device="cuda")
            cand = torch.empty((self.batch, T, kp), dtype=torch.int32, device="cuda")
            comp = torch.empty((self.batch, T, kp), dtype=torch.float32, device="cuda")
            idx = torch.empty((self.batch, T, k), dtype=torch.int32, device="cuda")
            keep += [qh, wh, ah, routed, cand, comp, idx]
            B.misa_route_score_topk(self.ix.args, c["block"], h, k, kp, idx, None, None, cand, self.ws)
            f_routed = lambda: B.indexer_scores(ah, routed, L, ws)
            f_routed()
            out.append(("score_tc<bf16,h=%d> (routed)" % h, f_routed, self.pairs * 2.0 * d * h, "tensor"))
            out.append(("topk_rows (k'=%d over routed rows)" % kp,
                        lambda: B.indexer_topk_rows(routed, rows, L, T, self.inp.q_offset, 1, L, kp, None,
                                                    0, 1, cand, None, ws),
                        self.pairs * 4 + rows * kp * 4, "hbm"))
            f_gather = lambda: B.indexer_score_gathered(self.ix.args, cand, kp, 1, comp, kp, ws)
            f_gather()
            out.append(("score_tc<bf16> gathered (MISA-dagger re-score)", f_gather,
                        rows * kp * 2.0 * d * H, "tensor"))
            out.append(("topk_rows (k=%d over k' candidates)" % k,
                        lambda: B.indexer_topk_rows(comp, rows, kp, T, self.inp.q_offset, 0, kp, k, cand,
                                                    kp, 1, idx, None, ws),
                        rows * kp * 4 + rows * k * 8, "hbm"))
        else:
            m, blk = c["m"], c["block"]
            nc = m * blk
            blocks = torch.empty((self.batch, T, m), dtype=torch.int32, device="cuda")
            comp = torch.empty((self.batch, T, nc), dtype=torch.float32, device="cuda")
            idx = torch.empty((self.batch, T, k), dtype=torch.int32, device="cuda")
            keep += [blocks, comp, idx]
            B.hisa_block_filter_topk(self.ix.args, blk, m, k, idx, None, blocks, self.ws)
            f_gather = lambda: B.indexer_score_gathered(self.ix.args, blocks, m, blk, comp, nc, ws)
            f_gather()
            out.append(("score_tc<bf16> gathered (HISA kept blocks)", f_gather,
                        rows * nc * 2.0 * d * H, "tensor"))
            out.append(("topk_rows (k=%d over m*block tokens)" % k,
                        lambda: B.indexer_topk_rows(comp, rows, nc, T, self.inp.q_offset, 0, nc, k, blocks,
                                                    m, blk, idx, None, ws),
                        rows * nc * 4 + rows * k * 8, "hbm"))
        self._keep = keep
        return out


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# one ncu capture of the kernel named, valid only while its sources hash to
# the value recorded with it (None otherwise). Full-size captures unless the
# profile summary says it was scaled from a smaller case.
_SC, _TK = "483be90f01b3", "b877d4d6299f"   # score_tc / topk_rows sources of the captures
TRAFFIC = {
    ("dsa", "score_tc<bf16>"): (86.33e6 + 448.97e6, _SC),
    ("dsa", "topk_rows"): (504.22e6 + 28.66e6, _TK),
    ("decode", "score_tc<fp8>"): (1.11e9 + 33.55e6, _SC),
    ("decode", "topk_rows"): (33.62e6, _TK),
    ("misa", "topk_rows (k'=8192 over routed rows)"): (1.98e9 + 61.00e6, _TK),
    ("misa", "score_tc<bf16> gathered (MISA-dagger re-score)"): (138.21e6 + 54.98e6, _SC),
    ("misa", "topk_rows (k=2048 over k' candidates)"): (134.28e6 + 8.11e6, _TK),
    ("hisa", "score_tc<bf16> gathered (HISA kept blocks)"): (264.02e6 + 66.76e6, _SC),
    ("hisa", "topk_rows (k=2048 over m*block tokens)"): (67.70e6 + 1.11e6, _TK),
}
KERNEL_SOURCES = {
    "score_tc": ("score_tc.cuh", "common.cuh"),
    "topk_rows": ("topk.cuh",),  # the top-k uses none of common.cuh's helpers
}


def source_hash(kernel_name):
    """Hash of the kernel's source lines, full-line comments and blank lines
    excluded (a comment edit does not invalidate a capture)."""
    import hashlib
    fam = "topk_rows" if kernel_name.startswith("topk_rows") else "score_tc"
    h = hashlib.sha1()
    for f in KERNEL_SOURCES[fam]:
        with open(os.path.join(ROOT, "sparse_attention_token_score_b200", "csrc", f)) as fh:
            for line in fh:
                t = line.strip()
                if t and not t.startswith("//"):
                    h.update(t.encode() + b"\n")
    return h.hexdigest()[:12]


def traffic_for(workload, kernel_name):
    t = TRAFFIC.get((workload, kernel_name))
    if t is None or t[1] != source_hash(kernel_name):
        return None
    return t[0]


def aggregate_ranks(total_ms: float, units_per_rank_step: int, steps: int, world: int, reduce_max=None):
    """Whole-job throughput of independent replicas: every rank processes
    `units_per_rank_step` units per step; the job takes as long as its slowest
    rank. reduce_max(x) returns the max of x over ranks (identity on one rank).
    Returns (max total ms, aggregate units per second)."""
    t = reduce_max(total_ms) if (reduce_max is not None and world > 1) else total_ms
    return t, world * units_per_rank_step * steps / (t / 1e3)


def dist_max(dist, device):
    """reduce_max over the default process group (NCCL on GPUs, gloo on CPU)."""
    import torch

    def f(x):
        v = torch.tensor([float(x)], dtype=torch.float64, device=device)
        dist.all_reduce(v, op=dist.ReduceOp.MAX)
        return float(v.item())
    return f


def l2_flush(buf):
    buf.add_(1)


def time_steps(fn, n, torch, flush):
    """Per-launch CUDA-event times (ms) on the current stream, L2 flushed before each."""
    st = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for e0, e1 in ev:
        l2_flush(flush)
        e0.record(st)
        fn()
        e1.record(st)
    torch.cuda.synchronize()
    return [e0.elapsed_time(e1) for e0, e1 in ev]


def run_e2e(r, inp, steps, torch, barrier):
    """Steps through the C-ABI call from host memory: every step copies its
    inputs host -> device from pinned memory, runs the call and copies its
    indices device -> host. Two buffer sets on three streams (copy in, call,
    copy out) let a step's copies overlap the previous step's call, as a
    server streaming batches would. Returns (device ms of the `steps` steps,
    H2D bytes per step, D2H bytes per step)."""
    from sparse_attention_token_score_b200 import binding as B
    srcs = r.dev
    host = [t.cpu().pin_memory() if t is not None else None for t in srcs]
    sets = []
    for _ in range(2):
        dev = [torch.empty_like(t) if t is not None else None for t in srcs]
        sets.append({"dev": dev, "args": B.make_args(dev[0], dev[1], dev[2], inp.q_offset, dev[3], dev[4]),
                     "idx": torch.empty_like(r.idx),
                     "out": torch.empty(r.idx.shape, dtype=torch.int32, pin_memory=True),
                     "loaded": torch.cuda.Event(), "done": torch.cuda.Event(), "copied": torch.cuda.Event()})
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def issue(i):
        b = sets[i % 2]
        s_in.wait_event(b["done"])      # the call of step i - 2 has read this set's inputs
        with torch.cuda.stream(s_in):
            for h, d in zip(host, b["dev"]):
                if h is not None:
                    d.copy_(h, non_blocking=True)
            b["loaded"].record(s_in)
        s_run.wait_event(b["loaded"])
        s_run.wait_event(b["copied"])   # step i - 2's indices have left this set's buffer
        with torch.cuda.stream(s_run):
            r.step(args=b["args"], out=b["idx"])
            b["done"].record(s_run)
        s_out.wait_event(b["done"])
        with torch.cuda.stream(s_out):
            b["out"].copy_(b["idx"], non_blocking=True)
            b["copied"].record(s_out)

    for i in range(3):
        issue(i)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(steps):
        issue(3 + i)
    e1.record(s_out)                    # after the last copy out, which follows every step's work
    torch.cuda.synchronize()
    barrier()
    h2d = sum(t.numel() * t.element_size() for t in host if t is not None)
    return float(e0.elapsed_time(e1)), h2d, r.idx.numel() * 4


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                       "-i", str(gpu_index), "-lms", "200"], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.p.terminate()
        self.p.wait(timeout=10)
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.count(",") >= 8]
        os.unlink(self.f.name)
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if "Active" in v and "Not" not in v})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ oracle (CPU) timing
def oracle_sample(name, inp, budget_s=10.0, max_q=4096):
    """Time the fp64 oracle, as it stands, on a bounded sample of this workload's
    queries (the same computation as one GPU step, restricted to the sample)."""
    import oracle
    from sparse_attention_token_score_b200 import workloads as wl
    c = wl.CONFIGS[name]
    T = c["T"]
    rng = np.random.default_rng(1)

    def run(qs, b=0):
        t0 = time.perf_counter()
        if name == "misa":
            oracle.misa(inp, c["block"], c["h"], c["topk"], kprime=c["kprime"], queries=qs, b=b)
        elif name == "hisa":
            oracle.hisa(inp, c["block"], c["m"], c["topk"], queries=qs, b=b)
        else:
            oracle.dense_topk(inp, c["topk"], queries=qs, b=b)
        return time.perf_counter() - t0

    def pairs(qs, b=0):
        off = inp.q_offset
        return int(sum(min(off + int(t) + 1, inp.L) for t in qs))

    if name == "decode":
        # one unit = one sequence's query; add sequences until budget_s is spent
        t, nb = 0.0, 0
        while t < budget_s and nb < inp.batch:
            t += run([0], b=nb)
            nb += 1
        return nb * inp.L / t / 1e9, f"{nb} of {inp.batch} sequences (all {inp.L} keys each)", nb, t
    # grow the sample until one run takes at least budget_s (or covers every query)
    n = 8
    while True:
        n = min(n, T, max_q)
        qs = np.sort(rng.choice(T, n, replace=False)) if n < T else np.arange(T)
        t = run(qs)
        if t >= budget_s or n >= min(T, max_q):
            break
        n = int(n * min(8.0, max(2.0, 1.2 * budget_s / max(t, 1e-3))))
    return pairs(qs) / t / 1e9, f"{len(qs)} of {T} queries (uniform sample)", len(qs), t


def run_reference(args):
    """The oracle arm: fp64 CPU oracle on host cores, bounded sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    from sparse_attention_token_score_b200 import workloads as wl
    c, batch, off, pairs, label = workload_desc(args.workload)
    inp = wl.make_inputs(args.workload, seed=0)
    per_step = max(2.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    vals, samples = [], None
    for i in range(args.warmup + args.steps):
        v, samples, _, _ = oracle_sample(args.workload, inp, budget_s=per_step / 2)
        if i >= args.warmup:
            vals.append(v)
    value = float(np.mean(vals))
    cores = oracle.num_threads()
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": pairs / (value * 1e9) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": label, "pairs_per_step": pairs, "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": samples},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def make_inputs(name, seed, queries=0, batch=0):
    """The workload's inputs; with `queries`, only the last `queries` queries
    of the chunk (same prefix, same distributions); with `batch`, only the
    first `batch` sequences."""
    from sparse_attention_token_score_b200 import workloads as wl
    if batch and name == "decode":
        c = wl.CONFIGS[name]
        return wl.decode_inputs(batch, c["L"], c["H"], c["d"], seed=seed)
    inp = wl.make_inputs(name, seed=seed)
    if queries and queries < inp.T:
        T0 = inp.T - queries
        inp.q = inp.q[:, T0:].copy()
        inp.w = inp.w[:, T0:].copy()
        if inp.q_scale is not None:
            inp.q_scale = inp.q_scale[:, T0:].copy()
        inp.q_offset += T0
    return inp


# ------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="dsa", choices=["tiny", "dsa", "decode", "misa", "hisa"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--queries", type=int, default=0,
                    help="profiling: use only the last N queries of the chunk")
    ap.add_argument("--batch", type=int, default=0,
                    help="profiling: use only the first N sequences (decode)")
    ap.add_argument("--kernel-only", action="store_true",
                    help="profiling: launch only one kernel of the step (W + K times)")
    ap.add_argument("--kernel", type=int, default=0,
                    help="with --kernel-only: index into the step's kernel list (0 = first)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist
    from sparse_attention_token_score_b200 import workloads as wl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    inp = make_inputs(args.workload, rank, args.queries, args.batch)
    r = Runner(args.workload, inp, torch, args.queries, args.batch)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    if args.kernel_only:
        kname, fn, _, _ = r.kernels()[args.kernel]
        kt = time_steps(fn, args.warmup + args.steps, torch, flush)[args.warmup:]
        print(json.dumps({"kernel": kname, "workload": r.label, "kernel_ms": kt}), flush=True)
        return 0
    for _ in range(args.warmup):
        r.step()
    torch.cuda.synchronize()

    # ---- timed region
    sampler = ClockSampler(local) if rank == 0 else None
    barrier()
    torch.cuda.synchronize()
    times = time_steps(r.step, args.steps, torch, flush)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop() if sampler else None
    rmax = dist_max(dist, "cuda") if world > 1 else None
    total_ms, pairs_per_s = aggregate_ranks(float(sum(times)), r.pairs, args.steps, world, rmax)
    ms_per_step = total_ms / args.steps
    value = pairs_per_s / 1e9
    assert r.ix.device_status() == 0, "device wait timed out"

    # ---- each kernel alone; the one with the largest time is the roofline's
    peaks, peak_src = load_peaks()
    per_kernel = []
    for kname, fn, units, bound in r.kernels():
        for _ in range(3):
            fn()
        kms = statistics.mean(time_steps(fn, args.steps, torch, flush))
        if bound == "tensor":
            achieved, peak, unit = units / (kms / 1e3) / 1e12, peaks["bf16_tflops"], "TFLOP/s"
        else:
            achieved, peak, unit = units / (kms / 1e3) / 1e9, peaks["hbm_gbs"], "GB/s"
        per_kernel.append({"kernel": kname, "bound": bound, "ms": kms, "achieved": achieved, "peak": peak,
                           "unit": unit, "frac": achieved / peak, "algorithmic_units_per_launch": units,
                           "traffic": traffic_for(args.workload, kname)})
    dom = max(per_kernel, key=lambda e: e["ms"])
    kernel_sum = sum(e["ms"] for e in per_kernel)
    for e in per_kernel:
        e["share_of_listed"] = e["ms"] / kernel_sum
    roof = {"bound": dom["bound"], "achieved": dom["achieved"], "peak": dom["peak"], "unit": dom["unit"],
            "frac": dom["frac"], "traffic": dom["traffic"], "kernel": dom["kernel"], "kernel_ms": dom["ms"],
            "algorithmic_units_per_launch": dom["algorithmic_units_per_launch"],
            "peak_source": f"{peak_src} ({'bf16 burst' if dom['bound'] == 'tensor' else 'HBM copy'})"}

    # ---- end to end: host buffers, H2D + call + D2H in every step
    e_total, h2d, d2h = run_e2e(r, inp, args.steps, torch, barrier)
    e_ms, e_pairs_per_s = aggregate_ranks(e_total, r.pairs, args.steps, world, rmax)
    e2e_value = e_pairs_per_s / 1e9

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, one GPU only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        v, sample, _, secs = oracle_sample(args.workload, inp)
        cpu = {"value": v, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
               "sample": sample, "seconds": round(secs, 2)}

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    c = r.c
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": r.dtype, "data": "synthetic",
        "config": {"workload": r.label, "batch": r.batch, "T": c["T"], "L": c["L"], "H": c["H"],
                   "d": c["d"], "topk": c["topk"], "q_offset": inp.q_offset,
                   "pairs_per_step": r.pairs, "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "256 MiB buffer written before every timed step"},
        "queries_per_s": world * r.batch * c["T"] * args.steps / (total_ms / 1e3),
        "roofline": roof,
        "kernels": per_kernel,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e_ms / args.steps,
                "pipeline": "2 buffer sets, copy-in / call / copy-out streams"},
        "gpu_launches": r.launches * args.steps,
        "clocks": clocks,
        "step_ms": {"min": min(times), "median": statistics.median(times), "max": max(times)},
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
