#!/usr/bin/env python
"""Benchmark of the B200 lightning indexer (score + top-k) on synthetic inputs.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one pass of the indexer hot path over one batch of resident inputs.
The headline line is the DeepSeek-V3.2-shaped prefill chunk (T=4096 queries at
the end of a 32768-token prefix, H_I=64, d=128, top-k=2048): tcgen05 scoring of
every visible (query, key) pair followed by the per-query radix top-k, both
through the C-ABI entry point indexer_score_topk. By default the same run also
measures the other four workloads (tiny prefill, FP8 decode, MISA-dagger,
HISA) and reports each under "workloads" with the same fields; --workload
NAME measures one workload alone as the headline.

The metric is scored query-key pairs per second (visible pairs of the dense
problem, so routed / filtered variants show their speed-up in the same unit).
Timing: W warm-up steps, then K steps (sub-records: at least 60 ms of steps),
each preceded by a 256 MiB L2 flush and timed with CUDA events on the
launching stream; a barrier + synchronize bracket the timed region; the max
over ranks is reported. With N > 1 every rank runs an independent replica on
its own GPU (the path has no exchange step), so the aggregate is weak scaling.

Extra keys: roofline of the dominant kernel (after the timed region, the
same number of steps runs again with the library's launch profiler on: every
launch bracketed by CUDA events on its stream; all kernels are listed under
"kernels" with their time per step, and the slowest one with known
algorithmic work is the roofline's), cpu_baseline (the fp64 oracle on a
bounded sample, host cores), e2e (host buffers: every step copies its inputs
in and its indices out inside the timed region, double-buffered so copies
overlap the previous step's call), clocks sampled by NVML every 5 ms during
the timed region, gpu_launches (counted by the profiler).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
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
    if name == "indexcache":  # pairs of the dense problem of every layer
        pairs *= len(c["pattern"])
    tag = {"tiny": "tiny_prefill", "dsa": "dsa_chunk", "decode": "decode_fp8",
           "misa": "misa_dagger", "hisa": "hisa", "dsa_fp8": "dsa_chunk_fp8",
           "indexcache": "indexcache_dsa_chunk", "dosa": "dosa_dsa_chunk",
           "dosa_lownorm": "dosa_lownorm_dsa_chunk", "dsa_lists": "dsa_chunk_lists",
           "hisa_decode": "hisa_decode_fp8", "misa_decode": "misa_dagger_decode_fp8"}[name]
    label = f"{tag}_B{batch}_T{c['T']}_L{c['L']}_H{c['H']}_d{c['d']}_k{c['topk']}"
    if name in ("misa", "misa_decode"):
        label += f"_blk{c['block']}_h{c['h']}_kp{c['kprime']}"
    if name in ("hisa", "hisa_decode"):
        label += f"_blk{c['block']}_m{c['m']}"
    if name in POOLED_CACHE:  # pooled keys kept across steps, the last block re-pooled per step
        label += "_pooledcache"
    if name == "indexcache":
        label += f"_layers{c['pattern']}"
    if name in ("dosa", "dosa_lownorm"):
        label += f"_screen{c['n_screen']}"
    return c, batch, off, pairs, label


DENSE = ("tiny", "dsa", "decode", "dsa_fp8", "indexcache")  # workloads whose F layer is indexer_score_topk
DOSA = ("dosa", "dosa_lownorm")                              # dosa_score_topk
LISTS = ("dsa_lists",)                                       # indexer_score_topk_lists
POOLED_CACHE = ("hisa_decode", "misa_decode")                # *_pooled calls on a pooled-key cache


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
        if name in DENSE:
            self.ws = B.alloc_workspace(B.indexer_workspace_size(a, self.topk))
            if name == "indexcache":
                pat = c["pattern"]
                assert pat.count("F") == 1, "the bench's IndexCache slice has one F layer"
                self.shared = B.IndexerArgs(batch=self.batch, T=c["T"])  # S layers: shape only
        elif name in LISTS:
            self.ws = B.alloc_workspace(B.indexer_lists_workspace_size(a, self.topk))
        elif name in DOSA:
            self.ws = B.alloc_workspace(B.dosa_workspace_size(a, self.topk, c["n_screen"]))
            qpt = 256 // c["H"]
            self.live = torch.empty((self.batch, -(-c["T"] // qpt), -(-c["L"] // 128)), dtype=torch.uint8,
                                    device="cuda")
            self.live_pairs = None
        elif name in ("misa", "misa_decode"):
            self.ws = B.alloc_workspace(B.misa_workspace_size(a, c["block"], c["h"], self.topk, c["kprime"]))
        else:
            self.ws = B.alloc_workspace(B.hisa_workspace_size(a, c["block"], c["m"], self.topk))
        if name in POOLED_CACHE:
            # decode: the pooled keys live in a cache next to the key cache;
            # completed blocks are pooled once (here), the last block again
            # at every step
            self.M = -(-c["L"] // c["block"])
            self.kbar, self.ksc = B.pooled_cache(a, c["block"], device="cuda")
            B.dsa_pool_keys(a, c["block"], 0, self.M, self.kbar, self.ksc)
        self.dtype = "e4m3" if inp.dtype != "bf16" else "bf16"

    def step(self, args=None, out=None):
        B, c = self.B, self.c
        a = self.ix.args if args is None else args
        o = self.idx if out is None else out
        if self.name == "indexcache":
            # S layers share the F layer's index buffer (the page's index cache)
            layers = [a if r == "F" else self.shared for r in c["pattern"]]
            B.indexcache_score_topk(layers, c["pattern"], self.topk, [o] * len(layers), None, self.ws)
        elif self.name in DENSE:
            B.indexer_score_topk(a, self.topk, o, None, self.ws)
        elif self.name in LISTS:
            B.indexer_score_topk_lists(a, self.topk, o, None, self.ws)
        elif self.name in DOSA:
            B.dosa_score_topk(a, self.topk, c["n_screen"], o, None, self.live, self.ws)
        elif self.name in POOLED_CACHE:
            B.dsa_pool_keys(a, c["block"], self.M - 1, self.M, self.kbar, self.ksc)
            if self.name == "misa_decode":
                B.misa_route_score_topk_pooled(a, c["block"], c["h"], self.topk, c["kprime"], self.kbar, self.ksc,
                                               o, None, None, None, self.ws)
            else:
                B.hisa_block_filter_topk_pooled(a, c["block"], c["m"], self.topk, self.kbar, self.ksc, o, None,
                                                None, self.ws)
        elif self.name == "misa":
            B.misa_route_score_topk(a, c["block"], c["h"], self.topk, c["kprime"], o, None, None,
                                    None, self.ws)
        else:
            B.hisa_block_filter_topk(a, c["block"], c["m"], self.topk, o, None, None, self.ws)

    # ---- algorithmic units of the step's kernels (per step), by the name the
    # library's launch profiler files them under
    def kernel_units(self, name):
        """(units per step, bound) of a profiled kernel, or (None, None) when
        its work depends on data the host does not see (list lengths, sample
        sizes). Units: FLOPs (2 * d per head per scored pair) for the tensor
        core kernels, bytes for the HBM-bound ones."""
        c, inp = self.c, self.inp
        T, L, H, d, k = c["T"], c["L"], c["H"], c["d"], self.topk
        rows = self.batch * T
        pos = inp.q_offset + np.arange(T, dtype=np.int64)
        label = name.split(": ")[-1]
        stage = name.split(": ")[0] if ": " in name else ""
        if "sample pass" in stage or "fallback" in stage or "candidate lists)" in label:
            return None, None
        if self.name in DENSE + DOSA + LISTS:
            pairs = self.pairs // len(c.get("pattern", "F"))  # the F layer's pairs (indexcache)
            if stage == "bounds" and label.startswith("score_tc"):
                return pairs * 2.0 * d * 8, "tensor"          # 8 augmented heads per pair
            if label.startswith("score_tc"):
                if self.name == "decode":
                    return pairs * (d + 4), "hbm"          # one FP8 key row + its scale per pair
                if self.name in DOSA:                      # the live tiles' pairs only
                    return self.live_pairs * 2.0 * d * H if self.live_pairs is not None else None, "tensor"
                return pairs * 2.0 * d * H, ("tensor_fp8" if self.name == "dsa_fp8" else "tensor")
            if label == "topk_rows":
                return pairs * 4 + rows * k * 4, "hbm"    # every visible score read, k ids written
        if self.name in ("misa", "misa_decode"):
            fp8 = self.name == "misa_decode"
            blk, h, kp = c["block"], c["h"], c["kprime"]
            M = -(-L // blk)
            vis_blocks = int(self.batch * np.minimum(pos // blk + 1, M).sum())
            if stage == "router" and label.startswith("score_tc"):
                return vis_blocks * 2.0 * d * H, "tensor_fp8" if fp8 else "tensor"
            if stage == "routed" and label.startswith("score_tc"):
                if fp8:                                    # the key stream: one FP8 row + scale per pair
                    return self.pairs * (d + 4), "hbm"
                return self.pairs * 2.0 * d * h, "tensor"
            if stage == "routed" and label == "topk_rows":
                return self.pairs * 4 + rows * kp * 4, "hbm"
            if stage == "re-score" and label.startswith("score_tc"):
                if fp8:                                    # one query per sequence: the gathered rows + scales
                    return rows * kp * (d + 4), "hbm"
                return rows * kp * 2.0 * d * H, "tensor"
            if stage == "re-score" and label == "topk_rows":
                return rows * kp * 4 + rows * k * 8, "hbm"
        if self.name in ("hisa", "hisa_decode"):
            fp8 = self.name == "hisa_decode"
            blk, m = c["block"], c["m"]
            M = -(-L // blk)
            vis_blocks = int(self.batch * np.minimum(pos // blk + 1, M).sum())
            if stage == "blocks" and label.startswith("score_tc"):
                if fp8:                                    # decode: one query per sequence, pooled rows + scales
                    return vis_blocks * (d + 4), "hbm"
                return vis_blocks * 2.0 * d * H, "tensor"
            if stage == "tokens" and label.startswith("score_"):
                if fp8:                                    # decode: the kept blocks' key rows + scales
                    return rows * m * blk * (d + 4), "hbm"
                return rows * m * blk * 2.0 * d * H, "tensor"
            if stage == "tokens" and label == "topk_rows":
                return rows * m * blk * 4 + rows * k * 8, "hbm"
        return None, None

    def dosa_live(self):
        """Fraction of the visible (query group, key tile) pairs the bound kept,
        and the visible pairs of the kept tiles (from the last step's mask)."""
        c = self.c
        live = self.live.cpu().numpy()[0]
        qpt, T, L = 256 // c["H"], c["T"], c["L"]
        kept = total = 0
        pairs = 0
        for g in range(live.shape[0]):
            t0, t1 = g * qpt, min(T, (g + 1) * qpt)
            pos = self.inp.q_offset + np.arange(t0, t1)
            nt = -(-min(pos[-1] + 1, L) // 128)
            kept += int(live[g, :nt].sum())
            total += nt
            for j in np.flatnonzero(live[g, :nt]):
                lo, hi = 128 * j, min(128 * (j + 1), L)
                pairs += int(np.clip(pos + 1 - lo, 0, hi - lo).sum())
        self.live_pairs = pairs
        return kept / total, pairs


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# one ncu capture of the kernel named, valid only while its sources hash to
# the value recorded with it (None otherwise). Full-size captures unless the
# profile summary says it was scaled from a smaller case.
_SC, _INV, _TK = "98af7e7b7253", "c482859cb74d", "c51353878d82"   # score_tc / score_inv / topk_rows sources
TRAFFIC = {
    ("dsa", "score_tc"): (87.25e6 + 449.52e6, _SC),
    ("dsa", "topk_rows"): (505.61e6 + 28.82e6, _TK),
    ("tiny", "topk_rows"): (8.56e6, _TK),
    ("decode", "score_tc fp8"): (1108.43e6 + 33.14e6, _SC),
    ("decode", "topk_rows"): (33.63e6, _TK),
    ("misa", "routed: score_tc"): (275.97e6 + 1016.91e6, _SC),
    ("misa", "routed: topk_rows"): (1350.05e6 + 61.08e6, _TK),
    ("misa", "re-score: score_tc gathered"): (137.70e6 + 54.82e6, _SC),
    ("hisa", "blocks: topk_rows"): (8.43e6, _TK),
    ("hisa", "tokens: score_inv (block-major)"): (81.49e6 + 33.05e6, _INV),
    ("hisa", "tokens: topk_rows"): (67.72e6 + 1.26e6, _TK),
    ("dsa_fp8", "score_tc fp8"): (45.55e6 + 445.67e6, _SC),
    ("hisa_decode", "tokens: score_tc gathered"): (139.25e6 + 3.93e6, _SC),
    ("misa_decode", "routed: score_tc fp8"): (1107.88e6 + 33.24e6, _SC),
}
KERNEL_SOURCES = {
    "score_tc": ("score_tc.cuh", "common.cuh"),
    "score_inv": ("score_inv.cuh", "common.cuh"),
    "topk_rows": ("topk.cuh",),  # the top-k uses none of common.cuh's helpers
}


def source_hash(kernel_name):
    """Hash of the kernel's source lines, full-line comments and blank lines
    excluded (a comment edit does not invalidate a capture)."""
    import hashlib
    label = kernel_name.split(": ")[-1]
    fam = "topk_rows" if label.startswith("topk_rows") else ("score_inv" if label.startswith("score_inv")
                                                             else "score_tc")
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
    server streaming batches would. Decode workloads keep the key cache
    resident (it is the model's cache): a step copies its queries, weights
    and query scales and the one new key row (and scale) per sequence, which
    it writes at the cache's last position. Returns (device ms of the `steps`
    steps, H2D bytes per step, D2H bytes per step)."""
    from sparse_attention_token_score_b200 import binding as B
    decode = r.c.get("kind") == "decode"
    srcs = r.dev
    host = [t.cpu().pin_memory() if t is not None else None for t in srcs]
    L = inp.L
    if decode:  # the cache stays on the device; only the newest row per sequence travels
        host[1] = srcs[1][:, L - 1:L].cpu().pin_memory()
        host[4] = srcs[4][:, L - 1:L].cpu().pin_memory()
        cache_k, cache_ks = srcs[1].clone(), srcs[4].clone()
    sets = []
    for _ in range(2):
        dev = [torch.empty_like(t) if t is not None else None for t in srcs]
        if decode:
            dev[1], dev[4] = cache_k, cache_ks
        sets.append({"dev": dev, "args": B.make_args(dev[0], dev[1], dev[2], inp.q_offset, dev[3], dev[4]),
                     "idx": torch.empty_like(r.idx),
                     "out": torch.empty(r.idx.shape, dtype=torch.int32, pin_memory=True),
                     "loaded": torch.cuda.Event(), "done": torch.cuda.Event(), "copied": torch.cuda.Event()})
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def issue(i):
        b = sets[i % 2]
        s_in.wait_event(b["done"])      # the call of step i - 2 has read this set's inputs
        if decode:                       # and step i - 1's call has read the shared cache
            s_in.wait_event(sets[(i + 1) % 2]["done"])
        with torch.cuda.stream(s_in):
            for j, (h, d) in enumerate(zip(host, b["dev"])):
                if h is None:
                    continue
                if decode and j in (1, 4):
                    d[:, L - 1:L].copy_(h, non_blocking=True)
                else:
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
    """SM clock and throttle reasons sampled while the GPU works: NVML polled
    from a thread every 5 ms (nvidia-smi at 200 ms where NVML is missing).
    Only samples taken between mark_start() and mark_stop() are reported, so
    the record covers exactly the timed region."""
    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4}

    def __init__(self, device_index):
        import threading
        self.samples = []          # (monotonic s, sm MHz, max MHz, reason bits)
        self.t0 = self.t1 = None
        self.stop_flag = threading.Event()
        self.nvml = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            self.nvml = pynvml
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        except Exception:
            self.nvml = None
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _reasons(self):
        p = self.nvml
        f = getattr(p, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(p, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return int(f(self.h))

    def _run(self):
        if self.nvml is None:
            return
        p = self.nvml
        while not self.stop_flag.is_set():
            try:
                sm = float(p.nvmlDeviceGetClockInfo(self.h, p.NVML_CLOCK_SM))
                self.samples.append((time.monotonic(), sm, self.max_mhz, self._reasons()))
            except Exception:
                pass
            time.sleep(0.005)

    def mark_start(self):
        self.t0 = time.monotonic()

    def mark_stop(self):
        self.t1 = time.monotonic()

    def stop(self):
        self.stop_flag.set()
        self.thread.join(timeout=5)
        if self.nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["NVML unavailable"], "samples": 0}
        return self.summarize(self.samples, self.t0, self.t1, self.max_mhz)

    @classmethod
    def summarize(cls, samples, t0, t1, max_mhz):
        """Median SM clock and the throttle reasons seen in samples with
        t0 <= time <= t1; the samples just before t0 and just after t1 are kept
        too, so a region shorter than the polling interval still has a record."""
        if t0 is None:
            return {"sm_mhz": None, "sm_max_mhz": max_mhz, "reasons": [], "samples": 0}
        t1 = t1 if t1 is not None else float("inf")
        inside = [r for r in samples if t0 <= r[0] <= t1]
        before = [r for r in samples if r[0] < t0][-1:]
        after = [r for r in samples if r[0] > t1][:1]
        rows = before + inside + after
        sm = [r[1] for r in rows]
        reasons = sorted({n for r in rows for n, bit in cls.REASONS.items() if r[3] & bit})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max_mhz,
                "reasons": reasons, "samples": len(rows), "samples_inside": len(inside),
                "source": "NVML, every 5 ms"}


# ------------------------------------------------------------------ oracle (CPU) timing
def oracle_sample(name, inp, budget_s=10.0, max_q=4096, with_pairs=False):
    """Time the fp64 oracle, as it stands, on a bounded sample of this workload's
    queries (the same computation as one GPU step, restricted to the sample)."""
    import oracle
    from sparse_attention_token_score_b200 import workloads as wl
    c = wl.CONFIGS[name]
    T = c["T"]
    rng = np.random.default_rng(1)

    def run(qs, b=0):
        t0 = time.perf_counter()
        if name in ("misa", "misa_decode"):
            oracle.misa(inp, c["block"], c["h"], c["topk"], kprime=c["kprime"], queries=qs, b=b)
        elif name in ("hisa", "hisa_decode"):
            oracle.hisa(inp, c["block"], c["m"], c["topk"], queries=qs, b=b)
        else:
            oracle.dense_topk(inp, c["topk"], queries=qs, b=b)
        return time.perf_counter() - t0

    def pairs(qs, b=0):
        # IndexCache: the oracle runs the F layer; its S layers reuse the indices
        # (as on the GPU), and the dense pairs of every layer count
        off = inp.q_offset
        return int(sum(min(off + int(t) + 1, inp.L) for t in qs)) * len(c.get("pattern", "F"))

    if name in ("decode", "hisa_decode", "misa_decode"):
        # one unit = one sequence's query; add sequences until budget_s is spent
        t, nb = 0.0, 0
        while t < budget_s and nb < inp.batch:
            t += run([0], b=nb)
            nb += 1
        res = (nb * inp.L / t / 1e9, f"{nb} of {inp.batch} sequences (all {inp.L} keys each)", nb, t)
        return res + (nb * inp.L,) if with_pairs else res
    # grow the sample until one run takes at least budget_s (or covers every query)
    n = 8
    while True:
        n = min(n, T, max_q)
        qs = np.sort(rng.choice(T, n, replace=False)) if n < T else np.arange(T)
        t = run(qs)
        if t >= budget_s or n >= min(T, max_q):
            break
        n = int(n * min(8.0, max(2.0, 1.2 * budget_s / max(t, 1e-3))))
    res = (pairs(qs) / t / 1e9, f"{len(qs)} of {T} queries (uniform sample)", len(qs), t)
    return res + (pairs(qs),) if with_pairs else res


def workload_config(r_c, batch, label, q_offset, pairs, world):
    """The `config` object of a JSON line (the same for both arms)."""
    return {"workload": label, "batch": batch, "T": r_c["T"], "L": r_c["L"], "H": r_c["H"],
            "d": r_c["d"], "topk": r_c["topk"], "q_offset": q_offset, "pairs_per_step": pairs,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "256 MiB buffer written before every timed step"}


def run_reference(args):
    """The oracle arm: the fp64 CPU oracle, as it stands, on the host cores; each
    step is a bounded query sample of the headline workload, timed as it runs
    (ms_per_step is that sample's time, value its pairs / time)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    import oracle
    from sparse_attention_token_score_b200 import workloads as wl
    name = "dsa" if args.workload == "all" else args.workload
    c, batch, off, pairs, label = workload_desc(name)
    inp = wl.make_inputs(name, seed=0)
    per_step = max(2.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    vals, secs, npairs, samples = [], [], [], None
    for i in range(args.warmup + args.steps):
        v, samples, _, t, p = oracle_sample(name, inp, budget_s=per_step / 2, with_pairs=True)
        if i >= args.warmup:
            vals.append(v)
            secs.append(t)
            npairs.append(p)
    value = float(sum(npairs) / sum(secs) / 1e9)
    cores = oracle.num_threads()
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * float(np.mean(secs)), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": workload_config(c, batch, label, off, pairs, world),
            "sample": {"what": samples, "pairs_per_timed_step": int(np.mean(npairs)),
                       "note": "each step times the oracle on this query sample of the workload"},
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
SUB_WORKLOADS = ("tiny", "decode", "misa", "hisa", "hisa_decode", "misa_decode", "dsa_fp8", "indexcache",
                 "dsa_lists", "dosa", "dosa_lownorm")
MIN_TIMED_MS = 60.0  # sub-records run enough steps that the clock sampler sees the GPU busy


def measure_workload(name, args, torch, world, rank, local, flush, barrier, rmax, steps,
                     cpu_budget_s, min_timed_ms=0.0):
    """Everything one JSON record says about a workload, measured in this
    process: timed steps, each kernel alone (roofline), end to end through
    host buffers, clocks during the timed region, and the oracle's CPU rate."""
    inp = make_inputs(name, rank, args.queries, args.batch)
    r = Runner(name, inp, torch, args.queries, args.batch)
    for _ in range(args.warmup):
        r.step()
    torch.cuda.synchronize()
    if min_timed_ms > 0:  # lengthen short workloads' timed regions (same count on every rank)
        probe = statistics.median(time_steps(r.step, 3, torch, flush))
        steps = max(steps, int(np.ceil(min_timed_ms / max(probe, 1e-3))))
        if world > 1:
            steps = int(rmax(steps))

    # ---- timed region
    sampler = ClockSampler(local) if rank == 0 else None
    barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.mark_start()
    times = time_steps(r.step, steps, torch, flush)
    torch.cuda.synchronize()
    if sampler:
        sampler.mark_stop()
    barrier()
    clocks = sampler.stop() if sampler else None
    total_ms, pairs_per_s = aggregate_ranks(float(sum(times)), r.pairs, steps, world, rmax)
    assert r.ix.device_status() == 0, "device wait timed out"

    dosa = None
    if name in DOSA:
        frac_live, live_pairs = r.dosa_live()
        dosa = {"live_tile_fraction": frac_live, "pruned_tile_fraction": 1.0 - frac_live,
                "refined_pairs_per_step": live_pairs,
                "pruned_pair_fraction": 1.0 - live_pairs / (r.pairs / len(r.c.get("pattern", "F")))}
    # ---- every launch of the step, timed by the library's launch profiler
    # (CUDA events on the launching stream) over `steps` more steps with the
    # same L2 flush; the kernel with the largest time per step is the roofline's
    peaks, peak_src = load_peaks()
    from sparse_attention_token_score_b200 import binding as B
    B.dsa_profile_begin()
    for _ in range(steps):
        l2_flush(flush)
        r.step()
    recs = B.dsa_profile_end()
    per_name = {}
    for nm, ms in recs:
        e = per_name.setdefault(nm, [0.0, 0])
        e[0] += ms
        e[1] += 1
    per_kernel = []
    for nm, (ms_tot, n) in per_name.items():
        kms = ms_tot / steps
        units, bound = r.kernel_units(nm)
        rec_k = {"kernel": nm, "ms": kms, "launches_per_step": n / steps, "bound": bound,
                 "algorithmic_units_per_step": units, "traffic": traffic_for(name, nm)}
        if units is not None:
            if bound == "tensor":
                rec_k.update(achieved=units / (kms / 1e3) / 1e12, peak=peaks["bf16_tflops"], unit="TFLOP/s")
            elif bound == "tensor_fp8":  # measured bf16 burst x the nominal dense fp8 : bf16 ratio (2)
                rec_k.update(achieved=units / (kms / 1e3) / 1e12, peak=2.0 * peaks["bf16_tflops"], unit="TFLOP/s")
            else:
                rec_k.update(achieved=units / (kms / 1e3) / 1e9, peak=peaks["hbm_gbs"], unit="GB/s")
            rec_k["frac"] = rec_k["achieved"] / rec_k["peak"]
        per_kernel.append(rec_k)
    kernel_sum = sum(e["ms"] for e in per_kernel)
    for e in per_kernel:
        e["share_of_step"] = e["ms"] / kernel_sum
    launches_per_step = len(recs) / steps
    dom = max((e for e in per_kernel if "frac" in e), key=lambda e: e["ms"])
    psrc = {"tensor": "bf16 burst", "tensor_fp8": "bf16 burst x 2, the nominal fp8:bf16 dense ratio",
            "hbm": "HBM copy"}[dom["bound"]]
    roof = {"bound": "tensor" if dom["bound"].startswith("tensor") else dom["bound"],
            "achieved": dom["achieved"], "peak": dom["peak"], "unit": dom["unit"],
            "frac": dom["frac"], "traffic": dom["traffic"], "kernel": dom["kernel"], "kernel_ms": dom["ms"],
            "algorithmic_units_per_launch": dom["algorithmic_units_per_step"] / dom["launches_per_step"],
            "largest_kernel": max(per_kernel, key=lambda e: e["ms"])["kernel"],
            "peak_source": f"{peak_src} ({psrc})"}

    # ---- end to end: host buffers, H2D + call + D2H in every step
    e_total, h2d, d2h = run_e2e(r, inp, steps, torch, barrier)
    e_ms, e_pairs_per_s = aggregate_ranks(e_total, r.pairs, steps, world, rmax)

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, one GPU only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        v, sample, _, secs = oracle_sample(name, inp, budget_s=cpu_budget_s)
        cpu = {"value": v, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
               "sample": sample, "seconds": round(secs, 2)}
    c = r.c
    rec = {
        "value": pairs_per_s / 1e9, "unit": UNIT, "steps": steps, "ms_per_step": total_ms / steps,
        "dtype": r.dtype,
        "config": workload_config(c, r.batch, r.label, inp.q_offset, r.pairs, world),
        "queries_per_s": world * r.batch * c["T"] * steps / (total_ms / 1e3),
        "roofline": roof, "kernels": per_kernel, "cpu_baseline": cpu,
        "e2e": {"value": e_pairs_per_s / 1e9, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e_ms / steps, "pipeline": "2 buffer sets, copy-in / call / copy-out streams",
                **({"key_cache": "resident; each step copies one new key row (and scale) per sequence"}
                   if r.c.get("kind") == "decode" else {})},
        "gpu_launches": int(round(launches_per_step * steps)), "clocks": clocks,
        "step_ms": {"min": min(times), "median": statistics.median(times), "max": max(times)},
    }
    if dosa is not None:
        rec["dosa"] = dosa
    del r, inp
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="all", choices=["all", "tiny", "dsa", "decode", "misa", "hisa", "dsa_fp8", "indexcache", "dosa",
                             "dosa_lownorm", "dsa_lists", "hisa_decode", "misa_decode"],
                    help="all (default): the dsa chunk is the headline line, the other four "
                         "workloads are measured in the same run under 'workloads'")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--queries", type=int, default=0,
                    help="profiling: use only the last N queries of the chunk")
    ap.add_argument("--batch", type=int, default=0,
                    help="profiling: use only the first N sequences (decode)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

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

    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    head = "dsa" if args.workload == "all" else args.workload
    rmax = dist_max(dist, "cuda") if world > 1 else None

    rec = measure_workload(head, args, torch, world, rank, local, flush, barrier, rmax, args.steps, 10.0)
    subs = {}
    if args.workload == "all":
        for name in SUB_WORKLOADS:
            subs[name] = measure_workload(name, args, torch, world, rank, local, flush, barrier, rmax,
                                          args.steps, 5.0, min_timed_ms=MIN_TIMED_MS)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": rec["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": rec["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": rec["dtype"], "data": "synthetic",
        "config": rec["config"], "queries_per_s": rec["queries_per_s"], "roofline": rec["roofline"],
        "kernels": rec["kernels"], "cpu_baseline": rec["cpu_baseline"], "e2e": rec["e2e"],
        "gpu_launches": rec["gpu_launches"], "clocks": rec["clocks"], "step_ms": rec["step_ms"],
    }
    if subs:
        line["workloads"] = subs
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
