"""Seeded synthetic inputs for the lightning-indexer workloads.

This module only draws random numbers and rounds them to the storage types the
indexer reads (bf16 bit patterns, FP8 e4m3 bytes with fp32 scales, fp32 head
weights). It holds none of the indexer's arithmetic: no scores, no ReLU, no
selection. Both the CUDA path (through the C-ABI) and the fp64 oracle consume
exactly the buffers built here, so every comparison starts from the same
rounded inputs.

Distributions follow the five workloads the indexer is measured on:

* ``tiny``   causal prefill, T=L=2048, H_I=8, d=64, top-k=256
* ``dsa``    DSA-shaped chunk: T=4096 queries at the end of a 32768 prefix,
             H_I=64 (DeepSeek-V3.2 head count), d=128, top-k=2048, 64 planted
             needle keys
* ``decode`` 64 one-token queries over a 131072-token FP8 e4m3 K cache
             (per-token scale absmax/448), 1% of tokens copies of 16 shared
             cluster centres
* ``misa``   T=2048 at the end of a 131072 prefix, H_I=64, block 64, top-8
             heads, top-k=2048, MISA-dagger k'=8192
* ``hisa``   T=1024 at the end of a 262144 prefix, H_I=32 (GLM-5 head count),
             block 128, top-128 blocks, top-k=2048, recency ramp on key dim 0
* ``indexcache`` four layers of ``dsa`` chunks with the IndexCache pattern
             FSSS: one layer runs the indexer, three reuse its indices (only
             the F layer has inputs: S layers compute no indexer projections)
* ``hisa_decode`` HISA (block 128, top-128 blocks) on the ``decode`` FP8 cache
* ``misa_decode`` MISA-dagger (block 64, top-8 heads, k'=8192) on the ``decode``
             FP8 cache
* ``dsa_lists`` the ``dsa`` chunk through the candidate-list selection
* ``dosa``   the ``dsa`` chunk through DoSA's certified pruning (5 screened heads)
* ``dosa_lownorm`` the ``dsa`` shape with three of every four key tiles shrunk
             100x and non-negative head weights: most tiles can be pruned
* ``dsa_fp8`` the ``dsa`` chunk quantised to FP8 e4m3 the way the decode cache
             is (per-token key scale, per-(query, head) query scale)

Random streams: one numpy PCG64 stream per tensor, spawned from
``SeedSequence(seed)``; the decode K cache uses one child stream per sequence so
the values do not depend on how generation is chunked.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

E4M3_MAX = 448.0


# ----------------------------------------------------------------- rounding
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); return the
    16-bit patterns. Inputs here are finite and far from the fp32 overflow
    threshold, so the carry never reaches the sign bit."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_e4m3_bytes(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to OCP FP8 e4m3 (finite-only variant), saturating at
    +-448. Uses torch's round-to-nearest-even conversion on the host."""
    import torch

    x = np.clip(np.asarray(x, dtype=np.float32), -E4M3_MAX, E4M3_MAX)
    t = torch.from_numpy(np.ascontiguousarray(x)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy().copy()


def absmax_scale(x: np.ndarray, axis: int = -1) -> np.ndarray:
    """Per-row quantisation scale absmax/448 in fp32; 1 where the row is all zero."""
    amax = np.max(np.abs(x), axis=axis).astype(np.float32)
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    s[amax == 0] = np.float32(1.0)
    return s


def quantize_rows_e4m3(x: np.ndarray):
    """Per-row (last axis) e4m3 quantisation: returns (bytes, fp32 scale)."""
    s = absmax_scale(x, axis=-1)
    q = f32_to_e4m3_bytes(x / s[..., None])
    return q, s


# ----------------------------------------------------------------- containers
@dataclass
class IndexerInputs:
    """Host buffers of one indexer problem.

    q:  [batch, T, H, d]  uint16 (bf16 bits) or uint8 (e4m3 bytes)
    k:  [batch, L, d]     uint16 (bf16 bits) or uint8 (e4m3 bytes)
    w:  [batch, T, H]     float32, signed
    q_scale: [batch, T, H] float32 (e4m3 only)
    k_scale: [batch, L]    float32 (e4m3 only)
    q_offset: absolute position of query 0 of every sequence; query t sees
              keys s <= q_offset + t.
    """

    q: np.ndarray
    k: np.ndarray
    w: np.ndarray
    q_offset: int
    dtype: str = "bf16"  # "bf16" or "fp8_e4m3"
    q_scale: Optional[np.ndarray] = None
    k_scale: Optional[np.ndarray] = None
    meta: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return self.q.shape[0]

    @property
    def T(self) -> int:
        return self.q.shape[1]

    @property
    def H(self) -> int:
        return self.q.shape[2]

    @property
    def d(self) -> int:
        return self.q.shape[3]

    @property
    def L(self) -> int:
        return self.k.shape[1]


def _streams(seed: int, n: int):
    return [np.random.Generator(np.random.PCG64(s)) for s in np.random.SeedSequence(seed).spawn(n)]


def prefill_inputs(T: int, L: int, H: int, d: int, q_offset: Optional[int] = None,
                   seed: int = 0, batch: int = 1, w_std: Optional[float] = None,
                   needles: int = 0, recency: float = 0.0) -> IndexerInputs:
    """bf16 prefill chunk: q, k ~ N(0,1)/sqrt(d), w ~ N(0,1)*w_std (default
    1/sqrt(H)). ``q_offset`` defaults to L - T (chunk at the end of the prefix).

    needles: per sequence, that many distinct key positions uniform in
      [0, q_offset) are overwritten with bf16(0.5 * mean over heads of the
      bf16 query vectors of a uniformly drawn chunk query).
    recency: adds recency * s / L to key component 0 before rounding.
    """
    if q_offset is None:
        q_offset = L - T
    if w_std is None:
        w_std = 1.0 / np.sqrt(H)
    rq, rk, rw, rn = _streams(seed, 4)
    inv = np.float32(1.0 / np.sqrt(d))
    q32 = rq.standard_normal((batch, T, H, d), dtype=np.float32) * inv
    k32 = rk.standard_normal((batch, L, d), dtype=np.float32) * inv
    if recency:
        k32[:, :, 0] += (np.float32(recency) * np.arange(L, dtype=np.float32) / np.float32(L))[None, :]
    w = (rw.standard_normal((batch, T, H), dtype=np.float32) * np.float32(w_std)).astype(np.float32)
    q = f32_to_bf16_bits(q32)
    k = f32_to_bf16_bits(k32)
    meta = {}
    if needles:
        hi = min(q_offset, L)
        assert hi >= needles, "needle range [0, q_offset) too small"
        pos_all, src_all = [], []
        for b in range(batch):
            pos = rn.choice(hi, size=needles, replace=False)
            src = rn.integers(0, T, size=needles)
            qv = bf16_bits_to_f32(q[b, src])  # [needles, H, d]
            k[b, pos] = f32_to_bf16_bits(np.float32(0.5) * qv.mean(axis=1, dtype=np.float32))
            pos_all.append(pos)
            src_all.append(src)
        meta["needle_pos"] = np.stack(pos_all)
        meta["needle_src"] = np.stack(src_all)
    return IndexerInputs(q=q, k=k, w=w, q_offset=int(q_offset), dtype="bf16", meta=meta)


def decode_inputs(batch: int, L: int, H: int, d: int, seed: int = 0,
                  cluster_frac: float = 0.01, n_centres: int = 16,
                  w_std: float = 0.125) -> IndexerInputs:
    """FP8 decode: one query per sequence at position L-1.

    Keys ~ N(0,1); each token independently (prob ``cluster_frac``) is replaced
    by an exact copy of one of ``n_centres`` shared centres ~ N(0,1). Keys are
    quantised per token to e4m3 with scale absmax/448. q ~ N(0,1)/sqrt(d),
    quantised per head. w ~ N(0,1) * w_std.
    """
    streams = _streams(seed, 4 + batch)
    rq, rw, rc, rsel = streams[:4]
    kst = streams[4:]
    centres = rc.standard_normal((n_centres, d), dtype=np.float32)
    k8 = np.empty((batch, L, d), dtype=np.uint8)
    ks = np.empty((batch, L), dtype=np.float32)

    def one_sequence(b):
        kb = kst[b].standard_normal((L, d), dtype=np.float32)
        pick = kst[b].random(L) < cluster_frac
        which = kst[b].integers(0, n_centres, size=L)
        kb[pick] = centres[which[pick]]
        k8[b], ks[b] = quantize_rows_e4m3(kb)
        return int(pick.sum())

    # every sequence draws from its own stream, so the values do not depend
    # on the order the threads run in
    with ThreadPoolExecutor(max_workers=max(1, min(16, os.cpu_count() or 1, batch))) as ex:
        n_clustered = sum(ex.map(one_sequence, range(batch)))
    q32 = rq.standard_normal((batch, 1, H, d), dtype=np.float32) * np.float32(1.0 / np.sqrt(d))
    q8, qs = quantize_rows_e4m3(q32)
    w = (rw.standard_normal((batch, 1, H), dtype=np.float32) * np.float32(w_std)).astype(np.float32)
    return IndexerInputs(q=q8, k=k8, w=w, q_offset=L - 1, dtype="fp8_e4m3",
                         q_scale=qs, k_scale=ks, meta={"clustered_tokens": n_clustered})


def fp8_prefill_inputs(T: int, L: int, H: int, d: int, q_offset: Optional[int] = None,
                       seed: int = 0, batch: int = 1, w_std: Optional[float] = None,
                       needles: int = 0) -> IndexerInputs:
    """FP8 prefill chunk: the bf16 chunk of ``prefill_inputs`` (same streams,
    needles included), widened to fp32 and quantised the way the decode cache
    is: keys per token, queries per (query, head) row, e4m3 with scale
    absmax/448."""
    base = prefill_inputs(T, L, H, d, q_offset=q_offset, seed=seed, batch=batch, w_std=w_std,
                          needles=needles)
    q8, qs = quantize_rows_e4m3(bf16_bits_to_f32(base.q))
    k8, ks = quantize_rows_e4m3(bf16_bits_to_f32(base.k))
    return IndexerInputs(q=q8, k=k8, w=base.w, q_offset=base.q_offset, dtype="fp8_e4m3",
                         q_scale=qs, k_scale=ks, meta=base.meta)


def lownorm_inputs(T: int, L: int, H: int, d: int, q_offset: Optional[int] = None, seed: int = 0,
                   w_std: Optional[float] = None, live_every: int = 4, shrink: float = 0.01) -> IndexerInputs:
    """A prefill chunk where most keys cannot rank high for any query: the
    keys of every 128-key tile except each live_every-th one are scaled by
    ``shrink`` before rounding, and the head weights are non-negative (|w|),
    so every query's best scores come from the full-norm tiles."""
    base = prefill_inputs(T, L, H, d, q_offset=q_offset, seed=seed, w_std=w_std)
    kf = bf16_bits_to_f32(base.k)
    tile = np.arange(L) // 128
    kf[:, tile % live_every != 0] *= np.float32(shrink)
    base.k = f32_to_bf16_bits(kf)
    base.w = np.abs(base.w)
    return base


# ----------------------------------------------------------------- workloads
CONFIGS = {
    "tiny": dict(kind="dense", T=2048, L=2048, H=8, d=64, q_offset=0, topk=256),
    "dsa": dict(kind="dense", T=4096, L=32768, H=64, d=128, q_offset=28672, topk=2048,
                needles=64, w_std=0.125),
    "decode": dict(kind="decode", batch=64, T=1, L=131072, H=64, d=128, topk=2048),
    "indexcache": dict(kind="indexcache", pattern="FSSS", T=4096, L=32768, H=64, d=128, q_offset=28672,
                       topk=2048, needles=64, w_std=0.125),
    "hisa_decode": dict(kind="decode", batch=64, T=1, L=131072, H=64, d=128, topk=2048, block=128, m=128),
    "misa_decode": dict(kind="decode", batch=64, T=1, L=131072, H=64, d=128, topk=2048, block=64, h=8,
                        kprime=8192),
    "dsa_lists": dict(kind="dosa", T=4096, L=32768, H=64, d=128, q_offset=28672, topk=2048, needles=64,
                      w_std=0.125),
    "dosa": dict(kind="dosa", T=4096, L=32768, H=64, d=128, q_offset=28672, topk=2048, needles=64,
                 w_std=0.125, n_screen=5),
    "dosa_lownorm": dict(kind="dosa_lownorm", T=4096, L=32768, H=64, d=128, q_offset=28672, topk=2048,
                         w_std=0.125, n_screen=5, live_every=4, shrink=0.01),
    "dsa_fp8": dict(kind="dense_fp8", T=4096, L=32768, H=64, d=128, q_offset=28672, topk=2048,
                    needles=64, w_std=0.125),
    "misa": dict(kind="misa", T=2048, L=131072, H=64, d=128, q_offset=129024, topk=2048,
                 block=64, h=8, kprime=8192, w_std=0.125),
    "hisa": dict(kind="hisa", T=1024, L=262144, H=32, d=128, q_offset=261120, topk=2048,
                 block=128, m=128, recency=0.1),
}


def make_inputs(name: str, seed: int = 0) -> IndexerInputs:
    """Build the host inputs of a named workload (see module docstring)."""
    c = CONFIGS[name]
    if c["kind"] == "decode":
        return decode_inputs(c["batch"], c["L"], c["H"], c["d"], seed=seed)
    if c["kind"] == "dosa_lownorm":
        return lownorm_inputs(c["T"], c["L"], c["H"], c["d"], q_offset=c["q_offset"], seed=seed,
                              w_std=c["w_std"], live_every=c["live_every"], shrink=c["shrink"])
    if c["kind"] in ("indexcache", "dosa"):  # the dsa chunk (indexcache: its single F layer)
        return prefill_inputs(c["T"], c["L"], c["H"], c["d"], q_offset=c["q_offset"], seed=seed,
                              w_std=c.get("w_std"), needles=c.get("needles", 0))
    if c["kind"] == "dense_fp8":
        return fp8_prefill_inputs(c["T"], c["L"], c["H"], c["d"], q_offset=c["q_offset"], seed=seed,
                                  w_std=c.get("w_std"), needles=c.get("needles", 0))
    return prefill_inputs(c["T"], c["L"], c["H"], c["d"], q_offset=c["q_offset"], seed=seed,
                          w_std=c.get("w_std"), needles=c.get("needles", 0),
                          recency=c.get("recency", 0.0))


def visible_pairs(T: int, L: int, q_offset: int, batch: int = 1) -> int:
    """Number of (query, key) pairs with key <= query position, over all sequences."""
    p = q_offset + np.arange(T, dtype=np.int64)
    return int(batch * np.minimum(p + 1, L).clip(min=0).sum())
