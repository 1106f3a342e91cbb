"""fp64 CPU oracle for the lightning indexer and its MISA / HISA variants.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may use it. The CUDA path never imports it, and
it imports nothing from the CUDA path. It reads the same rounded host buffers
that the GPU reads (built by ``sparse_attention_token_score_b200.workloads``),
widens them exactly to fp64 and follows the pages' steps in order:

* dense indexer + top-k ("MISA: Mixture of Indexer Sparse Attention for
  Long-Context LLM Inference", section "Problem statement"): score every
  causal-prefix token with all H_I heads, keep the k best.
* MISA (same page, section "Methodology"): split the prefix into
  M = ceil(L/B) blocks, mean-pool the keys of each block, compute a per-head
  affinity from the pooled keys, keep the top-h heads per query, score all
  tokens with those heads only, keep the top-k.
* MISA-dagger (same page, "Hierarchical variant"): the routed pass keeps k'
  candidates, the full H_I-head indexer re-scores them, keep the top-k.
* HISA ("HISA: Efficient Hierarchical Indexing for Fine-Grained Sparse
  Attention" review, section 3): score pooled block keys, keep the top-m
  blocks, score the tokens of the surviving blocks, keep the top-k. On an
  FP8 key cache the pooled keys of MISA and HISA are kept in the cache's
  format (e4m3 with a per-block scale).
* IndexCache ("IndexCache: Accelerating Sparse Attention via Cross-Layer
  Index Reuse", section 2): layers marked F run their own indexer and cache
  its top-k; layers marked S skip the indexer and reuse the cache of the
  nearest preceding F layer.
* DoSA certified pruning ("DoSA: Dots Sparse Attention" review, section 3):
  a seed set scored with all heads bounds the k-th score from below, a
  screened subset of heads bounds every other key's score from above, keys
  whose bound is below the seeds' threshold are pruned, the survivors are
  scored with all heads; the selection equals the dense one.

Readings where the pages are silent (each is listed in the design notes):
* Ties in any selection go to the lower index; a selection over fewer
  candidates than asked returns all of them, padded with -1; selected indices
  are returned in ascending order.
* A query at absolute position p sees keys s <= p; a pooled block m is visible
  when its first token is (m*B <= p). Pooled keys are the bf16-rounded fp64
  mean of all tokens of the block (fewer in a partial last block).
* Routed scoring uses the chosen heads' original signed weights, with no
  renormalisation.
* FP8 inputs are dequantised exactly (scale * decoded byte) and scored in the
  unfactored form.
* DoSA: the page names its bounds but gives no formulas; the upper bound
  here keeps the screened heads' exact terms, bounds the unscreened
  positive-weight heads jointly through ReLU(x) = (x + |x|) / 2 (one
  aggregated dot product plus Cauchy-Schwarz on |x|) and subtracts ReLU of
  one aggregated dot product for the unscreened negative-weight heads
  (subadditivity of ReLU); the seeds are the keys with the largest screened
  partial scores.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "indexer_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C core with gcc (-O2, no fast-math: sums stay sequential)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _core():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        lib.or_score_pairs.argtypes = [P, P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_longlong,
                                       P, P, P, P]
        lib.or_score_pairs.restype = None
        lib.or_router.argtypes = [P, P, P, ctypes.c_longlong, ctypes.c_int, ctypes.c_int,
                                  ctypes.c_longlong, P, P]
        lib.or_router.restype = None
        lib.or_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_core().or_num_threads())


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# ------------------------------------------------------------ number formats
def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp64 (exact): the pattern is the top half of an fp32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _e4m3_value(code: int) -> float:
    """Value of an OCP FP8 E4M3 code: 1 sign, 4 exponent (bias 7), 3 mantissa
    bits; exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; no infinities."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    """FP8 e4m3 bytes -> fp64 (exact)."""
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


# e4m3 codes 0x00 .. 0x7E (non-negative finite values, increasing with the code)
_E4M3_POS = E4M3_TABLE[:0x7F]


def f64_to_e4m3(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to OCP FP8 E4M3 codes: nearest representable value,
    ties to the even code (even mantissa), saturating at +-448; zero keeps its
    sign. Brute force over the 127 non-negative finite codes."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), 448.0)
    d = np.abs(a[..., None] - _E4M3_POS)                     # distance to every code
    best = d.min(axis=-1, keepdims=True)
    cand = d == best
    # ties: two neighbours at the same distance; take the even code
    code = np.where(cand.sum(-1) > 1, np.argmax(cand & (np.arange(0x7F) % 2 == 0), axis=-1),
                    np.argmax(cand, axis=-1)).astype(np.uint8)
    sign = np.signbit(x).astype(np.uint8) << 7
    return code | sign


def meanpool_e4m3(k_codes: np.ndarray, k_scale: np.ndarray, B: int):
    """Pooled keys of an FP8 cache, stored in the cache's format: the fp64
    mean of the block's dequantised keys, a scale absmax/448 (fp32 absmax
    divided in fp32; 1 when the mean is zero), codes e4m3(mean / scale).
    Returns (codes [M, d] uint8, scales [M] fp32)."""
    k = decode_e4m3(k_codes) * np.asarray(k_scale, dtype=np.float64)[:, None]
    L, d = k.shape
    M = -(-L // B)
    codes = np.empty((M, d), dtype=np.uint8)
    scales = np.empty(M, dtype=np.float32)
    for m in range(M):
        blk = k[m * B:min((m + 1) * B, L)]
        mean = blk.sum(axis=0) / blk.shape[0]
        amax = np.float32(np.max(np.abs(mean)))
        sc = np.float32(amax / np.float32(448.0)) if amax > 0 else np.float32(1.0)
        scales[m] = sc
        codes[m] = f64_to_e4m3(mean / np.float64(sc))
    return codes, scales


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 to bf16 directly (nearest, ties to even), no intermediate fp32.

    bf16 keeps 7 of fp64's 52 fraction bits; rounding adds half an ulp minus one
    plus the kept lsb to the 45 dropped bits, then truncates. Valid for zero and
    for normal values inside the bf16 exponent range (all the pooled keys here)."""
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    if np.any((ax != 0) & ((ax < 2.0 ** -126) | (ax >= 2.0 ** 127))):
        raise ValueError("f64_to_bf16_bits: value outside the normal bf16 range")
    u = x.view(np.uint64)
    lsb = (u >> np.uint64(45)) & np.uint64(1)
    u = (u + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    f32 = u.view(np.float64).astype(np.float32)  # exact: 8 significant bits, in range
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# ------------------------------------------------------------ inputs -> fp64
def dequant(inp, b: int = 0):
    """fp64 (q [T,H,d], k [L,d], w [T,H]) of sequence ``b``."""
    if inp.dtype == "bf16":
        q = widen_bf16(inp.q[b])
        k = widen_bf16(inp.k[b])
    else:
        q = decode_e4m3(inp.q[b]) * inp.q_scale[b].astype(np.float64)[..., None]
        k = decode_e4m3(inp.k[b]) * inp.k_scale[b].astype(np.float64)[:, None]
    return q, k, inp.w[b].astype(np.float64)


# ------------------------------------------------------------ primitives
def score_pairs(q: np.ndarray, k: np.ndarray, w: np.ndarray, pq: np.ndarray, pk: np.ndarray,
                hmask: Optional[np.ndarray] = None):
    """Indexer score of pairs (pq[i], pk[i]): returns (score, cond), fp64.

    score = sum_h w[t,h] ReLU(q[t,h].k[s]);  cond = sum_h |w[t,h]| ReLU(q[t,h].k[s]).
    ``hmask`` [T,H] (uint8) restricts the sum to the marked heads."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    w = np.ascontiguousarray(w, dtype=np.float64)
    T, H, d = q.shape
    assert k.shape[1] == d and w.shape == (T, H)
    pq = np.ascontiguousarray(pq, dtype=np.int64)
    pk = np.ascontiguousarray(pk, dtype=np.int64)
    assert pq.shape == pk.shape
    if pq.size:
        assert pq.min() >= 0 and pq.max() < T and pk.min() >= 0 and pk.max() < k.shape[0]
    hm = None if hmask is None else np.ascontiguousarray(hmask, dtype=np.uint8)
    if hm is not None:
        assert hm.shape == (T, H)
    out = np.empty(pq.shape, dtype=np.float64)
    cond = np.empty(pq.shape, dtype=np.float64)
    _core().or_score_pairs(_ptr(q), _ptr(k), _ptr(w), _ptr(hm), H, d, pq.size, _ptr(pq), _ptr(pk),
                           _ptr(out), _ptr(cond))
    return out, cond


def select_topk(scores: np.ndarray, k: int, index: Optional[np.ndarray] = None) -> np.ndarray:
    """The k best candidates by (score descending, index ascending).

    NaN scores mark candidates that do not exist. Returns their indices
    (``index[j]`` if given, else j) in ascending order, padded with -1 to k."""
    scores = np.asarray(scores, dtype=np.float64)
    idx = np.arange(scores.size, dtype=np.int64) if index is None else np.asarray(index, dtype=np.int64)
    ok = ~np.isnan(scores)
    s, ix = scores[ok], idx[ok]
    order = np.lexsort((ix, -s))  # primary: -score ascending; secondary: index ascending
    chosen = np.sort(ix[order[:k]])
    out = np.full(k, -1, dtype=np.int64)
    out[:chosen.size] = chosen
    return out


def kth_score(scores: np.ndarray, k: int, index: Optional[np.ndarray] = None) -> float:
    """Score of the k-th best candidate (NaN if there are fewer than k)."""
    s = np.asarray(scores, dtype=np.float64)
    s = s[~np.isnan(s)]
    if s.size < k or k <= 0:
        return float("nan")
    return float(np.sort(s)[::-1][k - 1])


def visible_count(p: np.ndarray, L: int) -> np.ndarray:
    """Keys visible to queries at absolute positions p: s <= p and s < L."""
    return np.clip(np.asarray(p, dtype=np.int64) + 1, 0, L)


def meanpool_bf16(k_bits: np.ndarray, B: int) -> np.ndarray:
    """Pooled keys kbar[m] = bf16(mean of k[mB : min((m+1)B, L)]) from bf16 keys
    [L, d] (MISA page, "Methodology", step 1: M = ceil(L/B) blocks, mean-pooled
    indexing keys). The mean is taken in fp64 and rounded once."""
    k = widen_bf16(k_bits)
    L, d = k.shape
    M = -(-L // B)
    out = np.empty((M, d), dtype=np.float64)
    for m in range(M):
        blk = k[m * B:min((m + 1) * B, L)]
        out[m] = blk.sum(axis=0) / blk.shape[0]
    return f64_to_bf16_bits(out)


# ------------------------------------------------------------ dense indexer
def dense_scores_row(q, k, w, t: int, p: int, keys: Optional[np.ndarray] = None):
    """Scores of query t (absolute position p) on ``keys`` (default: the whole
    visible prefix). Returns (keys, score, cond)."""
    L = k.shape[0]
    if keys is None:
        keys = np.arange(int(visible_count(p, L)), dtype=np.int64)
    pq = np.full(keys.shape, t, dtype=np.int64)
    s, c = score_pairs(q, k, w, pq, keys)
    return keys, s, c


def dense_topk(inp, topk: int, queries: Optional[Sequence[int]] = None, b: int = 0):
    """Dense lightning indexer + top-k for queries of sequence b.

    Returns dict with 'idx' [nq, topk] (ascending, -1 padded) and per query
    'scores' / 'cond' over the visible prefix."""
    q, k, w = dequant(inp, b)
    if queries is None:
        queries = range(q.shape[0])
    res = {"idx": [], "scores": [], "cond": [], "queries": list(queries)}
    for t in queries:
        keys, s, c = dense_scores_row(q, k, w, t, inp.q_offset + t)
        res["idx"].append(select_topk(s, topk))
        res["scores"].append(s)
        res["cond"].append(c)
    res["idx"] = np.array(res["idx"], dtype=np.int64).reshape(len(res["queries"]), topk)
    return res


# ------------------------------------------------------------ MISA
def router_affinity(q: np.ndarray, kbar: np.ndarray, w: np.ndarray, nvis_blocks: np.ndarray):
    """a[t,h] = |w[t,h]| * sum_{m < nvis[t]} ReLU(q[t,h].kbar[m]) (fp64)."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    kbar = np.ascontiguousarray(kbar, dtype=np.float64)
    w = np.ascontiguousarray(w, dtype=np.float64)
    T, H, d = q.shape
    nv = np.ascontiguousarray(nvis_blocks, dtype=np.int64)
    assert nv.shape == (T,)
    a = np.empty((T, H), dtype=np.float64)
    _core().or_router(_ptr(q), _ptr(kbar), _ptr(w), T, H, d, kbar.shape[0], _ptr(nv), _ptr(a))
    return a


def visible_blocks(p: np.ndarray, B: int, M: int) -> np.ndarray:
    """Blocks whose first token is visible: m*B <= p, m < M."""
    return np.clip(np.asarray(p, dtype=np.int64) // B + 1, 0, M)


def misa(inp, block: int, h: int, topk: int, kprime: int = 0,
         queries: Optional[Sequence[int]] = None, b: int = 0,
         heads_given: Optional[np.ndarray] = None, cand_given: Optional[np.ndarray] = None):
    """MISA routed indexer (kprime == 0) or MISA-dagger (kprime > 0).

    bf16 or FP8 inputs: with an FP8 cache every stage reads the dequantised
    values (q = q_scale * e4m3(q), k = k_scale * e4m3(k)) and the pooled keys
    stay in the cache's format (``meanpool_e4m3``), as in ``hisa``.

    heads_given [nq, h] / cand_given [nq, kprime]: run the later stages on these
    choices instead of the oracle's own (lets a test condition each stage on
    the GPU's previous discrete choice). Returns a dict with every stage."""
    q, k, w = dequant(inp, b)
    T, H, d = q.shape
    L = k.shape[0]
    if queries is None:
        queries = np.arange(T)
    queries = np.asarray(queries, dtype=np.int64)
    if inp.dtype == "bf16":
        kbar_bits = meanpool_bf16(inp.k[b], block)
        kbar = widen_bf16(kbar_bits)
    else:  # FP8 cache: pooled keys in the cache's format, as for HISA
        codes, scales = meanpool_e4m3(inp.k[b], inp.k_scale[b], block)
        kbar_bits = (codes, scales)
        kbar = decode_e4m3(codes) * scales.astype(np.float64)[:, None]
    M = kbar.shape[0]
    p = inp.q_offset + queries
    a = router_affinity(q[queries], kbar, w[queries], visible_blocks(p, block, M))
    heads = np.stack([select_topk(a[i], h) for i in range(len(queries))]) if heads_given is None \
        else np.asarray(heads_given, dtype=np.int64)
    out = {"kbar_bits": kbar_bits, "affinity": a, "heads": heads, "queries": queries,
           "routed_scores": [], "routed_cond": [], "idx": [], "cand": [], "scores": [], "cond": []}
    for i, t in enumerate(queries):
        hm = np.zeros((T, H), dtype=np.uint8)
        hm[t, heads[i][heads[i] >= 0]] = 1
        V = int(visible_count(p[i], L))
        keys = np.arange(V, dtype=np.int64)
        sr, cr = score_pairs(q, k, w, np.full(V, t, dtype=np.int64), keys, hmask=hm)
        out["routed_scores"].append(sr)
        out["routed_cond"].append(cr)
        if kprime <= 0:
            out["idx"].append(select_topk(sr, topk))
            continue
        cand = select_topk(sr, kprime) if cand_given is None else np.asarray(cand_given[i], dtype=np.int64)
        out["cand"].append(cand)
        cv = cand[cand >= 0]
        _, s, c = dense_scores_row(q, k, w, int(t), int(p[i]), keys=cv)
        out["scores"].append(s)
        out["cond"].append(c)
        out["idx"].append(select_topk(s, topk, index=cv))
    out["idx"] = np.array(out["idx"], dtype=np.int64).reshape(len(queries), topk)
    return out


# ------------------------------------------------------------ HISA
def hisa(inp, block: int, m: int, topk: int, queries: Optional[Sequence[int]] = None, b: int = 0,
         blocks_given: Optional[np.ndarray] = None):
    """HISA: block-level coarse filter on pooled keys (top-m blocks), then
    token-level scoring inside the surviving blocks (top-k).

    blocks_given [nq, m]: run the token stage on these blocks instead of the
    oracle's own choice."""
    q, k, w = dequant(inp, b)
    T, H, d = q.shape
    L = k.shape[0]
    if queries is None:
        queries = np.arange(T)
    queries = np.asarray(queries, dtype=np.int64)
    if inp.dtype == "bf16":
        kbar_bits = meanpool_bf16(inp.k[b], block)
        kbar = widen_bf16(kbar_bits)
    else:  # FP8 cache: pooled keys in the cache's format (meanpool_e4m3)
        codes, scales = meanpool_e4m3(inp.k[b], inp.k_scale[b], block)
        kbar_bits = (codes, scales)
        kbar = decode_e4m3(codes) * scales.astype(np.float64)[:, None]
    M = kbar.shape[0]
    p = inp.q_offset + queries
    nvb = visible_blocks(p, block, M)
    out = {"kbar_bits": kbar_bits, "queries": queries, "block_scores": [], "block_cond": [],
           "blocks": [], "idx": [], "tokens": [], "scores": [], "cond": []}
    for i, t in enumerate(queries):
        bidx = np.arange(nvb[i], dtype=np.int64)
        sb, cb = score_pairs(q[t][None], kbar, w[t][None], np.zeros(bidx.size, dtype=np.int64), bidx)
        out["block_scores"].append(sb)
        out["block_cond"].append(cb)
        blocks = select_topk(sb, m) if blocks_given is None else np.asarray(blocks_given[i], dtype=np.int64)
        out["blocks"].append(blocks)
        bv = blocks[blocks >= 0]
        toks = (bv[:, None] * block + np.arange(block, dtype=np.int64)[None, :]).reshape(-1)
        toks = np.sort(toks[toks < visible_count(p[i], L)])
        _, s, c = dense_scores_row(q, k, w, int(t), int(p[i]), keys=toks)
        out["tokens"].append(toks)
        out["scores"].append(s)
        out["cond"].append(c)
        out["idx"].append(select_topk(s, topk, index=toks))
    out["blocks"] = np.array(out["blocks"], dtype=np.int64).reshape(len(queries), m)
    out["idx"] = np.array(out["idx"], dtype=np.int64).reshape(len(queries), topk)
    return out


# ------------------------------------------------------------ IndexCache
def indexcache(layer_inputs, pattern: str, topk: int):
    """Per-layer top-k indices [batch, T, topk] of an F/S layer pattern: an F
    layer runs the dense indexer on its own inputs (dense_topk, every sequence)
    and becomes the cache; an S layer returns the cache of the nearest F layer
    before it. pattern[0] must be 'F'."""
    if len(pattern) != len(layer_inputs) or not pattern or pattern[0] != "F" or set(pattern) - {"F", "S"}:
        raise ValueError("pattern: one 'F' or 'S' per layer, starting with 'F'")
    out, cache = [], None
    for inp, role in zip(layer_inputs, pattern):
        if role == "F":
            cache = np.stack([dense_topk(inp, topk, b=b)["idx"] for b in range(inp.batch)])
        out.append(cache)
    return out


# ------------------------------------------------------------ DoSA (certified pruning)
def dosa_upper_bound(q, k, w, t: int, keys: np.ndarray, screen: Sequence[int]):
    """Upper bound on I[t,s] for each key s in ``keys`` from a subset of
    heads ("DoSA: Dots Sparse Attention" review, section 3: screening dot
    products and bound evaluation; the page names a seed-set threshold,
    nonnegative head projection, joint residual bounds and an aggregate of the
    omitted negative heads, without formulas). With x_h = q_h.k_s:
      - screened heads contribute their exact terms w_h ReLU(x_h);
      - unscreened heads with w_h > 0 (set P): ReLU(x) = (x + |x|) / 2 gives
        sum_P w_h ReLU(x_h) <= (k_s.v_P + A_P ||k_s||) / 2 with the aggregate
        v_P = sum_P w_h q_h and A_P = sum_P w_h ||q_h|| (|x_h| <= ||q_h|| ||k_s||);
      - unscreened heads with w_h < 0 (set N): ReLU is subadditive, so
        sum_N |w_h| ReLU(x_h) >= ReLU(k_s.v_N) with v_N = sum_N |w_h| q_h, and
        their (negative) contribution is at most -ReLU(k_s.v_N).
    A relative slack of 1e-12 covers fp64 rounding. Returns (bound, screened
    part of the score)."""
    T, H, _ = q.shape
    screen = np.unique(np.asarray(screen, dtype=np.int64))
    hmask = np.zeros((T, H), dtype=np.uint8)
    hmask[t, screen] = 1
    keys = np.asarray(keys, dtype=np.int64)
    part, pcond = score_pairs(q, k, w, np.full(keys.shape, t, dtype=np.int64), keys, hmask)
    rest = np.setdiff1d(np.arange(H), screen)
    wt = np.asarray(w[t], dtype=np.float64)
    qt = np.asarray(q[t], dtype=np.float64)
    kk = np.asarray(k, dtype=np.float64)[keys]
    pos, neg = rest[wt[rest] > 0], rest[wt[rest] < 0]
    v_p = (wt[pos, None] * qt[pos]).sum(0)
    a_p = float(np.sum(wt[pos] * np.linalg.norm(qt[pos], axis=1))) if pos.size else 0.0
    v_n = (-wt[neg, None] * qt[neg]).sum(0)
    kn = np.linalg.norm(kk, axis=1)
    lin_p = kk @ v_p
    up = 0.5 * (lin_p + a_p * kn)
    down = np.maximum(kk @ v_n, 0.0)
    slack = 1e-12 * (pcond + a_p * kn + np.abs(lin_p) + down) + 1e-300
    return part + up - down + slack, part


def dosa_topk(inp, topk: int, screen: Sequence[int], n_seed: int,
              queries: Optional[Sequence[int]] = None, b: int = 0):
    """Certified exact top-k (DoSA review, section 3), per query:
      1. the n_seed visible keys with the largest screened part of the score
         (ties -> lower index) are scored with all heads; the topk-th best of
         them, tau, is a lower bound on the row's k-th best score (-inf when
         the seeds are fewer than topk);
      2. every other visible key whose upper bound (dosa_upper_bound) is below
         tau cannot be selected and is pruned;
      3. the surviving keys are scored with all heads;
      4. top-k (score descending, index ascending) over seeds and survivors.
    The result equals dense_topk (lossless). Returns dict with 'idx'
    [nq, topk], per query 'tau', 'survivors' (keys scored in step 3) and
    'visible'."""
    q, k, w = dequant(inp, b)
    if queries is None:
        queries = range(q.shape[0])
    res = {"idx": [], "tau": [], "survivors": [], "visible": [], "queries": list(queries)}
    for t in queries:
        keys = np.arange(int(visible_count(inp.q_offset + t, k.shape[0])), dtype=np.int64)
        bound, part = dosa_upper_bound(q, k, w, t, keys, screen)
        order = np.lexsort((keys, -part))
        seeds = np.sort(keys[order[:n_seed]])
        _, s_seed, _ = dense_scores_row(q, k, w, t, inp.q_offset + t, keys=seeds)
        tau = kth_score(s_seed, topk) if seeds.size >= topk else -np.inf
        rest = np.setdiff1d(keys, seeds)
        keep = rest[~(bound[rest] < tau)]
        _, s_keep, _ = dense_scores_row(q, k, w, t, inp.q_offset + t, keys=keep)
        cand = np.concatenate([seeds, keep])
        res["idx"].append(select_topk(np.concatenate([s_seed, s_keep]), topk, index=cand))
        res["tau"].append(tau)
        res["survivors"].append(int(keep.size))
        res["visible"].append(int(keys.size))
    res["idx"] = np.array(res["idx"], dtype=np.int64).reshape(len(res["queries"]), topk)
    return res



def dosa_screen_heads(q_t: np.ndarray, w_t: np.ndarray, n_screen: int) -> np.ndarray:
    """The screened heads of one query: the n_screen heads with the largest
    |w_h| * ||q_h|| (the heads that can move the score most; ties -> lower h),
    ascending."""
    g = np.abs(np.asarray(w_t, dtype=np.float64)) * np.linalg.norm(np.asarray(q_t, dtype=np.float64), axis=1)
    sel = select_topk(g, n_screen)
    return sel[sel >= 0]


def sample_threshold(sample_scores: np.ndarray, k: int, V: int) -> float:
    """A threshold the k-th best of V scores is very likely to reach, from the
    scores of every S-th key (ns of them): the r_lo-th best sample with r_lo =
    ceil(ns p + 4 sqrt(ns p (1 - p)) + 4), p = k / V; -inf when V <= k or the
    sample is too small. Any value is safe for the exact selection that uses
    it (the count of scores reaching it is checked); it only decides how much
    work is skipped."""
    ns = int(np.size(sample_scores))
    if V <= k:
        return -np.inf
    p = k / V
    r_lo = int(np.ceil(ns * p + 4.0 * np.sqrt(ns * p * (1.0 - p)) + 4.0))
    if r_lo > ns:
        return -np.inf
    return float(np.sort(np.asarray(sample_scores, dtype=np.float64))[::-1][r_lo - 1])


def dosa_tile_topk(inp, topk: int, n_screen: int, S: int, qpt: int, tile: int = 128, b: int = 0,
                   groups: Optional[Sequence[int]] = None):
    """DoSA certified pruning at tile granularity ("DoSA: Dots Sparse
    Attention" review, section 3: screening dot products, bound evaluation,
    pruning and candidate compaction, full-head dot products of the survivors,
    original-score reduction with sparse writeback, exact selection), for the
    queries of sequence b grouped qpt at a time (the queries that share a
    tensor-core tile) and keys in tiles of `tile`:
      1. per query, a threshold thr from the full scores of every S-th visible
         key (sample_threshold);
      2. per query and key, the upper bound of dosa_upper_bound with the
         query's n_screen screened heads (dosa_screen_heads);
      3. a key tile stays live for a group when some query of the group has a
         visible key in it whose bound reaches that query's thr; other tiles
         are pruned (every key in them scores below thr for every query);
      4. each query scores the visible keys of its group's live tiles; if at
         least min(k, V) of those scores reach thr (the certificate: the k-th
         best of the row then reaches thr, so no pruned key can be a winner),
         the top-k comes from them, else from the whole row (fallback);
      5. top-k (score descending, index ascending).
    The result equals dense_topk. Returns dict with 'idx' [nq, topk] (queries
    of the groups, in order), 'queries', 'thr', 'live' [n_groups, n_tiles]
    (1 live, 0 pruned), 'fallback' per query and 'groups'."""
    q, k, w = dequant(inp, b)
    T, H, _ = q.shape
    L = k.shape[0]
    n_groups = -(-T // qpt)
    n_tiles = -(-L // tile)
    groups = range(n_groups) if groups is None else groups
    out = {"idx": [], "queries": [], "thr": [], "fallback": [], "groups": list(groups),
           "live": np.zeros((len(groups), n_tiles), dtype=np.uint8)}
    for gi, g in enumerate(groups):
        qs = list(range(g * qpt, min(T, (g + 1) * qpt)))
        rows = []
        for t in qs:
            p = inp.q_offset + t
            V = int(visible_count(p, L))
            _, samp, _ = dense_scores_row(q, k, w, t, p, keys=np.arange(0, V, S, dtype=np.int64))
            thr = sample_threshold(samp, topk, V)
            keys = np.arange(V, dtype=np.int64)
            bound, _ = dosa_upper_bound(q, k, w, t, keys, dosa_screen_heads(q[t], w[t], n_screen))
            live_keys = keys[bound >= thr]
            out["live"][gi, np.unique(live_keys // tile)] = 1
            rows.append((t, p, V, thr))
        for t, p, V, thr in rows:
            keys = np.arange(V, dtype=np.int64)
            cand = keys[out["live"][gi, keys // tile] == 1]
            _, s, _ = dense_scores_row(q, k, w, t, p, keys=cand)
            fb = int(np.sum(s >= thr)) < min(topk, V)
            if fb:
                _, s, _ = dense_scores_row(q, k, w, t, p)
                cand = keys
            out["idx"].append(select_topk(s, topk, index=cand))
            out["queries"].append(t)
            out["thr"].append(thr)
            out["fallback"].append(fb)
    out["idx"] = np.array(out["idx"], dtype=np.int64).reshape(len(out["queries"]), topk)
    return out
