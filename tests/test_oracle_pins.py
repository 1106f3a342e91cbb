"""Pins of the fp64 oracle against facts fixed by the pages and by mathematics,
not against a retyped copy of its own formulas:

* a hand-worked example (tests/golden/hand_example.json);
* algebraic identities of ReLU (ReLU(x) - ReLU(-x) = x, ReLU(x) + ReLU(-x) = |x|)
  evaluated through numpy matmuls, which catch a dropped ReLU, a flipped sign,
  a transposed operand or a wrong head weight;
* brute-force ranking (count of better candidates) for the selection rule;
* special cases where a variant provably reduces to the dense indexer
  (MISA with h = H_I, MISA-dagger with k' >= visible prefix, HISA with m = M or
  block size 1; MISA and HISA pages, sections "Methodology" / section 3);
* number formats checked against torch's own conversions.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_token_score_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_problem(T=5, L=40, H=3, d=8, q_offset=20, seed=1):
    return wl.prefill_inputs(T, L, H, d, q_offset=q_offset, seed=seed)


# ------------------------------------------------------------------ formats
def test_e4m3_table_matches_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = oracle.decode_e4m3(np.arange(256, dtype=np.uint8))
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours))
    assert nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(ref[~nan], ours[~nan])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9


def test_generator_bf16_rounding_matches_torch():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(100000).astype(np.float32) * np.float32(7.0)
    # exact ties: bf16 value + half ulp
    base = wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(x[:1000]))
    ties = (base.view(np.uint32) | np.uint32(0x8000)).view(np.float32)
    x = np.concatenate([x, ties, np.float32([0.0, -0.0, 1.0, -3.5])])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(wl.f32_to_bf16_bits(x), ref)


def test_f64_to_bf16_is_nearest_even():
    rng = np.random.default_rng(4)
    x = rng.standard_normal(20000) * 3.0
    lo_bits = wl.f32_to_bf16_bits(x.astype(np.float32))
    # add exact midpoints between neighbouring bf16 values (ties)
    a = oracle.widen_bf16(lo_bits[:500])
    b = oracle.widen_bf16((lo_bits[:500].astype(np.uint32) + 1).astype(np.uint16))
    x = np.concatenate([x, (a + b) / 2, np.array([0.0, 1.0, -2.0, 0.1])])
    got = oracle.widen_bf16(oracle.f64_to_bf16_bits(x))
    # brute force: nearest of the bf16 values bracketing x (truncation and next up)
    trunc = (x.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    cands = []
    for delta in (-1, 0, 1):
        c = (trunc.astype(np.int32) + delta).astype(np.uint16)
        cands.append(oracle.widen_bf16(c))
    cands = np.stack(cands)  # [3, n]
    dist = np.abs(cands - x[None])  # exact (Sterbenz); NaN where a bit pattern wrapped
    best = np.nanmin(dist, axis=0)
    assert np.all(np.abs(got - x) == best)
    # ties: the chosen value has an even mantissa
    tie = (dist == best[None]).sum(axis=0) > 1
    assert tie.sum() >= 400
    got_bits = oracle.f64_to_bf16_bits(x[tie])
    assert np.all((got_bits & 1) == 0)


def test_e4m3_quantisation_of_generator():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((64, 128)).astype(np.float32)
    q8, s = wl.quantize_rows_e4m3(x)
    deq = oracle.decode_e4m3(q8) * s[:, None].astype(np.float64)
    # every row's absmax maps to the largest code 448 (up to fp32 rounding of x/s)
    assert np.all(np.abs(oracle.decode_e4m3(q8)).max(axis=1) == 448.0)
    # e4m3 has 3 fraction bits: relative error <= 2^-4 for normal values
    big = np.abs(x) > 2.0 ** -6 * s[:, None] * 4
    assert np.all(np.abs(deq - x)[big] <= 2.0 ** -4 * np.abs(x)[big] + 1e-12)


# ------------------------------------------------------------------ score
def _golden():
    with open(os.path.join(GOLDEN, "hand_example.json")) as f:
        return json.load(f)


def _golden_inputs(g):
    q = wl.f32_to_bf16_bits(np.array(g["q"], dtype=np.float32))[None]
    k = wl.f32_to_bf16_bits(np.array(g["k"], dtype=np.float32))[None]
    w = np.array(g["w"], dtype=np.float32)[None]
    return wl.IndexerInputs(q=q, k=k, w=w, q_offset=g["q_offset"])


def test_hand_worked_example():
    g = _golden()
    inp = _golden_inputs(g)
    for kk, want in g["topk"].items():
        res = oracle.dense_topk(inp, int(kk))
        assert res["idx"].tolist() == want
        for t in range(g["T"]):
            assert res["scores"][t].tolist() == g["scores"][t]
            assert res["cond"][t].tolist() == g["cond"][t]


def _all_pairs(q, k):
    T, L = q.shape[0], k.shape[0]
    pq = np.repeat(np.arange(T), L)
    pk = np.tile(np.arange(L), T)
    return pq, pk


def test_relu_identities_pin_score():
    inp = _rand_problem(T=6, L=30, H=4, d=16)
    q, k, w = oracle.dequant(inp)
    pq, pk = _all_pairs(q, k)
    s_pos, c_pos = oracle.score_pairs(q, k, w, pq, pk)
    s_neg, c_neg = oracle.score_pairs(-q, k, w, pq, pk)
    dots = np.einsum("thd,sd->tsh", q, k).reshape(-1, q.shape[1])  # [T*L, H]
    wt = w[pq]
    lin = (wt * dots).sum(axis=1)
    ab = (wt * np.abs(dots)).sum(axis=1)
    tol = 1e-12 * (np.abs(wt) * np.abs(dots)).sum(axis=1) + 1e-300
    assert np.all(np.abs((s_pos - s_neg) - lin) <= tol)  # ReLU(x) - ReLU(-x) = x
    assert np.all(np.abs((s_pos + s_neg) - ab) <= tol)  # ReLU(x) + ReLU(-x) = |x|
    assert np.all(np.abs((c_pos - c_neg) - (np.abs(wt) * dots).sum(axis=1)) <= tol)
    assert np.all(c_pos >= np.abs(s_pos) - tol)


def test_score_invariances():
    inp = _rand_problem(T=4, L=25, H=5, d=8, seed=7)
    q, k, w = oracle.dequant(inp)
    pq, pk = _all_pairs(q, k)
    s, _ = oracle.score_pairs(q, k, w, pq, pk)
    perm = np.array([3, 0, 4, 1, 2])
    s_perm, _ = oracle.score_pairs(q[:, perm], k, w[:, perm], pq, pk)
    assert np.allclose(s_perm, s, rtol=1e-13, atol=1e-15)
    s_scaled, _ = oracle.score_pairs(q * 4.0, k, w, pq, pk)  # positive scaling passes through ReLU
    assert np.allclose(s_scaled, 4.0 * s, rtol=1e-13, atol=1e-15)
    w2 = np.random.default_rng(1).standard_normal(w.shape)
    s_w2, _ = oracle.score_pairs(q, k, w2, pq, pk)
    s_sum, _ = oracle.score_pairs(q, k, w + w2, pq, pk)  # linear in w
    assert np.allclose(s_sum, s + s_w2, rtol=1e-12, atol=1e-14)


def test_single_head_mask_is_that_head():
    inp = _rand_problem(T=3, L=20, H=4, d=8, seed=9)
    q, k, w = oracle.dequant(inp)
    pq, pk = _all_pairs(q, k)
    for h in range(4):
        hm = np.zeros((3, 4), dtype=np.uint8)
        hm[:, h] = 1
        s, _ = oracle.score_pairs(q, k, w, pq, pk, hmask=hm)
        dots = np.einsum("td,sd->ts", q[:, h], k).reshape(-1)
        assert np.allclose(s, w[pq, h] * np.maximum(dots, 0.0), rtol=1e-13, atol=1e-15)


# ------------------------------------------------------------------ selection
def _brute_topk(scores, k):
    """Candidate j is selected iff fewer than k candidates beat it, where i
    beats j when s_i > s_j, or s_i == s_j and i < j. NaN = absent."""
    n = scores.size
    sel = []
    for j in range(n):
        if np.isnan(scores[j]):
            continue
        better = 0
        for i in range(n):
            if np.isnan(scores[i]) or i == j:
                continue
            if scores[i] > scores[j] or (scores[i] == scores[j] and i < j):
                better += 1
        if better < k:
            sel.append(j)
    return sel + [-1] * (k - len(sel))


@pytest.mark.parametrize("seed", range(12))
def test_select_topk_brute_force(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 40))
    s = rng.integers(-3, 4, size=n).astype(np.float64)  # many exact ties
    s[rng.random(n) < 0.15] = np.nan
    if seed % 3 == 0:
        s[rng.random(n) < 0.3] = -0.0
    for k in (1, 2, 5, n, n + 3):
        assert oracle.select_topk(s, k).tolist() == _brute_topk(s, k)


def test_causal_prefix_and_short_rows():
    inp = _rand_problem(T=6, L=12, H=2, d=4, q_offset=3, seed=2)
    res = oracle.dense_topk(inp, 8)
    for t in range(6):
        V = min(3 + t + 1, 12)
        row = res["idx"][t]
        assert row[row >= 0].max() <= 3 + t
        if V <= 8:
            assert row.tolist() == list(range(V)) + [-1] * (8 - V)
        assert len(res["scores"][t]) == V


def test_all_negative_weights_tie_to_lowest_index():
    inp = _rand_problem(T=3, L=128, H=2, d=4, q_offset=120, seed=11)
    inp.w[:] = -np.abs(inp.w)
    res = oracle.dense_topk(inp, 5)
    for t in range(3):
        s = res["scores"][t]
        assert s.max() == 0.0
        zeros = np.flatnonzero(s == 0.0)
        assert zeros.size >= 5
        assert res["idx"][t].tolist() == zeros[:5].tolist()


# ------------------------------------------------------------------ FP8
def test_fp8_unfactored_equals_factored():
    inp = wl.decode_inputs(batch=2, L=300, H=4, d=16, seed=3, cluster_frac=0.1, n_centres=3)
    for b in range(2):
        q, k, w = oracle.dequant(inp, b)
        pq = np.zeros(300, dtype=np.int64)
        pk = np.arange(300)
        s, _ = oracle.score_pairs(q, k, w, pq, pk)
        q8 = oracle.decode_e4m3(inp.q[b, 0])  # [H, d]
        k8 = oracle.decode_e4m3(inp.k[b])  # [L, d]
        coef = inp.w[b, 0].astype(np.float64) * inp.q_scale[b, 0].astype(np.float64)
        fac = inp.k_scale[b].astype(np.float64) * (np.maximum(k8 @ q8.T, 0.0) * coef[None]).sum(axis=1)
        assert np.allclose(s, fac, rtol=1e-12, atol=1e-15)
    # exact copies of a cluster centre quantise identically -> exactly tied scores
    res = oracle.dense_topk(inp, 300, b=0)
    s = res["scores"][0]
    kb = inp.k[0]
    _, inv, cnt = np.unique(kb, axis=0, return_inverse=True, return_counts=True)
    dup = cnt[inv.reshape(-1)] > 1
    assert dup.sum() >= 2
    for u in np.unique(inv.reshape(-1)[dup]):
        members = np.flatnonzero(inv.reshape(-1) == u)
        assert np.all(s[members] == s[members[0]])


# ------------------------------------------------------------------ pooling + router
def test_meanpool_closed_forms():
    L, d, B = 10, 4, 4
    k = np.zeros((L, d), dtype=np.float32)
    k[0:4] = 0.375  # constant block -> same value
    k[4:8, 0] = np.arange(4) * 0.25 + 1.0  # arithmetic series 1, 1.25, 1.5, 1.75 -> 1.375
    k[4:8, 1] = -2.0
    k[8:10, 2] = [3.0, 5.0]  # partial last block: mean over its 2 tokens
    kbar = oracle.widen_bf16(oracle.meanpool_bf16(wl.f32_to_bf16_bits(k), B))
    assert kbar.shape == (3, d)
    assert np.all(kbar[0] == 0.375)
    assert kbar[1].tolist() == [1.375, -2.0, 0.0, 0.0]
    assert kbar[2].tolist() == [0.0, 0.0, 4.0, 0.0]


def test_router_closed_form_with_equal_pooled_keys():
    H, d, M, B = 3, 4, 6, 8
    rng = np.random.default_rng(0)
    v = rng.standard_normal(d)
    kbar = np.tile(v, (M, 1))
    q = rng.standard_normal((4, H, d))
    w = rng.standard_normal((4, H))
    p = np.array([0, 7, 8, 100])  # block m visible iff m*B <= p
    nvis = oracle.visible_blocks(p, B, M)
    assert nvis.tolist() == [1, 1, 2, 6]
    a = oracle.router_affinity(q, kbar, w, nvis)
    want = np.abs(w) * nvis[:, None] * np.maximum(np.einsum("thd,d->th", q, v), 0.0)
    assert np.allclose(a, want, rtol=1e-13, atol=0)


# ------------------------------------------------------------------ variant reductions
def test_misa_all_heads_is_dense():
    inp = _rand_problem(T=6, L=70, H=4, d=8, q_offset=50, seed=21)
    dense = oracle.dense_topk(inp, 10)
    m = oracle.misa(inp, block=8, h=4, topk=10)
    assert np.array_equal(m["idx"], dense["idx"])
    for t in range(6):
        assert np.array_equal(m["routed_scores"][t], dense["scores"][t])


def test_misa_one_head_brute_force():
    inp = _rand_problem(T=4, L=50, H=5, d=8, q_offset=30, seed=22)
    q, k, w = oracle.dequant(inp)
    m = oracle.misa(inp, block=8, h=1, topk=6)
    kbar = oracle.widen_bf16(m["kbar_bits"])
    for t in range(4):
        p = 30 + t
        nb = p // 8 + 1
        aff = [abs(w[t, h]) * sum(max(0.0, float(q[t, h] @ kbar[j])) for j in range(nb)) for h in range(5)]
        best = int(np.argmax(aff))  # first maximum = lowest head on ties
        assert m["heads"][t].tolist() == [best]
        s = [w[t, best] * max(0.0, float(q[t, best] @ k[s_])) for s_ in range(p + 1)]
        assert np.allclose(m["routed_scores"][t], s, rtol=1e-13, atol=1e-15)
        assert m["idx"][t].tolist() == _brute_topk(np.array(s), 6)


def test_misa_dagger_full_candidates_is_dense():
    inp = _rand_problem(T=5, L=40, H=4, d=8, q_offset=30, seed=23)
    dense = oracle.dense_topk(inp, 7)
    m = oracle.misa(inp, block=8, h=2, topk=7, kprime=40)
    assert np.array_equal(m["idx"], dense["idx"])


def test_hisa_all_blocks_is_dense():
    inp = _rand_problem(T=5, L=64, H=3, d=8, q_offset=50, seed=24)
    dense = oracle.dense_topk(inp, 9)
    hs = oracle.hisa(inp, block=8, m=8, topk=9)
    assert np.array_equal(hs["idx"], dense["idx"])


def test_hisa_block_one_is_dense():
    inp = _rand_problem(T=5, L=48, H=3, d=8, q_offset=30, seed=25)
    dense = oracle.dense_topk(inp, 6)
    hs = oracle.hisa(inp, block=1, m=6, topk=6)
    assert np.array_equal(hs["idx"], dense["idx"])
    # with B = 1 the pooled key is the key itself
    assert np.array_equal(hs["kbar_bits"], inp.k[0])


# ------------------------------------------------------------------ generator
def test_generator_deterministic_and_needles():
    a = wl.prefill_inputs(16, 256, 4, 8, q_offset=200, seed=5, needles=6)
    b = wl.prefill_inputs(16, 256, 4, 8, q_offset=200, seed=5, needles=6)
    assert np.array_equal(a.q, b.q) and np.array_equal(a.k, b.k) and np.array_equal(a.w, b.w)
    pos = a.meta["needle_pos"][0]
    assert len(set(pos.tolist())) == 6 and pos.max() < 200
    qv = wl.bf16_bits_to_f32(a.q[0, a.meta["needle_src"][0]])
    assert np.array_equal(a.k[0, pos], wl.f32_to_bf16_bits(np.float32(0.5) * qv.mean(axis=1, dtype=np.float32)))
    assert wl.visible_pairs(16, 256, 200) == sum(min(201 + t, 256) for t in range(16))


# ------------------------------------------------------------ DoSA certified pruning
def _dosa_inp(seed, H=8, d=32, T=6, L=300, w_sign=0):
    inp = wl.prefill_inputs(T=T, L=L, H=H, d=d, q_offset=L - T, seed=seed)
    if w_sign < 0:
        inp.w = -np.abs(inp.w)  # all heads negative: scores <= 0, mass ties at 0
    return inp


@pytest.mark.parametrize("screen", [[], [0], [1, 5], [0, 2, 4, 6], list(range(8))])
def test_dosa_bound_is_sound(screen):
    inp = _dosa_inp(41)
    q, k, w = oracle.dequant(inp)
    for t in range(inp.T):
        p = inp.q_offset + t
        keys = np.arange(p + 1)
        bound, _ = oracle.dosa_upper_bound(q, k, w, t, keys, screen)
        # exact scores by brute force (numpy, fp64), not through the oracle's core
        x = np.einsum("hd,sd->hs", q[t], k[keys])
        exact = (w[t][:, None] * np.maximum(x, 0.0)).sum(0)
        assert np.all(bound >= exact)


def test_dosa_bound_is_tight_with_every_head_screened():
    inp = _dosa_inp(42)
    q, k, w = oracle.dequant(inp)
    keys = np.arange(inp.q_offset + 1)
    bound, part = oracle.dosa_upper_bound(q, k, w, 0, keys, range(8))
    x = np.einsum("hd,sd->hs", q[0], k[keys])
    exact = (w[0][:, None] * np.maximum(x, 0.0)).sum(0)
    assert np.allclose(bound, exact, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("seed,screen,n_seed,w_sign", [
    (43, [0, 1], 64, 0), (44, [3], 32, 0), (45, [], 64, 0),       # no screened head: bounds from norms only
    (46, [0, 1, 2, 3], 8, 0),                                      # fewer seeds than k: tau = -inf, no pruning
    (47, [2, 6], 64, -1),                                          # all-negative weights: ties at 0
])
def test_dosa_equals_dense(seed, screen, n_seed, w_sign):
    inp = _dosa_inp(seed, w_sign=w_sign)
    if seed == 44:
        inp.k[0, 100:110] = inp.k[0, 50]  # duplicate keys: exact ties across positions
    topk = 16
    dense = oracle.dense_topk(inp, topk)
    dosa = oracle.dosa_topk(inp, topk, screen, n_seed)
    assert np.array_equal(dense["idx"], dosa["idx"])
    for i, t in enumerate(dense["queries"]):
        kth = oracle.kth_score(dense["scores"][i], topk)
        assert dosa["tau"][i] <= kth            # the seeds' k-th score bounds the row's from below
    if n_seed < topk:
        assert dosa["survivors"] == [v - min(n_seed, v) for v in dosa["visible"]]


def test_dosa_planted_mistake_is_caught(monkeypatch):
    # a bound that forgets the unscreened positive-weight heads is unsound;
    # the selection then loses winners and no longer equals the dense one
    real = oracle.dosa_upper_bound

    def forgetful(q, k, w, t, keys, screen):
        bound, part = real(q, k, w, t, keys, screen)
        return part, part

    monkeypatch.setattr(oracle, "dosa_upper_bound", forgetful)
    inp = _dosa_inp(48, H=8, T=8, L=400)
    dense = oracle.dense_topk(inp, 16)
    dosa = oracle.dosa_topk(inp, 16, [0], 32)
    assert not np.array_equal(dense["idx"], dosa["idx"])


def test_indexcache_layers_follow_the_pattern():
    # F layers are the dense indexer on their own inputs; an S layer is the
    # nearest preceding F layer's result, whatever its own inputs are
    layers = [wl.prefill_inputs(6, 300, 8, 64, q_offset=294, seed=100 + i, batch=2) for i in range(5)]
    got = oracle.indexcache(layers, "FSFSS", 20)
    dense = [np.stack([oracle.dense_topk(x, 20, b=b)["idx"] for b in range(2)]) for x in layers]
    for i, j in enumerate([0, 0, 2, 2, 2]):
        assert np.array_equal(got[i], dense[j])
    assert not np.array_equal(dense[0], dense[1])  # the layers differ, so reuse is visible
    all_f = oracle.indexcache(layers, "FFFFF", 20)
    assert all(np.array_equal(a, b) for a, b in zip(all_f, dense))
    for bad in ("SFFFF", "FFF", "FXFFF"):
        with pytest.raises(ValueError):
            oracle.indexcache(layers, bad, 20)


# ------------------------------------------------------------ DoSA at tile granularity
def test_sample_threshold_closed_form():
    # V = 1000 keys, k = 50: p = 0.05; 100 samples -> r_lo = ceil(5 + 4 sqrt(4.75) + 4) = 18
    samp = np.arange(100, dtype=np.float64)[::-1] * 0.5          # 49.5, 49.0, ...
    assert oracle.sample_threshold(samp, 50, 1000) == 49.5 - 17 * 0.5
    assert oracle.sample_threshold(samp, 1000, 1000) == -np.inf  # V <= k keeps every key
    assert oracle.sample_threshold(samp[:6], 50, 1000) == -np.inf  # r_lo = 7 beyond the sample


def test_dosa_screen_heads_rank_by_weighted_norm():
    q = np.zeros((4, 2))
    q[:, 0] = [1.0, 2.0, 1.0, 4.0]
    w = np.array([-3.0, 1.0, 2.0, 0.25])     # |w| ||q||: 3, 2, 2, 1
    assert oracle.dosa_screen_heads(q, w, 2).tolist() == [0, 1]   # tie 2 = 2 -> lower head
    assert oracle.dosa_screen_heads(q, w, 4).tolist() == [0, 1, 2, 3]


def _low_norm_population(seed, T=8, L=4096, H=8, d=32, live_every=4):
    """Keys of most 128-key tiles shrunk 100x (a low-norm population no query
    can rank high); every live_every-th tile keeps its norm. Non-negative head
    weights, so every query's best scores are clearly positive."""
    inp = wl.prefill_inputs(T=T, L=L, H=H, d=d, q_offset=L - T, seed=seed)
    inp.w = np.abs(inp.w)
    kf = wl.bf16_bits_to_f32(inp.k)
    tile = np.arange(L) // 128
    kf[0, tile % live_every != 0] *= np.float32(0.01)
    inp.k = wl.f32_to_bf16_bits(kf)
    return inp


@pytest.mark.parametrize("seed,n_screen,S,qpt,w_sign", [
    (51, 3, 16, 4, 0), (52, 0, 8, 2, 0), (53, 8, 16, 4, 0),   # no screened head / every head screened
    (54, 2, 16, 8, -1),                                         # all-negative weights: ties at 0
])
def test_dosa_tile_equals_dense(seed, n_screen, S, qpt, w_sign):
    inp = _dosa_inp(seed, w_sign=w_sign, T=12, L=700)
    if seed == 52:
        inp.k[0, 300:320] = inp.k[0, 40]  # duplicate keys: exact ties across positions
    dense = oracle.dense_topk(inp, 16)
    got = oracle.dosa_tile_topk(inp, 16, n_screen, S, qpt)
    assert got["queries"] == list(range(12))
    assert np.array_equal(dense["idx"], got["idx"])


def test_dosa_tile_prunes_a_low_norm_population():
    inp = _low_norm_population(55)
    dense = oracle.dense_topk(inp, 16)
    got = oracle.dosa_tile_topk(inp, 16, 3, 16, 4)
    assert np.array_equal(dense["idx"], got["idx"])
    assert got["live"].mean() <= 0.5          # at least half of the tiles pruned
    assert not any(got["fallback"])
    # the live tiles hold every winner
    for i, t in enumerate(got["queries"]):
        assert np.all(got["live"][t // 4, dense["idx"][i] // 128] == 1)


def test_dosa_tile_short_certificate_falls_back():
    # the sampled keys (every 16th) are the strongest: thresholds come out so
    # high that fewer than k scores reach them; the rows fall back to all keys
    inp = _dosa_inp(56, T=8, L=900)
    q, _, _ = oracle.dequant(inp)
    kf = wl.bf16_bits_to_f32(inp.k)
    inp.w = np.abs(inp.w)
    kf[0, ::16] = 3.0 * q.mean(axis=(0, 1)) / np.linalg.norm(q.mean(axis=(0, 1)))
    inp.k = wl.f32_to_bf16_bits(kf)
    dense = oracle.dense_topk(inp, 100)
    got = oracle.dosa_tile_topk(inp, 100, 3, 16, 4)
    assert any(got["fallback"])
    assert np.array_equal(dense["idx"], got["idx"])


def test_dosa_tile_planted_mistake_is_caught(monkeypatch):
    # a bound without the unscreened positive heads prunes tiles that hold
    # winners; the certificate still rescues rows whose count comes out short,
    # so the mistake must show as a different selection somewhere
    real = oracle.dosa_upper_bound

    def forgetful(q, k, w, t, keys, screen):
        bound, part = real(q, k, w, t, keys, screen)
        return part, part

    monkeypatch.setattr(oracle, "dosa_upper_bound", forgetful)
    inp = _dosa_inp(57, T=16, L=1500)
    dense = oracle.dense_topk(inp, 16)
    got = oracle.dosa_tile_topk(inp, 16, 1, 16, 4)
    assert not np.array_equal(dense["idx"], got["idx"])


# ------------------------------------------------------------ FP8 pooled keys
def test_e4m3_encoder_is_nearest_even_and_matches_torch():
    import torch
    # exact midpoints go to the even code: 1.0625 between 1.0 (0x38) and 1.125 (0x39)
    assert oracle.f64_to_e4m3(np.array([1.0625, -1.0625, 1.1875]))[:3].tolist() == [0x38, 0xB8, 0x3A]
    assert oracle.f64_to_e4m3(np.array([1000.0, -1000.0, 0.0]))[:3].tolist() == [0x7E, 0xFE, 0x00]
    x = np.random.default_rng(3).standard_normal(20000).astype(np.float32) * np.float32(40.0)
    ref = torch.from_numpy(np.clip(x, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.f64_to_e4m3(x.astype(np.float64)), ref)
    # every code decodes and re-encodes to itself
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    back = oracle.f64_to_e4m3(oracle.decode_e4m3(codes))
    assert np.array_equal(back[codes != 0x80], codes[codes != 0x80])


def test_meanpool_e4m3_closed_form():
    # block of two tokens (scale 1): the mean (2, 1, -0.5, 0, ...) is representable
    # after scaling by amax / 448 = 2 / 448, so it decodes back exactly
    d = 16
    k = np.zeros((4, d), dtype=np.float64)
    k[0, :3], k[1, :3] = [1.0, 0.5, -0.25], [3.0, 1.5, -0.75]
    k[2:] = 0.0                                       # an all-zero block: scale 1, codes 0
    codes = oracle.f64_to_e4m3(k)
    got, sc = oracle.meanpool_e4m3(codes, np.ones(4, dtype=np.float32), 2)
    assert sc[0] == np.float32(2.0) / np.float32(448.0) and sc[1] == np.float32(1.0)
    # mean / scale = (448, 224, -112) up to the fp32 rounding of the scale
    assert got[0][:3].tolist() == oracle.f64_to_e4m3(np.array([448.0, 224.0, -112.0])).tolist()
    mean = oracle.decode_e4m3(got[0]) * np.float64(sc[0])
    assert np.allclose(mean[:3], [2.0, 1.0, -0.5], rtol=1e-6, atol=0) and np.all(mean[3:] == 0)
    assert np.all(got[1] == 0)


def test_hisa_fp8_all_blocks_is_dense():
    inp = wl.decode_inputs(batch=2, L=900, H=32, d=128, seed=77)
    for b in range(2):
        dense = oracle.dense_topk(inp, 40, b=b)
        h = oracle.hisa(inp, 128, 8, 40, b=b)   # 8 blocks of 128 cover all 900 keys
        assert np.array_equal(dense["idx"], h["idx"])


def test_misa_fp8_all_heads_and_all_candidates_are_dense():
    # MISA on an FP8 cache reduces to the dense FP8 indexer when every head is
    # routed (h = H) or every visible key is a MISA-dagger candidate (k' >= V)
    inp = wl.decode_inputs(batch=2, L=700, H=32, d=128, seed=78)
    for b in range(2):
        dense = oracle.dense_topk(inp, 30, b=b)
        m = oracle.misa(inp, 64, 32, 30, b=b)
        assert np.array_equal(dense["idx"], m["idx"])
        assert np.array_equal(m["routed_scores"][0], dense["scores"][0])
        md = oracle.misa(inp, 64, 4, 30, kprime=700, b=b)
        assert np.array_equal(dense["idx"], md["idx"])


def test_misa_fp8_router_brute_force():
    # affinity of every head from the decoded pooled keys, summed by hand
    inp = wl.decode_inputs(batch=1, L=300, H=32, d=128, seed=79)
    q, k, w = oracle.dequant(inp)
    m = oracle.misa(inp, 64, 3, 10)
    codes, scales = m["kbar_bits"]
    assert codes.shape == (5, 128) and scales.shape == (5,)
    kbar = oracle.decode_e4m3(codes) * scales.astype(np.float64)[:, None]
    p = inp.q_offset                        # one query, at the end of the cache
    nb = p // 64 + 1
    aff = [abs(w[0, h]) * sum(max(0.0, float(q[0, h] @ kbar[j])) for j in range(nb)) for h in range(32)]
    assert np.allclose(m["affinity"][0], aff, rtol=1e-12, atol=0)
    want = sorted(range(32), key=lambda h: (-aff[h], h))[:3]
    assert sorted(m["heads"][0].tolist()) == sorted(want)
