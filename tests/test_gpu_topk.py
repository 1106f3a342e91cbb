"""The top-k stage alone (indexer_topk_rows) on crafted fp32 rows: the scores
are given, so the selection must equal the oracle's exactly (ties to the
lower position, -inf absent, fewer candidates than k padded with -1, output in
ascending order). Covers rows staged in shared memory and rows streamed from
global memory, the sampled-band path and its fallback (mass ties), unaligned
row starts, per-query causal lengths and the index maps used by MISA-dagger
and HISA."""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_token_score_b200 import binding as B

pytestmark = pytest.mark.gpu


def _run(scores, T, q_offset, pstride, row_len, k, cand=None, n_slots=0, blk=1, ld=None):
    rows = scores.shape[0]
    ld = scores.shape[1] if ld is None else ld
    dev = torch.from_numpy(np.ascontiguousarray(scores, dtype=np.float32)).cuda()
    c = torch.from_numpy(np.ascontiguousarray(cand, dtype=np.int32)).cuda() if cand is not None else None
    idx = torch.full((rows, k), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((rows, k), float("nan"), dtype=torch.float32, device="cuda")
    ws = B.alloc_workspace(256)
    B.indexer_topk_rows(dev, rows, ld, T, q_offset, pstride, row_len, k, c, n_slots, blk, idx, sc, ws)
    assert B.dsa_device_status(ws) == 0
    return idx.cpu().numpy(), sc.cpu().numpy()


def _expect(scores, T, q_offset, pstride, row_len, k, cand=None, blk=1):
    out = []
    for r in range(scores.shape[0]):
        t = r % T
        n = row_len if pstride == 0 else int(np.clip((q_offset + t) // pstride + 1, 0, row_len))
        row = scores[r, :n].astype(np.float64)
        row[np.isneginf(row)] = np.nan
        sel = oracle.select_topk(row, k)
        if cand is not None:
            m = sel >= 0
            sel[m] = cand[r, sel[m] // blk] * blk + sel[m] % blk
        out.append(sel)
    return np.array(out).reshape(scores.shape[0], k)


def _check(scores, idx, sc, expect, what):
    assert np.array_equal(idx, expect), what
    pad = expect < 0
    assert np.all(np.isneginf(sc[pad])), what


# (20000, 5000) and (40000, 13000): more selected than the shared-memory output
# staging holds (direct writes); (140000, 1000): longer than the band path's
# bitmap (fallback only)
@pytest.mark.parametrize("n,k", [(33, 5), (1000, 100), (32768, 2048), (32769, 2048), (40000, 3000),
                                 (131072, 8192), (131072, 2048), (4096, 4096), (5000, 6000),
                                 (20000, 5000), (40000, 13000), (140000, 1000)])
def test_random_rows(n, k):
    rng = np.random.default_rng(n + k)
    s = (rng.standard_normal((6, n)) * 0.05).astype(np.float32)
    idx, sc = _run(s, 6, 0, 0, n, k)
    exp = _expect(s, 6, 0, 0, n, k)
    _check(s, idx, sc, exp, f"n={n} k={k}")
    sel = exp >= 0
    rows = np.repeat(np.arange(6)[:, None], k, axis=1)
    assert np.array_equal(sc[sel], s[rows[sel], exp[sel]])


@pytest.mark.parametrize("n", [20000, 100000])
def test_mass_ties_fall_back(n):
    rng = np.random.default_rng(7)
    s = rng.integers(-3, 4, size=(4, n)).astype(np.float32) * np.float32(0.25)  # 7 distinct values
    s[1, : n // 2] = -0.0
    s[1, n // 2:] = 0.0  # one value, signed zeros
    idx, sc = _run(s, 4, 0, 0, n, 1500)
    _check(s, idx, sc, _expect(s, 4, 0, 0, n, 1500), f"ties n={n}")


def test_absent_entries_and_short_rows():
    rng = np.random.default_rng(3)
    s = rng.standard_normal((5, 9000)).astype(np.float32)
    s[0, rng.random(9000) < 0.7] = -np.inf
    s[1, :] = -np.inf
    s[2, 100:] = -np.inf  # only 100 present
    idx, sc = _run(s, 5, 0, 0, 9000, 500)
    _check(s, idx, sc, _expect(s, 5, 0, 0, 9000, 500), "absent")


def test_causal_row_lengths_and_unaligned_rows():
    rng = np.random.default_rng(4)
    T, L = 7, 3001
    s = rng.standard_normal((T, L)).astype(np.float32)
    # ld = L (odd): rows after the first start off a 16-byte boundary
    idx, sc = _run(s, T, 2990, 1, L, 64)
    _check(s, idx, sc, _expect(s, T, 2990, 1, L, 64), "causal")
    # pooled blocks: row length (q_offset + t) // 64 + 1
    idx, sc = _run(s, T, 1000, 64, L, 9)
    _check(s, idx, sc, _expect(s, T, 1000, 64, L, 9), "block stride")


def test_index_maps():
    rng = np.random.default_rng(5)
    rows, m, blk = 3, 6, 128
    s = rng.standard_normal((rows, m * blk)).astype(np.float32)
    cand = np.sort(rng.choice(500, size=(rows, m), replace=True), axis=1).astype(np.int32)
    idx, sc = _run(s, rows, 0, 0, m * blk, 100, cand=cand, n_slots=m, blk=blk)
    _check(s, idx, sc, _expect(s, rows, 0, 0, m * blk, 100, cand=cand, blk=blk), "block map")
    cand1 = np.sort(rng.choice(100000, size=(rows, 700), replace=False), axis=1).astype(np.int32)
    s1 = rng.standard_normal((rows, 700)).astype(np.float32)
    idx, sc = _run(s1, rows, 0, 0, 700, 64, cand=cand1, n_slots=700, blk=1)
    _check(s1, idx, sc, _expect(s1, rows, 0, 0, 700, 64, cand=cand1, blk=1), "token map")


def test_many_long_rows():
    # enough rows longer than 32768 to fill the GPU with 256-thread CTAs
    rng = np.random.default_rng(11)
    rows, n, k = 320, 33000, 2048
    s = (rng.standard_normal((rows, n)) * 0.05).astype(np.float32)
    s[::7, : n // 3] = -np.inf  # some rows with absent entries
    idx, sc = _run(s, rows, 0, 0, n, k)
    exp = _expect(s, rows, 0, 0, n, k)
    _check(s, idx, sc, exp, "many long rows")


def test_many_short_rows():
    # more rows (of at most 32768 scores) than SMs: the 256-thread short-row
    # layout, 4 CTAs per SM (fewer rows take one 512-thread CTA each)
    rng = np.random.default_rng(13)
    rows, n, k = 400, 20000, 2048
    s = (rng.standard_normal((rows, n)) * 0.05).astype(np.float32)
    s[::5, n // 2:] = -np.inf
    s[3::11] = np.round(s[3::11] * 8) / 8  # rows with many ties
    idx, sc = _run(s, rows, 0, 0, n, k)
    _check(s, idx, sc, _expect(s, rows, 0, 0, n, k), "many short rows")


def test_many_long_rows_mass_ties():
    # the long-row layout's fallback path: few distinct values, enough rows
    # longer than 32768 to fill the GPU
    rng = np.random.default_rng(12)
    rows, n, k = 300, 36000, 1000
    s = rng.integers(-3, 4, size=(rows, n)).astype(np.float32) * np.float32(0.5)
    idx, sc = _run(s, rows, 0, 0, n, k)
    _check(s, idx, sc, _expect(s, rows, 0, 0, n, k), "long rows, mass ties")


@pytest.mark.parametrize("n,k", [(2048, 256), (2048, 2047), (1500, 1500), (2000, 3000), (64, 7), (1, 1),
                                 (3000, 100), (8192, 2048), (12000, 13000), (16384, 2048)])
def test_short_rows_one_cta_each(n, k):
    # rows of at most 2048 scores take one CTA per row (keys in registers),
    # longer ones the sampled-band CTAs: random values, mass ties with signed zeros, absent entries, NaN,
    # all-equal rows, k >= n
    rng = np.random.default_rng(n * 7 + k)
    rows = 40
    s = (rng.standard_normal((rows, n)) * 0.05).astype(np.float32)
    s[1] = rng.integers(-3, 4, size=n).astype(np.float32) * np.float32(0.25)
    s[2] = np.where(rng.random(n) < 0.5, np.float32(-0.0), np.float32(0.0))
    s[3, rng.random(n) < 0.6] = -np.inf
    s[4] = -np.inf
    s[5] = np.float32(1.5)
    s[6, rng.random(n) < 0.2] = np.nan
    s[7, : n // 2] = -np.inf
    idx, sc = _run(s, rows, 0, 0, n, k)
    exp_in = s.copy()
    exp_in[np.isnan(exp_in)] = -np.inf  # NaN is absent too
    exp = _expect(exp_in, rows, 0, 0, n, k)
    _check(s, idx, sc, exp, f"short n={n} k={k}")
    sel = exp >= 0
    r_ = np.repeat(np.arange(rows)[:, None], k, axis=1)
    want = exp_in[r_[sel], exp[sel]]
    assert np.array_equal(sc[sel], np.where(want == 0, np.float32(0.0), want))


def test_short_rows_causal_lengths_and_maps():
    # many short rows (more than one row per warp of the grid), per-query
    # causal lengths, pooled-block strides and a block index map
    rng = np.random.default_rng(21)
    T, L = 3000, 2048
    s = rng.standard_normal((T, L)).astype(np.float32)
    idx, sc = _run(s, T, 100, 1, L, 128)
    _check(s, idx, sc, _expect(s, T, 100, 1, L, 128), "short causal")
    idx, sc = _run(s[:50], 50, 5000, 4, L, 300)
    _check(s[:50], idx, sc, _expect(s[:50], 50, 5000, 4, L, 300), "short block stride")
    m, blk = 8, 128
    cand = np.sort(rng.choice(4000, size=(20, m), replace=False), axis=1).astype(np.int32)
    s2 = rng.standard_normal((20, m * blk)).astype(np.float32)
    idx, sc = _run(s2, 20, 0, 0, m * blk, 200, cand=cand, n_slots=m, blk=blk)
    _check(s2, idx, sc, _expect(s2, 20, 0, 0, m * blk, 200, cand=cand, blk=blk), "short block map")
