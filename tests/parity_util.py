"""Comparison rules between the CUDA path and the fp64 oracle.

Scores: |S_gpu - S_oracle| <= rtol * C + 1e-30, where C = sum_h |w| ReLU(q.k) is
the score's condition scale (signed heads can cancel to ~0, where a plain
relative bound means nothing). rtol = 1e-2 for bf16 inputs, 3e-2 for FP8.

Selections: both sides return min(k, #candidates) distinct candidates, in
ascending order, padded with -1. A candidate may be in one set and not the
other only if its oracle score lies within 1e-3 * max(|tau|, C_tau) of the
oracle's k-th score tau (a near-tie that rounding may flip).
"""
import collections

import numpy as np

RTOL_BF16 = 1e-2
RTOL_FP8 = 3e-2
TIE_REL = 1e-3
PLAIN_FLOOR = 1e-3  # |S| below this fraction of C is too cancelled for a plain relative bound

# Per-label record of how much of each tolerance the checks used (filled when a
# check is given `stats=`): the largest |err| / C, how many scores also meet the
# plain relative bound |err| <= rtol * |S| (for |S| >= PLAIN_FLOOR * C), how
# many selections were compared, and how many ids differed as allowed near-ties
# (and of those, how many fall inside the plain slack 1e-3 * |tau|).
STATS = collections.defaultdict(lambda: {"scores": 0, "max_err_over_cond": 0.0, "plain_checked": 0,
                                         "plain_ok": 0, "rows": 0, "exempt_ids": 0,
                                         "exempt_plain_ok": 0, "max_exempt_rows": 0})


def check_scores(gpu, ref, cond, rtol, what="", stats=None):
    gpu = np.asarray(gpu, dtype=np.float64)
    err = np.abs(gpu - ref)
    bound = rtol * cond + 1e-30
    if stats is not None and err.size:
        st = STATS[stats]
        st["scores"] += int(err.size)
        st["max_err_over_cond"] = max(st["max_err_over_cond"], float(np.max(err / (cond + 1e-300))))
        big = np.abs(ref) >= PLAIN_FLOOR * cond
        st["plain_checked"] += int(big.sum())
        st["plain_ok"] += int(np.sum(err[big] <= rtol * np.abs(ref[big])))
    bad = ~(err <= bound)
    if bad.any():
        i = int(np.flatnonzero(bad)[0])
        raise AssertionError(f"{what}: {bad.sum()} scores out of tolerance; first at {i}: "
                             f"gpu={gpu[i]!r} oracle={ref[i]!r} cond={cond[i]!r}")


def check_selection(gpu_row, cand, scores, cond, k, what="", rel=TIE_REL, stats=None):
    """gpu_row: [k] selected ids from the GPU; cand/scores/cond: the oracle's
    candidate ids and their fp64 scores and condition scales."""
    gpu_row = np.asarray(gpu_row, dtype=np.int64)
    cand = np.asarray(cand, dtype=np.int64)
    n = min(k, cand.size)
    sel = gpu_row[:n]
    assert np.all(gpu_row[n:] == -1), f"{what}: padding is not -1"
    assert np.all(sel >= 0), f"{what}: {np.sum(sel < 0)} missing selections"
    assert np.all(np.diff(sel) > 0), f"{what}: not strictly ascending (duplicates?)"
    pos = {int(c): i for i, c in enumerate(cand)}
    assert all(int(s) in pos for s in sel), f"{what}: selected an id that is not a candidate"
    # oracle selection: (score desc, id asc)
    order = np.lexsort((cand, -scores))
    ref = np.sort(cand[order[:n]])
    st = STATS[stats] if stats is not None else None
    if st is not None:
        st["rows"] += 1
    if n < k or n == cand.size:
        assert np.array_equal(sel, ref), f"{what}: selection differs with no threshold"
        return 0
    kth = order[n - 1]
    tau = scores[kth]
    slack = rel * max(abs(tau), cond[kth])
    diff = np.setxor1d(sel, ref)
    for c in diff:
        i = pos[int(c)]
        assert abs(scores[i] - tau) <= slack, (
            f"{what}: id {c} (score {scores[i]!r}) differs but is not a near-tie of tau={tau!r}")
        if st is not None:
            st["exempt_ids"] += 1
            st["exempt_plain_ok"] += int(abs(scores[i] - tau) <= rel * abs(tau))
    if st is not None:
        st["max_exempt_rows"] = max(st["max_exempt_rows"], int(diff.size // 2))
    return diff.size // 2


def stats_table():
    """One line per label of STATS (printed at the end of a test session)."""
    lines = []
    for k in sorted(STATS):
        st = STATS[k]
        pl = st["plain_ok"] / st["plain_checked"] if st["plain_checked"] else float("nan")
        lines.append(f"{k}: scores={st['scores']} max|err|/C={st['max_err_over_cond']:.2e} "
                     f"plain-rtol ok={pl:.4f} of {st['plain_checked']} rows={st['rows']} "
                     f"near-tie ids={st['exempt_ids']} (within 1e-3|tau|: {st['exempt_plain_ok']}) "
                     f"max swaps/row={st['max_exempt_rows']}")
    return lines
