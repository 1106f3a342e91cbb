"""The C-ABI library loads on a machine without a GPU, exports every function
include/dsa_indexer.h declares, and its host-side validation rejects bad
arguments before any CUDA call (so these run on CPU)."""
import ctypes

import pytest

from sparse_attention_token_score_b200 import binding as B
from sparse_attention_token_score_b200 import build as build_mod


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.lib()


def test_exports_every_declared_symbol(lib):
    names = B.header_symbols()
    assert len(names) == 28
    assert set(names) == set(B._SIGS)
    for n in names:
        assert getattr(lib, n) is not None


def test_status_strings(lib):
    assert lib.dsa_status_string(0) == b"ok"
    assert lib.dsa_status_string(-3) == b"workspace too small"
    assert lib.dsa_status_string(-5) == b"device wait timed out"


def _args(**kw):
    a = B.IndexerArgs(batch=1, T=4, L=256, H=64, d=128, q_offset=252, qk_dtype=B.DSA_BF16)
    a.q, a.k, a.w = 0x10000, 0x20000, 0x30000  # never dereferenced: validation fails first
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_workspace_sizes(lib):
    a = _args()
    assert lib.indexer_workspace_size(ctypes.byref(a), 16) == 256 + 4 * 256 * 4
    assert lib.indexer_workspace_size(None, 16) == 0
    m = lib.misa_workspace_size(ctypes.byref(a), 64, 8, 16, 0)
    m2 = lib.misa_workspace_size(ctypes.byref(a), 64, 8, 16, 128)
    assert m2 == m + 2 * 256 * 4 * 2  # candidates + their scores, [T, kprime] each
    assert lib.hisa_workspace_size(ctypes.byref(a), 128, 2, 16) > 256


@pytest.mark.parametrize("bad", [
    dict(batch=0), dict(T=0), dict(L=0), dict(q_offset=-1), dict(q=None), dict(w=None),
    dict(q=0x10008),  # q not 16-byte aligned
    dict(qk_dtype=7),
    dict(qk_dtype=B.DSA_FP8_E4M3),  # FP8 without scales
])
def test_invalid_arguments_rejected(lib, bad):
    a = _args(**bad)
    st = lib.indexer_score_topk(ctypes.byref(a), 16, ctypes.c_void_p(0x40000), None,
                                ctypes.c_void_p(0x50000), 1 << 30, None)
    assert st == -1


@pytest.mark.parametrize("shape", [dict(H=48), dict(d=96), dict(H=128)])
def test_unsupported_shapes(lib, shape):
    a = _args(**shape)
    st = lib.indexer_score_topk(ctypes.byref(a), 16, ctypes.c_void_p(0x40000), None,
                                ctypes.c_void_p(0x50000), 1 << 30, None)
    assert st == -2


def test_workspace_checks(lib):
    a = _args()
    out = ctypes.c_void_p(0x40000)
    assert lib.indexer_score_topk(ctypes.byref(a), 16, out, None, None, 1 << 30, None) == -3
    assert lib.indexer_score_topk(ctypes.byref(a), 16, out, None, ctypes.c_void_p(0x50000), 100, None) == -3
    assert lib.indexer_score_topk(ctypes.byref(a), 16, out, None, ctypes.c_void_p(0x50010), 1 << 30, None) == -1
    assert lib.indexer_score_topk(ctypes.byref(a), 0, out, None, ctypes.c_void_p(0x50000), 1 << 30, None) == -1


def test_variant_argument_checks(lib):
    a = _args()
    out = ctypes.c_void_p(0x40000)
    ws = ctypes.c_void_p(0x50000)
    big = 1 << 40
    # h > H, unsupported h, bad block
    assert lib.misa_route_score_topk(ctypes.byref(a), 64, 65, 16, 0, out, None, None, None, ws, big, None) == -1
    assert lib.misa_route_score_topk(ctypes.byref(a), 64, 12, 16, 0, out, None, None, None, ws, big, None) == -2
    assert lib.misa_route_score_topk(ctypes.byref(a), 0, 8, 16, 0, out, None, None, None, ws, big, None) == -1
    # FP8 MISA: d = 128 and H in {32, 64} only (rejected before any launch)
    f = _args(qk_dtype=B.DSA_FP8_E4M3, q_scale=0x60000, k_scale=0x70000, H=16)
    assert lib.misa_route_score_topk(ctypes.byref(f), 64, 8, 16, 0, out, None, None, None, ws, big, None) == -2
    f = _args(qk_dtype=B.DSA_FP8_E4M3, q_scale=0x60000, k_scale=0x70000, d=64)
    assert lib.misa_route_score_topk(ctypes.byref(f), 64, 8, 16, 0, out, None, None, None, ws, big, None) == -2
    assert lib.hisa_block_filter_topk(ctypes.byref(a), 128, 0, 16, out, None, None, ws, big, None) == -1
    h8 = _args(H=8)
    assert lib.hisa_block_filter_topk(ctypes.byref(h8), 128, 2, 16, out, None, None, ws, big, None) == -2
    assert lib.indexer_topk_rows(None, 4, 256, 4, 0, 1, 256, 16, None, 0, 1, out, None, ws, big, None) == -1
    assert lib.dsa_meanpool_keys(None, 1, 256, 128, 64, ws, None) == -1
    # pooled-key cache: missing buffers, bad block ranges (rejected before any launch)
    kb = ctypes.c_void_p(0x90000)
    assert lib.dsa_pool_keys(ctypes.byref(a), 64, 0, 4, None, None, None) == -1
    assert lib.dsa_pool_keys(ctypes.byref(a), 64, 3, 2, kb, None, None) == -1
    assert lib.dsa_pool_keys(ctypes.byref(a), 64, -1, 2, kb, None, None) == -1
    assert lib.dsa_pool_keys(ctypes.byref(a), 0, 0, 2, kb, None, None) == -1
    f = _args(qk_dtype=B.DSA_FP8_E4M3, q_scale=0x60000, k_scale=0x70000)
    assert lib.dsa_pool_keys(ctypes.byref(f), 64, 0, 4, kb, None, None) == -1  # FP8 needs the scales
    assert lib.misa_route_score_topk_pooled(ctypes.byref(a), 64, 8, 16, 0, None, None, out, None, None, None,
                                            ws, big, None) == -1
    assert lib.misa_route_score_topk_pooled(ctypes.byref(f), 64, 8, 16, 0, kb, None, out, None, None, None,
                                            ws, big, None) == -1
    assert lib.hisa_block_filter_topk_pooled(ctypes.byref(a), 128, 2, 16, None, None, out, None, None, ws, big,
                                             None) == -1
    assert lib.hisa_block_filter_topk_pooled(ctypes.byref(h8), 128, 2, 16, kb, None, out, None, None, ws, big,
                                             None) == -2


def test_stage_entry_point_checks(lib):
    a = _args()
    out = ctypes.c_void_p(0x40000)
    ws = ctypes.c_void_p(0x50000)
    big = 1 << 40
    # indexer_scores: row pitch below L, missing output, missing workspace
    assert lib.indexer_scores(ctypes.byref(a), out, 255, ws, big, None) == -1
    assert lib.indexer_scores(ctypes.byref(a), None, 256, ws, big, None) == -1
    assert lib.indexer_scores(ctypes.byref(a), out, 256, None, big, None) == -3
    # indexer_score_gathered: missing candidates, empty slots, pitch below the
    # compact row, head counts / dims / dtype the gather does not support
    cand = ctypes.c_void_p(0x60000)
    assert lib.indexer_score_gathered(ctypes.byref(a), None, 8, 1, out, 8, ws, big, None) == -1
    assert lib.indexer_score_gathered(ctypes.byref(a), cand, 0, 1, out, 8, ws, big, None) == -1
    assert lib.indexer_score_gathered(ctypes.byref(a), cand, 8, 128, out, 1000, ws, big, None) == -1
    assert lib.indexer_score_gathered(ctypes.byref(_args(H=16)), cand, 8, 1, out, 8, ws, big, None) == -2
    assert lib.indexer_score_gathered(ctypes.byref(_args(d=64)), cand, 8, 1, out, 8, ws, big, None) == -2
    f = _args(qk_dtype=B.DSA_FP8_E4M3, q_scale=0x60000, k_scale=0x70000, H=8)
    assert lib.indexer_score_gathered(ctypes.byref(f), cand, 8, 1, out, 8, ws, big, None) == -2
    # indexer_topk_rows: pitch below the row, index map shorter than the row,
    # k out of range, negative position stride
    sc = ctypes.c_void_p(0x80000)
    assert lib.indexer_topk_rows(sc, 4, 100, 4, 0, 0, 256, 16, None, 0, 1, out, None, ws, big, None) == -1
    assert lib.indexer_topk_rows(sc, 4, 256, 4, 0, 0, 256, 16, cand, 3, 64, out, None, ws, big, None) == -1
    assert lib.indexer_topk_rows(sc, 4, 256, 4, 0, 0, 256, (1 << 24) + 1, None, 0, 1, out, None, ws, big,
                                 None) == -1
    assert lib.indexer_topk_rows(sc, 4, 256, 4, 0, -1, 256, 16, None, 0, 1, out, None, ws, big, None) == -1


def test_selftest_and_noalloc_checks(lib):
    assert lib.dsa_selftest_wait_timeout(None, 256, None) == -3
    assert lib.dsa_selftest_wait_timeout(ctypes.c_void_p(0x50010), 256, None) == -1
    assert lib.dsa_selftest_wait_timeout(ctypes.c_void_p(0x50000), 100, None) == -3
    # the static scratch holds the scores of at most 16 M pairs: larger problems
    # are refused before any CUDA call
    a = _args(T=4, L=5_000_000, q_offset=4_999_996)
    assert lib.indexer_score_topk_noalloc(ctypes.byref(a), 16, ctypes.c_void_p(0x40000), None, None) == -3


def test_indexcache_checks(lib):
    F = _args()
    S = B.IndexerArgs(batch=1, T=4, L=0, H=0, d=0, q_offset=0, qk_dtype=0)  # only batch, T read
    arr = (B.IndexerArgs * 3)(F, S, F)
    P = ctypes.c_void_p
    outs = (P * 3)(0x40000, 0x40000, 0x41000)
    ws, big = ctypes.c_void_p(0x50000), 1 << 30
    one = lib.indexer_workspace_size(ctypes.byref(F), 16)
    assert lib.indexcache_workspace_size(arr, 3, b"FSF", 16) == one
    assert lib.indexcache_workspace_size(arr, 3, b"FXF", 16) == 0
    # rejected before any launch: bad pattern, first layer shared, mismatched
    # S shape, missing output, unsupported F layer, small workspace
    assert lib.indexcache_score_topk(arr, 3, b"SFF", 16, outs, None, ws, big, None) == -1
    assert lib.indexcache_score_topk(arr, 3, b"FXF", 16, outs, None, ws, big, None) == -1
    assert lib.indexcache_score_topk(arr, 3, b"FS", 16, outs, None, ws, big, None) == -1
    bad_s = (B.IndexerArgs * 3)(F, B.IndexerArgs(batch=1, T=5), F)
    assert lib.indexcache_score_topk(bad_s, 3, b"FSF", 16, outs, None, ws, big, None) == -1
    assert lib.indexcache_score_topk(arr, 3, b"FSF", 16, (P * 3)(0x40000, None, 0x41000), None, ws, big,
                                     None) == -1
    bad_f = (B.IndexerArgs * 3)(F, S, _args(H=48))
    assert lib.indexcache_score_topk(bad_f, 3, b"FSF", 16, outs, None, ws, big, None) == -2
    assert lib.indexcache_score_topk(arr, 3, b"FSF", 16, outs, None, ws, one - 1, None) == -3
    # scores requested for an S layer whose F layer has none
    assert lib.indexcache_score_topk(arr, 3, b"FSF", 16, outs, (P * 3)(None, 0x60000, None), ws, big,
                                     None) == -1


def test_hisa_refine_checks(lib):
    a = _args(L=1000, q_offset=996)
    blocks, out, ws, big = ctypes.c_void_p(0x40000), ctypes.c_void_p(0x60000), ctypes.c_void_p(0x50000), 1 << 30
    need = lib.hisa_refine_workspace_size(ctypes.byref(a), 4, 128)
    assert need > 256
    assert lib.hisa_refine_scores(ctypes.byref(a), None, 4, 128, out, 512, ws, big, None) == -1
    assert lib.hisa_refine_scores(ctypes.byref(a), blocks, 4, 128, out, 511, ws, big, None) == -1  # ld < m*blk
    assert lib.hisa_refine_scores(ctypes.byref(a), blocks, 4, 96, out, 512, ws, big, None) == -2  # blk % 128
    f8 = _args(L=1000, q_offset=996, qk_dtype=B.DSA_FP8_E4M3, q_scale=0x60000, k_scale=0x70000)
    assert lib.hisa_block_filter_topk(ctypes.byref(f8), 96, 4, 16, out, None, None, ws, big, None) == -2
    assert lib.hisa_refine_scores(ctypes.byref(_args(H=16, L=1000, q_offset=996)), blocks, 4, 128, out, 512,
                                  ws, big, None) == -2
    assert lib.hisa_refine_scores(ctypes.byref(a), blocks, 4, 128, out, 512, ws, need - 1, None) == -3
    # the HISA workspace grows by the inverted lists when blocks are whole key tiles
    assert lib.hisa_workspace_size(ctypes.byref(a), 128, 4, 16) > lib.hisa_workspace_size(ctypes.byref(a), 96, 4, 16)


def test_dosa_checks(lib):
    a = _args(T=64, L=8192, q_offset=8128)
    big, ws = 1 << 34, ctypes.c_void_p(0x50000)
    out = ctypes.c_void_p(0x40000)
    assert lib.dosa_workspace_size(ctypes.byref(a), 512, 5) > lib.indexer_workspace_size(ctypes.byref(a), 512)
    assert lib.dosa_score_topk(ctypes.byref(a), 512, 5, None, None, None, ws, big, None) == -1
    assert lib.dosa_score_topk(ctypes.byref(a), 512, 14, out, None, None, ws, big, None) == -2    # > 13 screened
    assert lib.dosa_score_topk(ctypes.byref(_args(T=64, L=2048, q_offset=1984)), 128, 5, out, None, None, ws, big,
                               None) == -2                                                       # rows too short
    assert lib.dosa_score_topk(ctypes.byref(_args(H=8, T=64, L=8192, q_offset=8128)), 512, 5, out, None, None, ws,
                               big, None) == -2                                                  # H = 8
    assert lib.dosa_workspace_size(ctypes.byref(_args(T=64, L=2048, q_offset=1984)), 128, 5) == 0
    need = lib.dosa_workspace_size(ctypes.byref(a), 512, 5)
    assert lib.dosa_score_topk(ctypes.byref(a), 512, 5, out, None, None, ws, need - 1, None) == -3


def test_lists_checks(lib):
    a = _args(T=64, L=8192, q_offset=8128)
    ws, big, out = ctypes.c_void_p(0x50000), 1 << 34, ctypes.c_void_p(0x40000)
    need = lib.indexer_lists_workspace_size(ctypes.byref(a), 512)
    assert need > lib.indexer_workspace_size(ctypes.byref(a), 512)
    assert lib.indexer_lists_workspace_size(ctypes.byref(_args(T=4, L=2048, q_offset=2044)), 64) == 0
    assert lib.indexer_score_topk_lists(ctypes.byref(_args(T=4, L=2048, q_offset=2044)), 64, out, None, ws, big,
                                        None) == -2                     # rows too short for the sample
    assert lib.indexer_score_topk_lists(ctypes.byref(a), 2048, out, None, ws, big, None) == -2   # k > L / 8
    assert lib.indexer_score_topk_lists(ctypes.byref(a), 512, None, None, ws, big, None) == -1
    assert lib.indexer_score_topk_lists(ctypes.byref(a), 512, out, None, ws, need - 1, None) == -3
