"""indexer_score_topk_noalloc: the dense score + top-k for callers that cannot
allocate device memory (a plugin whose host runtime owns every device
allocation, a loop where cudaMalloc and its possible device synchronisation
are not allowed, or code with no allocator at all). It uses the library's own
static scratch instead of a caller workspace. These checks compare it, through
the C ABI, with the workspace entry point on the same inputs, twice in a row
(the second call reuses scratch that still holds the first call's scores),
check after each call that the scratch's status word (dsa_noalloc_status)
reads "ok", and check that a problem too large for the scratch is refused
before any launch.

This file is collected last so that a run stopping at the first failure has
already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

from sparse_attention_token_score_b200 import binding as B
from sparse_attention_token_score_b200 import workloads as wl
from tests.parity_util import RTOL_BF16, RTOL_FP8

pytestmark = pytest.mark.gpu


def _compare(inp, topk, rtol):
    q, k, w, qs, ks = B.to_device(inp)
    args = B.make_args(q, k, w, inp.q_offset, qs, ks)
    shape = (inp.batch, inp.T, topk)
    ref_idx = torch.empty(shape, dtype=torch.int32, device="cuda")
    ref_sc = torch.empty(shape, dtype=torch.float32, device="cuda")
    ws = B.alloc_workspace(B.indexer_workspace_size(args, topk))
    B.indexer_score_topk(args, topk, ref_idx, ref_sc, ws)
    idx = torch.full(shape, -7, dtype=torch.int32, device="cuda")
    sc = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
    st = B.lib().indexer_score_topk_noalloc(ctypes.byref(args), topk, ctypes.c_void_p(idx.data_ptr()),
                                            ctypes.c_void_p(sc.data_ptr()),
                                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, B.STATUS.get(st, st)
    # a bounded device wait that gave up inside the call would show here
    st = B.lib().dsa_noalloc_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, B.STATUS.get(st, st)
    ref_idx, ref_sc, idx, sc = (t.cpu().numpy() for t in (ref_idx, ref_sc, idx, sc))
    assert np.array_equal(idx, ref_idx)
    pad = ref_idx < 0
    assert np.all(np.isneginf(sc[pad]))
    assert np.all(np.abs(sc[~pad] - ref_sc[~pad]) <= rtol * np.abs(ref_sc[~pad]))


def test_noalloc_matches_workspace_entry_point_twice():
    # first: a bf16 prefill chunk (several key tiles, ragged tail)
    _compare(wl.prefill_inputs(37, 3000, 64, 128, q_offset=2963, seed=31), 100, RTOL_BF16)
    # second, right after: a smaller FP8 decode batch on the same scratch
    _compare(wl.decode_inputs(batch=3, L=1000, H=32, d=128, seed=32), 77, RTOL_FP8)


def test_noalloc_rejects_problems_larger_than_its_scratch():
    a = B.IndexerArgs(batch=1, T=4096, L=32768, H=64, d=128, q_offset=28672, qk_dtype=B.DSA_BF16)
    a.q, a.k, a.w = 0x10000, 0x20000, 0x30000  # never dereferenced: the size check comes first
    st = B.lib().indexer_score_topk_noalloc(ctypes.byref(a), 2048, ctypes.c_void_p(0x40000), None, None)
    assert st == -3
