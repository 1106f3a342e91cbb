"""Calls from several host threads: each thread owns its stream and
workspace; results must equal the same calls made one after another."""
import threading

import numpy as np
import pytest
import torch

from sparse_attention_token_score_b200 import binding as B
from sparse_attention_token_score_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _inputs(seed):
    inp = wl.prefill_inputs(T=300, L=2500, H=64, d=128, q_offset=2200, seed=seed)
    q, k, w, _, _ = B.to_device(inp)
    return q, k, w, inp.q_offset


def test_two_threads_match_sequential():
    data = [_inputs(s) for s in (21, 22)]
    ref = [B.Indexer(q, k, w, off).dense(64)[0].cpu().numpy() for (q, k, w, off) in data]
    torch.cuda.synchronize()
    out = [None, None]
    errors = []

    def work(i):
        try:
            s = torch.cuda.Stream()
            q, k, w, off = data[i]
            with torch.cuda.stream(s):
                for _ in range(5):
                    idx, _ = B.Indexer(q, k, w, off).dense(64, stream=s)
                s.synchronize()
            out[i] = idx.cpu().numpy()
        except Exception as e:  # reported below
            errors.append(e)

    th = [threading.Thread(target=work, args=(i,)) for i in range(2)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert not errors, errors
    for i in range(2):
        assert np.array_equal(out[i], ref[i])
