"""Failure detection without a GPU fault: a bounded device wait that runs out
(a barrier nothing completes) is reported through the workspace status word,
and the context stays usable for the next call."""
import numpy as np
import pytest

import oracle
from sparse_attention_token_score_b200 import binding as B
from sparse_attention_token_score_b200 import workloads as wl
from tests.parity_util import check_selection

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    ws = B.alloc_workspace(256)
    B.dsa_selftest_wait_timeout(ws)
    assert B.dsa_device_status(ws) == -5  # DSA_ERR_TIMEOUT
    assert B.dsa_device_status(ws) == 0   # reading the status clears it
    inp = wl.prefill_inputs(T=40, L=700, H=64, d=128, q_offset=660, seed=31)
    q, k, w, _, _ = B.to_device(inp)
    ix = B.Indexer(q, k, w, inp.q_offset)
    idx, _ = ix.dense(50)
    assert ix.device_status() == 0
    idx = idx.cpu().numpy()
    res = oracle.dense_topk(inp, 50, queries=[0, 17, 39])
    for i, t in enumerate(res["queries"]):
        s, c = res["scores"][i], res["cond"][i]
        check_selection(idx[0, t], np.arange(s.size), s, c, 50, what=f"after timeout t={t}")
