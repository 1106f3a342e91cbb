"""Host-side logic of bench.py (no GPU): workload sizes, replica
aggregation, and the captured-traffic table's invalidation rule."""
import os
import shutil

import pytest

import bench
from sparse_attention_token_score_b200 import workloads as wl


@pytest.mark.parametrize("name", ["tiny", "dsa", "decode", "misa", "hisa"])
def test_pairs_are_the_dense_visible_pairs(name):
    c, batch, off, pairs, label = bench.workload_desc(name)
    T = c["T"]
    # query t at position off + t sees off + t + 1 keys (never more than L)
    expect = batch * sum(min(c["L"], off + t + 1) for t in range(T))
    assert pairs == expect
    assert label.startswith({"tiny": "tiny_prefill", "dsa": "dsa_chunk", "decode": "decode_fp8",
                              "misa": "misa_dagger", "hisa": "hisa"}[name])


def test_dsa_chunk_size():
    c, batch, off, pairs, _ = bench.workload_desc("dsa")
    assert (c["T"], c["L"], off, pairs) == (4096, 32768, 28672, 125831168)


def test_profiling_subsets_keep_the_prefix():
    c, batch, off, pairs, _ = bench.workload_desc("dsa", queries=1024)
    assert c["T"] == 1024 and off == c["L"] - 1024
    c, batch, off, pairs, _ = bench.workload_desc("decode", batch=8)
    assert batch == 8 and pairs == 8 * c["L"]


def test_aggregate_ranks():
    t, v = bench.aggregate_ranks(10.0, 1000, 5, 1)
    assert t == 10.0 and v == pytest.approx(5000 / 0.01)
    t, v = bench.aggregate_ranks(10.0, 1000, 5, 4, reduce_max=lambda x: 2 * x)
    assert t == 20.0 and v == pytest.approx(4 * 5000 / 0.02)


def test_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    src = os.path.join(bench.ROOT, "sparse_attention_token_score_b200", "csrc")
    dst = tmp_path / "sparse_attention_token_score_b200" / "csrc"
    shutil.copytree(src, dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    key = ("dsa", "score_tc<bf16>")
    assert bench.traffic_for(*key) == bench.TRAFFIC[key][0]
    f = dst / "score_tc.cuh"
    f.write_text("// a comment line\n" + f.read_text())         # comments do not count
    assert bench.traffic_for(*key) == bench.TRAFFIC[key][0]
    f.write_text(f.read_text() + "\nstatic int changed_code = 1;\n")  # code does
    assert bench.traffic_for(*key) is None
    assert bench.traffic_for("dsa", "no such kernel") is None


def test_reference_arm_json_line():
    # the oracle arm needs no GPU: one JSON line with the contract's keys
    import json
    import subprocess
    import sys
    out = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, check=True).stdout
    line = json.loads(out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["warmup"] == 3
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["config"]["workload"].startswith("tiny_prefill")
