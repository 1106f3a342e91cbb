"""Host-side logic of bench.py (no GPU): workload sizes, replica
aggregation, and the captured-traffic table's invalidation rule."""
import os
import shutil

import pytest

import bench
from sparse_attention_token_score_b200 import workloads as wl


@pytest.mark.parametrize("name", ["tiny", "dsa", "decode", "misa", "hisa", "dsa_fp8", "indexcache", "dosa",
                                  "dosa_lownorm", "dsa_lists", "hisa_decode"])
def test_pairs_are_the_dense_visible_pairs(name):
    c, batch, off, pairs, label = bench.workload_desc(name)
    T = c["T"]
    # query t at position off + t sees off + t + 1 keys (never more than L)
    expect = batch * sum(min(c["L"], off + t + 1) for t in range(T)) * len(c.get("pattern", "F"))
    assert pairs == expect
    assert label.startswith({"tiny": "tiny_prefill", "dsa": "dsa_chunk", "decode": "decode_fp8",
                              "misa": "misa_dagger", "hisa": "hisa", "dsa_fp8": "dsa_chunk_fp8",
                              "indexcache": "indexcache_dsa_chunk", "dosa": "dosa_dsa_chunk",
                              "dosa_lownorm": "dosa_lownorm_dsa_chunk", "dsa_lists": "dsa_chunk_lists",
                              "hisa_decode": "hisa_decode_fp8"}[name])


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
    # a capture recorded against the current source stays valid ...
    monkeypatch.setitem(bench.TRAFFIC, key, (123.0e6, bench.source_hash(key[1])))
    assert bench.traffic_for(*key) == bench.TRAFFIC[key][0]
    f = dst / "score_tc.cuh"
    f.write_text("// a comment line\n" + f.read_text())         # comments do not count
    assert bench.traffic_for(*key) == bench.TRAFFIC[key][0]
    f.write_text(f.read_text() + "\nstatic int changed_code = 1;\n")  # code does
    assert bench.traffic_for(*key) is None
    assert bench.traffic_for("dsa", "no such kernel") is None
    # a staged name ("stage: kernel") hashes its own kernel family's sources
    key = ("hisa", "tokens: score_inv (block-major)")
    monkeypatch.setitem(bench.TRAFFIC, key, (7.0e6, bench.source_hash(key[1])))
    assert bench.traffic_for(*key) == 7.0e6
    f.write_text(f.read_text() + "\nstatic int changed_again = 2;\n")  # score_tc.cuh: not its source
    assert bench.traffic_for(*key) == 7.0e6
    g = dst / "score_inv.cuh"
    g.write_text(g.read_text() + "\nstatic int changed_inv = 3;\n")
    assert bench.traffic_for(*key) is None


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
    # same config object as the GPU arm's line, and a step time that is the
    # sampled step's own (not an extrapolation to the full workload)
    c, batch, off, pairs, label = bench.workload_desc("tiny")
    assert line["config"] == bench.workload_config(c, batch, label, off, pairs, 1)
    assert line["ms_per_step"] * line["steps"] / 1e3 < 600
    assert line["sample"]["pairs_per_timed_step"] <= pairs


def test_clock_summary_keeps_the_timed_window():
    S = bench.ClockSampler
    rows = [(0.00, 1900.0, 1965.0, 0), (0.01, 1950.0, 1965.0, 0x4), (0.02, 1960.0, 1965.0, 0),
            (0.03, 1000.0, 1965.0, 0x40), (0.10, 1100.0, 1965.0, 0x8)]
    st = S.summarize(rows, 0.005, 0.025, 1965.0)
    # the sample before the window, the two inside and the first one after
    assert st["samples"] == 4 and st["samples_inside"] == 2
    assert st["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert st["sm_mhz"] == 1925.0
    assert S.summarize(rows, None, None, 1965.0)["samples"] == 0
