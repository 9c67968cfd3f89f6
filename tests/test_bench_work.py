"""The algorithmic work bench.py divides by device time (the roofline's `achieved`), checked
against sizes written out from the layer's definition.  No GPU.

- The container of the colibrì README stores an int4 expert as packed codes plus one fp32 scale
  per output row; the iliria page gives about 19 MB per GLM expert, scales 0.22 % of the bytes.
- The expert FFN is three d x f matrices per expert (gate, up, down): 2 flops per multiply-add
  and per token slot.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synthetic as syn  # noqa: E402

GLM = syn.CONFIGS["glm_decode"]
EXPERT = 18_915_328          # 3 * 2048 * 6144 / 2 bytes of codes + (2 * 2048 + 6144) * 4 bytes of scales


def test_expert_bytes_match_the_container():
    assert bench.expert_bytes(GLM) == EXPERT
    codes = 3 * 2048 * 6144 // 2
    assert abs((EXPERT - codes) / codes - 0.00217) < 1e-5        # the page's 0.22 % of scales


def test_single_token_step_bytes():
    w = bench.kernel_work(GLM, 1, 8)
    kind, fused = w["fused"]
    assert kind == "hbm"
    router = 256 * 6144 * 4 + 256 * 4                  # fp32 router matrix and bias
    x, h, out = 6144 * 2, 9 * 2048 * 2, 6144 * 4       # x read, h written and read back, y written
    assert fused == 9 * EXPERT + router + x + 2 * h + out


def test_gemm_flops_count_every_token_slot():
    cfg = syn.CONFIGS["glm_prefill"]
    w = bench.kernel_work(cfg, 2048, 200)              # flops do not depend on the unique experts
    slots = 2048 * 8 + 2048                             # routed slots + the shared expert's
    assert w["gemm_gateup"] == ("tensor", 2 * 2 * slots * 6144 * 2048)
    assert w["gemm_down"] == ("tensor", 2 * slots * 6144 * 2048)
    total = w["gemm_gateup"][1] + w["gemm_down"][1]
    assert total == pytest.approx(1.392e12, rel=1e-3)  # 2 T (k + 1) 3 d f


def test_job_throughput_counts_all_ranks():
    assert bench.job_tokens_per_s(4, 100, 2, 50.0) == pytest.approx(4 * 100 * 2 / 0.05)
    assert bench.replica_token_base(3) != bench.replica_token_base(2)


def test_step_percentiles():
    assert bench.step_percentiles([]) == {}
    p = bench.step_percentiles([5.0, 1.0, 3.0, 2.0, 4.0])
    assert p == {"p10": 1.0, "p50": 3.0, "p90": 5.0}
    q = bench.step_percentiles(range(101))
    assert (q["p10"], q["p50"], q["p90"]) == (10.0, 50.0, 90.0)


def test_cpu_baseline_times_all_cores_and_one():
    import oracle
    cores = oracle.num_threads()
    res = bench.cpu_baseline(syn.CONFIGS["tiny"], "tiny", 0, 0.2)
    assert res["kind"] == "oracle" and res["unit"] == "tokens/s" and res["value"] > 0
    assert res["cores"] == cores and "layer" not in res
    one = res["single_core"]
    assert one["cores"] == 1 and one["value"] > 0 and "one host core" in one["sample"]
    assert oracle.num_threads() == cores                # the thread count is put back


def test_oracle_result_does_not_depend_on_threads():
    import oracle
    cfg = syn.CONFIGS["tiny"]
    x = syn.gen_x(cfg, 0, T=cfg.T)
    L = bench.oracle_sample_layer(cfg, 0, x)
    cores = oracle.num_threads()
    many = L.forward(x)
    oracle.set_num_threads(1)
    try:
        one = L.forward(x)
    finally:
        oracle.set_num_threads(cores)
    for key in ("out", "idx", "w", "gap"):
        assert many[key].tobytes() == one[key].tobytes()


def test_traffic_is_reported_only_for_unchanged_sources():
    import json
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    keys = [key for key in rec if not key.startswith("_")]
    assert {"glm_decode:fused", "glm_prefill:gemm_gateup", "glm_prefill:gemm_down"} <= set(keys)
    for key in keys:
        workload, kernel = key.split(":")
        assert workload in bench.WORKLOADS
        r = rec[key]
        fresh = bench.source_sha(r["sources"]) == r["source_sha"]
        assert bench.traffic_for(kernel, workload) == (r["bytes_per_launch"] if fresh else None)
        assert r["bytes_per_launch"] > 0
    assert bench.traffic_for("no_such_kernel", "glm_decode") is None
    assert bench.traffic_for("fused", "no_such_workload") is None


def test_traffic_is_null_once_a_source_changes(monkeypatch):
    monkeypatch.setattr(bench, "source_sha", lambda paths: "0" * 16)
    assert bench.traffic_for("fused", "glm_decode") is None


def test_every_workload_is_measured_once_with_the_headline_first():
    import argparse
    a = argparse.Namespace(workload="glm_decode", workloads="all")
    names = bench.selected_workloads(a)
    assert names[0] == "glm_decode" and sorted(names) == sorted(bench.WORKLOADS)
    a = argparse.Namespace(workload="granite", workloads="none")
    assert bench.selected_workloads(a) == ["granite"]
    a = argparse.Namespace(workload="tiny", workloads="glm_prefill,tiny")
    assert bench.selected_workloads(a) == ["tiny", "glm_prefill"]
