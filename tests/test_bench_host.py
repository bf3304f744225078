"""Host logic of bench.py that needs no GPU: the reference arm (the oracle timed on the host
cores) and the bounded samples it is timed on."""
from __future__ import annotations

import os
import sys
import time
from types import SimpleNamespace

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def test_first_rows_cuts_segments_in_order():
    import bench

    seg = np.array([0, 3, 5, 9], np.int32)
    idx = np.array([7, 2, 4], np.int32)
    cases = {1: ([0, 1], [7]), 3: ([0, 3], [7]), 4: ([0, 3, 4], [7, 2]), 5: ([0, 3, 5], [7, 2]),
             8: ([0, 3, 5, 8], [7, 2, 4]), 9: ([0, 3, 5, 9], [7, 2, 4])}
    for n, (want_seg, want_idx) in cases.items():
        got_seg, got_idx = bench.OracleSampler.first_rows(seg, idx, n)
        assert got_seg.tolist() == want_seg and got_idx.tolist() == want_idx, n


def test_first_rows_sample_equals_the_call_it_cuts():
    # the sampled rows are the first rows of the whole call, bit for bit
    import bench
    import oracle
    from adapter_matmul_b200 import inputs

    w = inputs.small_random(40, 3, 64, 48, 8, "f16", seed=11)
    seg, idx, _ = oracle.group_segments(w.ids, w.num_adapters)
    X, Y = w.x(), w.y_random()
    A = [w.adapter_a(i) for i in range(3)]
    B = [w.adapter_b(i) for i in range(3)]
    full, _ = oracle.apply_f32(Y, X, A, B, seg, idx, w.scale, w.dtype)
    for n in (1, int(seg[1]), int(seg[1]) + 1, 40):
        s2, i2 = bench.OracleSampler.first_rows(seg, idx, n)
        part, _ = oracle.apply_f32(Y[:n], X[:n], A, B, s2, i2, w.scale, w.dtype)
        assert np.array_equal(part, full[:n]), n


def test_reference_arm_line_and_bounded_time(monkeypatch):
    import bench

    monkeypatch.setattr(bench, "REFERENCE_BUDGET_S", 1.0)
    spec = bench.make_spec("tiny")
    args = SimpleNamespace(steps=20000, warmup=200)
    t0 = time.perf_counter()
    out = bench.run_reference(args, spec, 0)
    elapsed = time.perf_counter() - t0
    # 20200 steps share the budget: the run stays near it, not 20000 x a minimum step
    assert elapsed < 20.0
    assert out["impl"] == "reference" and out["steps"] == 20000 and out["warmup"] == 200
    assert out["value"] > 0 and out["unit"] == bench.UNIT and out["metric"] == bench.METRIC
    assert out["cpu_baseline"]["kind"] == "oracle" and out["cpu_baseline"]["value"] == out["value"]
    assert out["e2e"] == {"value": out["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}


def test_reference_arm_partial_rows_on_a_large_workload(monkeypatch):
    # a call far above a step's share: each step runs the first rows of one call
    import bench

    monkeypatch.setattr(bench, "REFERENCE_BUDGET_S", 0.5)
    spec = bench.make_spec("llama70b_decode_h8192")
    out = bench.run_reference(SimpleNamespace(steps=50, warmup=3), spec, 0)
    assert out["cpu_baseline"]["sample"].startswith("first ")
    assert out["value"] > 0


def test_make_roofline_arithmetic():
    import bench

    r = bench.make_roofline(36700160, 3.0e9, 10.975e-6, 6544.7, 1630.0, "measured", 35726336, "k")
    assert r["achieved"] == round(36700160 / 10.975e-6 / 1e9, 1)
    assert r["frac"] == round(36700160 / 10.975e-6 / 1e9 / 6544.7, 4)
    assert r["frac_nominal"] == round(36700160 / 10.975e-6 / 1e9 / 8000.0, 4)
    assert r["tflops"] == round(3.0e9 / 10.975e-6 / 1e12, 3)
    assert r["tensor_frac"] == round(3.0e9 / 10.975e-6 / 1e12 / 1630.0, 4)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6544.7 and r["traffic"] == 35726336
    assert r["launch_us"] == 10.975 and r["algorithmic_bytes_per_launch"] == 36700160


def test_rows_share_partitions_a_call():
    import bench
    import oracle
    from adapter_matmul_b200 import inputs

    seg = np.array([0, 3, 5, 9], np.int32)
    idx = np.array([7, 2, 4], np.int32)
    s, i = bench.rows_share(seg, idx, 2, 7)
    assert s.tolist() == [0, 1, 3, 5] and i.tolist() == [7, 2, 4]
    s, i = bench.rows_share(seg, idx, 3, 5)
    assert s.tolist() == [0, 2] and i.tolist() == [2]
    # shares computed apart and put side by side equal the whole call, bit for bit
    w = inputs.small_random(37, 4, 48, 40, 8, "bf16", seed=5)
    seg, idx, _ = oracle.group_segments(w.ids, w.num_adapters)
    X, Y = w.x(), w.y_random()
    A = [w.adapter_a(k) for k in range(4)]
    B = [w.adapter_b(k) for k in range(4)]
    full, _ = oracle.apply_f32(Y, X, A, B, seg, idx, w.scale, w.dtype)
    bounds = [0, 5, 6, 20, 37]
    parts = []
    for a, b in zip(bounds[:-1], bounds[1:]):
        s, i = bench.rows_share(seg, idx, a, b)
        part, _ = oracle.apply_f32(Y[a:b], X[a:b], A, B, s, i, w.scale, w.dtype)
        parts.append(part)
    assert np.array_equal(np.concatenate(parts), full)


def test_all_cores_baseline_runs_in_spawned_processes():
    import bench

    out = bench.oracle_all_cores(bench.make_spec("tiny"), 0.3, max_procs=4)
    assert "unavailable" not in out, out
    assert out["kind"] == "oracle" and out["value"] > 0 and 1 <= out["cores"] <= 4


def test_dispatch_name_of_the_batched_default_line():
    import bench
    from adapter_matmul_b200 import sgmv

    spec = bench.make_spec("distinct")
    assert bench.dispatch_name(spec, 32, 1, sgmv.F16, 0) == "batched FUSED (4 projections per launch)"
    assert set(bench.VARIANT_NAMES.values()) == {"SPLIT", "GROUPED_TC", "FUSED", "FUSED_TC", "SPLIT_TC"}
    assert all(getattr(sgmv, "VARIANT_" + name) == v for v, name in bench.VARIANT_NAMES.items())
