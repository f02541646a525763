"""Host-side pieces of bench.py on the CPU: the algorithmic byte count behind
every GB/s figure, the reference arm's bounded sample, and the rule that a
committed ncu summary's DRAM traffic is reported only for the kernel sources it
was captured from."""

import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads  # noqa: E402


def test_algorithmic_bytes_of_the_workloads():
    # codes N K / 2 + scales N K / 16 + sign bits (N + K) r / 8 + BF16 x and y + FP32
    # alpha, tabulated independently for the decode and MLP shapes
    want = {"decode": 15_423_488, "mlp_up": 41_633_792, "mlp_down": 42_240_000}
    for name, b in want.items():
        w = workloads.CONFIGS[name]
        assert bench.algo_bytes(w.M, w.N, w.K, w.r) == b, name


def test_algorithmic_bytes_grow_with_each_term():
    base = bench.algo_bytes(1, 128, 256, 32)
    assert bench.algo_bytes(1, 256, 256, 32) - base == 128 * 256 // 2 + 128 * 256 // 16 + 128 * 32 // 8 + 2 * 128
    assert bench.algo_bytes(2, 128, 256, 32) - base == 2 * 256 + 2 * 128
    assert bench.algo_bytes(1, 128, 256, 64) - base == (128 + 256) * 32 // 8 + 4 * 32


def test_reference_sample_is_the_same_problem_smaller():
    w = workloads.CONFIGS["tiny"]
    s = bench._oracle_sample(w, 3, 128, 8)
    assert s["x"].shape == (w.M, 128)
    assert s["wq"].shape == (3, 64) and s["ws"].shape == (3, 8)
    assert s["U"].shape == (3, 8) and s["V"].shape == (128, 8) and s["alpha"].shape == (8,)
    y = bench._oracle_step(s)
    assert y.shape == (w.M, 3) and np.all(np.isfinite(y))
    # the full sample reproduces the oracle's output rows on the same inputs
    full = bench._oracle_step(bench._oracle_sample(w, w.N))
    part = bench._oracle_step(bench._oracle_sample(w, 5))
    np.testing.assert_array_equal(part, full[:, :5])


def test_ncu_traffic_follows_the_source_digest(monkeypatch):
    got = bench.ncu_traffic("decode", 1)
    if got is not None:
        assert got > 14_000_000                      # about the 15.4 MB a decode call moves
    monkeypatch.setattr(bench, "kernel_source_digest", lambda: "0000000000000000")
    assert bench.ncu_traffic("decode", 1) is None
    assert bench.ncu_traffic("no_such_workload", 1) is None


def test_every_committed_profile_names_its_workload_and_kernel():
    # each summary under profiles/ carries the two fields the bench reads, and its
    # workload resolves to a configuration or a sweep point of the bench
    prof = os.path.join(ROOT, "profiles")
    names = [f for f in os.listdir(prof) if f.startswith("decode_kernel_") and f.endswith(".md")]
    assert names
    for f in names:
        text = open(os.path.join(prof, f)).read()
        assert "- source_digest: `" in text and "- dram_bytes_per_launch: " in text, f
        wl = f[len("decode_kernel_"):-3]
        if wl.startswith("sweep_M"):
            M, r = (int(v) for v in wl[len("sweep_M"):].split("_r"))
            assert workloads.sweep_config(M, r).name == wl
        else:
            assert wl in workloads.CONFIGS, f


def test_metric_range_reports_the_worst_point():
    extra = {"sweep_M8_r512": {"us": 17.6, "frac": 0.137}, "sweep_M16_r512": {"us": 19.0, "frac": 0.128},
             "sweep_M32_r512": {"us": 23.7, "frac": 0.105}, "mlp_up": {"us": 22.0, "frac": 0.293}}
    got = bench.metric_range(11.4, 0.21, extra)
    assert sorted(got["points"]) == ["M1", "M16", "M32", "M8"]
    assert got["worst"] == {"M": 32, "us": 23.7, "frac": 0.105}
    # with only the headline, the headline is the worst point
    assert bench.metric_range(11.4, 0.21, {})["worst"]["M"] == 1


def test_sweep_option_selects_a_sweep_point():
    class A:
        sweep = "64,512"
        workload = "decode"
    w = bench.selected_workload(A)
    assert (w.name, w.M, w.N, w.K, w.r) == ("sweep_M64_r512", 64, 5120, 5120, 512)
    A.sweep = None
    assert bench.selected_workload(A).name == "decode"
