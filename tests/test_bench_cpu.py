"""The arithmetic behind bench.py's JSON line, on CPU.

The roofline fraction, the work-done throughput, the pre-pass bandwidth and
the SFU rate are all derived from a count of visible (query, key) pairs and
a few per-element byte counts.  These tests hold those counts to brute force
and closed forms, the percentiles to NumPy's linear interpolation, the
traffic record to its source-hash rule, and the kernel name to the
library's persistent-kernel rule, so that a wrong count (a causal mask
counted as the full matrix, a missing diagonal) fails here.
"""

import hashlib
import json
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from quantized_attention_quant_b200.workloads import WORKLOADS  # noqa: E402


@pytest.mark.parametrize("N", [1, 2, 77, 128, 300])
@pytest.mark.parametrize("causal", [False, True])
def test_visible_pairs_against_brute_force(N, causal):
    w = WORKLOADS["tiny"].with_(N=N, causal=causal)
    i, j = np.meshgrid(np.arange(N), np.arange(N), indexing="ij")
    want = int(((j <= i) if causal else np.ones_like(i, bool)).sum())
    assert bench.visible_pairs(w) == want
    # 4 d operations per pair (2 d for the score, 2 d for its share of P~V)
    assert bench.work_ops(w, 3) == 4.0 * w.d * want * 3


def test_work_counts_of_the_target_shape():
    w = WORKLOADS["n16k"]
    heads = w.B * w.H
    assert bench.work_ops(w, heads) == pytest.approx(4 * 128 * 16384 ** 2 * 64)
    # non-causal: the metric's 4 B H N^2 d and the work done agree
    assert w.ops == pytest.approx(bench.work_ops(w, heads))
    # causal: the work done is N (N + 1) / 2 of the N^2 pairs
    c = w.with_(causal=True)
    assert bench.work_ops(c, heads) / c.ops == pytest.approx((16384 + 1) / (2 * 16384))


@pytest.mark.parametrize("mode,write", [("int8_fp8", 1.0), ("fp8", 1.0), ("fp4", 0.5 + 1 / 16)])
def test_prepass_bytes(mode, write):
    # Q, K and V read once as 16-bit values, their codes written once
    w = WORKLOADS["tiny"].with_(mode=mode)
    elem = w.N * w.d * 5
    assert bench.prepass_bytes(w, 5) == pytest.approx(3 * elem * (2 + write))


def test_percentile_matches_numpy_linear_interpolation():
    rng = np.random.default_rng(3)
    for n in (1, 2, 7, 20):
        xs = list(rng.standard_normal(n))
        for p in (0, 50, 95, 100):
            assert bench.percentile(xs, p) == pytest.approx(float(np.percentile(xs, p)))
    assert bench.percentile([], 50) is None


def test_summarize_roofline_is_work_over_time_over_peak(monkeypatch):
    peaks = {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0, "sm_max_mhz": 2000.0}
    monkeypatch.setattr(bench, "measured_peaks", lambda: (peaks, "measured"))
    monkeypatch.setattr(bench, "read_traffic", lambda name: None)
    for name, ratio in (("n16k", 2.0), ("fp4", 4.0)):
        w = WORKLOADS[name]
        heads = w.B * w.H
        times = [(8.0, 0.4, 7.0), (8.2, 0.5, 7.2), (7.8, 0.3, 6.8)]
        s = bench.summarize(w, 1, times, 148)
        t_attn = 7.0e-3
        achieved = bench.work_ops(w, heads) / t_attn / 1e12
        assert s["roofline"]["achieved"] == pytest.approx(achieved, abs=0.05)
        assert s["roofline"]["peak"] == pytest.approx(1000.0 * ratio)
        assert s["roofline"]["frac"] == pytest.approx(achieved / (1000.0 * ratio), abs=1e-4)
        assert s["value"] == pytest.approx(w.ops / 8.0e-3 / 1e12, abs=0.01)
        assert s["prepass_gbs"] == pytest.approx(bench.prepass_bytes(w, heads) / 0.4e-3 / 1e9,
                                                 abs=0.05)
        # one exponential per visible pair against 16 per clock per SM
        per_clk = bench.visible_pairs(w) * heads / t_attn / (148 * 2000e6)
        assert s["exp_rate"]["exps_per_clk_per_sm"] == pytest.approx(per_clk, abs=0.005)
        assert s["exp_rate"]["sfu_frac"] == pytest.approx(per_clk / 16, abs=1e-4)


def test_traffic_record_is_used_only_for_the_source_it_was_taken_on(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("// one kernel\n")
    digest = hashlib.sha256(src.read_bytes()).hexdigest()
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"n16k": {"bytes": 1234, "kernel_source": "kernel.cu", "kernel_source_sha256": digest}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.read_traffic("n16k") == 1234
    assert bench.read_traffic("llm") is None           # no record for that workload
    src.write_text("// the kernel, changed\n")
    assert bench.read_traffic("n16k") is None          # record older than the source


def test_attention_kernel_name_follows_the_persistent_rule():
    # short items over more tiles than SMs run persistent; long ones one
    # CTA per (query tile, head); FP4 has its own kernel
    assert bench.attention_kernel(WORKLOADS["llm"], 148) == "attn_i8f8_persist_kernel"
    assert bench.attention_kernel(WORKLOADS["n16k"], 148) == "attn_i8f8_kernel"
    assert bench.attention_kernel(WORKLOADS["fp4"], 148) == "attn_fp4_kernel"
    # too few tiles to fill the SMs: one CTA each
    assert bench.attention_kernel(WORKLOADS["tiny"], 148) == "attn_i8f8_kernel"
