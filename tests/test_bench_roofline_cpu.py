"""bench.py's roofline arithmetic (host logic, no GPU): algorithmic work per launch over the
event-timed duration, the peak it is compared with, and when the captured DRAM traffic is
attached."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from workloads import WORKLOADS  # noqa: E402

PK = {"hbm_gbs": 6650.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}


def test_pair_count_causal_and_full():
    assert bench.pair_count(8, False) == 64
    assert bench.pair_count(8, True) == 36     # n (n + 1) / 2: the diagonal included


def test_backward_roofline_arithmetic():
    w = WORKLOADS[bench.DEFAULT_WORKLOAD]
    flop = 10.0 * w.d * w.n * (w.n + 1) / 2 * w.B * w.H
    r = bench.roofline(w, "attn_bwd_tc", 2.5, PK, "measured", sustained=False)
    assert r["algorithmic_per_launch"] == pytest.approx(flop)
    assert r["achieved"] == pytest.approx(flop / 2.5e-3 / 1e12, rel=1e-6)
    assert r["peak"] == PK["bf16_tflops"] and r["bound"] == "tensor"
    assert r["frac"] == pytest.approx(r["achieved"] / 1600.0, abs=1e-4)
    s = bench.roofline(w, "attn_bwd_tc", 2.5, PK, "measured", sustained=True)
    assert s["peak"] == PK["bf16_tflops_sustained"]
    assert s["frac_of_burst"] == r["frac"]


def test_forward_is_two_fifths_of_the_backward_work():
    w = WORKLOADS["b4_h16_n2048_d64_bf16"]
    f = bench.roofline(w, "attn_fwd_tc", 1.0, PK, "measured")
    b = bench.roofline(w, "attn_bwd_tc", 1.0, PK, "measured")
    assert f["algorithmic_per_launch"] * 10 == pytest.approx(b["algorithmic_per_launch"] * 4)


def test_traffic_only_for_the_captured_workload_and_mode(monkeypatch):
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as fh:
        rec = json.load(fh)["attn_bwd_tc"]
    monkeypatch.setattr(bench, "kernel_source_sha", lambda k: rec["source_sha"])
    w = WORKLOADS[bench.DEFAULT_WORKLOAD]
    assert bench.roofline(w, "attn_bwd_tc", 2.5, PK, "m")["traffic"] == \
        rec["dram_bytes_per_launch"]
    assert bench.roofline(w, "attn_bwd_tc", 2.5, PK, "m", deterministic=True)["traffic"] is None
    other = WORKLOADS["b4_h16_n2048_d64_bf16"]
    assert bench.roofline(other, "attn_bwd_tc", 2.5, PK, "m")["traffic"] is None
    # a kernel source changed since the capture: no traffic figure
    monkeypatch.setattr(bench, "kernel_source_sha", lambda k: "0" * 16)
    assert bench.roofline(w, "attn_bwd_tc", 2.5, PK, "m")["traffic"] is None


def test_memory_bound_kernel_rooflines():
    w = WORKLOADS[bench.DEFAULT_WORKLOAD]
    act = w.B * w.H * w.n * w.d
    r = bench.kernel_roofline(w, "dq_unrotate", 0.05, PK)
    assert r["bound"] == "hbm"
    assert r["achieved"] == pytest.approx(6.0 * act / 0.05e-3 / 1e9, rel=1e-3)
    assert bench.kernel_roofline(w, "rope_table", 0.01, PK) is None
