"""Host-side accounting of bench.py, on CPU: the algorithmic bytes per token of each operator
of the pass (what every GB/s figure divides by), the roofline's DRAM traffic taken from the
committed ncu summary, and the per-workload throughput arithmetic."""
from __future__ import annotations

import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from dit_block_b200 import workloads as wl  # noqa: E402


def test_bytes_per_token_follow_each_operators_reads_and_writes():
    w = wl.WORKLOADS["fullres_10s"]
    e = 2  # bf16
    d, hd, inner = 5120, 40 * 128, 13824
    assert (w.d, w.hd, w.inner) == (d, hd, inner)
    want = {
        "adaln_modulate": (d + d) * e,            # read x, write h
        "dit_epilogue": (2 * hd + 2 * hd) * e,    # read q and k, write them back (v untouched)
        "dit_prologue": (2 * d + 2 * d) * e,      # read x and y, write x' and h
        "swiglu": (2 * inner + inner) * e,        # read [a | b], write silu(a) * b
        "gated_residual": (2 * d + d) * e,        # read x and y, write out
    }
    assert bench.bytes_per_token(w) == want
    assert sum(want.values()) == 216064
    # the pass over the 245,952-token grid moves 53.1 GB
    assert abs(sum(want.values()) * w.n_tokens / 1e9 - 53.14) < 0.01
    tiny = wl.WORKLOADS["tiny"]  # fp32: 4 bytes an element
    assert bench.bytes_per_token(tiny)["swiglu"] == 3 * tiny.inner * 4


def test_roofline_traffic_comes_from_the_committed_capture():
    with open(bench.TRAFFIC_FILE) as f:
        t = json.load(f)
    assert t["kernel_source_sha256_16"] == bench.source_digest(), "SwiGLU source changed since the capture"
    n = 245952
    traffic = bench.ncu_traffic(n)
    assert traffic is not None
    per_token = traffic / n
    # DRAM bytes of the launch equal its algorithmic bytes to well under 1%
    assert abs(per_token / t["algorithmic_bytes_per_token"] - 1) < 0.005
    # the stored per-launch figures are the two-capture difference scaled to one capture
    a, b = t["captures"]
    slope = (b["dram_bytes_read"] + b["dram_bytes_write"] - a["dram_bytes_read"] - a["dram_bytes_write"]) / (
        b["tokens"] - a["tokens"])
    assert abs(per_token - slope) / slope < 1e-6


def test_config_entry_arithmetic():
    w = wl.WORKLOADS["lowres"]
    n = w.n_tokens
    bpt = bench.bytes_per_token(w)
    op_ms = {"adaln_modulate": 0.1, "dit_epilogue": 0.2, "dit_prologue": 0.2, "swiglu": 0.4, "gated_residual": 0.15}
    op_times = {k: [v, v] for k, v in op_ms.items()}
    peak = 6535.7
    e = bench.config_entry(w, n, total_ms=2 * 1.05, steps=2, op_times=op_times, peak=peak)
    assert e["chain_ms"] == pytest.approx(1.05)
    gbs = sum(bpt.values()) * n / 1.05e-3 / 1e9
    assert e["GB_s"] == pytest.approx(gbs, abs=0.1)
    assert e["tokens_per_s"] == pytest.approx(n / 1.05e-3, rel=1e-6)
    assert e["frac_of_measured_peak"] == pytest.approx(gbs / peak, abs=1e-4)
    assert e["frac_of_spec_peak"] == pytest.approx(gbs / 8000.0, abs=1e-4)
    for op, ms in op_ms.items():
        g = bpt[op] * n / (ms * 1e-3) / 1e9
        assert e["per_op"][op]["GB_s"] == pytest.approx(g, abs=0.1)
        assert e["per_op"][op]["ms"] == pytest.approx(ms)
