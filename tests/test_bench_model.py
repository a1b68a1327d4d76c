"""bench.py host logic on the CPU: the algorithmic byte model behind the roofline, and the
lookup of ncu DRAM counters, which must ignore counters taken on another kernel source."""
import hashlib
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

B, S = 4, 16384
TOK = B * S
QB = TOK * 32 * 128 * 2   # one [B,S,32,128] bf16 tensor
KB = TOK * 8 * 128 * 2    # one [B,S,8,128] bf16 tensor
LSE = TOK * 32 * 4


def test_step_bytes_are_each_tensor_once():
    """Forward: read q, k, v, g, write out, lse; backward: read q, k, v, g, out, dout, lse,
    write dq, dk, dv, dg.  5.65e9 B at the 16K sliding workload: the roofline step."""
    w = bench.work(B, S, 128, True)
    assert w["fwd_bytes"] == 3 * QB + 2 * KB + LSE
    assert w["bwd_bytes"] == 6 * QB + 4 * KB + LSE
    assert w["fwd_bytes"] + w["bwd_bytes"] == pytest.approx(5.654e9, rel=1e-3)
    assert bench.work(B, S, 128, False)["bwd_bytes"] == 0


def test_kept_activations_change_kernels_not_the_step():
    plain = bench.work(B, S, 128, True)
    kept = bench.work(B, S, 128, True, saved=True)
    # the forward that keeps q~ (fp16) and every q and k row's inverse RMS writes them once more
    extra = QB + TOK * 32 * 4 + TOK * 8 * 4
    assert kept["kernels"]["fwd_tc_kernel"][0] - plain["kernels"]["fwd_tc_kernel"][0] == extra
    # the strip forward normalises its keys in shared memory; in the training pair it reads the
    # q~ and k~ fp16 that the preparation kernels wrote, the same bytes as raw q and k
    assert kept["kernels"]["fwd_strip_kernel"][0] == plain["kernels"]["fwd_strip_kernel"][0]
    assert plain["kernels"]["fwd_strip_kernel"][0] == plain["fwd_bytes"]
    # the V-only preparation: read v, write V fp16 and a norm per row
    assert kept["kernels"]["bwd_prep_v_kernel"][0] == 2 * KB + TOK * 8 * 4
    # the roofline is the layer's, not this implementation's
    assert (kept["fwd_bytes"], kept["bwd_bytes"]) == (plain["fwd_bytes"], plain["bwd_bytes"])


def test_traffic_lookup_drops_counters_of_another_source(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "k.cu"
    src.write_text("kernel as captured")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    entry = {"kernel": "k", "workload": "w", "source": "k.cu", "source_sha": sha, "bytes_per_launch": 5.0}
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps([entry]))
    assert bench.traffic_for("k", "w") == 5.0
    assert bench.traffic_for("k", "other workload") is None
    src.write_text("kernel changed since")
    assert bench.traffic_for("k", "w") is None


def _row(sm, reasons=()):
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    flags = ["Active" if n in reasons else "Not Active" for n in names]
    return ["0", str(sm), "1965", "900.0", "0x0"] + flags


def test_clock_summary_median_and_reasons():
    """The clocks record of the JSON line: median SM clock over the samples, the maximum, and
    every throttle reason seen active (a run showing a hardware or thermal one is re-taken)."""
    cs = bench.ClockSampler("GPU-test")
    rows = [_row(1965), _row(1320, ("sw_power_cap",)), _row(1500, ("sw_power_cap",)), ["malformed"], []]
    cs.rows = [(float(i), r) for i, r in enumerate(rows)]
    assert cs.summary() == {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3,
                            "window": "all"}
    cs.rows = [(0.0, _row(1100, ("hw_slowdown",))), (1.0, _row(1200, ("sw_thermal_slowdown", "sw_power_cap")))]
    assert cs.summary()["reasons"] == ["hw_slowdown", "sw_power_cap", "sw_thermal_slowdown"]
    cs.rows = []
    assert cs.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_clock_summary_keeps_the_timed_region():
    """Rows inside the marked region count; the idle rows before it and the rows after it do
    not.  A region shorter than the sampling interval takes the two rows around it."""
    cs = bench.ClockSampler("GPU-test")
    cs.rows = [(0.0, _row(900)), (1.0, _row(1900, ("sw_power_cap",))), (1.5, _row(1880)), (3.0, _row(700))]
    cs.t_start, cs.t_end = 0.5, 2.0
    assert cs.summary() == {"sm_mhz": 1890.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 2,
                            "window": "timed region"}
    cs.t_start, cs.t_end = 1.1, 1.2
    sm = cs.summary()
    assert (sm["samples"], sm["window"], sm["sm_mhz"]) == (2, "bracketing", 1890.0)