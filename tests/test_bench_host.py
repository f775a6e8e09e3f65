"""Host logic of the benchmark (no GPU): the algorithmic bytes per step that the
roofline divides by, the lookup of profiled DRAM traffic, and the summary of
the clock samples taken during the timed region.

The byte counts are worked out here by hand from each workload's shapes: codes
and scales read and written, the input vectors and gates, and the fp32 output
(plus Mamba-2's per-request B and C and per-head A and D).
"""
import json
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.join(os.path.dirname(__file__), ".."))
import bench  # noqa: E402
import workloads as W  # noqa: E402


def _gdn_head(dk, dv, bits):
    codes = dk * dv * bits // 8
    return 2 * codes + 2 * 4 * dv + 2 * (2 * dk + dv) + 8 + 4 * dv


def test_algorithmic_bytes_of_the_benchmark_workloads():
    # Gated DeltaNet INT8, B=64, H=16, d=128, bf16 inputs: 35,080 bytes per head update
    assert _gdn_head(128, 128, 8) == 35080
    w = W.BY_NAME["gdn_b64_h16_d128_int8_sr"]
    assert bench.step_bytes(w, np.full(w.H, 8)) == 35080 * 64 * 16 == 35_921_920
    # packed INT4, B=1024
    assert _gdn_head(128, 128, 4) == 18696
    w = W.BY_NAME["gdn_b1024_h16_d128_int4_sr_long"]
    assert bench.step_bytes(w, np.full(w.H, 4)) == 18696 * 1024 * 16 == 306_315_264
    # mixed: 8 INT8 + 24 INT4 heads per request, B=256
    w = W.BY_NAME["gdn_b256_h32_d128_mixed_sr"]
    bits = np.array([8] * 8 + [4] * 24)
    assert bench.step_bytes(w, bits) == (8 * 35080 + 24 * 18696) * 256 == 186_712_064
    # Mamba-2 INT8, B=128, H=80, P=64, N=128: per head codes N*P read and written,
    # P scales, x (bf16) and dt, the output; per request B and C (bf16, one group);
    # per head A and D
    w = W.BY_NAME["mamba2_b128_h80_p64_n128_int8_sr"]
    per_head = 2 * 128 * 64 + 2 * 4 * 64 + 2 * 64 + 4 + 4 * 64
    assert per_head == 17284
    total = per_head * 128 * 80 + 128 * 2 * 128 * 2 + 8 * 80
    assert bench.step_bytes(w, np.full(w.H, 8)) == total == 177_054_336


def test_profiled_traffic_follows_the_kernel_sources(tmp_path, monkeypatch):
    """DRAM bytes from a committed capture are reported only for the workload and
    kernel they were measured on, and only while the kernel sources are the ones
    captured."""
    csrc = tmp_path / "ssm_decode_02_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("// kernel v1\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.source_hash()
    tag = "rsq_decode_kernel<gdn,dk=128,blocks=4,sr>"
    entry = {"kernel": tag, "source_hash": h, "dram_bytes_per_launch": 123.0}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"wl": entry}))
    assert bench.profiled_traffic("wl", tag) == 123.0
    assert bench.profiled_traffic("other", tag) is None
    assert bench.profiled_traffic("wl", "rsq_decode_kernel<mamba2,dk=128,blocks=4,sr>") is None
    (csrc / "k.cu").write_text("// kernel v2\n")       # the sources changed since the capture
    assert bench.source_hash() != h
    assert bench.profiled_traffic("wl", tag) is None


class _FakeProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


class _FakeThread:
    def join(self, timeout=None):
        pass


def _summary(lines):
    s = bench.ClockSampler("0")
    s.proc, s.thread, s.lines = _FakeProc(), _FakeThread(), lines
    return s.stop()


def test_clock_summary_reports_median_max_and_throttle_reasons():
    ok = "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active"
    capped = "0, 1800, 1965, 999.9, 0x0000000000000004, Not Active, Not Active, Not Active, Active"
    hot = "0, 1500, 1965, 900.0, 0x0000000000000008, Active, Not Active, Not Active, Not Active"
    r = _summary([ok, ok, capped])
    assert r["sm_mhz"] == 1965 and r["sm_max_mhz"] == 1965 and r["samples"] == 3
    assert r["reasons"] == ["sw_power_cap"]
    r = _summary([ok, hot, "garbage", "0, [N/A], 1965, 1, 0, a, b, c, d"])
    assert r["samples"] == 2 and r["reasons"] == ["hw_slowdown"]
    assert r["sm_mhz"] == pytest.approx((1965 + 1500) / 2)
    r = _summary([])
    assert r["sm_mhz"] is None and r["samples"] == 0 and r["reasons"] == []
