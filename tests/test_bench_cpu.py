"""Host-side logic of the benchmark (no GPU): the roofline bound choice, the guard on recorded
ncu traffic, and the reference arm's JSON line (the fp64 oracle on the host)."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from mxfp4_quantized_moe_b200 import inputs  # noqa: E402


def test_algorithmic_work_and_bound():
    ridge = 1403.3e12 / 6550.4e9
    big = bench.gemm_work(inputs.WORKLOADS["gpt-oss-20b-moe-T8192"])
    small = bench.gemm_work(inputs.WORKLOADS["gpt-oss-20b-moe-T256"])
    T, H, I, E, k = 8192, 2880, 2880, 32, 4
    A = T * k
    # FLOP: 2 * rows * N * K for each GEMM; the step is 12 A H I
    assert sum(f for f, _ in big.values()) == pytest.approx(12.0 * A * H * I)
    # packed gate_up weights alone are 0.5 + 1/32 bytes per element
    assert big["gemm_dx"][1] >= E * 2 * I * H * (0.5 + 1 / 32)
    assert all(f / b > ridge for f, b in big.values())      # tensor-bound at T=8192
    assert all(f / b < ridge for f, b in small.values())    # weight streaming at T=256


def test_recorded_traffic_only_for_the_captured_sources(monkeypatch):
    key = ("gemm_gate_up_glu", "gpt-oss-20b-moe-T8192")
    monkeypatch.setitem(bench.NCU_TRAFFIC, key, {"bytes": 1.0e9, "sources": "0" * 16})
    assert bench.recorded_traffic(*key) is None  # sources differ from the capture
    monkeypatch.setitem(bench.NCU_TRAFFIC, key,
                        {"bytes": 1.0e9, "sources": bench.kernel_sources_digest()})
    assert bench.recorded_traffic(*key) == 1.0e9
    assert bench.recorded_traffic("gemm_gate_up_glu", "another-workload") is None


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny-moe-T64-H256-E8-k2", "--steps", "2", "--warmup", "1"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"] == "tiny-moe-T64-H256-E8-k2"


def test_peak_choice_follows_region_length_and_clocks():
    pk = {"bf16_tflops": 1644.9, "bf16_tflops_sustained": 1403.3, "hbm_gbs": 6550.0,
          "source": "measured"}
    boost = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}
    capped = {"sm_mhz": 1680.0, "sm_max_mhz": 1965.0}
    assert bench.choose_peak(pk, 0.08, boost)[:2] == (1644.9, "burst")
    assert bench.choose_peak(pk, 0.08, capped)[:2] == (1403.3, "sustained")
    assert bench.choose_peak(pk, 0.85, boost)[:2] == (1644.9, "burst")
    assert bench.choose_peak(pk, 3.0, boost)[:2] == (1403.3, "sustained")
    assert bench.choose_peak(pk, 0.08, None)[:2] == (1403.3, "sustained")


def test_clock_sampler_keeps_only_samples_inside_the_region():
    s = bench.ClockSampler(0)
    s.thread = type("T", (), {"join": lambda self, timeout=None: None})()
    s.source = "nvml"
    s.rows = [(1.0, 1000.0, 1965.0, set()), (2.0, 1900.0, 1965.0, {"sw_power_cap"}),
              (3.0, 1950.0, 1965.0, set()), (9.0, 500.0, 1965.0, set())]
    s.mark(1.5, 3.5)
    c = s.stop()
    assert c["samples_in_timed_region"] == 2 and c["sm_mhz"] == 1925.0
    assert c["reasons"] == ["sw_power_cap"] and c["sm_max_mhz"] == 1965.0
