"""Host logic of bench.py without a GPU: clock-record parsing, the roofline arithmetic of a
forward line (device timing replaced by a fixed duration) and the traffic-record hash."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from exact_attention_128_b200 import workloads as W  # noqa: E402


def test_clock_lines_median_max_and_reasons():
    lines = [
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active\n",
        "0, 1950, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active\n",
        "0, 1900, 1965, 999.5, 0x4, Not Active, Not Active, Not Active, Active\n",
        "garbage line\n",
        "0, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active\n",
    ]
    c = bench.parse_clock_lines(lines)
    assert c == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    hot = bench.parse_clock_lines(["0, 1500, 1965, 800, 0x8, Active, Not Active, Active, Not Active"])
    assert hot["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert bench.parse_clock_lines([]) is None


@pytest.fixture
def fake_timing(monkeypatch):
    """Every forward step takes 31.5 us; no device is touched."""
    def fns(case, dev, rot=None):
        return [lambda: None], [], case.make(), 1
    monkeypatch.setattr(bench, "dense_fwd_step_fns", fns)
    monkeypatch.setattr(bench, "timed_loop", lambda f, steps, warmup, world: 0.0315 * steps)
    return {"hbm_gbs": 6545.3, "bf16_tflops": 1645.7, "bf16_tflops_sustained": 1385.8, "sm_max_mhz": 1965.0}


def test_headline_roofline_arithmetic(fake_timing):
    c = W.VIT_BATCHED_BF16
    r = bench.measure_dense_fwd(c, None, 100, 3, 1, fake_timing)
    roof = r["roofline"]
    flops = 4 * 64 * 64 * 12 * 196 * 196
    nbytes = 4 * 64 * 12 * 196 * 64 * 2 + 64 * 12 * 196 * 4  # q, k, v, o bf16 + lse fp32
    assert roof["algorithmic_flops_per_launch"] == flops and roof["algorithmic_bytes_per_launch"] == nbytes
    assert roof["bound"] == "hbm"  # 98 FLOP/B is under the ridge of either peak
    assert roof["achieved"] == pytest.approx(nbytes / 31.5e-6 / 1e9, rel=1e-3)
    assert roof["frac"] == pytest.approx(roof["achieved"] / 6545.3, abs=1e-4)
    assert r["tflops"] == pytest.approx(flops / 31.5e-6 / 1e12)
    # one SFU exponential per (query, key) pair and head at 16 per clock per SM
    exp_s = 64 * 12 * 196 * 196 / (16 * 148 * 1965e6)
    assert roof["exp_bound"]["tflops"] == pytest.approx(flops / exp_s / 1e12, rel=1e-3)
    json.dumps(r)  # the line stays serialisable


def test_fp32_line_is_alu_bound(fake_timing):
    r = bench.measure_dense_fwd(W.VIT_LAYER_F32, None, 10, 3, 1, fake_timing)
    # the ViT layer's 196 keys fit the one-pass fp32 kernel
    assert r["roofline"]["bound"] == "alu" and r["roofline"]["kernel"] == "fa_fwd_f32_small_kernel"
    assert r["roofline"]["peak"] == pytest.approx(148 * 128 * 2 * 1965e6 / 1e12, abs=0.1)


def test_traffic_hash_ignores_comments_only(tmp_path, monkeypatch):
    csrc = tmp_path / "exact_attention_128_b200" / "csrc"
    csrc.mkdir(parents=True)
    f = csrc / "k.cuh"
    f.write_text("// header\nint a = 1;  // why\n/* block */ int b;\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_sources_sha(["k.cuh"])
    f.write_text("// a longer header\n\nint a = 1;\n int b;  /* note */\n")
    assert bench.kernel_sources_sha(["k.cuh"]) == h0
    f.write_text("int a = 2;\nint b;\n")
    assert bench.kernel_sources_sha(["k.cuh"]) != h0


def test_oracle_row_units_count_the_workload_flops():
    """One pass over every row unit of a small causal GQA workload (ragged last unit) counts
    exactly the workload's algorithmic FLOPs, and the units cover every query row once."""
    c = W.DenseCase("units", 2, 4, 2, 300, 300, 64, "bf16", True, 5)
    orc = bench.OracleRows(c, rows=128)
    assert orc.per_head == 3 and orc.units == 2 * 4 * 3
    for _ in range(orc.units):
        orc.step()
    assert orc.rows_done == 2 * 4 * 300
    assert orc.flops == pytest.approx(c.fwd_flops(), rel=1e-12)


def test_compact_secondary_record():
    r = {"tflops": 1157.123, "per_step_ms": 3.80123,
         "roofline": {"frac": 0.7031, "traffic": 640e6, "algorithmic_bytes_per_launch": 540e6}}
    assert bench.compact(r, "tflops") == [1157.12, "TFLOP/s", 3.8012, 0.7031, 1.19]
    r2 = {"gbs": 5334.04, "per_step_ms": 0.05411, "roofline": {"frac": 0.8138}}
    assert bench.compact(r2, "gbs", 1) == [5334.0, "GB/s", 0.0541, 0.8138, None]
