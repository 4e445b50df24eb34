"""Host-side logic of bench.py that needs no GPU: the workload and config objects
both arms print, the L2 rule, and the reference arm's JSON line on a tiny sample."""
import json
import subprocess
import sys
import types

import pytest

import bench
from diffusion_transformer_video_b200 import workloads as wl


def _args(**kw):
    base = dict(workload="480p", seed=0, heads=0)
    base.update(kw)
    return types.SimpleNamespace(**base)


def test_config_is_the_workload_and_the_l2_rule():
    w = bench.resolve_workload(_args())
    cfg = bench.workload_config(w, 1)
    assert cfg["workload"] == "480p" and cfg["rows"] == 32760 and cfg["heads"] == 40
    assert cfg["d_model"] == 5120 and cfg["rope_bands"] == [44, 42, 42]
    assert cfg["l2"].startswith("inputs larger than L2")      # 335 MB per tensor
    img = bench.resolve_workload(_args(workload="image"))
    assert not bench.l2_resident_free(img)                     # 50 MB per tensor
    assert bench.workload_config(img, 8)["l2"].startswith("L2 flushed")
    assert bench.workload_config(img, 8)["parallelism"].startswith("dp8")


def test_heads_override_renames_the_workload():
    w = bench.resolve_workload(_args(heads=16))
    assert w.heads == 16 and w.name == "480p-h16"
    assert w.attn_flops() == pytest.approx(wl.get_workload("480p").attn_flops() * 16 / 40)


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                          "--steps", "1", "--warmup", "1", "--ref-rows", "4"],
                         capture_output=True, text=True, timeout=300, check=True).stdout
    line = json.loads(out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s"
    assert line["config"] == bench.workload_config(bench.resolve_workload(_args(workload="tiny")), 1)
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_clock_summary_reports_reasons_power_and_the_active_mask(tmp_path):
    # rows as nvidia-smi prints them: index, clocks.sm, clocks.max.sm, power.draw,
    # reasons bitmask, then the four yes/no reason fields
    p = tmp_path / "clk.csv"
    p.write_text("0, 1965, 1965, 612.40, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"
                 "0, 1590, 1965, 998.10, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
                 "0, 1605, 1965, 996.00, 0x0000000000000004, Not Active, Not Active, Not Active, Not Active\n"
                 "0, [N/A], 1965, [N/A], [N/A], Not Active, Not Active, Not Active, Not Active\n")
    c = bench.ClockSampler(0)
    c.path = str(p)
    s = c.summary()
    assert s["sm_mhz"] == 1605 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"] and s["active_mask"] == "0x4"
    assert s["power_w"] == 996.0 and s["samples"] == 4


def test_oracle_memory_steps_baseline_on_the_tiny_workload():
    w = wl.get_workload("tiny")
    x = wl.make_inputs(w, seed=0, which=("x",))["x"]
    r = bench.cpu_oracle_memory_steps(w, x, 0)
    for name in ("adaln_modulate", "gated_residual"):
        assert r[name]["GB/s"] > 0 and r[name]["rows"] == w.rows // 2
    assert "threads" in r["sample"]
