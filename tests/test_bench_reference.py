"""The benchmark's reference arm (the CPU oracle on the host cores): one JSON line with the
engine arm's metric, unit and config, the requested step counts, and its own description
of the sample.  Runs on CPU only."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def reference_line(*extra):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          *extra], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


def test_reference_decode_line_matches_the_engine_arm():
    sys.path.insert(0, ROOT)
    import bench
    from persistent_tile_pipelined_b200.synth import workloads as W
    d = reference_line("--workload", "tiny-2L-d256", "--steps", "5", "--warmup", "3",
                       "--tokens-per-step", "2")
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["steps"] == 5 and d["warmup"] == 3 and d["value"] > 0
    # the engine arm builds its config with the same function and the same workload
    wl = W.WORKLOADS["tiny-2L-d256"].replace(decode_steps=8, tokens_per_step=2)
    assert d["config"] == bench.decode_config(wl, 2, {}, 1)
    # two tokens per step: a step is two tokens of oracle time
    assert d["ms_per_step"] == pytest.approx(2e3 / d["value"], rel=1e-9)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert "5 timed after 3 warm-up" in cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_layers_line():
    sys.path.insert(0, ROOT)
    import bench
    from persistent_tile_pipelined_b200.synth import workloads as W
    d = reference_line("--workload", "moe-4L-d7168", "--steps", "3", "--warmup", "3")
    assert d["metric"] == bench.LAYERS_METRIC and d["unit"] == "steps/s"
    assert d["steps"] == 3 and d["warmup"] == 3
    wl = W.WORKLOADS["moe-4L-d7168"].replace(decode_steps=6)
    assert d["config"] == bench.layers_config(wl, 1)
    assert "moe layers" in d["cpu_baseline"]["sample"]


def test_plan_step_bytes_in_config():
    """The config's statement of streamed bytes comes from the host planner: weights plus
    the KV rows read at the workload's position."""
    sys.path.insert(0, ROOT)
    import bench
    from persistent_tile_pipelined_b200 import tre
    from persistent_tile_pipelined_b200.synth import workloads as W
    wl = W.LLAMA8B.replace(decode_steps=16)
    info = tre.tre_plan_inspect(tre.config_from_workload(wl))
    kv = 2 * wl.n_layers * wl.n_kv_heads * wl.head_dim * 2 * wl.prefill
    assert bench.plan_step_gb(wl) == pytest.approx((info.weight_bytes + kv) / 1e9, rel=1e-3)
    assert bench.plan_step_gb(wl) == pytest.approx(15.55, abs=0.01)
