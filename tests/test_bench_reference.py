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


def test_clock_samples_inside_the_timed_windows():
    """The `clocks` entry: median SM clock and throttle reasons of the samples taken inside
    the timed windows; malformed and out-of-window samples are ignored."""
    import datetime
    sys.path.insert(0, ROOT)
    import bench

    def row(sec, clk, reasons=("Not Active",) * 4):
        ts = datetime.datetime(2026, 1, 1, 12, 0, 0) + datetime.timedelta(seconds=sec)
        return ", ".join([ts.strftime("%Y/%m/%d %H:%M:%S.%f")[:-3], "0", str(clk), "1965",
                          "700.5", *reasons])
    t0 = datetime.datetime(2026, 1, 1, 12, 0, 0).timestamp()
    text = "\n".join([
        row(0.0, 1200),                                      # before the window: ignored
        row(1.0, 1965), row(1.2, 1950),
        row(1.4, 1965, ("Not Active", "Not Active", "Not Active", "Active")),
        "garbage line", row(1.5, "[N/A]"),                   # malformed: ignored
        row(3.0, 900, ("Active", "Not Active", "Not Active", "Not Active")),  # after: ignored
    ])
    c = bench.parse_clocks(text, [(t0 + 0.9, t0 + 1.6)])
    assert c == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                 "samples": 3}
    every = bench.parse_clocks(text, [])
    assert every["samples"] == 5 and every["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert bench.parse_clocks("", [(t0, t0 + 1)])["samples"] == 0


def test_workload_step_bytes_match_the_planner():
    """The bytes `config` states come from the workload shape alone (the reference arm
    loads no engine library); they equal the planner's weight bytes plus the KV rows read
    at the workload's length, the new rows written, the embedding row and the logits."""
    sys.path.insert(0, ROOT)
    import bench
    from persistent_tile_pipelined_b200 import tre
    from persistent_tile_pipelined_b200.synth import workloads as W
    for wl in W.WORKLOADS.values():
        info = tre.tre_plan_inspect(tre.config_from_workload(wl))
        row = (wl.kv_lora + wl.rope_dim) * 2 if wl.kind == "mla" else wl.n_kv_heads * wl.head_dim * 4
        read = info.kv_bytes_at_capacity * wl.prefill // (wl.kv_capacity - 1)
        lm = wl.vocab * 4 + 2 * wl.hidden if wl.vocab else 0
        if wl.index_topk and wl.prefill + 1 > wl.index_topk:
            # sparse MLA: every index key (+ the new one), the K chosen latent rows + the new one
            read = wl.n_layers * (wl.prefill * wl.index_dim * 2 + wl.index_topk * row)
            row += wl.index_dim * 2
        assert bench.workload_step_bytes(wl) == info.weight_bytes + read + wl.n_layers * row + lm


def test_reference_arm_loads_no_engine_library():
    """The CPU baseline describes and times its workload without libtre.so."""
    code = ("import sys, runpy; sys.argv = ['bench.py', '--impl', 'reference', '--workload', "
            "'tiny-2L-d256', '--steps', '3', '--warmup', '3'];\n"
            "try:\n runpy.run_path('bench.py', run_name='__main__')\n"
            "finally:\n print('LOADED', any('libtre.so' in l for l in open('/proc/self/maps')))")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    assert "LOADED False" in out.stdout, out.stdout[-2000:]
