"""The plan report (python -m persistent_tile_pipelined_b200.plan): CPU only."""
import json
import subprocess
import sys

import pytest

from persistent_tile_pipelined_b200 import tre
from persistent_tile_pipelined_b200.synth import workloads as W


@pytest.mark.parametrize("wl,over,tiles", [
    (W.LLAMA8B, {}, False),
    (W.LLAMA8B.replace(tokens_per_step=2), {}, False),
    (W.LLAMA8B.replace(tokens_per_step=3), {}, False),
    (W.LLAMA8B.replace(tokens_per_step=4), {}, True),
    (W.LLAMA8B.replace(tokens_per_step=4), {"multi_token_gemv": 1}, False),
    (W.TINY.replace(tokens_per_step=2), {"multi_token_gemv": 2}, True),
    (W.TINY.replace(tokens_per_step=4, hidden=264, ffn=696), {}, False),
])
def test_gemv_form_rule_matches_the_plan(wl, over, tiles):
    """The documented form rule (tre.h, multi_token_gemv) is what the planner reports, and
    tile plans carry one 16-row tile of 1024 padded columns per stage, row plans (32 KB
    stages here) do not."""
    cfg = tre.config_from_workload(wl, **over)
    info = tre.tre_plan_inspect(cfg)
    assert bool(info.gemv_tiles) == tiles
    assert (info.stage_bytes >= 16 * (1024 * 2 + 16)) == tiles


def test_plan_reports_sparse_splits():
    info = tre.tre_plan_inspect(tre.config_from_workload(W.MLA4_SPARSE128K))
    assert info.index_splits == info.num_sms == 148
    assert tre.tre_plan_inspect(tre.config_from_workload(W.MLA4)).index_splits == 0


def test_plan_report_cli():
    out = subprocess.run([sys.executable, "-m", "persistent_tile_pipelined_b200.plan",
                          "--tokens-per-step", "4", "--num-sms", "132", "--config", "kv_splits=8"],
                         capture_output=True, text=True, check=True, timeout=120)
    r = json.loads(out.stdout)
    assert r["gemv_form"].startswith("tensor-core") and r["num_sms"] == 132
    assert r["kv_splits"] == 8 and r["tasks_by_kind_per_step"]["attention"] == 32 * 8 * 8
    assert r["weight_gb_per_step"] == pytest.approx(15.01, abs=0.01)
    assert 1.0 <= r["sm_bytes_max_over_min"] < 1.1


def test_plan_report_names_the_weight_format():
    out = subprocess.run([sys.executable, "-m", "persistent_tile_pipelined_b200.plan",
                          "--workload", "moe-4L-d7168-fp4"],
                         capture_output=True, text=True, check=True, timeout=120)
    r = json.loads(out.stdout)
    assert r["weights"].startswith("MXFP4") and r["weight_gb_per_step"] == pytest.approx(2.173, abs=1e-3)
