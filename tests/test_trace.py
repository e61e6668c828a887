"""The trace summary and Chrome-trace export on a synthetic trace over a real plan (the
device side of tracing runs in the GPU tests; this checks the host arithmetic).  CPU only."""
import json
import os

import numpy as np
import pytest

from persistent_tile_pipelined_b200 import trace as T
from persistent_tile_pipelined_b200 import tre
from persistent_tile_pipelined_b200.synth import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def synthetic(nsm=7):
    cfg = tre.config_from_workload(W.TINY)
    tasks, begin = tre.tre_plan_tasks(cfg, num_sms=nsm)
    n = len(tasks)
    tr = np.zeros((n, tre.TRACE_COLS), dtype=np.int64)
    for q in range(nsm):
        for k in range(begin[q], begin[q + 1]):
            i = int(tasks[k, 7])                      # rows by task id
            start = 1000 + 100 * i
            tr[i] = (start, start + 10, start + 60, q, start + 15, start + 55, 0, 0)
    return tr, tasks


def test_summary_of_a_synthetic_trace():
    tr, tasks = synthetic()
    s = T.summarize(tr, tasks)
    n = len(tasks)
    assert s["step_us"] == pytest.approx((100 * (n - 1) + 60) / 1e3)
    tt = T.task_table(tasks)
    names = [T.op_name(tt, i) for i in range(n)]
    for op, d in s["per_op"].items():
        assert d["tasks"] == names.count(op)
        assert d["mean_wait_us"] == pytest.approx(0.010)
        assert d["mean_busy_us"] == pytest.approx(0.050)
    for op, d in s["phases_us"].items():
        assert (d["prep"], d["stages"], d["tail"]) == pytest.approx((0.005, 0.040, 0.005))
    # task i starts at 100 i ns: an op's span in a layer is from its first task's ready
    # (+10) to its last task's end (+60); its finish spread is last minus median end
    layers = tt["layer"]
    for op in s["op_span_us"]:
        ids = [[i for i in range(n) if names[i] == op and layers[i] == l]
               for l in sorted(set(layers.tolist()))]
        ids = [v for v in ids if v]
        span = np.mean([100 * (max(v) - min(v)) + 50 for v in ids]) / 1e3
        spread = [100 * (max(v) - np.median(v)) / 1e3 for v in ids]
        assert s["op_span_us"][op] == pytest.approx(span)
        assert s["finish_spread_us"][op]["max"] == pytest.approx(max(spread))
        assert s["finish_spread_us"][op]["mean"] == pytest.approx(np.mean(spread))


def test_sparse_plan_op_names():
    """Index scoring and selection tasks and the W_o K-slices are named in the summary."""
    cfg = tre.config_from_workload(W.MLA4_SPARSE128K.replace(n_layers=1))
    tasks, begin = tre.tre_plan_tasks(cfg, num_sms=148)
    tt = T.task_table(tasks)
    names = {T.op_name(tt, i) for i in range(len(tasks))}
    assert {"index_score", "index_select", "mla_attention", "uk", "uv", "mla_o"} <= names
    assert "?" not in names


def test_chrome_trace_export():
    tr, tasks = synthetic()
    out = os.path.join(ROOT, "tests", "_build")
    os.makedirs(out, exist_ok=True)
    path = os.path.join(out, "trace.json")
    T.chrome_trace(tr, tasks, path)
    ev = json.load(open(path))["traceEvents"]
    assert len(ev) == 2 * len(tasks)                  # a wait and a busy span per task
    busy = [e for e in ev if e["cat"] != "wait"]
    assert all(e["dur"] == pytest.approx(0.050) for e in busy)
    assert {e["tid"] for e in ev} == set(range(7))
