"""Per-task trace of one engine step: statistics and a Chrome-trace (chrome://tracing) file.

An engine created with TRE_DEBUG_TRACE records, for every task, the global-timer
nanoseconds when its consumer warps started waiting for its dependency, when the
dependency was met, when the task finished, and the SM it ran on.  Combined with the plan
(``tre_plan_tasks``), this gives per-op time, dependency-wait (idle) time and the spread
of finish times across SMs — the straggler effect at every op boundary.
"""
from __future__ import annotations

import json
from collections import defaultdict

import numpy as np

OP_NAMES = {0: "qkv", 1: "o_proj", 2: "gate_up", 3: "down", 4: "lm_head", 5: "router",
            6: "shared_gate_up", 7: "routed_gate_up", 8: "moe_down", 9: "mla_down",
            10: "q_up", 11: "uk", 12: "uv", 13: "mla_o", 14: "mla_o"}


def task_table(tasks: np.ndarray) -> dict:
    """Decode the 8-int32 task descriptors of ``tre_plan_tasks`` into columns by task id."""
    w0 = tasks[:, 0].astype(np.int64) & 0xFFFFFFFF
    order = np.argsort(tasks[:, 7])
    cols = {"type": w0 & 0xFF, "op": (w0 >> 8) & 0xFF, "layer": (w0 >> 16) & 0xFFFF,
            "r0": tasks[:, 4], "r1": tasks[:, 5]}
    return {k: v[order] for k, v in cols.items()}


def op_name(tt: dict, i: int) -> str:
    if tt["type"][i] == 1:
        return "attention"
    if tt["type"][i] == 2:
        return "mla_attention"
    if tt["type"][i] == 3:
        return "index_score"
    if tt["type"][i] == 4:
        return "index_select"
    return OP_NAMES.get(int(tt["op"][i]), "?")


def summarize(trace: np.ndarray, tasks: np.ndarray) -> dict:
    """trace: [n_tasks][8] int64 (start, ready, end, sm, phase marks) by task id."""
    tt = task_table(tasks)
    t0 = trace[:, 0].min()
    start, ready, end = trace[:, 0] - t0, trace[:, 1] - t0, trace[:, 2] - t0
    step_ns = float(end.max())
    per_op = defaultdict(lambda: {"tasks": 0, "wait_ns": 0.0, "busy_ns": 0.0})
    spans = defaultdict(list)
    for i in range(len(trace)):
        name = op_name(tt, i)
        d = per_op[name]
        d["tasks"] += 1
        d["wait_ns"] += float(ready[i] - start[i])
        d["busy_ns"] += float(end[i] - ready[i])
        spans[(int(tt["layer"][i]), name)].append((start[i], ready[i], end[i]))
    # straggler spread: for each (layer, op), last finish minus median finish; op span:
    # first dependency met to last finish (the op's share of the step's critical path)
    spread = defaultdict(list)
    span = defaultdict(list)
    for (layer, name), v in spans.items():
        ends = np.array([e for _, _, e in v], dtype=np.float64)
        spread[name].append(float(ends.max() - np.median(ends)))
        span[name].append(float(ends.max() - min(r for _, r, _ in v)))
    nsm = int(trace[:, 3].max()) + 1
    busy = np.zeros(nsm)
    waitt = np.zeros(nsm)
    for i in range(len(trace)):
        busy[int(trace[i, 3])] += end[i] - ready[i]
        waitt[int(trace[i, 3])] += ready[i] - start[i]
    phases = defaultdict(lambda: [0.0, 0.0, 0.0, 0])
    if trace.shape[1] >= 7:
        for i in range(len(trace)):
            r, e, a, b, c = (int(trace[i, k]) for k in (1, 2, 4, 5, 6))
            d = phases[op_name(tt, i)]
            if a and b:
                d[0] += a - r          # input staged / q ready
                d[1] += b - a          # stages consumed
                d[2] += e - (c if c else b)   # tail: epilogue, ticket, combine, publish
                d[3] += 1
    # op boundaries, in global task order (the op groups of the kernel-per-op form): the
    # hand-off from the last task of one op to the first task of the next one to start
    # computing (dependency met) — a launch boundary in the kernel-per-op form, a counter
    # publish and wake-up in the persistent form
    ids = np.arange(len(trace))
    key = np.stack([tt["layer"], tt["type"], tt["op"]], axis=1)
    new_group = np.ones(len(ids), dtype=bool)
    new_group[1:] = (key[1:] != key[:-1]).any(axis=1)
    gid = np.cumsum(new_group) - 1
    G = int(gid.max()) + 1
    g_end = np.full(G, -np.inf)
    g_ready = np.full(G, np.inf)
    np.maximum.at(g_end, gid, end.astype(np.float64))
    np.minimum.at(g_ready, gid, ready.astype(np.float64))
    gaps = g_ready[1:] - g_end[:-1]
    return {
        "op_groups": G,
        "op_gap_us": {"mean": float(np.mean(gaps)) / 1e3, "median": float(np.median(gaps)) / 1e3,
                      "sum": float(np.sum(np.maximum(gaps, 0))) / 1e3},
        "phases_us": {k: {"prep": v[0] / v[3] / 1e3, "stages": v[1] / v[3] / 1e3,
                          "tail": v[2] / v[3] / 1e3} for k, v in phases.items() if v[3]},
        "step_us": step_ns / 1e3,
        "per_op": {k: {"tasks": v["tasks"], "mean_wait_us": v["wait_ns"] / v["tasks"] / 1e3,
                       "mean_busy_us": v["busy_ns"] / v["tasks"] / 1e3}
                   for k, v in per_op.items()},
        "finish_spread_us": {k: {"mean": float(np.mean(v)) / 1e3, "max": float(np.max(v)) / 1e3}
                             for k, v in spread.items()},
        "op_span_us": {k: float(np.mean(v)) / 1e3 for k, v in span.items()},
        "sm_wait_frac_mean": float(np.mean(waitt) / step_ns),
        "sm_busy_frac_mean": float(np.mean(busy) / step_ns),
    }


def chrome_trace(trace: np.ndarray, tasks: np.ndarray, path: str) -> None:
    tt = task_table(tasks)
    t0 = trace[:, 0].min()
    ev = []
    for i in range(len(trace)):
        s, r, e, sm = (int(x) for x in trace[i, :4])
        name = f"L{int(tt['layer'][i])}.{op_name(tt, i)}"
        if r > s:
            ev.append({"name": "wait", "ph": "X", "ts": (s - t0) / 1e3, "dur": (r - s) / 1e3,
                       "pid": 0, "tid": sm, "cat": "wait"})
        ev.append({"name": name, "ph": "X", "ts": (r - t0) / 1e3, "dur": (e - r) / 1e3,
                   "pid": 0, "tid": sm, "cat": op_name(tt, i)})
    with open(path, "w") as f:
        json.dump({"traceEvents": ev, "displayTimeUnit": "ns"}, f)
