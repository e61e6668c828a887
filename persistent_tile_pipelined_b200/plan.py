"""Print what the host planner makes of a workload — no GPU needed.

    python -m persistent_tile_pipelined_b200.plan [--workload NAME] [--tokens-per-step M]
                                                  [--num-sms N] [--config FIELD=VALUE ...]

Reports the launch shape (ring stages x stage bytes, shared memory per CTA), the GEMV
form (whole-row stages on CUDA cores, or 16-row tensor-core tiles), the KV splits, the
task count and per-op task counts, the bytes a step streams, and how evenly the streamed
bytes fall on the SMs.
"""
from __future__ import annotations

import argparse
import json
from collections import Counter

from . import tre
from .synth import workloads as W
from .trace import OP_NAMES

def report(wl, num_sms: int = 148, **overrides) -> dict:
    cfg = tre.config_from_workload(wl, **overrides)
    info = tre.tre_plan_inspect(cfg, num_sms=num_sms)
    tasks, begin = tre.tre_plan_tasks(cfg, num_sms=num_sms)
    w0 = tasks[:, 0].astype("int64") & 0xFFFFFFFF
    kinds = Counter()
    for typ, op in zip((w0 & 0xFF).tolist(), ((w0 >> 8) & 0xFF).tolist()):
        kinds[{1: "attention", 2: "mla_attention", 3: "index_score",
               4: "index_select"}.get(typ) or OP_NAMES.get(op, str(op))] += 1
    M = max(1, cfg.max_tokens_per_step)
    tiles = bool(info.gemv_tiles)  # the planner's choice of GEMV form
    kv_at_prefill = info.kv_bytes_at_capacity * wl.prefill / max(1, cfg.kv_capacity - M)
    return {
        "workload": wl.name, "kind": wl.kind, "tokens_per_step": M,
        "gemv_form": "tensor-core tiles (16 x 1024)" if tiles else "CUDA-core rows",
        "weights": {1: "E4M3 projections, 128 x 128 fp32 block scales",
                    2: "MXFP4 routed experts (E2M1 + E8M0 per 32)"}.get(cfg.weight_format, "bf16"),
        "num_sms": info.num_sms, "ring": f"{info.ring_stages} x {info.stage_bytes} B",
        "smem_bytes_per_cta": info.smem_bytes, "kv_splits": info.kv_splits,
        "tasks": info.num_tasks, "tasks_by_kind_per_step": dict(sorted(kinds.items())),
        "max_tasks_per_sm": info.max_tasks_per_sm, "counters": info.num_counters,
        "weight_gb_per_step": info.weight_bytes / 1e9,
        "kv_gb_per_step_at_prefill": kv_at_prefill / 1e9,
        "sm_bytes_max_over_min": info.max_sm_bytes / max(1, info.min_sm_bytes),
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", default="llama3-8b-shaped", choices=sorted(W.WORKLOADS))
    ap.add_argument("--tokens-per-step", type=int, default=1)
    ap.add_argument("--num-sms", type=int, default=148)
    ap.add_argument("--config", action="append", default=[],
                    help="tre_config FIELD=VALUE (repeatable), e.g. kv_splits=8")
    args = ap.parse_args(argv)
    over = {}
    for item in args.config:
        k, v = item.split("=", 1)
        over[k] = int(v)
    wl = W.WORKLOADS[args.workload].replace(tokens_per_step=args.tokens_per_step)
    print(json.dumps(report(wl, args.num_sms, **over), indent=1))


if __name__ == "__main__":
    main()
