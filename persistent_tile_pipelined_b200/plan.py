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

TILE_STAGE_BYTES = 16 * (1024 * 2 + 16)  # one 16-row tile of 1024 padded columns


def gemv_tiles(cfg) -> bool:
    """The GEMV form rule of tre_config.multi_token_gemv: tensor-core tiles when asked for
    (2), or by the planner's choice (0) at 4 tokens per step when hidden and ffn are
    multiples of 16; CUDA-core rows otherwise (and always at one token)."""
    M = max(1, cfg.max_tokens_per_step)
    if M == 1 or cfg.multi_token_gemv == 1:
        return False
    return cfg.multi_token_gemv == 2 or (M >= 4 and cfg.hidden % 16 == 0 and cfg.ffn % 16 == 0)


def report(wl, num_sms: int = 148, **overrides) -> dict:
    cfg = tre.config_from_workload(wl, **overrides)
    info = tre.tre_plan_inspect(cfg, num_sms=num_sms)
    tasks, begin = tre.tre_plan_tasks(cfg, num_sms=num_sms)
    w0 = tasks[:, 0].astype("int64") & 0xFFFFFFFF
    kinds = Counter()
    for typ, op in zip((w0 & 0xFF).tolist(), ((w0 >> 8) & 0xFF).tolist()):
        kinds["attention" if typ == 1 else "mla_attention" if typ == 2
              else OP_NAMES.get(op, str(op))] += 1
    M = max(1, cfg.max_tokens_per_step)
    tiles = gemv_tiles(cfg)
    kv_at_prefill = info.kv_bytes_at_capacity * wl.prefill / max(1, cfg.kv_capacity - M)
    return {
        "workload": wl.name, "kind": wl.kind, "tokens_per_step": M,
        "gemv_form": "tensor-core tiles (16 x 1024)" if tiles else "CUDA-core rows",
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
