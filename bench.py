"""Benchmark: batch-1 decode tokens/s and achieved HBM GB/s of the persistent engine.

Workload: the Llama-3-8B-shaped stack (32 layers, hidden 4096, 32 q / 8 kv heads of dim
128, SwiGLU 14336, vocab 128256), bf16 random-init weights N(0, 0.02), KV cache of 4096
positions N(0, 1) bf16, batch 1.  One step = one decode step of the whole stack = one
launch of the persistent engine kernel.  Inputs are synthetic (seeded generator) and
resident in HBM; every step streams ~15.5 GB, far more than the 126 MB L2, so no flush
is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl engine|reference]

For N > 1 it runs under torch.distributed.run, one process per GPU; the path does not
shard, so every rank runs an independent replica (no collective on the data path) and
`value` is the sum over ranks of tokens / the slowest rank's time.

Numbers printed (one JSON line on rank 0):
  value        tokens/s over the K timed steps, launches back to back on the device
               (CUDA events on the launching stream, barrier + synchronize on both sides,
               max over ranks)
  e2e          the greedy generation loop through the C ABI call tre_decode_step_host:
               the token goes in as a kernel argument, the argmax token comes back to the
               host every step; host wall time, max over ranks
  roofline     the engine kernel's algorithmic bytes per launch / average launch time,
               against the measured HBM copy bandwidth of this machine
  cpu_baseline the CPU oracle (tests-only code) timed on this machine's cores on a bounded
               sample of the same workload (rank 0, N = 1)
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "batch-1 decode tokens/s and achieved HBM GB/s (fraction of ~8 TB/s roofline)"
LAYERS_METRIC = "layer-stack step time and achieved HBM GB/s over the bytes a token reads"
NOMINAL_HBM_GBS = 8000.0
REFERENCE_SECONDS = 120.0  # oracle work of a whole reference-arm run
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="engine", choices=["engine", "reference"])
    ap.add_argument("--workload", default="llama3-8b-shaped")
    ap.add_argument("--tokens-per-step", type=int, default=1,
                    help="tokens per launch (1..4): multi-token verify steps via tre_decode_tokens")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-layers", type=int, default=4)
    ap.add_argument("--trace", default="", help="write a per-task trace of one step (JSON)")
    ap.add_argument("--config", action="append", default=[], metavar="FIELD=VALUE",
                    help="engine config override (launch shape, K-part limit); repeatable")
    ap.add_argument("--flags", type=int, default=0,
                    help="engine debug flags for the timed engine (8 = no cross-op prefetch)")
    ap.add_argument("--launch-mode", default="persistent", choices=["persistent", "per-op"],
                    help="persistent: one launch per step (the product); per-op: the same "
                         "tiles, one plain launch per op (measurement form)")
    ap.add_argument("--wl", action="append", default=[], metavar="FIELD=VALUE",
                    help="workload shape override (e.g. n_layers=1, n_experts=16: a small "
                         "case of the same kernel for profiler captures); repeatable")
    ap.add_argument("--no-ablation", action="store_true",
                    help="skip the kernel-per-op comparison and the device-loop timing")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "persistent_tile_pipelined_b200", "csrc")
    for fn in sorted(os.listdir(csrc)):
        if fn.endswith((".cu", ".cuh", ".h", ".cpp")):
            with open(os.path.join(csrc, fn), "rb") as f:
                h.update(fn.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


PROFILES = {("llama3-8b-shaped", 1): "engine_kernel_llama8b.md",
            ("llama3-8b-shaped", 4): "engine_kernel_llama8b_4tok.md"}


def profiled_traffic(workload: str, tokens_per_step: int = 1):
    """DRAM bytes per launch from the committed ncu summary of this workload's kernel (one
    per token count), if it was taken on the current kernel source (else None)."""
    name = PROFILES.get((workload, tokens_per_step))
    path = os.path.join(ROOT, "profiles", name) if name else ""
    if not name or not os.path.exists(path):
        return None
    txt = open(path).read()
    m_src = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", txt)
    m_tr = re.search(r"dram_bytes_per_launch_full_workload:\s*([0-9.eE+]+)", txt)
    if not (m_src and m_tr) or m_src.group(1) != kernel_source_hash():
        return None
    return float(m_tr.group(1))


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the timed regions run."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.windows = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.index), "-lms", "50"], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def mark(self, t0, t1):
        self.windows.append((t0, t1))

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        return parse_clocks(out, self.windows)


def parse_clocks(text: str, windows) -> dict:
    """The `clocks` entry from nvidia-smi CSV samples (the ClockSampler fields, no header,
    no units): the median SM clock and the throttle reasons seen during the timed windows
    (wall-clock (start, end) pairs; every sample when there are none)."""
    sm, mx, reasons = [], None, set()
    names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    for line in text.splitlines():
        parts = [x.strip() for x in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            continue
        if windows and not any(a - 0.05 <= ts <= b + 0.05 for a, b in windows):
            continue
        try:
            clk, top = float(parts[2]), float(parts[3])
        except ValueError:
            continue
        sm.append(clk)
        mx = top
        for n, v in zip(names, parts[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    if not sm:
        return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
    return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
            "samples": len(sm)}


# ---------------------------------------------------------------- workload -------------

def max_over_ranks(values, world: int, device: str = "cpu"):
    """Element-wise maximum of per-rank timings over all ranks (the slowest rank sets the
    job's time); identity on one rank.  Collective: every rank calls it once."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(world: int, steps: int, tokens_per_step: int, slowest_s: float) -> float:
    """Whole-job tokens/s: every rank runs its own replica, so the job processes world x
    steps x tokens_per_step tokens in the slowest rank's time."""
    return world * steps * tokens_per_step / slowest_s


def workload_of(args):
    """The named workload with the --wl shape overrides applied (renamed to show them)."""
    from persistent_tile_pipelined_b200.synth import workloads as W
    wl = W.WORKLOADS[args.workload]
    over = config_overrides(args.wl)
    if over:
        wl = wl.replace(name=wl.name + "".join(f",{k}={v}" for k, v in sorted(over.items())),
                        **over)
    return wl


def config_overrides(items):
    """FIELD=VALUE strings -> {field: int}."""
    out = {}
    for it in items or []:
        k, v = it.split("=", 1)
        out[k.strip()] = int(v)
    return out


def build_engine(wl, device: int, debug_flags: int = 0, overrides=None):
    """Generate the synthetic model tensor by tensor (host generator -> device) so the
    host holds at most one tensor at a time."""
    import torch

    from persistent_tile_pipelined_b200 import tre
    from persistent_tile_pipelined_b200.synth import (TID_EMBED, TID_FINAL_NORM, TID_LM_HEAD,
                                                      tid_layer)
    from persistent_tile_pipelined_b200.synth import workloads as W

    dev = f"cuda:{device}"

    def up(words):
        if words.dtype in (np.uint8, np.float32):  # E4M3 bytes, fp32 block scales
            return torch.from_numpy(words).to(dev)
        t = torch.from_numpy(words.view(np.int16)).view(torch.bfloat16)
        return t.to(dev)

    model = {"layers": [], "k_cache": [], "v_cache": []}
    for l in range(wl.n_layers):
        if wl.weight_format == "fp8":  # one layer's E4M3 bytes and scales at a time
            model["layers"].append({slot: up(a) for slot, a in W.gen_gqa_layer(wl, l).items()})
        else:
            model["layers"].append({slot: up(W.gen_tensor(wl, tid_layer(l, slot), shape, kind))
                                    for slot, shape, kind in W.gqa_layer_shapes(wl)})
        model["k_cache"].append(up(W.gen_kv_cache(wl, l, "k")))
        model["v_cache"].append(up(W.gen_kv_cache(wl, l, "v")))
    model["embed"] = up(W.gen_tensor(wl, TID_EMBED, (wl.vocab, wl.hidden), "w"))
    model["final_norm"] = up(W.gen_tensor(wl, TID_FINAL_NORM, (wl.hidden,), "g"))
    model["lm_head"] = up(W.gen_tensor(wl, TID_LM_HEAD, (wl.vocab, wl.hidden), "w"))
    torch.cuda.synchronize(device)
    cfg = tre.config_from_workload(wl, debug_flags=debug_flags, **(overrides or {}))
    return tre.Engine(cfg, model, device), model


def build_layers_engine(wl, device: int, debug_flags: int = 0, overrides=None):
    """A layers-only stack (MoE or MLA layers, no embedding / LM head): non-expert tensors
    and caches from the workload generator, routed experts generated one at a time and
    stacked on the device."""
    import torch

    from persistent_tile_pipelined_b200 import tre
    from persistent_tile_pipelined_b200.synth import workloads as W

    dev = f"cuda:{device}"
    if wl.kind == "moe":
        model = W.gen_moe_model(wl)
        dmodel = tre.upload_moe_model(wl, model, dev)
    elif wl.kind == "mla":
        dmodel = tre.upload_mla_model(W.gen_mla_model(wl), dev)
    else:
        raise SystemExit(f"layers-only workload kind {wl.kind!r} is not built")
    torch.cuda.synchronize(device)
    cfg = tre.config_from_workload(wl, debug_flags=debug_flags, **(overrides or {}))
    return tre.Engine(cfg, dmodel, device), dmodel


def run_layers(args, rank, world, local_rank):
    """Timed layers-only steps: each step takes a different seeded hidden vector (so MoE
    routing changes from step to step, as in decode) at the next KV position."""
    import torch
    import torch.distributed as dist

    from persistent_tile_pipelined_b200.synth import TID_X_IN, normal_f32
    from persistent_tile_pipelined_b200.synth import workloads as W

    torch.cuda.set_device(local_rank)
    K, Wm = args.steps, args.warmup
    wl = workload_of(args).replace(decode_steps=K + Wm)
    wl = wl.replace(seed=wl.seed + rank)
    eng, dmodel = build_layers_engine(wl, local_rank, args.flags, config_overrides(args.config))
    stream = torch.cuda.current_stream(local_rank)
    s_ptr = stream.cuda_stream
    xs_host = [normal_f32(wl.seed + i, TID_X_IN, (wl.hidden,)) for i in range(K + Wm)]
    xs = torch.from_numpy(np.stack(xs_host)).to(f"cuda:{local_rank}")
    out = torch.empty(wl.hidden, dtype=torch.float32, device=f"cuda:{local_rank}")
    positions = [wl.prefill + i for i in range(K + Wm)]

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(local_rank)

    for i in range(Wm):
        eng.layers_step(xs[i], out, positions[i], stream=s_ptr)
    torch.cuda.synchronize(local_rank)
    assert eng.status() == (0, 0), eng.status()
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.2)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    barrier()
    tw0 = time.time()
    ev[0].record(stream)
    for i in range(K):
        eng.layers_step(xs[Wm + i], out, positions[Wm + i], stream=s_ptr)
        ev[i + 1].record(stream)
    torch.cuda.synchronize(local_rank)
    tw1 = time.time()
    barrier()
    sampler.mark(tw0, tw1)
    dev_s = ev[0].elapsed_time(ev[K]) / 1e3
    launch_ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(K)]
    assert eng.status() == (0, 0)
    # end to end: the hidden vector from pinned host memory in, the result back out
    x_pin = torch.empty(wl.hidden, dtype=torch.float32).pin_memory()
    o_pin = torch.empty(wl.hidden, dtype=torch.float32).pin_memory()
    x_dev = torch.empty(wl.hidden, dtype=torch.float32, device=f"cuda:{local_rank}")
    barrier()
    tw0 = time.time()
    t0 = time.perf_counter()
    for i in range(K):
        x_pin.copy_(torch.from_numpy(xs_host[Wm + i]))
        x_dev.copy_(x_pin, non_blocking=True)
        eng.layers_step(x_dev, out, positions[Wm + i], stream=s_ptr)
        o_pin.copy_(out, non_blocking=True)
        torch.cuda.synchronize(local_rank)
    e2e_s = time.perf_counter() - t0
    tw1 = time.time()
    barrier()
    sampler.mark(tw0, tw1)
    clocks = sampler.stop()
    step_bytes = float(np.mean([eng.step_bytes(positions[Wm + i]) for i in range(K)]))
    eng.close()
    if args.trace and rank == 0:
        # a fresh engine with the trace flag on the same device memory: three steps
        from persistent_tile_pipelined_b200 import trace as trace_mod
        from persistent_tile_pipelined_b200 import tre
        cfg = tre.config_from_workload(wl, debug_flags=tre.TRE_DEBUG_TRACE | args.flags)
        teng = tre.Engine(cfg, dmodel, local_rank)
        for i in range(3):
            teng.layers_step(xs[i], out, positions[i], stream=s_ptr)
        torch.cuda.synchronize(local_rank)
        tr = teng.trace()
        nsm = torch.cuda.get_device_properties(local_rank).multi_processor_count
        tasks, begin = tre.tre_plan_tasks(cfg, num_sms=nsm)
        teng.close()
        summ = trace_mod.summarize(tr, tasks)
        with open(args.trace, "w") as f:
            json.dump({"workload": wl.name, "summary": summ, "trace": tr.tolist(),
                       "tasks": tasks.tolist(), "sm_begin": begin.tolist()}, f)
        print(json.dumps(summ), file=sys.stderr)
    del dmodel
    torch.cuda.empty_cache()
    dev_s, e2e_s, launch_ms_avg = max_over_ranks(
        [dev_s, e2e_s, float(np.mean(launch_ms))], world, f"cuda:{local_rank}")
    return wl, dev_s, e2e_s, launch_ms_avg, step_bytes, clocks


def workload_step_bytes(wl, pos=None) -> int:
    """Bytes a one-token step streams at `pos` (default: the workload's KV length), from
    the workload's shape alone: every weight and norm gain the token reads (MoE: the
    router, the shared and the selected experts only), the K / V (latent) rows read and
    the new rows written, the embedding row and the logits.  Both arms state it in
    `config` without loading the engine library."""
    pos = wl.prefill if pos is None else pos
    d, L = wl.hidden, wl.n_layers
    if wl.kind == "mla":
        H, C = wl.n_q_heads, wl.kv_lora + wl.rope_dim
        w = ((wl.q_lora + C) * d + H * (wl.nope_dim + wl.rope_dim) * wl.q_lora +
             H * wl.nope_dim * wl.kv_lora + H * wl.v_dim * wl.kv_lora + d * H * wl.v_dim)
        HI, DI, KI = wl.index_heads, wl.index_dim, wl.index_topk
        if KI:  # the indexer's projections
            w += HI * DI * wl.q_lora + (DI + HI) * d
        total = (w * 2 + (d + wl.q_lora + wl.kv_lora) * 2) * L
        if KI and pos + 1 > KI:
            # every index key read (+ this one written), the K chosen latent rows read and
            # this position's latent row written
            total += L * ((pos + 1) * DI * 2 + (KI + 1) * C * 2)
        else:
            total += L * (pos + 1) * C * 2 + (L * (pos + 1) * DI * 2 if KI else 0)
    else:
        Hq, Hkv, D = wl.n_q_heads, wl.n_kv_heads, wl.head_dim
        mlp = (wl.n_experts * d + 3 * (wl.n_shared + wl.top_k) * wl.expert_ffn * d
               if wl.kind == "moe" else 3 * wl.ffn * d)
        proj = (Hq + 2 * Hkv) * D * d + d * Hq * D + mlp
        per_layer = proj * 2 + 2 * d * 2
        if getattr(wl, "weight_format", "bf16") == "fp4":  # the selected experts as MXFP4 rows
            from persistent_tile_pipelined_b200.synth import mxfp4_pitch
            Fe = wl.expert_ffn
            per_layer += wl.top_k * (2 * Fe * mxfp4_pitch(d) + d * mxfp4_pitch(Fe) - 3 * Fe * d * 2)
        if getattr(wl, "weight_format", "bf16") == "fp8":  # E4M3 + a scale per 128x128 block
            def blocks(N, K):
                return -(-N // 128) * -(-K // 128)
            nq, nk = Hq * D, Hkv * D
            per_layer = proj + 4 * (blocks(nq, d) + 2 * blocks(nk, d) + blocks(d, nq) +
                                    2 * blocks(wl.ffn, d) + blocks(d, wl.ffn)) + 2 * d * 2
        total = per_layer * L + L * Hkv * (pos + 1) * D * 2 * 2
    if wl.vocab > 0:
        total += wl.vocab * d * 2 + d * 2 + d * 2 + wl.vocab * 4
    return total


def plan_step_gb(wl) -> float:
    """GB a step streams at the workload's KV length (weights + KV), for `config`."""
    return workload_step_bytes(wl) / 1e9


def decode_config(wl, M: int, overrides: dict, world: int) -> dict:
    """`config` of a decode workload (the engine arm and the reference arm report the same)."""
    return {
        "workload": f"{wl.name} decode, batch 1, KV {wl.prefill} positions" +
                    (f", {M} tokens per step (causal verify tiles)" if M > 1 else ""),
        "tokens_per_step": M,
        "weights": ("E4M3 projections, 128x128 fp32 block scales; bf16 embedding, norms, LM head"
                    if wl.weight_format == "fp8" else "bf16"),
        "engine_config": overrides,
        "layers": wl.n_layers, "hidden": wl.hidden, "q_heads": wl.n_q_heads,
        "kv_heads": wl.n_kv_heads, "head_dim": wl.head_dim, "ffn": wl.ffn,
        "vocab": wl.vocab, "kv_positions": wl.prefill, "batch": 1,
        "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
        "l2": f"not flushed: each step streams {plan_step_gb(wl):.2f} GB >> 126 MB L2",
    }


def layers_config(wl, world: int) -> dict:
    """`config` of a layers-only workload (MoE, MLA); both arms report the same."""
    cfg = {"workload": f"{wl.name} layers-only step, batch 1, KV {wl.prefill} positions",
           "kind": wl.kind, "layers": wl.n_layers, "hidden": wl.hidden,
           "heads": wl.n_q_heads, "batch": 1,
           "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
           "l2": f"not flushed: each step streams {plan_step_gb(wl):.2f} GB >> 126 MB L2"}
    if wl.kind == "moe":
        cfg.update(experts=wl.n_experts, top_k=wl.top_k, shared=wl.n_shared,
                   expert_ffn=wl.expert_ffn, kv_heads=wl.n_kv_heads, head_dim=wl.head_dim)
        if getattr(wl, "weight_format", "bf16") == "fp4":
            cfg.update(weights="routed experts MXFP4 (E2M1 + E8M0 scale per 32); the rest bf16")
    if wl.kind == "mla":
        cfg.update(q_lora=wl.q_lora, kv_lora=wl.kv_lora, rope_dim=wl.rope_dim,
                   nope_dim=wl.nope_dim, v_dim=wl.v_dim, latent_positions=wl.prefill)
    return cfg


class DecodeSample:
    """One bounded sample of the oracle (as it stands, fp32, on this machine's cores) on a
    decode workload: a decode step of an `n`-layer slice (same layer shapes, same LM head,
    same KV length) and the slice's layers alone, scaled to the full stack as
    per-layer time x layers + the embedding / final-norm / LM-head time."""

    def __init__(self, wl, layers: int):
        self.wl = wl
        self.set_layers(layers)

    def set_layers(self, n: int):
        import oracle
        from persistent_tile_pipelined_b200.synth import workloads as W
        self.n = n
        self.sw = self.wl.replace(n_layers=n, decode_steps=1, tokens_per_step=1)
        self.model = W.gen_gqa_model(self.sw)
        self.orc = oracle.Oracle(32)
        self.tok = W.first_token(self.sw)
        self.x = np.full(self.sw.hidden, 0.01, dtype=np.float32)

    def step(self) -> float:
        """Seconds per token of the full stack, from one sample."""
        t0 = time.perf_counter()
        self.orc.decode_step(self.sw, self.model, self.tok, self.sw.prefill, want_hidden=False)
        t_step = time.perf_counter() - t0
        t0 = time.perf_counter()
        self.orc.layers_step(self.sw, self.model, self.x, self.sw.prefill)
        t_layers = time.perf_counter() - t0
        return t_layers / self.n * self.wl.n_layers + max(t_step - t_layers, 0.0)

    def describe(self) -> str:
        return (f"fp32 oracle, {self.n} of {self.wl.n_layers} layers + LM head, decode step "
                f"at pos {self.sw.prefill} (and the layers alone), scaled to the full stack")


class LayerSample:
    """One bounded sample of the oracle on a layers-only workload (MoE, MLA): one layer
    step of the stack's first layer at `prefill`, scaled by the number of layers."""

    def __init__(self, wl):
        import oracle
        from persistent_tile_pipelined_b200.synth import TID_X_IN, normal_f32
        from persistent_tile_pipelined_b200.synth import workloads as W
        self.wl = wl
        self.n = 1
        self.sw = wl.replace(n_layers=1, decode_steps=1)
        self.orc = oracle.Oracle(32)
        self.x = normal_f32(wl.seed, TID_X_IN, (wl.hidden,))
        if wl.kind == "moe":
            self.model = W.gen_moe_model(self.sw)
            self.experts = {}

            def expert(e):
                if e not in self.experts:
                    self.experts[e] = W.gen_expert(self.sw, 0, e)
                return self.experts[e]
            self.expert = expert
            self.step()  # the selected experts are generated once, outside the timed samples
        else:
            self.model = W.gen_mla_model(self.sw)

    def step(self) -> float:
        """Seconds per step of the full layer stack, from one sample."""
        m, pos = self.model, self.sw.prefill
        t0 = time.perf_counter()
        if self.wl.kind == "moe":
            self.orc.moe_layer_step(self.sw, m["layers"][0], m["k_cache"][0], m["v_cache"][0],
                                    self.expert, pos, self.x)
        else:
            ic = m["index_cache"][0] if self.sw.index_topk else None  # sparse: the indexer too
            self.orc.mla_layer_step(self.sw, m["layers"][0], m["latent_cache"][0], pos, self.x,
                                    index_cache=ic)
        return (time.perf_counter() - t0) * self.wl.n_layers

    def describe(self) -> str:
        return (f"fp32 oracle, 1 of {self.wl.n_layers} {self.wl.kind} layers at pos "
                f"{self.sw.prefill}, scaled to the full stack")


def cpu_cores() -> int:
    """Threads the OpenMP oracle runs on: OMP_NUM_THREADS, else the CPUs this process may
    run on (the OpenMP runtime's default)."""
    env = os.environ.get("OMP_NUM_THREADS", "").split(",")[0].strip()
    if env.isdigit() and int(env) > 0:
        return int(env)
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(wl, sample_layers: int, min_seconds: float = 10.0):
    """The oracle timed on a bounded sample of the workload (about `min_seconds` of CPU
    work): the median of repeated samples, scaled to the full stack."""
    smp = DecodeSample(wl, sample_layers)
    vals, t_start = [], time.perf_counter()
    while time.perf_counter() - t_start < min_seconds or len(vals) < 2:
        vals.append(smp.step())
    t_full = float(np.median(vals))
    work = time.perf_counter() - t_start
    return {"value": 1.0 / t_full, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
            "sample": f"{smp.describe()}; {len(vals)} samples ({work:.1f} s of CPU work), "
                      f"median {t_full:.3f} s/token",
            "seconds_per_token": t_full}


def run_engine(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from persistent_tile_pipelined_b200.synth import token_id
    from persistent_tile_pipelined_b200.synth import workloads as W

    torch.cuda.set_device(local_rank)
    wl = workload_of(args)
    K, Wm, M = args.steps, args.warmup, args.tokens_per_step
    wl = wl.replace(decode_steps=K + Wm, tokens_per_step=M, seed=wl.seed + rank)
    eng, model = build_engine(wl, local_rank, args.flags, config_overrides(args.config))
    from persistent_tile_pipelined_b200 import tre
    timed_launches = eng.set_launch_mode(tre.TRE_LAUNCH_PER_OP if args.launch_mode == "per-op"
                                         else tre.TRE_LAUNCH_PERSISTENT)
    stream = torch.cuda.current_stream(local_rank)
    s_ptr = stream.cuda_stream
    # step i takes tokens i M .. i M + M - 1 of the seeded stream at positions prefill + i M ..
    tokens = [[token_id(wl.seed, wl.vocab, i * M + v) for v in range(M)] for i in range(K + Wm)]
    positions = [wl.prefill + i * M for i in range(K + Wm)]

    def launch(i):
        if M == 1:
            eng.step(tokens[i][0], positions[i], stream=s_ptr)
        else:
            eng.step_tokens(tokens[i], positions[i], stream=s_ptr)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(local_rank)

    # warm-up
    for i in range(Wm):
        launch(i)
    torch.cuda.synchronize(local_rank)
    assert eng.status() == (0, 0), eng.status()

    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.2)

    # ---- device-timed region: K launches back to back
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    barrier()
    tw0 = time.time()
    ev[0].record(stream)
    for i in range(K):
        launch(Wm + i)
        ev[i + 1].record(stream)
    torch.cuda.synchronize(local_rank)
    tw1 = time.time()
    barrier()
    sampler.mark(tw0, tw1)
    dev_s = ev[0].elapsed_time(ev[K]) / 1e3
    launch_ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(K)]
    st = eng.status()
    assert st == (0, 0), st

    # ---- end to end through the C ABI: greedy loop, token(s) back to the host every step
    tok = tokens[0][0]
    tok_dev = torch.empty(M, dtype=torch.int32, device=f"cuda:{local_rank}")
    barrier()
    tw0 = time.time()
    t0 = time.perf_counter()
    for i in range(K):
        if M == 1:
            tok = eng.step_host(tok, positions[Wm + i], stream=s_ptr)
        else:   # verify the next M tokens, read the M argmax tokens back
            eng.step_tokens(tokens[Wm + i], positions[Wm + i], tokens_out=tok_dev, stream=s_ptr)
            tok = tok_dev.cpu()
    e2e_s = time.perf_counter() - t0
    tw1 = time.time()
    barrier()
    sampler.mark(tw0, tw1)
    clocks = sampler.stop()

    step_bytes = float(np.mean([eng.step_bytes(positions[Wm + i], M) for i in range(K)]))
    extra = {}
    if M == 1 and not args.no_ablation and args.launch_mode == "persistent":
        extra = ablation(eng, wl, tokens, positions, Wm, K, stream, local_rank, barrier)
    trace_path = args.trace if rank == 0 else ""
    eng.close()
    del model
    torch.cuda.empty_cache()

    if trace_path:
        write_trace(wl, local_rank, trace_path, args.flags, config_overrides(args.config),
                    per_op=args.launch_mode == "per-op")

    dev_s, e2e_s, launch_ms_avg = max_over_ranks(
        [dev_s, e2e_s, float(np.mean(launch_ms))], world, f"cuda:{local_rank}")
    if extra:
        keys = sorted(k for k, v in extra.items() if isinstance(v, float))
        worst = max_over_ranks([extra[k] for k in keys], world, f"cuda:{local_rank}")
        extra.update(zip(keys, worst))
    extra["timed_launches_per_step"] = timed_launches
    return wl, dev_s, e2e_s, launch_ms_avg, step_bytes, clocks, extra


def ablation(eng, wl, tokens, positions, Wm, K, stream, local_rank, barrier):
    """Beside the timed persistent steps: (1) the kernel-per-op form of the same step (the
    same tiles on the same plan, one plain launch per op) enqueued launch by launch and
    replayed from CUDA graphs, timed with CUDA events over steps at the same positions
    (each step streams the same bytes); (2) the device-resident greedy loop
    (tre_decode_loop): n steps enqueued at once, each step's argmax feeding the next on the
    device, timed end to end on the host up to the n tokens back in pinned host memory."""
    import torch

    from persistent_tile_pipelined_b200 import tre
    n = min(K, 16)
    s_ptr = stream.cuda_stream
    out = {}

    def timed(run):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        barrier()
        ev[0].record(stream)
        for i in range(n):
            run(i)
        ev[1].record(stream)
        torch.cuda.synchronize(local_rank)
        return ev[0].elapsed_time(ev[1]) / n

    out["launches_per_step"] = eng.set_launch_mode(tre.TRE_LAUNCH_PER_OP)
    for i in range(3):
        eng.step(tokens[Wm + i][0], positions[Wm + i], stream=s_ptr)
    out["per_op_ms_per_step"] = timed(lambda i: eng.step(tokens[Wm + i][0], positions[Wm + i],
                                                         stream=s_ptr))
    # the same per-op steps captured once and replayed (host launch cost removed)
    graphs = []
    side = torch.cuda.Stream(local_rank)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for i in range(n):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                eng.step(tokens[Wm + i][0], positions[Wm + i], stream=side.cuda_stream)
            graphs.append(g)
    stream.wait_stream(side)
    torch.cuda.synchronize(local_rank)
    for i in range(3):
        graphs[i].replay()
    out["per_op_graph_ms_per_step"] = timed(lambda i: graphs[i].replay())
    del graphs
    st = eng.status()
    assert st == (0, 0), st
    # per-op steps (direct or replayed) leave the persistent form's counters untouched
    eng.set_launch_mode(tre.TRE_LAUNCH_PERSISTENT)
    for i in range(3):
        eng.step(tokens[Wm + i][0], positions[Wm + i], stream=s_ptr)
    out["persistent_ms_per_step"] = timed(lambda i: eng.step(tokens[Wm + i][0], positions[Wm + i],
                                                             stream=s_ptr))
    # device-resident greedy loop: n steps, one call, tokens back once
    toks_dev = torch.empty(n, dtype=torch.int32, device=f"cuda:{local_rank}")
    toks_pin = torch.empty(n, dtype=torch.int32).pin_memory()
    eng.decode_loop(tokens[Wm][0], positions[Wm], 3, toks_dev, stream=s_ptr)
    barrier()
    t0 = time.perf_counter()
    eng.decode_loop(tokens[Wm][0], positions[Wm], n, toks_dev, stream=s_ptr)
    toks_pin.copy_(toks_dev, non_blocking=True)
    torch.cuda.synchronize(local_rank)
    out["device_loop_s_per_step"] = (time.perf_counter() - t0) / n
    st = eng.status()
    assert st == (0, 0), st
    out["steps"] = n
    return out


def write_trace(wl, device, path, flags=0, overrides=None, per_op=False):
    """Three traced steps on a fresh engine (debug flag): per-task start / ready / end of
    the last one, with the plan and its summary.  Steps take the workload's tokens per step;
    per_op: the kernel-per-op launch form."""
    import torch

    from persistent_tile_pipelined_b200 import trace as trace_mod
    from persistent_tile_pipelined_b200 import tre
    M = max(1, wl.tokens_per_step)
    eng, model = build_engine(wl.replace(decode_steps=3 * M), device, tre.TRE_DEBUG_TRACE | flags,
                              overrides)
    if per_op:
        eng.set_launch_mode(tre.TRE_LAUNCH_PER_OP)
    for i in range(3):
        if M > 1:
            eng.step_tokens([1 + i * M + v for v in range(M)], wl.prefill + i * M)
        else:
            eng.step(1 + i, wl.prefill + i)
    torch.cuda.synchronize(device)
    tr = eng.trace()
    nsm = torch.cuda.get_device_properties(device).multi_processor_count
    tasks, begin = tre.tre_plan_tasks(eng.cfg, num_sms=nsm)
    eng.close()
    summ = trace_mod.summarize(tr, tasks)
    with open(path, "w") as f:
        json.dump({"workload": wl.name, "summary": summ, "trace": tr.tolist(),
                   "tasks": tasks.tolist(), "sm_begin": begin.tolist()}, f)
    print(json.dumps(summ), file=sys.stderr)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if world != args.gpus:
        args.gpus = world

    if args.impl == "reference":
        return main_reference(args, rank, world)

    import torch
    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device(f"cuda:{local_rank}"))
    from persistent_tile_pipelined_b200.synth import workloads as W
    if workload_of(args).kind != "gqa":
        return main_layers(args, rank, world, local_rank)
    wl, dev_s, e2e_s, launch_ms, step_bytes, clocks, abl = run_engine(args, rank, world,
                                                                      local_rank)
    K, M = args.steps, args.tokens_per_step
    peak, peak_kind = peaks()
    achieved = step_bytes / (launch_ms / 1e3) / 1e9
    line = {
        "metric": METRIC,
        "value": job_throughput(world, K, M, dev_s),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": dev_s / K * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8e4m3" if wl.weight_format == "fp8" else "bf16",
        "data": "synthetic (seeded random-init weights N(0,0.02), KV N(0,1))" +
                ("; projections block-quantised to E4M3 (128x128 fp32 scales)"
                 if wl.weight_format == "fp8" else ""),
        "config": decode_config(wl, M, config_overrides(args.config), world),
        "hbm_gbs": step_bytes / (dev_s / K) / 1e9,
        "hbm_frac_of_8tbs": step_bytes / (dev_s / K) / 1e9 / NOMINAL_HBM_GBS,
        "roofline": {
            "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "peak_kind": peak_kind,
            "traffic": profiled_traffic(args.workload, M),
            "kernel": "tre::engine_kernel",
            "algorithmic_bytes_per_launch": step_bytes,
        },
        "e2e": {"value": job_throughput(world, K, M, e2e_s), "unit": "tokens/s",
                "h2d_bytes_per_step": 4 * M,
                "d2h_bytes_per_step": 4 * M,
                "note": "greedy loop via tre_decode_step_host: token in as a kernel argument, "
                        "argmax token back to pinned-less host memory, host wall time"},
        "gpu_launches": K * abl["timed_launches_per_step"],
        "launch_mode": args.launch_mode,
        "clocks": clocks,
    }
    if "steps" in abl:
        n = abl["steps"]
        line["ablation"] = {
            "what": "the same tiles on the same plan: one persistent launch per step vs one "
                    "plain launch per op (QKV, attention + combine, O, gate/up, down per layer, "
                    "LM head), enqueued launch by launch and replayed from CUDA graphs; "
                    f"{n} steps each at the timed positions, CUDA events",
            "launches_per_step": abl["launches_per_step"],
            "persistent_ms_per_step": abl["persistent_ms_per_step"],
            "per_op_ms_per_step": abl["per_op_ms_per_step"],
            "per_op_graph_ms_per_step": abl["per_op_graph_ms_per_step"],
            "per_op_extra_us_per_launch": (abl["per_op_ms_per_step"] -
                                           abl["persistent_ms_per_step"]) * 1e3 /
                                          abl["launches_per_step"],
        }
        line["e2e_device_loop"] = {
            "value": world / abl["device_loop_s_per_step"], "unit": "tokens/s",
            "h2d_bytes_per_step": 4.0 / n, "d2h_bytes_per_step": 4,
            "note": f"tre_decode_loop: {n} greedy steps in one call, each step's argmax feeds "
                    "the next step on the device; host wall time up to the tokens back in "
                    "pinned memory"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        try:
            line["cpu_baseline"] = cpu_baseline(wl, args.cpu_sample_layers)
        except Exception as exc:  # report, do not hide
            line["cpu_baseline"] = {"error": repr(exc)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main_layers(args, rank, world, local_rank):
    """Layers-only workloads (MoE, MLA): step time of the whole layer stack and the HBM
    bandwidth it achieves over the bytes a token actually reads."""
    import torch.distributed as dist
    wl, dev_s, e2e_s, launch_ms, step_bytes, clocks = run_layers(args, rank, world, local_rank)
    K = args.steps
    peak, peak_kind = peaks()
    achieved = step_bytes / (launch_ms / 1e3) / 1e9
    cfg = layers_config(wl, world)
    line = {
        "metric": LAYERS_METRIC,
        "value": job_throughput(world, K, 1, dev_s), "unit": "steps/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": dev_s / K * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "fp4e2m1-experts" if wl.weight_format == "fp4" else "bf16",
        "data": "synthetic (seeded random-init weights N(0,0.02), KV N(0,1))" +
                ("; routed experts random MXFP4 codes, scales 2^-8 / 2^-7"
                 if wl.weight_format == "fp4" else ""),
        "config": cfg,
        "hbm_gbs": step_bytes / (dev_s / K) / 1e9,
        "hbm_frac_of_8tbs": step_bytes / (dev_s / K) / 1e9 / NOMINAL_HBM_GBS,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind, "traffic": None,
                     "kernel": "tre::engine_kernel",
                     "algorithmic_bytes_per_launch": step_bytes},
        "e2e": {"value": job_throughput(world, K, 1, e2e_s), "unit": "steps/s",
                "h2d_bytes_per_step": 4 * wl.hidden, "d2h_bytes_per_step": 4 * wl.hidden},
        "gpu_launches": K,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main_reference(args, rank, world):
    """The reference arm: the CPU oracle as it stands, on this machine's host cores, for the
    engine arm's workload, metric, unit and config.  W untimed and K timed steps, each step
    one bounded sample of the workload (a layer slice, scaled to the full stack), the slice
    sized so the whole run takes about two minutes.  Rank 0 only."""
    if rank != 0:
        return
    from persistent_tile_pipelined_b200.synth import workloads as W
    K, Wm, M = args.steps, args.warmup, args.tokens_per_step
    wl = workload_of(args).replace(decode_steps=K + Wm)
    budget = REFERENCE_SECONDS / max(1, K + Wm)  # seconds of oracle work per step
    if wl.kind == "gqa":
        wl = wl.replace(tokens_per_step=M)
        smp = DecodeSample(wl, args.cpu_sample_layers)
        while smp.n > 1:  # one sample must fit the per-step budget (untimed calibration)
            t0 = time.perf_counter()
            smp.step()
            if time.perf_counter() - t0 <= budget:
                break
            smp.set_layers(max(1, smp.n // 2))
        metric, unit, per = METRIC, "tokens/s", M  # tokens per step
        config = decode_config(wl, M, config_overrides(args.config), world)
    else:
        M = 1
        smp = LayerSample(wl)
        metric, unit, per = LAYERS_METRIC, "steps/s", 1
        config = layers_config(wl, world)
    for _ in range(Wm):
        smp.step()
    t_start = time.perf_counter()
    vals = [smp.step() for _ in range(K)]
    work = time.perf_counter() - t_start
    t = float(np.median(vals))  # seconds per token (decode) or per stack step (layers)
    v = 1.0 / t
    sample = (f"{smp.describe()}; one sample per step, {K} timed after {Wm} warm-up "
              f"({work:.1f} s of CPU work), median {t:.4f} s per "
              f"{'token' if wl.kind == 'gqa' else 'stack step'}")
    line = {
        "metric": metric, "value": v, "unit": unit, "n_gpus": world, "steps": K,
        "warmup": Wm, "ms_per_step": t * per * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded random-init weights N(0,0.02), KV N(0,1))",
        "config": config,
        "impl": "reference",
        "cpu_baseline": {"value": v, "unit": unit, "cores": cpu_cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
