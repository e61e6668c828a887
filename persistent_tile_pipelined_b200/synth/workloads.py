"""Workload recipes: shapes, seeds and value distributions of the synthetic decode inputs.

Every tensor is drawn from the seeded generator in this package (one stream per tensor
id), so the engine's device copy and the oracle's host copy are bit-identical.

Distributions (the workloads' own statement): bf16 weights N(0, 0.02); RMSNorm gains
1 + N(0, 0.01); KV cache positions [0, prefill) N(0, 1) bf16, later positions zero until
a decode step writes them; layer-only workloads start from a hidden vector N(0, 1) fp32.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np

from . import (TID_EMBED, TID_FINAL_NORM, TID_LM_HEAD, TID_X_IN, e4m3_blocks, mxfp4_rows,
               normal_bf16, normal_f32, tid_kcache, tid_layer, tid_vcache, token_id)

W_STD = 0.02
GAIN_STD = 0.01


@dataclasses.dataclass
class Workload:
    name: str
    kind: str                 # "gqa" | "mla" | "moe"
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int = 0
    head_dim: int = 0
    ffn: int = 0
    vocab: int = 0
    prefill: int = 0          # KV positions filled before the first decode step
    decode_steps: int = 1     # decode steps the workload runs (KV capacity = prefill + steps)
    rope_theta: float = 1e4
    norm_eps: float = 1e-5
    tokens_per_step: int = 1
    seed: int = 1234
    weight_format: str = "bf16"  # "fp8": GQA projections as E4M3 bytes + 128x128 block scales;
    #                              "fp4": MoE routed experts as MXFP4 rows (E2M1 + E8M0 per 32)
    # MLA sparse attention (0 = dense): index heads, index dim, positions kept per step
    index_heads: int = 0
    index_dim: int = 0
    index_topk: int = 0
    # MLA
    q_lora: int = 0
    kv_lora: int = 0
    rope_dim: int = 0
    nope_dim: int = 0
    v_dim: int = 0
    # MoE
    n_experts: int = 0
    top_k: int = 0
    n_shared: int = 0
    expert_ffn: int = 0

    @property
    def kv_capacity(self) -> int:
        return self.prefill + self.decode_steps * self.tokens_per_step

    @property
    def has_embed_lm_head(self) -> bool:
        return self.vocab > 0

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# Tiny 2-layer decoder: hidden 256, 4 q / 2 kv heads of dim 64, RoPE theta 1e4, SwiGLU 688,
# vocab 1024, KV cache 128 positions.
TINY = Workload(name="tiny-2L-d256", kind="gqa", n_layers=2, hidden=256, n_q_heads=4,
                n_kv_heads=2, head_dim=64, ffn=688, vocab=1024, prefill=128, decode_steps=64,
                rope_theta=1e4, norm_eps=1e-5)

# Llama-3-8B-shaped stack: 32 layers, hidden 4096, 32 q / 8 kv heads of dim 128, SwiGLU 14336,
# vocab 128256, KV cache 4096 positions, 64 greedy decode steps.
LLAMA8B = Workload(name="llama3-8b-shaped", kind="gqa", n_layers=32, hidden=4096, n_q_heads=32,
                   n_kv_heads=8, head_dim=128, ffn=14336, vocab=128256, prefill=4096,
                   decode_steps=64, rope_theta=5e5, norm_eps=1e-5)

# The same layer shapes with 4 layers: a ~3.8 GB case (well above the 126 MB L2) for
# profiler captures that must stay small.
LLAMA8B_4L = LLAMA8B.replace(name="llama3-8b-shaped-4L", n_layers=4)

# Absorbed-MLA decode layers x4 (attention only): hidden 7168, 128 heads, q_lora 1536,
# kv_lora 512, rope 64, nope 128, v 128; latent KV cache 8192 positions; theta 1e4, eps 1e-6.
MLA4 = Workload(name="mla-4L-d7168", kind="mla", n_layers=4, hidden=7168, n_q_heads=128,
                q_lora=1536, kv_lora=512, rope_dim=64, nope_dim=128, v_dim=128, prefill=8192,
                decode_steps=1, rope_theta=1e4, norm_eps=1e-6)

# MoE decode layers x4: hidden 7168, 256 routed experts top-8 + 1 shared, expert SwiGLU 2048,
# sigmoid router; GQA attention 64 q / 8 kv heads of dim 128 over 4096 positions.
MOE4 = Workload(name="moe-4L-d7168", kind="moe", n_layers=4, hidden=7168, n_q_heads=64,
                n_kv_heads=8, head_dim=128, prefill=4096, decode_steps=1, rope_theta=1e4,
                norm_eps=1e-6, n_experts=256, top_k=8, n_shared=1, expert_ffn=2048)

# Long-context sweep on the 8B-shaped stack: 8192 / 32768 / 131072 cached positions.
LLAMA8B_KV8K = LLAMA8B.replace(name="llama3-8b-shaped-kv8k", prefill=8192)
LLAMA8B_KV32K = LLAMA8B.replace(name="llama3-8b-shaped-kv32k", prefill=32768)
LLAMA8B_KV128K = LLAMA8B.replace(name="llama3-8b-shaped-kv128k", prefill=131072)

# The 8B-shaped stack with FP8 projections (E4M3, one scale per 128 x 128 block); the
# embedding, norms and LM head stay bf16.
LLAMA8B_FP8 = LLAMA8B.replace(name="llama3-8b-shaped-fp8", weight_format="fp8")

# Absorbed-MLA layers x4 with the sparse-attention indexer (64 index heads of dim 128 keep
# the top 2048 of 131072 cached positions: the pages' 160K-context setting), and the same
# layers dense at that length for comparison.
MLA4_SPARSE128K = MLA4.replace(name="mla-4L-d7168-sparse-kv128k", prefill=131072, index_heads=64,
                               index_dim=128, index_topk=2048)
MLA4_KV128K = MLA4.replace(name="mla-4L-d7168-kv128k", prefill=131072)

# The MoE layers with FP4 routed experts (MXFP4 rows: E2M1 codes, one power-of-two scale per
# 32 weights); attention, router and shared expert stay bf16.
MOE4_FP4 = MOE4.replace(name="moe-4L-d7168-fp4", weight_format="fp4")

WORKLOADS = {w.name: w for w in (TINY, LLAMA8B, LLAMA8B_4L, MLA4, MOE4, LLAMA8B_KV8K,
                                 LLAMA8B_KV32K, LLAMA8B_KV128K, LLAMA8B_FP8, MLA4_SPARSE128K,
                                 MLA4_KV128K, MOE4_FP4)}


def gqa_layer_shapes(w: Workload) -> List[tuple]:
    """(slot, shape, kind) of every GQA layer tensor; kind 'w' = weight, 'g' = gain."""
    d, hq, hkv, dh, f = w.hidden, w.n_q_heads, w.n_kv_heads, w.head_dim, w.ffn
    return [
        (0, (d,), "g"),                 # attention RMSNorm gain
        (1, (hq * dh, d), "w"),         # Wq
        (2, (hkv * dh, d), "w"),        # Wk
        (3, (hkv * dh, d), "w"),        # Wv
        (4, (d, hq * dh), "w"),         # Wo
        (5, (d,), "g"),                 # MLP RMSNorm gain
        (6, (f, d), "w"),               # W_gate
        (7, (f, d), "w"),               # W_up
        (8, (d, f), "w"),               # W_down
    ]


def mla_layer_shapes(w: Workload) -> List[tuple]:
    """(slot, shape, kind) of every absorbed-MLA layer tensor."""
    d, H, ql, kl, r = w.hidden, w.n_q_heads, w.q_lora, w.kv_lora, w.rope_dim
    nope, v = w.nope_dim, w.v_dim
    return [
        (0, (d,), "g"),                     # attention RMSNorm gain
        (1, (ql, d), "w"),                  # W_dq
        (2, (ql,), "g"),                    # q_lora RMSNorm gain
        (3, (H * (nope + r), ql), "w"),     # W_uq: per head [nope | rope] rows
        (4, (kl + r, d), "w"),              # W_dkv: [kv_lora | rope] rows
        (5, (kl,), "g"),                    # kv_lora RMSNorm gain
        (6, (H * nope, kl), "w"),           # W_uk
        (7, (H * v, kl), "w"),              # W_uv
        (8, (d, H * v), "w"),               # W_o
    ] + ([
        (9, (w.index_heads * w.index_dim, ql), "w"),      # indexer queries W_iq
        (10, (w.index_dim + w.index_heads, d), "w"),      # indexer key rows, head-weight rows
    ] if w.index_topk else [])


def moe_layer_shapes(w: Workload) -> List[tuple]:
    """(slot, shape, kind) of the non-expert tensors of a MoE layer."""
    d, hq, hkv, dh = w.hidden, w.n_q_heads, w.n_kv_heads, w.head_dim
    fs = w.expert_ffn * w.n_shared
    return [
        (0, (d,), "g"), (1, (hq * dh, d), "w"), (2, (hkv * dh, d), "w"),
        (3, (hkv * dh, d), "w"), (4, (d, hq * dh), "w"),
        (5, (d,), "g"),                     # MLP RMSNorm gain
        (6, (w.n_experts, d), "w"),         # router
        (7, (fs, d), "w"), (8, (fs, d), "w"), (9, (d, fs), "w"),   # shared expert
    ]


def tid_expert(layer: int, expert: int, which: int) -> int:
    """Tensor id of routed expert `expert` of `layer`: which 0 = gate, 1 = up, 2 = down."""
    return 1_000_000 + int(layer) * 100_000 + int(expert) * 4 + int(which)


def gen_expert(w: Workload, layer: int, expert: int) -> tuple:
    """(W_gate [F][d], W_up [F][d], W_down [d][F]) of one routed expert, on demand: bf16
    words N(0, 0.02), or (weight_format "fp4") MXFP4 rows of bytes [F][pitch(d)], [F][pitch(d)],
    [d][pitch(F)] with scales 2^-8 / 2^-7 (rms about 0.018)."""
    F, d = w.expert_ffn, w.hidden
    if w.weight_format == "fp4":
        return (mxfp4_rows(w.seed, tid_expert(layer, expert, 0), F, d),
                mxfp4_rows(w.seed, tid_expert(layer, expert, 1), F, d),
                mxfp4_rows(w.seed, tid_expert(layer, expert, 2), d, F))
    return (gen_tensor(w, tid_expert(layer, expert, 0), (F, d), "w"),
            gen_tensor(w, tid_expert(layer, expert, 1), (F, d), "w"),
            gen_tensor(w, tid_expert(layer, expert, 2), (d, F), "w"))


def gen_mla_model(w: Workload) -> dict:
    assert w.kind == "mla"
    C = w.kv_lora + w.rope_dim
    model = {"layers": [], "latent_cache": [], "x_in": normal_f32(w.seed, TID_X_IN, (w.hidden,))}
    for l in range(w.n_layers):
        model["layers"].append({slot: gen_tensor(w, tid_layer(l, slot), shape, kind)
                                for slot, shape, kind in mla_layer_shapes(w)})
        cache = np.zeros((w.kv_capacity, C), dtype=np.uint16)
        if w.prefill:
            cache[: w.prefill] = normal_bf16(w.seed, tid_kcache(l), (w.prefill, C), 0.0, 1.0)
        model["latent_cache"].append(cache)
        if w.index_topk:  # the indexer's key cache [capacity][index_dim], N(0, 1) like the latents
            icache = np.zeros((w.kv_capacity, w.index_dim), dtype=np.uint16)
            if w.prefill:
                icache[: w.prefill] = normal_bf16(w.seed, tid_vcache(l), (w.prefill, w.index_dim),
                                                  0.0, 1.0)
            model.setdefault("index_cache", []).append(icache)
    return model


def gen_moe_model(w: Workload, with_experts: bool = False) -> dict:
    """Non-expert tensors, KV caches and x_in; routed experts come from gen_expert on
    demand (all of them when with_experts)."""
    assert w.kind == "moe"
    model = {
        "layers": [{slot: gen_tensor(w, tid_layer(l, slot), shape, kind)
                    for slot, shape, kind in moe_layer_shapes(w)} for l in range(w.n_layers)],
        "k_cache": [gen_kv_cache(w, l, "k") for l in range(w.n_layers)],
        "v_cache": [gen_kv_cache(w, l, "v") for l in range(w.n_layers)],
        "x_in": normal_f32(w.seed, TID_X_IN, (w.hidden,), 0.0, 1.0),
    }
    if with_experts:
        model["experts"] = [[gen_expert(w, l, e) for e in range(w.n_experts)]
                            for l in range(w.n_layers)]
    return model


def gen_tensor(w: Workload, tensor_id: int, shape, kind: str,
               out: Optional[np.ndarray] = None) -> np.ndarray:
    if kind == "g":
        return normal_bf16(w.seed, tensor_id, shape, 1.0, GAIN_STD, out)
    if kind == "w":
        return normal_bf16(w.seed, tensor_id, shape, 0.0, W_STD, out)
    if kind == "kv":
        return normal_bf16(w.seed, tensor_id, shape, 0.0, 1.0, out)
    raise ValueError(kind)


# FP8 GQA layers: the block scales of projection slot s sit in slot FP8_SCALE_SLOT[s]
FP8_SCALE_SLOT = {1: 9, 2: 10, 3: 11, 4: 12, 6: 13, 7: 14, 8: 15}


def gen_gqa_layer(w: Workload, layer: int) -> Dict[int, np.ndarray]:
    """bf16 words per slot; FP8 workloads: the projection slots hold E4M3 bytes (uint8) of
    the same N(0, 0.02) values and slots 9 .. 15 their fp32 block scales."""
    out = {}
    for slot, shape, kind in gqa_layer_shapes(w):
        if w.weight_format == "fp8" and slot in FP8_SCALE_SLOT:
            out[slot], out[FP8_SCALE_SLOT[slot]] = e4m3_blocks(w.seed, tid_layer(layer, slot),
                                                               shape, W_STD)
        else:
            out[slot] = gen_tensor(w, tid_layer(layer, slot), shape, kind)
    return out


def gen_kv_cache(w: Workload, layer: int, which: str) -> np.ndarray:
    """[Hkv][capacity][D] bf16 words; positions < prefill drawn N(0,1), the rest zero."""
    cap, hkv, dh = w.kv_capacity, w.n_kv_heads, w.head_dim
    out = np.zeros((hkv, cap, dh), dtype=np.uint16)
    tid = tid_kcache(layer) if which == "k" else tid_vcache(layer)
    if w.prefill:
        pre = normal_bf16(w.seed, tid, (hkv, w.prefill, dh), 0.0, 1.0)
        out[:, : w.prefill, :] = pre
    return out


def gen_gqa_model(w: Workload) -> dict:
    """All host tensors of a GQA decoder workload (bf16 words as uint16 arrays)."""
    assert w.kind == "gqa"
    model = {
        "layers": [gen_gqa_layer(w, l) for l in range(w.n_layers)],
        "k_cache": [gen_kv_cache(w, l, "k") for l in range(w.n_layers)],
        "v_cache": [gen_kv_cache(w, l, "v") for l in range(w.n_layers)],
    }
    if w.has_embed_lm_head:
        model["embed"] = gen_tensor(w, TID_EMBED, (w.vocab, w.hidden), "w")
        model["final_norm"] = gen_tensor(w, TID_FINAL_NORM, (w.hidden,), "g")
        model["lm_head"] = gen_tensor(w, TID_LM_HEAD, (w.vocab, w.hidden), "w")
    else:
        model["x_in"] = normal_f32(w.seed, TID_X_IN, (w.hidden,), 0.0, 1.0)
    return model


def first_token(w: Workload) -> int:
    return token_id(w.seed, w.vocab)
