"""Python binding of the engine's C ABI (``include/tre.h``): argument marshalling only.

Every step of the decode path runs inside ``libtre.so``; this module converts Python
objects to the C structs, passes device pointers from torch tensors and raises on error.
There is no fallback: if the native library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtre.so")

# ---- constants mirrored from tre.h ------------------------------------------------------
TRE_OK = 0
TRE_ERR_INVALID_ARG = -1
TRE_ERR_CUDA = -2
TRE_ERR_OCCUPANCY = -3
TRE_ERR_DEP_TIMEOUT = -4
TRE_ERR_POS_RANGE = -5
TRE_ERR_UNSUPPORTED = -6
TRE_ERR_BOUNDS = -7
TRE_ERR_STATE = -8
TRE_LAYER_GQA, TRE_LAYER_MLA, TRE_LAYER_MOE = 0, 1, 2
TRE_WEIGHTS_BF16, TRE_WEIGHTS_FP8_BLOCK128, TRE_WEIGHTS_FP4_EXPERTS = 0, 1, 2
TRE_DEBUG_HIDDEN, TRE_DEBUG_TRACE, TRE_DEBUG_FAULT_INJECT, TRE_DEBUG_NO_OVERLAP = 1, 2, 4, 8
TRE_W_SLOTS = 16
TRACE_COLS = 8
GQA_SLOTS = {"attn_norm": 0, "wq": 1, "wk": 2, "wv": 3, "wo": 4, "ffn_norm": 5, "wgate": 6,
             "wup": 7, "wdown": 8}
MOE_SLOTS = {"attn_norm": 0, "wq": 1, "wk": 2, "wv": 3, "wo": 4, "ffn_norm": 5, "router": 6,
             "shared_gate": 7, "shared_up": 8, "shared_down": 9, "expert_gate": 10,
             "expert_up": 11, "expert_down": 12}

STATUS_NAMES = {0: "TRE_OK", -1: "TRE_ERR_INVALID_ARG", -2: "TRE_ERR_CUDA",
                -3: "TRE_ERR_OCCUPANCY", -4: "TRE_ERR_DEP_TIMEOUT", -5: "TRE_ERR_POS_RANGE",
                -6: "TRE_ERR_UNSUPPORTED", -7: "TRE_ERR_BOUNDS", -8: "TRE_ERR_STATE"}


class tre_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "kind", "n_layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim", "ffn", "vocab",
        "q_lora", "kv_lora", "rope_dim", "nope_dim", "v_dim",
        "n_experts", "top_k", "n_shared", "expert_ffn",
        "kv_capacity", "max_tokens_per_step")] + [
        ("rope_theta", ctypes.c_float), ("norm_eps", ctypes.c_float)] + [
        (n, ctypes.c_int32) for n in (
            "has_embed_lm_head", "debug_flags", "dep_timeout_us", "num_sms", "kv_splits",
            "stage_bytes", "ring_stages", "l2_prefetch_kb", "gemv_kpart_max",
            "stream_policy", "multi_token_gemv", "weight_format", "index_heads", "index_dim",
            "index_topk")]


class tre_weights(ctypes.Structure):
    _fields_ = [("embed", ctypes.c_void_p), ("final_norm", ctypes.c_void_p),
                ("lm_head", ctypes.c_void_p), ("layer_w", ctypes.POINTER(ctypes.c_void_p)),
                ("k_cache", ctypes.POINTER(ctypes.c_void_p)),
                ("v_cache", ctypes.POINTER(ctypes.c_void_p))]


class tre_plan_info(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "num_sms", "num_tasks", "num_counters", "kv_splits", "ring_stages", "stage_bytes",
        "smem_bytes", "max_tasks_per_sm", "gemv_tiles", "index_splits")] + [
        (n, ctypes.c_int64) for n in ("weight_bytes", "kv_bytes_at_capacity", "max_sm_bytes",
                                      "min_sm_bytes")]


TRE_LAUNCH_PERSISTENT, TRE_LAUNCH_PER_OP = 0, 1

EXPORTED = ("tre_create", "tre_destroy", "tre_decode_step", "tre_decode_step_host",
            "tre_decode_step_static", "tre_layers_step", "tre_debug_routing", "tre_debug_index",
            "tre_debug_check",
            "tre_decode_tokens", "tre_decode_loop", "tre_set_launch_mode", "tre_get_status",
            "tre_reset", "tre_debug_hidden", "tre_debug_trace", "tre_step_bytes",
            "tre_plan_inspect", "tre_plan_tasks", "tre_plan_op_groups", "tre_last_error")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m persistent_tile_pipelined_b200.build` (needs nvcc)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    L.tre_create.argtypes = [ctypes.POINTER(tre_config), ctypes.POINTER(tre_weights), ctypes.c_int,
                             ctypes.POINTER(vp)]
    L.tre_destroy.argtypes = [vp]
    L.tre_destroy.restype = None
    L.tre_decode_step.argtypes = [vp, i32, i32, vp, vp, vp]
    L.tre_decode_step_host.argtypes = [vp, i32, i32, vp, vp, vp]
    L.tre_decode_step_static.argtypes = [ctypes.POINTER(tre_config), ctypes.POINTER(tre_weights),
                                         i32, i32, vp, vp, vp, vp]
    L.tre_layers_step.argtypes = [vp, vp, vp, i32, vp]
    L.tre_decode_tokens.argtypes = [vp, vp, i32, i32, vp, vp, vp]
    L.tre_decode_loop.argtypes = [vp, i32, i32, i32, vp, vp, vp]
    L.tre_set_launch_mode.argtypes = [vp, i32, ctypes.POINTER(i32)]
    L.tre_plan_op_groups.argtypes = [ctypes.POINTER(tre_config), i32, i32, vp, i32]
    L.tre_plan_op_groups.restype = i32
    L.tre_debug_routing.argtypes = [vp, vp, vp]
    L.tre_debug_index.argtypes = [vp, i32, i32, vp, vp, ctypes.POINTER(i32)]
    L.tre_debug_check.argtypes = [vp, ctypes.POINTER(i32), ctypes.POINTER(i32)]
    L.tre_get_status.argtypes = [vp, ctypes.POINTER(i32), ctypes.POINTER(i32)]
    L.tre_reset.argtypes = [vp, vp]
    L.tre_debug_hidden.argtypes = [vp, vp, vp]
    L.tre_debug_trace.argtypes = [vp, vp, ctypes.POINTER(i32)]
    L.tre_step_bytes.argtypes = [vp, i32, i32, ctypes.POINTER(i64)]
    L.tre_plan_inspect.argtypes = [ctypes.POINTER(tre_config), i32, i32,
                                   ctypes.POINTER(tre_plan_info)]
    L.tre_plan_tasks.argtypes = [ctypes.POINTER(tre_config), i32, i32, vp, i32, vp]
    L.tre_plan_tasks.restype = i32
    L.tre_last_error.argtypes = []
    L.tre_last_error.restype = ctypes.c_char_p
    for name in ("tre_create", "tre_decode_step", "tre_decode_step_host",
                 "tre_decode_step_static", "tre_layers_step", "tre_debug_routing",
                 "tre_debug_index", "tre_debug_check", "tre_decode_tokens", "tre_decode_loop", "tre_set_launch_mode", "tre_get_status",
                 "tre_reset", "tre_debug_hidden", "tre_debug_trace", "tre_step_bytes",
                 "tre_plan_inspect"):
        getattr(L, name).restype = ctypes.c_int
    return L


lib = _load()


class TreError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.tre_last_error().decode(errors="replace")
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")


def check(status: int, where: str) -> None:
    if status != TRE_OK:
        raise TreError(status, where)


# ---- same-named thin wrappers ----------------------------------------------------------------
def tre_create(cfg: tre_config, weights: tre_weights, device: int = 0) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    check(lib.tre_create(ctypes.byref(cfg), ctypes.byref(weights), device, ctypes.byref(h)),
          "tre_create")
    return h


def tre_destroy(h) -> None:
    lib.tre_destroy(h)


def tre_decode_step(h, token: int, pos: int, stream: int = 0, logits_dev: int = 0,
                    token_dev: int = 0) -> int:
    return lib.tre_decode_step(h, int(token), int(pos), ctypes.c_void_p(stream or None),
                               ctypes.c_void_p(logits_dev or None), ctypes.c_void_p(token_dev or None))


def tre_decode_step_host(h, token: int, pos: int, stream: int = 0,
                         logits_host: Optional[np.ndarray] = None) -> int:
    tok = ctypes.c_int32()
    lp = None
    if logits_host is not None:
        assert logits_host.dtype == np.float32 and logits_host.flags.c_contiguous
        lp = logits_host.ctypes.data_as(ctypes.c_void_p)
    check(lib.tre_decode_step_host(h, int(token), int(pos), ctypes.c_void_p(stream or None), lp,
                                   ctypes.byref(tok)), "tre_decode_step_host")
    return tok.value


def tre_decode_step_static(cfg: tre_config, weights: tre_weights, token: int, pos: int,
                           stream: int = 0, logits_dev: int = 0, token_dev: int = 0,
                           status_dev: int = 0) -> int:
    """One decode step that allocates no GPU memory (see include/tre.h); returns the status."""
    return lib.tre_decode_step_static(ctypes.byref(cfg), ctypes.byref(weights), int(token),
                                      int(pos), ctypes.c_void_p(stream or None),
                                      ctypes.c_void_p(logits_dev or None),
                                      ctypes.c_void_p(token_dev or None),
                                      ctypes.c_void_p(status_dev or None))


def tre_layers_step(h, x_in_dev: int, x_out_dev: int, pos: int, stream: int = 0) -> int:
    return lib.tre_layers_step(h, ctypes.c_void_p(x_in_dev or None), ctypes.c_void_p(x_out_dev or None),
                               int(pos), ctypes.c_void_p(stream or None))


def tre_debug_routing(h, n_layers: int, top_k: int):
    """(idx int32[L][top_k], w float32[L][top_k]) of the last step of a MoE engine."""
    idx = np.zeros((n_layers, top_k), dtype=np.int32)
    w = np.zeros((n_layers, top_k), dtype=np.float32)
    check(lib.tre_debug_routing(h, idx.ctypes.data_as(ctypes.c_void_p),
                                w.ctypes.data_as(ctypes.c_void_p)), "tre_debug_routing")
    return idx, w


def tre_debug_index(h, layer: int, pos: int, index_topk: int):
    """(scores float32[pos + 1], chosen positions int32[n], unordered) of layer `layer` at
    the last step (position pos) of a sparse MLA engine."""
    sc = np.zeros(pos + 1, dtype=np.float32)
    sel = np.zeros(max(index_topk, pos + 1), dtype=np.int32)
    n = ctypes.c_int32()
    check(lib.tre_debug_index(h, int(layer), int(pos), sc.ctypes.data_as(ctypes.c_void_p),
                              sel.ctypes.data_as(ctypes.c_void_p), ctypes.byref(n)),
          "tre_debug_index")
    return sc, sel[:n.value].copy()


def tre_debug_check(h):
    """(first counter off its per-step invariant or -1, first overwritten guard or -1)."""
    c, g = ctypes.c_int32(), ctypes.c_int32()
    check(lib.tre_debug_check(h, ctypes.byref(c), ctypes.byref(g)), "tre_debug_check")
    return c.value, g.value


def tre_get_status(h):
    st, det = ctypes.c_int32(), ctypes.c_int32()
    check(lib.tre_get_status(h, ctypes.byref(st), ctypes.byref(det)), "tre_get_status")
    return st.value, det.value


def tre_reset(h, stream: int = 0) -> None:
    check(lib.tre_reset(h, ctypes.c_void_p(stream or None)), "tre_reset")


def tre_step_bytes(h, pos: int, m: int = 1) -> int:
    b = ctypes.c_int64()
    check(lib.tre_step_bytes(h, int(pos), int(m), ctypes.byref(b)), "tre_step_bytes")
    return b.value


def tre_decode_tokens(h, tokens, pos: int, stream: int = 0, logits_dev: int = 0,
                      tokens_dev: int = 0) -> int:
    arr = (ctypes.c_int32 * len(tokens))(*[int(t) for t in tokens])
    return lib.tre_decode_tokens(h, arr, len(tokens), int(pos), ctypes.c_void_p(stream or None),
                                 ctypes.c_void_p(logits_dev or None),
                                 ctypes.c_void_p(tokens_dev or None))


def tre_decode_loop(h, token: int, pos: int, n_steps: int, stream: int = 0, tokens_dev: int = 0,
                    logits_dev: int = 0) -> int:
    return lib.tre_decode_loop(h, int(token), int(pos), int(n_steps),
                               ctypes.c_void_p(stream or None), ctypes.c_void_p(tokens_dev or None),
                               ctypes.c_void_p(logits_dev or None))


def tre_set_launch_mode(h, mode: int) -> int:
    """Set the engine's launch mode; returns the kernel launches one step takes."""
    n = ctypes.c_int32()
    check(lib.tre_set_launch_mode(h, int(mode), ctypes.byref(n)), "tre_set_launch_mode")
    return n.value


def tre_plan_op_groups(cfg: tre_config, num_sms: int = 148, smem_per_block: int = 232448):
    """Returns ranges int32[groups][num_sms][2] of the kernel-per-op form."""
    nsm = min(cfg.num_sms, num_sms) if cfg.num_sms else num_sms
    g = lib.tre_plan_op_groups(ctypes.byref(cfg), num_sms, smem_per_block, None, 0)
    if g < 0:
        raise TreError(g, "tre_plan_op_groups")
    out = np.zeros((g, nsm, 2), dtype=np.int32)
    g2 = lib.tre_plan_op_groups(ctypes.byref(cfg), num_sms, smem_per_block,
                                out.ctypes.data_as(ctypes.c_void_p), g)
    assert g2 == g
    return out


def tre_plan_inspect(cfg: tre_config, num_sms: int = 148, smem_per_block: int = 232448):
    info = tre_plan_info()
    check(lib.tre_plan_inspect(ctypes.byref(cfg), num_sms, smem_per_block, ctypes.byref(info)),
          "tre_plan_inspect")
    return info


def tre_plan_tasks(cfg: tre_config, num_sms: int = 148, smem_per_block: int = 232448):
    """Returns (tasks int32[n][8], sm_begin int32[num_sms+1])."""
    nsm = min(cfg.num_sms, num_sms) if cfg.num_sms else num_sms
    begin = np.zeros(nsm + 1, dtype=np.int32)
    n = lib.tre_plan_tasks(ctypes.byref(cfg), num_sms, smem_per_block, None, 0,
                           begin.ctypes.data_as(ctypes.c_void_p))
    if n < 0:
        raise TreError(n, "tre_plan_tasks")
    tasks = np.zeros((n, 8), dtype=np.int32)
    n2 = lib.tre_plan_tasks(ctypes.byref(cfg), num_sms, smem_per_block,
                            tasks.ctypes.data_as(ctypes.c_void_p), n,
                            begin.ctypes.data_as(ctypes.c_void_p))
    assert n2 == n
    return tasks, begin


# ---- convenience ------------------------------------------------------------------------------
def config_from_workload(wl, **overrides) -> tre_config:
    c = tre_config()
    c.kind = {"gqa": TRE_LAYER_GQA, "mla": TRE_LAYER_MLA, "moe": TRE_LAYER_MOE}[wl.kind]
    for f in ("n_layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim", "ffn", "vocab",
              "q_lora", "kv_lora", "rope_dim", "nope_dim", "v_dim", "n_experts", "top_k",
              "n_shared", "expert_ffn", "index_heads", "index_dim", "index_topk"):
        setattr(c, f, int(getattr(wl, f, 0)))
    c.kv_capacity = wl.kv_capacity
    c.max_tokens_per_step = wl.tokens_per_step
    c.rope_theta = wl.rope_theta
    c.norm_eps = wl.norm_eps
    c.has_embed_lm_head = 1 if wl.has_embed_lm_head else 0
    c.weight_format = {"fp8": TRE_WEIGHTS_FP8_BLOCK128, "fp4": TRE_WEIGHTS_FP4_EXPERTS}.get(
        getattr(wl, "weight_format", "bf16"), TRE_WEIGHTS_BF16)
    for k, v in overrides.items():
        setattr(c, k, v)
    return c


def _dev_tensor(words: np.ndarray, device):
    """bf16 words (uint16) as a bf16 tensor; E4M3 bytes (uint8) and fp32 scales as they are."""
    import torch
    a = np.ascontiguousarray(words)
    if a.dtype == np.uint8 or a.dtype == np.float32:
        return torch.from_numpy(a).to(device, non_blocking=False)
    t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    return t.to(device, non_blocking=False)


def upload_gqa_model(model: dict, device="cuda:0") -> dict:
    """Copy a host model (bf16 words) to device tensors; the caller keeps them alive."""
    out = {"layers": [], "k_cache": [], "v_cache": []}
    for l, layer in enumerate(model["layers"]):
        out["layers"].append({slot: _dev_tensor(a, device) for slot, a in layer.items()})
        out["k_cache"].append(_dev_tensor(model["k_cache"][l], device))
        out["v_cache"].append(_dev_tensor(model["v_cache"][l], device))
    for k in ("embed", "final_norm", "lm_head"):
        if k in model:
            out[k] = _dev_tensor(model[k], device)
    return out


def upload_moe_model(wl, model: dict, device="cuda:0", expert_fn=None) -> dict:
    """Copy a host MoE model to device tensors: the non-expert slots as they are, and the
    routed experts of every layer stacked expert-major into slots 10-12 ([E][Fe][d] gate
    and up, [E][d][Fe] down; FP4 workloads: MXFP4 row bytes [E][Fe][pitch(d)] and
    [E][d][pitch(Fe)]).  `expert_fn(layer, e)` returns an expert's host tensors (default: the
    workload's generator, one expert at a time)."""
    import torch
    from .synth import mxfp4_pitch
    from .synth import workloads as W
    expert_fn = expert_fn or (lambda l, e: W.gen_expert(wl, l, e))
    E, Fe, d = wl.n_experts, wl.expert_ffn, wl.hidden
    fp4 = getattr(wl, "weight_format", "bf16") == "fp4"
    out = {"layers": [], "k_cache": [], "v_cache": []}
    for l, layer in enumerate(model["layers"]):
        dev = {slot: _dev_tensor(a, device) for slot, a in layer.items()
               if not (slot in (7, 8, 9) and a.size == 0)}
        if fp4:
            g = torch.empty((E, Fe, mxfp4_pitch(d)), dtype=torch.uint8, device=device)
            u = torch.empty_like(g)
            dn = torch.empty((E, d, mxfp4_pitch(Fe)), dtype=torch.uint8, device=device)
        else:
            g = torch.empty((E, Fe, d), dtype=torch.bfloat16, device=device)
            u = torch.empty((E, Fe, d), dtype=torch.bfloat16, device=device)
            dn = torch.empty((E, d, Fe), dtype=torch.bfloat16, device=device)
        for e in range(E):
            eg, eu, ed = expert_fn(l, e)
            if fp4:
                for dst, a in ((g[e], eg), (u[e], eu), (dn[e], ed)):
                    assert a.dtype == np.uint8 and tuple(a.shape) == tuple(dst.shape)
                    dst.copy_(torch.from_numpy(a))
                continue
            g[e].copy_(torch.from_numpy(eg.view(np.int16)).view(torch.bfloat16))
            u[e].copy_(torch.from_numpy(eu.view(np.int16)).view(torch.bfloat16))
            dn[e].copy_(torch.from_numpy(ed.view(np.int16)).view(torch.bfloat16))
        dev[10], dev[11], dev[12] = g, u, dn
        out["layers"].append(dev)
        out["k_cache"].append(_dev_tensor(model["k_cache"][l], device))
        out["v_cache"].append(_dev_tensor(model["v_cache"][l], device))
    return out


def upload_mla_model(model: dict, device="cuda:0") -> dict:
    """Copy a host absorbed-MLA model (bf16 words) to device tensors: the layer slots as
    they are, each layer's latent cache [capacity][kv_lora + rope] as its k_cache and (sparse
    attention) its index-key cache [capacity][index_dim] as its v_cache."""
    return {"layers": [{slot: _dev_tensor(a, device) for slot, a in layer.items()}
                       for layer in model["layers"]],
            "k_cache": [_dev_tensor(c, device) for c in model["latent_cache"]],
            "v_cache": [_dev_tensor(c, device) for c in model.get("index_cache", [])]}


def make_weights(cfg: tre_config, dev_model: dict):
    """A tre_weights struct over the device tensors of `dev_model`.  Returns (weights,
    keepalive): keep `keepalive` referenced while the struct is in use."""
    L = cfg.n_layers
    layer_w = (ctypes.c_void_p * (L * TRE_W_SLOTS))()
    for l in range(L):
        for slot, t in dev_model["layers"][l].items():
            layer_w[l * TRE_W_SLOTS + slot] = t.data_ptr()
    kc = (ctypes.c_void_p * L)(*[t.data_ptr() for t in dev_model["k_cache"]])
    vc = (ctypes.c_void_p * L)(*[t.data_ptr() for t in dev_model["v_cache"]]) \
        if dev_model.get("v_cache") else None
    w = tre_weights()
    for k in ("embed", "final_norm", "lm_head"):
        if k in dev_model:
            setattr(w, k, dev_model[k].data_ptr())
    w.layer_w = ctypes.cast(layer_w, ctypes.POINTER(ctypes.c_void_p))
    w.k_cache = ctypes.cast(kc, ctypes.POINTER(ctypes.c_void_p))
    if vc is not None:
        w.v_cache = ctypes.cast(vc, ctypes.POINTER(ctypes.c_void_p))
    return w, (layer_w, kc, vc, dev_model)


class Engine:
    """Owns one tre_engine; keeps references to the caller's device tensors."""

    def __init__(self, cfg: tre_config, dev_model: dict, device: int = 0):
        self.cfg = cfg
        self.dev_model = dev_model  # keep the caller-owned memory alive
        L = cfg.n_layers
        self._layer_w = (ctypes.c_void_p * (L * TRE_W_SLOTS))()
        for l in range(L):
            for slot, t in dev_model["layers"][l].items():
                self._layer_w[l * TRE_W_SLOTS + slot] = t.data_ptr()
        self._kc = (ctypes.c_void_p * L)(*[t.data_ptr() for t in dev_model["k_cache"]])
        self._vc = (ctypes.c_void_p * L)(*[t.data_ptr() for t in dev_model["v_cache"]]) \
            if dev_model.get("v_cache") else None
        self.weights = tre_weights()
        for k in ("embed", "final_norm", "lm_head"):
            if k in dev_model:
                setattr(self.weights, k, dev_model[k].data_ptr())
        self.weights.layer_w = ctypes.cast(self._layer_w, ctypes.POINTER(ctypes.c_void_p))
        self.weights.k_cache = ctypes.cast(self._kc, ctypes.POINTER(ctypes.c_void_p))
        if self._vc is not None:
            self.weights.v_cache = ctypes.cast(self._vc, ctypes.POINTER(ctypes.c_void_p))
        self.device = device
        self.h = tre_create(cfg, self.weights, device)

    def close(self):
        if getattr(self, "h", None):
            tre_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def step(self, token: int, pos: int, logits=None, token_out=None, stream=None) -> None:
        """Enqueue one decode step on `stream` (default: torch's current stream)."""
        import torch
        s = stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        check(tre_decode_step(self.h, token, pos, s,
                              logits.data_ptr() if logits is not None else 0,
                              token_out.data_ptr() if token_out is not None else 0),
              "tre_decode_step")

    def step_host(self, token: int, pos: int, logits_host: Optional[np.ndarray] = None,
                  stream=None) -> int:
        import torch
        s = stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        return tre_decode_step_host(self.h, token, pos, s, logits_host)

    def step_tokens(self, tokens, pos: int, logits=None, tokens_out=None, stream=None) -> None:
        """Enqueue one step over len(tokens) consecutive tokens at pos .. pos + m - 1."""
        import torch
        s = stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        check(tre_decode_tokens(self.h, tokens, pos, s,
                                logits.data_ptr() if logits is not None else 0,
                                tokens_out.data_ptr() if tokens_out is not None else 0),
              "tre_decode_tokens")

    def decode_loop(self, token: int, pos: int, n_steps: int, tokens_out, logits=None,
                    stream=None) -> None:
        """Enqueue n_steps greedy steps (each step's argmax feeds the next on the device);
        tokens_out: device int32[n_steps]."""
        import torch
        s = stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        check(tre_decode_loop(self.h, token, pos, n_steps, s, tokens_out.data_ptr(),
                              logits.data_ptr() if logits is not None else 0), "tre_decode_loop")

    def set_launch_mode(self, mode: int) -> int:
        """TRE_LAUNCH_PERSISTENT or TRE_LAUNCH_PER_OP; returns launches per step."""
        return tre_set_launch_mode(self.h, mode)

    def layers_step(self, x_in, x_out, pos: int, stream=None) -> None:
        """Enqueue one layers-only step: x_out = stack(x_in) (device fp32[hidden] tensors)."""
        import torch
        s = stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        check(tre_layers_step(self.h, x_in.data_ptr(), x_out.data_ptr(), pos, s), "tre_layers_step")

    def routing(self):
        return tre_debug_routing(self.h, self.cfg.n_layers, self.cfg.top_k)

    def check(self):
        """Per-step invariants: (bad counter or -1, overwritten guard or -1)."""
        return tre_debug_check(self.h)

    def index(self, layer: int, pos: int):
        """Sparse MLA: (index scores [pos + 1], chosen positions) of `layer` at the last step."""
        return tre_debug_index(self.h, layer, pos, self.cfg.index_topk)

    def status(self):
        return tre_get_status(self.h)

    def reset(self, stream=None):
        import torch
        s = stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        tre_reset(self.h, s)

    def hidden(self, m: int = 1):
        """Residual stream after every layer of the last step: [L][d] (m = 1) or [L][m][d]."""
        import torch
        shape = (self.cfg.n_layers, self.cfg.hidden) if m == 1 else \
            (self.cfg.n_layers, m, self.cfg.hidden)
        out = torch.empty(shape, dtype=torch.float32, device=f"cuda:{self.device}")
        check(lib.tre_debug_hidden(self.h, ctypes.c_void_p(out.data_ptr()),
                                   ctypes.c_void_p(torch.cuda.current_stream(self.device).cuda_stream)),
              "tre_debug_hidden")
        return out

    def trace(self) -> np.ndarray:
        n = ctypes.c_int32()
        check(lib.tre_debug_trace(self.h, None, ctypes.byref(n)), "tre_debug_trace")
        buf = np.zeros((n.value, TRACE_COLS), dtype=np.int64)
        check(lib.tre_debug_trace(self.h, buf.ctypes.data_as(ctypes.c_void_p), ctypes.byref(n)),
              "tre_debug_trace")
        return buf

    def step_bytes(self, pos: int, m: int = 1) -> int:
        return tre_step_bytes(self.h, pos, m)
