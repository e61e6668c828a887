"""CPU ORACLE of the batch-1 decode step — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package.  The product (``persistent_tile_pipelined_b200``) never imports it,
and it imports nothing from the product except the seeded input generator's recipes
(which hold no decode arithmetic).

``oracle.c`` is the plain definition of a decoder step (see its header for the readings
of the pages and for the pins).  This module only marshals numpy arrays through ctypes.
Every function here is pinned by ``tests/test_oracle_pins.py``; nothing is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")


def lib_path(bits: int) -> str:
    return os.path.join(_HERE, f"liboracle{bits}.so")


def build(force: bool = False) -> None:
    """Compile oracle.c twice (fp64 and fp32 `real`) with gcc + OpenMP."""
    for bits, real in ((64, "double"), (32, "float")):
        out = lib_path(bits)
        if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(_SRC):
            subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                                   f"-DORC_REAL={real}", _SRC, "-o", out, "-lm"])


class _GqaConfig(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("hidden", ctypes.c_int32),
                ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("ffn", ctypes.c_int32),
                ("vocab", ctypes.c_int32), ("kv_capacity", ctypes.c_int32),
                ("rope_theta", ctypes.c_double), ("norm_eps", ctypes.c_double),
                ("weight_fp8", ctypes.c_int32)]


class _GqaLayer(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "wgate", "wup", "wdown",
                 "k_cache", "v_cache", "sq", "sk", "sv", "so", "sgate", "sup", "sdown")]


_SLOT_NAMES = ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "wgate", "wup", "wdown")
# FP8 layers: the block scales of the seven projection matrices sit in slots 9 .. 15
_SCALE_SLOTS = {"sq": 9, "sk": 10, "sv": 11, "so": 12, "sgate": 13, "sup": 14, "sdown": 15}


class _MlaConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("hidden", "n_heads", "q_lora", "kv_lora",
                                               "rope_dim", "nope_dim", "v_dim", "kv_capacity")] + [
        ("rope_theta", ctypes.c_double), ("norm_eps", ctypes.c_double)] + [
        (n, ctypes.c_int32) for n in ("index_heads", "index_dim", "index_topk")]


class _MlaLayer(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("attn_norm", "w_dq", "q_norm", "w_uq", "w_dkv", "kv_norm", "w_uk", "w_uv", "w_o",
                 "latent_cache", "w_iq", "w_ik", "index_cache")]


def _ptr(a: np.ndarray) -> ctypes.c_void_p:
    assert a.flags.c_contiguous, "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """The oracle at one precision: bits=64 (parity reference) or bits=32."""

    def __init__(self, bits: int = 64):
        assert bits in (32, 64)
        build()
        self.bits = bits
        self.real = np.float64 if bits == 64 else np.float32
        self.lib = ctypes.CDLL(lib_path(bits))
        L = self.lib
        vp, i32, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        creal = ctypes.c_double if bits == 64 else ctypes.c_float
        L.orc_real_bytes.restype = ctypes.c_int
        assert L.orc_real_bytes() == bits // 8
        L.orc_bf16_to_real.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_real.restype = creal
        L.orc_e4m3_to_real.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_to_real.restype = creal
        L.orc_gemv_fp8.argtypes = [i32, i32, vp, vp, vp, vp]
        L.orc_e2m1_to_real.argtypes = [ctypes.c_uint8]
        L.orc_e2m1_to_real.restype = creal
        L.orc_e8m0_to_real.argtypes = [ctypes.c_uint8]
        L.orc_e8m0_to_real.restype = creal
        L.orc_mxfp4_pitch.argtypes = [i32]
        L.orc_mxfp4_pitch.restype = i32
        L.orc_gemv_mxfp4.argtypes = [i32, i32, vp, vp, vp]
        L.orc_swiglu_mlp_mxfp4.argtypes = [i32, i32, vp, vp, vp, vp, vp]
        L.orc_round_bf16.argtypes = [creal]
        L.orc_round_bf16.restype = ctypes.c_uint16
        L.orc_rmsnorm.argtypes = [i32, vp, vp, dbl, vp]
        L.orc_gemv.argtypes = [i32, i32, vp, vp, vp]
        L.orc_rope.argtypes = [i32, i32, dbl, vp]
        L.orc_silu.argtypes = [creal]
        L.orc_silu.restype = creal
        L.orc_attention.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, vp, vp]
        L.orc_argmax.argtypes = [i32, vp]
        L.orc_argmax.restype = i32
        L.orc_gqa_layer_step.argtypes = [vp, vp, i32, vp]
        L.orc_gqa_layers_step.argtypes = [vp, vp, i32, vp, vp]
        L.orc_decode_step.argtypes = [vp, vp, vp, vp, vp, i32, i32, vp, vp]
        L.orc_gqa_attn_block.argtypes = [vp, vp, i32, vp, vp]
        L.orc_swiglu_mlp.argtypes = [i32, i32, vp, vp, vp, vp, vp]
        L.orc_router_topk.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp]
        L.orc_mla_layer_step.argtypes = [vp, vp, i32, vp]
        L.orc_mla_layer_step_ex.argtypes = [vp, vp, i32, vp, vp, i32, vp, vp]
        L.orc_index_select.argtypes = [i32, i32, vp, vp]
        L.orc_index_select.restype = i32

    # -- pieces ------------------------------------------------------------------
    def _r(self, a) -> np.ndarray:
        return np.ascontiguousarray(a, dtype=self.real)

    def round_bf16(self, v: float) -> int:
        return int(self.lib.orc_round_bf16(v))

    def bf16_to_real(self, w: int) -> float:
        return float(self.lib.orc_bf16_to_real(w))

    def e4m3_to_real(self, b: int) -> float:
        return float(self.lib.orc_e4m3_to_real(b))

    def gemv_fp8(self, W_e4m3, S, x):
        """y = (e4m3(W) * S[n / 128][k / 128]) x for W [N][K] bytes, S fp32 block scales."""
        W = np.ascontiguousarray(W_e4m3, dtype=np.uint8)
        S = np.ascontiguousarray(S, dtype=np.float32)
        x = self._r(x)
        N, K = W.shape
        assert x.size == K and S.shape == ((N + 127) // 128, (K + 127) // 128)
        y = np.empty(N, dtype=self.real)
        self.lib.orc_gemv_fp8(N, K, _ptr(W), _ptr(S), _ptr(x), _ptr(y))
        return y

    def e2m1_to_real(self, c: int) -> float:
        return float(self.lib.orc_e2m1_to_real(c))

    def e8m0_to_real(self, s: int) -> float:
        return float(self.lib.orc_e8m0_to_real(s))

    def mxfp4_pitch(self, K: int) -> int:
        return int(self.lib.orc_mxfp4_pitch(K))

    def gemv_mxfp4(self, W_rows, K: int, x):
        """y = W x for W [N][K] as MXFP4 rows (uint8 [N][mxfp4_pitch(K)])."""
        W = np.ascontiguousarray(W_rows, dtype=np.uint8)
        x = self._r(x)
        N = W.shape[0]
        assert x.size == K and W.shape[1] == self.mxfp4_pitch(K)
        y = np.empty(N, dtype=self.real)
        self.lib.orc_gemv_mxfp4(N, K, _ptr(W), _ptr(x), _ptr(y))
        return y

    def swiglu_mlp_mxfp4(self, wgate, wup, wdown, hn):
        """SwiGLU of one FP4 expert: gate / up [F][pitch(d)], down [d][pitch(F)] rows."""
        wg, wu, wd = (np.ascontiguousarray(a, dtype=np.uint8) for a in (wgate, wup, wdown))
        F, d = wg.shape[0], wd.shape[0]
        assert wg.shape == wu.shape == (F, self.mxfp4_pitch(d))
        assert wd.shape == (d, self.mxfp4_pitch(F))
        hn = self._r(hn)
        y = np.empty(d, dtype=self.real)
        self.lib.orc_swiglu_mlp_mxfp4(d, F, _ptr(wg), _ptr(wu), _ptr(wd), _ptr(hn), _ptr(y))
        return y

    def rmsnorm(self, x, g_bf16, eps):
        x = self._r(x)
        g = np.ascontiguousarray(g_bf16, dtype=np.uint16)
        out = np.empty_like(x)
        self.lib.orc_rmsnorm(x.size, _ptr(x), _ptr(g), float(eps), _ptr(out))
        return out

    def gemv(self, W_bf16, x):
        W = np.ascontiguousarray(W_bf16, dtype=np.uint16)
        x = self._r(x)
        N, K = W.shape
        assert x.size == K
        y = np.empty(N, dtype=self.real)
        self.lib.orc_gemv(N, K, _ptr(W), _ptr(x), _ptr(y))
        return y

    def rope(self, v, pos, theta):
        v = self._r(v).copy()
        self.lib.orc_rope(v.size, int(pos), float(theta), _ptr(v))
        return v

    def silu(self, z: float) -> float:
        return float(self.lib.orc_silu(z))

    def attention(self, q, k_cache, v_cache, P, want_probs=False):
        """q [Hq][D]; caches [Hkv][cap][D] bf16 words; attends positions [0, P)."""
        q = self._r(q)
        kc = np.ascontiguousarray(k_cache, dtype=np.uint16)
        vc = np.ascontiguousarray(v_cache, dtype=np.uint16)
        Hq, D = q.shape
        Hkv, cap, D2 = kc.shape
        assert D2 == D and vc.shape == kc.shape and 0 <= P <= cap
        out = np.empty((Hq, D), dtype=self.real)
        probs = np.empty((Hq, max(P, 1)), dtype=self.real) if want_probs else None
        self.lib.orc_attention(Hq, Hkv, D, int(P), cap, _ptr(q), _ptr(kc), _ptr(vc), _ptr(out),
                               _ptr(probs) if probs is not None else None)
        return (out, probs[:, :P]) if want_probs else out

    def argmax(self, v) -> int:
        v = self._r(v)
        return int(self.lib.orc_argmax(v.size, _ptr(v)))

    # -- the stack ---------------------------------------------------------------
    def _gqa_structs(self, wl, model):
        fp8 = getattr(wl, "weight_format", "bf16") == "fp8"
        cfg = _GqaConfig(wl.n_layers, wl.hidden, wl.n_q_heads, wl.n_kv_heads, wl.head_dim,
                         wl.ffn, wl.vocab, wl.kv_capacity, float(wl.rope_theta),
                         float(wl.norm_eps), 1 if fp8 else 0)
        layers = (_GqaLayer * wl.n_layers)()
        for l in range(wl.n_layers):
            t = model["layers"][l]
            for slot, name in enumerate(_SLOT_NAMES):
                setattr(layers[l], name, _ptr(t[slot]).value)
            if fp8:
                for name, slot in _SCALE_SLOTS.items():
                    setattr(layers[l], name, _ptr(t[slot]).value)
            layers[l].k_cache = _ptr(model["k_cache"][l]).value
            layers[l].v_cache = _ptr(model["v_cache"][l]).value
        return cfg, layers

    def decode_step(self, wl, model, token: int, pos: int, want_hidden: bool = True):
        """One decode step; writes this token's k, v into model's caches at pos.
        Returns (logits[V], hidden[L][d] or None)."""
        cfg, layers = self._gqa_structs(wl, model)
        logits = np.empty(wl.vocab, dtype=self.real)
        hidden = np.empty((wl.n_layers, wl.hidden), dtype=self.real) if want_hidden else None
        self.lib.orc_decode_step(ctypes.byref(cfg), _ptr(model["embed"]),
                                 _ptr(model["final_norm"]), _ptr(model["lm_head"]), layers,
                                 int(token), int(pos), _ptr(logits),
                                 _ptr(hidden) if hidden is not None else None)
        return logits, hidden

    def swiglu_mlp(self, wgate, wup, wdown, hn):
        wg, wu, wd = (np.ascontiguousarray(a, dtype=np.uint16) for a in (wgate, wup, wdown))
        F, d = wg.shape
        assert wu.shape == (F, d) and wd.shape == (d, F)
        hn = self._r(hn)
        y = np.empty(d, dtype=self.real)
        self.lib.orc_swiglu_mlp(d, F, _ptr(wg), _ptr(wu), _ptr(wd), _ptr(hn), _ptr(y))
        return y

    def router_topk(self, wr, hn, top_k: int):
        """(idx[top_k], w[top_k], scores[E]) of the sigmoid top-k router."""
        wr = np.ascontiguousarray(wr, dtype=np.uint16)
        E, d = wr.shape
        hn = self._r(hn)
        idx = np.empty(top_k, dtype=np.int32)
        w = np.empty(top_k, dtype=self.real)
        sc = np.empty(E, dtype=self.real)
        self.lib.orc_router_topk(E, int(top_k), d, _ptr(wr), _ptr(hn), _ptr(idx), _ptr(w), _ptr(sc))
        return idx, w, sc

    def gqa_attn_block(self, wl, layer: dict, k_cache, v_cache, pos: int, x):
        """h1 = x + Wo attention(RMSNorm(x)); appends this token's k, v to the caches."""
        cfg = _GqaConfig(1, wl.hidden, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.ffn,
                         wl.vocab, wl.kv_capacity, float(wl.rope_theta), float(wl.norm_eps))
        L = _GqaLayer()
        for slot, name in enumerate(_SLOT_NAMES[:5]):
            setattr(L, name, _ptr(layer[slot]).value)
        L.k_cache = _ptr(k_cache).value
        L.v_cache = _ptr(v_cache).value
        x = self._r(x)
        h1 = np.empty_like(x)
        self.lib.orc_gqa_attn_block(ctypes.byref(cfg), ctypes.byref(L), int(pos), _ptr(x), _ptr(h1))
        return h1

    def moe_layer_step(self, wl, layer: dict, k_cache, v_cache, experts, pos: int, x,
                       want_scores: bool = False):
        """One MoE decoder layer: the GQA attention block, then
        x = h1 + sum_i w_i Expert_{idx_i}(hn) + Shared(hn), hn = RMSNorm(h1).
        `experts(e)` returns routed expert e's (W_gate, W_up, W_down): bf16 words, or MXFP4
        rows when the workload's weight_format is "fp4".
        Returns (x_out, idx, w), and the router's scores of all experts when want_scores."""
        h1 = self.gqa_attn_block(wl, layer, k_cache, v_cache, pos, x)
        hn = self.rmsnorm(h1, layer[5], wl.norm_eps)
        idx, w, scores = self.router_topk(layer[6], hn, wl.top_k)
        y = np.zeros(wl.hidden, dtype=self.real)
        mlp = self.swiglu_mlp_mxfp4 if getattr(wl, "weight_format", "bf16") == "fp4" \
            else self.swiglu_mlp
        for i, e in enumerate(idx):
            y += w[i] * mlp(*experts(int(e)), hn)
        y += self.swiglu_mlp(layer[7], layer[8], layer[9], hn)
        if want_scores:
            return h1 + y, idx, w, scores
        return h1 + y, idx, w

    def index_select(self, scores, k: int):
        """The k positions of largest score (ties to the lower position), increasing."""
        sc = self._r(scores)
        out = np.empty(max(1, min(k, sc.size)), dtype=np.int32)
        n = self.lib.orc_index_select(sc.size, int(k), _ptr(sc), _ptr(out))
        return out[:n]

    def mla_layer_step(self, wl, layer: dict, latent_cache, pos: int, x, index_cache=None,
                       sel=None, want_index: bool = False):
        """One absorbed-MLA layer (attention only); appends this token's latent row (and, with
        the sparse indexer, its index key).  sel (positions, increasing) overrides the
        indexer's choice.  want_index: also return (index scores [pos + 1], chosen positions)."""
        topk = getattr(wl, "index_topk", 0)
        cfg = _MlaConfig(wl.hidden, wl.n_q_heads, wl.q_lora, wl.kv_lora, wl.rope_dim,
                         wl.nope_dim, wl.v_dim, wl.kv_capacity, float(wl.rope_theta),
                         float(wl.norm_eps), getattr(wl, "index_heads", 0),
                         getattr(wl, "index_dim", 0), topk)
        L = _MlaLayer()
        for slot, name in enumerate(("attn_norm", "w_dq", "q_norm", "w_uq", "w_dkv", "kv_norm",
                                     "w_uk", "w_uv", "w_o")):
            setattr(L, name, _ptr(layer[slot]).value)
        L.latent_cache = _ptr(latent_cache).value
        P = pos + 1
        iscore = np.empty(P, dtype=self.real)
        chosen = np.empty(max(1, min(P, topk)) if topk else 1, dtype=np.int32)
        sel_arr = None
        if topk:
            assert index_cache is not None
            L.w_iq = _ptr(layer[9]).value
            L.w_ik = _ptr(layer[10]).value
            L.index_cache = _ptr(index_cache).value
            if sel is not None:
                sel_arr = np.ascontiguousarray(sel, dtype=np.int32)
        x = self._r(x).copy()
        self.lib.orc_mla_layer_step_ex(ctypes.byref(cfg), ctypes.byref(L), int(pos), _ptr(x),
                                       _ptr(sel_arr) if sel_arr is not None else None,
                                       int(sel_arr.size) if sel_arr is not None else 0,
                                       _ptr(iscore) if topk else None,
                                       _ptr(chosen) if topk else None)
        if want_index:
            return x, (iscore if topk else None), (chosen[:min(P, topk)] if topk else None)
        return x

    def layers_step(self, wl, model, x, pos: int):
        """Layers only: returns (x_out[d], hidden[L][d])."""
        cfg, layers = self._gqa_structs(wl, model)
        x = self._r(x).copy()
        hidden = np.empty((wl.n_layers, wl.hidden), dtype=self.real)
        self.lib.orc_gqa_layers_step(ctypes.byref(cfg), layers, int(pos), _ptr(x), _ptr(hidden))
        return x, hidden
