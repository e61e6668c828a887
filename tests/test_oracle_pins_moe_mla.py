"""Pins of the oracle's MoE router / experts and absorbed-MLA layer.

Each pin checks the oracle against something other than itself: a library routine
(numpy matmul, stable sort), a special case that reduces to an already-pinned layer, an
invariance, or an independent formulation (the naive, decompressed MLA).
"""
import math

import numpy as np
import torch

import oracle
from persistent_tile_pipelined_b200 import synth
from persistent_tile_pipelined_b200.synth import workloads as W

O64 = oracle.Oracle(64)
rng = np.random.default_rng(1)


def dec(words):
    return synth.bf16_to_f32(np.asarray(words, dtype=np.uint16)).astype(np.float64)


def mat(t):
    return dec(t).reshape(t.shape)


def bf16w(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def rand_bf16(shape, std=1.0):
    return bf16w(rng.normal(0, std, size=shape))


def np_rms(x, g, eps):
    return x / np.sqrt(np.mean(x * x) + eps) * dec(g)


def np_rope(v, pos, theta):
    D = v.size
    z = v[: D // 2] + 1j * v[D // 2:]
    z = z * np.exp(1j * pos * theta ** (-2.0 * np.arange(D // 2) / D))
    return np.concatenate([z.real, z.imag])


# ------------------------------------------------------------------ router ------------

def test_router_scores_are_sigmoid_of_numpy_matmul_and_topk_is_a_stable_sort():
    E, d, k = 37, 48, 8
    wr = rand_bf16((E, d), 0.5)
    hn = rng.normal(0, 1, size=d)
    idx, w, s = O64.router_topk(wr, hn, k)
    np.testing.assert_allclose(s, 1 / (1 + np.exp(-(mat(wr) @ hn))), rtol=1e-13)
    order = np.argsort(-s, kind="stable")
    np.testing.assert_array_equal(idx, order[:k])
    np.testing.assert_allclose(w, s[order[:k]] / s[order[:k]].sum(), rtol=1e-14)
    assert abs(w.sum() - 1) < 1e-14 and (w > 0).all()


def test_router_ties_go_to_the_lower_expert_index():
    E, d = 10, 16
    wr = rand_bf16((E, d), 0.5)
    wr[7] = wr[2]            # experts 2 and 7 score identically
    wr[4] = wr[2]            # and 4
    hn = rng.normal(0, 1, size=d)
    hn = np.sign(mat(wr)[2] @ hn) * hn  # make the tied score high
    idx, _, s = O64.router_topk(wr, hn, 3)
    assert s[2] == s[4] == s[7]
    tied = [i for i in idx if i in (2, 4, 7)]
    assert tied == sorted(tied)


# ------------------------------------------------------------------ experts -----------

def test_swiglu_mlp_matches_numpy():
    d, F = 24, 40
    wg, wu, wd = rand_bf16((F, d), 0.3), rand_bf16((F, d), 0.3), rand_bf16((d, F), 0.3)
    hn = rng.normal(0, 1, size=d)
    g, u = mat(wg) @ hn, mat(wu) @ hn
    ref = mat(wd) @ (g / (1 + np.exp(-g)) * u)
    np.testing.assert_allclose(O64.swiglu_mlp(wg, wu, wd, hn), ref, rtol=1e-12, atol=1e-14)


MOE = W.MOE4.replace(name="moe-pin", n_layers=1, hidden=64, n_q_heads=4, n_kv_heads=2,
                     head_dim=16, prefill=5, decode_steps=1, n_experts=6, top_k=2,
                     n_shared=1, expert_ffn=24, seed=91)


def moe_inputs(wl):
    m = W.gen_moe_model(wl, with_experts=True)
    x = m["x_in"].astype(np.float64)
    return m, x


def test_moe_with_one_expert_and_no_shared_expert_is_the_dense_swiglu_layer():
    wl = MOE.replace(n_experts=1, top_k=1)
    m, x = moe_inputs(wl)
    L = m["layers"][0]
    for t in (L[7], L[8], L[9]):
        t[...] = 0                      # the shared expert contributes nothing
    kc, vc = m["k_cache"][0].copy(), m["v_cache"][0].copy()
    out, idx, w = O64.moe_layer_step(wl, L, kc, vc, lambda e: m["experts"][0][e], wl.prefill, x)
    assert list(idx) == [0] and w[0] == 1.0
    # the same layer through the pinned dense GQA path, the expert as its MLP
    g = W.TINY.replace(n_layers=1, hidden=wl.hidden, n_q_heads=wl.n_q_heads,
                       n_kv_heads=wl.n_kv_heads, head_dim=wl.head_dim, ffn=wl.expert_ffn,
                       vocab=3, prefill=wl.prefill, decode_steps=1,
                       rope_theta=wl.rope_theta, norm_eps=wl.norm_eps)
    ex = m["experts"][0][0]
    dense = {"layers": [{0: L[0], 1: L[1], 2: L[2], 3: L[3], 4: L[4], 5: L[5],
                         6: ex[0], 7: ex[1], 8: ex[2]}],
             "k_cache": [m["k_cache"][0].copy()], "v_cache": [m["v_cache"][0].copy()]}
    ref, _ = O64.layers_step(g, dense, x, wl.prefill)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_moe_with_identical_experts_and_all_selected_is_one_expert():
    wl = MOE.replace(top_k=MOE.n_experts)
    m, x = moe_inputs(wl)
    L = m["layers"][0]
    same = m["experts"][0][3]
    kc, vc = m["k_cache"][0].copy(), m["v_cache"][0].copy()
    out, idx, w = O64.moe_layer_step(wl, L, kc, vc, lambda e: same, wl.prefill, x)
    assert abs(w.sum() - 1) < 1e-14
    kc2, vc2 = m["k_cache"][0].copy(), m["v_cache"][0].copy()
    h1 = O64.gqa_attn_block(wl, L, kc2, vc2, wl.prefill, x)
    hn = O64.rmsnorm(h1, L[5], wl.norm_eps)
    ref = h1 + O64.swiglu_mlp(*same, hn) + O64.swiglu_mlp(L[7], L[8], L[9], hn)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_moe_invariant_under_expert_relabelling():
    wl = MOE
    m, x = moe_inputs(wl)
    L = m["layers"][0]
    perm = rng.permutation(wl.n_experts)          # new label e holds old expert perm[e]
    L2 = dict(L)
    L2[6] = L[6][perm].copy()
    out1, idx1, w1 = O64.moe_layer_step(wl, L, m["k_cache"][0].copy(), m["v_cache"][0].copy(),
                                        lambda e: m["experts"][0][e], wl.prefill, x)
    out2, idx2, w2 = O64.moe_layer_step(wl, L2, m["k_cache"][0].copy(), m["v_cache"][0].copy(),
                                        lambda e: m["experts"][0][perm[e]], wl.prefill, x)
    np.testing.assert_array_equal(perm[idx2], idx1)
    np.testing.assert_allclose(out2, out1, rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------------ absorbed MLA ------

MLA = W.MLA4.replace(name="mla-pin", n_layers=1, hidden=64, n_q_heads=4, q_lora=24,
                     kv_lora=20, rope_dim=8, nope_dim=8, v_dim=12, prefill=5, decode_steps=1,
                     seed=17)


def naive_mla(wl, L, cache, pos, x):
    """Decompressed MLA: per head, keys [W_uk,h c_kv ; k_pe] and values W_uv,h c_kv, then
    ordinary softmax attention — an independent formulation of the absorbed layer."""
    H, KL, R, NP, VD = wl.n_q_heads, wl.kv_lora, wl.rope_dim, wl.nope_dim, wl.v_dim
    eps, th = wl.norm_eps, wl.rope_theta
    xn = np_rms(x, L[0], eps)
    cq = np_rms(mat(L[1]) @ xn, L[2], eps)
    q = (mat(L[3]) @ cq).reshape(H, NP + R)
    kv = mat(L[4]) @ xn
    row = np.concatenate([np_rms(kv[:KL], L[5], eps), np_rope(kv[KL:], pos, th)])
    cache = cache.copy()
    cache[pos] = bf16w(row)
    C = mat(cache[: pos + 1])
    Wuk, Wuv = mat(L[6]), mat(L[7])
    outs = []
    for h in range(H):
        Kh = np.concatenate([C[:, :KL] @ Wuk[h * NP:(h + 1) * NP].T, C[:, KL:]], axis=1)
        Vh = C[:, :KL] @ Wuv[h * VD:(h + 1) * VD].T
        qh = np.concatenate([q[h, :NP], np_rope(q[h, NP:], pos, th)])
        s = Kh @ qh / math.sqrt(NP + R)
        p = np.exp(s - s.max())
        p /= p.sum()
        outs.append(p @ Vh)
    return x + mat(L[8]) @ np.concatenate(outs), cache


def test_absorbed_mla_equals_naive_decompressed_mla():
    wl = MLA
    m = W.gen_mla_model(wl)
    x = m["x_in"].astype(np.float64)
    cache = m["latent_cache"][0].copy()
    out = O64.mla_layer_step(wl, m["layers"][0], cache, wl.prefill, x)
    ref, ref_cache = naive_mla(wl, m["layers"][0], m["latent_cache"][0], wl.prefill, x)
    np.testing.assert_array_equal(cache, ref_cache)       # the appended latent row
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)


def test_mla_at_pos0_is_the_value_path_of_the_new_latent():
    wl = MLA.replace(prefill=0)
    m = W.gen_mla_model(wl)
    x = m["x_in"].astype(np.float64)
    L = m["layers"][0]
    cache = m["latent_cache"][0].copy()
    out = O64.mla_layer_step(wl, L, cache, 0, x)
    c0 = dec(cache[0, : wl.kv_lora])                      # one position: softmax weight 1
    o = np.concatenate([mat(L[7])[h * wl.v_dim:(h + 1) * wl.v_dim] @ c0
                        for h in range(wl.n_q_heads)])
    np.testing.assert_allclose(out, x + mat(L[8]) @ o, rtol=1e-11, atol=1e-12)


def test_mla_invariant_under_head_permutation():
    wl = MLA
    m = W.gen_mla_model(wl)
    x = m["x_in"].astype(np.float64)
    L = m["layers"][0]
    H, NP, R, VD = wl.n_q_heads, wl.nope_dim, wl.rope_dim, wl.v_dim
    perm = rng.permutation(H)
    rows = lambda n: np.concatenate([np.arange(perm[h] * n, (perm[h] + 1) * n) for h in range(H)])
    L2 = dict(L)
    L2[3] = L[3][rows(NP + R)].copy()
    L2[6] = L[6][rows(NP)].copy()
    L2[7] = L[7][rows(VD)].copy()
    L2[8] = L[8][:, rows(VD)].copy()
    a = O64.mla_layer_step(wl, L, m["latent_cache"][0].copy(), wl.prefill, x)
    b = O64.mla_layer_step(wl, L2, m["latent_cache"][0].copy(), wl.prefill, x)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)
