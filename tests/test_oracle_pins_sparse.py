"""Pins of the oracle's sparse-attention indexer and sparse absorbed MLA against things
other than itself: the index scores by an independent numpy formulation, the selection by a
stable sort, the sparse layer by the naive decompressed MLA restricted to the chosen
positions, and the reductions to the dense layer."""
import math

import numpy as np
import pytest

import oracle
from persistent_tile_pipelined_b200.synth import workloads as W

from test_oracle_pins_moe_mla import dec, mat, bf16w, np_rms, np_rope  # noqa: E402

O64 = oracle.Oracle(64)
O32 = oracle.Oracle(32)
rng = np.random.default_rng(5)

SP = W.MLA4.replace(name="mla-sparse-tiny", n_layers=1, hidden=256, n_q_heads=16, q_lora=64,
                    kv_lora=128, rope_dim=64, nope_dim=32, v_dim=32, prefill=300,
                    decode_steps=2, index_heads=4, index_dim=32, index_topk=48, seed=91)


def naive_index_scores(wl, L, icache, pos, x):
    """I[t] = sum_j w_j / sqrt(H_I) relu(q_j . k_t / sqrt(D_I)), written with numpy on the
    layer's tensors (k_t read back from the bf16 cache, this position's key rounded)."""
    HI, DI = wl.index_heads, wl.index_dim
    xn = np_rms(x, L[0], wl.norm_eps)
    cq = np_rms(mat(L[1]) @ xn, L[2], wl.norm_eps)
    kw = mat(L[10]) @ xn
    qi = (mat(L[9]) @ cq).reshape(HI, DI)
    ic = icache.copy()
    ic[pos] = bf16w(kw[:DI])
    K = mat(ic[: pos + 1])                                   # [P][DI]
    dots = np.maximum(qi @ K.T / math.sqrt(DI), 0.0)       # [HI][P]
    return (kw[DI:] / math.sqrt(HI)) @ dots, ic


def naive_sparse_mla(wl, L, cache, pos, x, sel):
    """The decompressed MLA (per head keys [W_uk c_kv ; k_pe], values W_uv c_kv) with the
    softmax over the positions in sel only."""
    H, KL, R, NP, VD = wl.n_q_heads, wl.kv_lora, wl.rope_dim, wl.nope_dim, wl.v_dim
    eps, th = wl.norm_eps, wl.rope_theta
    xn = np_rms(x, L[0], eps)
    cq = np_rms(mat(L[1]) @ xn, L[2], eps)
    q = (mat(L[3]) @ cq).reshape(H, NP + R)
    kv = mat(L[4]) @ xn
    row = np.concatenate([np_rms(kv[:KL], L[5], eps), np_rope(kv[KL:], pos, th)])
    cache = cache.copy()
    cache[pos] = bf16w(row)
    C = mat(cache[np.asarray(sel)])
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
    return x + mat(L[8]) @ np.concatenate(outs)


def model(wl):
    m = W.gen_mla_model(wl)
    return m, m["layers"][0], m["x_in"].astype(np.float64)


def test_index_scores_match_numpy_and_the_key_is_appended():
    wl = SP
    m, L, x = model(wl)
    ic = m["index_cache"][0].copy()
    _, isc, _ = O64.mla_layer_step(wl, L, m["latent_cache"][0].copy(), wl.prefill, x,
                                   index_cache=ic, want_index=True)
    ref, ref_ic = naive_index_scores(wl, L, m["index_cache"][0], wl.prefill, x)
    np.testing.assert_array_equal(ic, ref_ic)
    np.testing.assert_allclose(isc, ref, rtol=1e-11, atol=1e-12 * np.abs(ref).max())


def test_selection_is_the_top_k_of_a_stable_sort():
    for P, k in [(300, 48), (1000, 1000), (50, 64), (4096, 2048)]:
        sc = rng.normal(size=P).round(1)  # many exact ties: the lower position wins
        got = O64.index_select(sc, k)
        order = np.lexsort((np.arange(P), -sc))[: min(k, P)]
        np.testing.assert_array_equal(got, np.sort(order))


def test_sparse_layer_equals_naive_mla_over_the_chosen_positions():
    wl = SP
    m, L, x = model(wl)
    ic = m["index_cache"][0].copy()
    cache = m["latent_cache"][0].copy()
    out, isc, sel = O64.mla_layer_step(wl, L, cache, wl.prefill, x, index_cache=ic,
                                       want_index=True)
    assert sel.size == wl.index_topk and np.all(np.diff(sel) > 0)
    ref = naive_sparse_mla(wl, L, m["latent_cache"][0], wl.prefill, x, sel)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)
    # the chosen positions are the top-k of the scores
    np.testing.assert_array_equal(sel, np.sort(np.lexsort((np.arange(sc := isc.size), -isc))[:wl.index_topk]))
    # an explicit choice overrides the indexer's
    alt = np.arange(0, wl.prefill + 1, 7, dtype=np.int32)
    out2 = O64.mla_layer_step(wl, L, m["latent_cache"][0].copy(), wl.prefill, x,
                              index_cache=m["index_cache"][0].copy(), sel=alt)
    np.testing.assert_allclose(out2, naive_sparse_mla(wl, L, m["latent_cache"][0], wl.prefill, x, alt),
                               rtol=1e-11, atol=1e-12)


def test_sparse_with_k_at_least_the_length_is_the_dense_layer():
    wl = SP.replace(index_topk=400)  # 301 positions <= 400
    m, L, x = model(wl)
    a = O64.mla_layer_step(wl, L, m["latent_cache"][0].copy(), wl.prefill, x,
                           index_cache=m["index_cache"][0].copy())
    dense = SP.replace(index_topk=0, index_heads=0, index_dim=0)
    b = O64.mla_layer_step(dense, L, m["latent_cache"][0].copy(), wl.prefill, x)
    np.testing.assert_array_equal(a, b)


def test_a_key_aligned_with_every_query_is_chosen():
    """A cached index key equal to a large multiple of the direction every index query
    agrees with (head weights all positive) scores highest and is kept."""
    wl = SP
    m, L, x = model(wl)
    L = dict(L)
    DI, HI = wl.index_dim, wl.index_heads
    ik = mat(L[10])
    ik[DI:] = np.abs(ik[DI:]) + 0.01          # positive head weights for this x ...
    xn = np_rms(x, L[0], wl.norm_eps)
    ik[DI:] *= np.sign(ik[DI:] @ xn)[:, None]  # ... made positive in sign
    L[10] = bf16w(ik)
    cq = np_rms(mat(L[1]) @ xn, L[2], wl.norm_eps)
    qi = (mat(L[9]) @ cq).reshape(HI, DI)
    ic = m["index_cache"][0].copy()
    t = 123
    ic[t] = bf16w(40.0 * qi.sum(axis=0) / np.linalg.norm(qi.sum(axis=0)))
    _, isc, sel = O64.mla_layer_step(wl, L, m["latent_cache"][0].copy(), wl.prefill, x,
                                     index_cache=ic, want_index=True)
    assert int(np.argmax(isc)) == t and t in sel


def test_fp32_and_fp64_sparse_layers_agree():
    wl = SP
    m, L, x = model(wl)
    a, _, s64 = O64.mla_layer_step(wl, L, m["latent_cache"][0].copy(), wl.prefill, x,
                                   index_cache=m["index_cache"][0].copy(), want_index=True)
    b = O32.mla_layer_step(wl, L, m["latent_cache"][0].copy(), wl.prefill, x,
                           index_cache=m["index_cache"][0].copy(), sel=s64)
    assert np.abs(a - b).max() <= 1e-5 * np.abs(a).max()
