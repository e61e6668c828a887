"""Pins of the CPU oracle against things other than itself.

The pages print no worked numbers for the decode math, so every pin here is a closed
form, an invariant, a library routine or a brute force on tiny inputs, chosen so that a
plausible slip (a dropped term, a wrong sign or index, a transposed operand, a wrong
head mapping) fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from persistent_tile_pipelined_b200 import synth
from persistent_tile_pipelined_b200.synth import workloads as W

O64 = oracle.Oracle(64)
O32 = oracle.Oracle(32)
rng = np.random.default_rng(0)


def dec(words):
    return synth.bf16_to_f32(np.asarray(words, dtype=np.uint16)).astype(np.float64)


def torch_bf16_words(x):
    t = torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def rand_bf16(shape, std=1.0):
    return torch_bf16_words(rng.normal(0, std, size=shape))


# ---------------------------------------------------------------- bf16 storage ------

def test_bf16_special_values():
    assert O64.round_bf16(1.0) == 0x3F80
    assert O64.round_bf16(-2.0) == 0xC000
    assert O64.round_bf16(0.0) == 0x0000
    # 1 + 2^-8 is halfway between 1 (even mantissa) and 1 + 2^-7: ties go to even
    assert O64.round_bf16(1.0 + 2.0 ** -8) == 0x3F80
    # 1 + 3*2^-8 is halfway between 1+2^-7 (odd) and 1+2^-6 (even)
    assert O64.round_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82
    assert O64.bf16_to_real(0x3F80) == 1.0
    assert O64.bf16_to_real(0xC000) == -2.0
    assert O64.bf16_to_real(0x0001) == 2.0 ** -133


def test_bf16_rounding_matches_torch_on_float32_inputs():
    x = rng.normal(0, 3, size=4000).astype(np.float32)
    # add exact ties: low 16 bits = 0x8000
    ties = (rng.integers(0x3000, 0x4F00, size=1000).astype(np.uint32) << 16) | 0x8000
    x = np.concatenate([x, ties.view(np.float32), -ties.view(np.float32)])
    ref = torch_bf16_words(x)
    for o in (O64, O32):
        got = np.array([o.round_bf16(float(v)) for v in x], dtype=np.uint16)
        np.testing.assert_array_equal(got, ref)


def test_bf16_rounding_is_nearest_neighbour_for_doubles():
    for v in rng.normal(0, 10, size=2000):
        w = O64.round_bf16(float(v))
        r = O64.bf16_to_real(w)
        # the neighbours one bf16 step either side are no closer
        for nb in (w - 1, w + 1):
            assert abs(O64.bf16_to_real(nb & 0xFFFF) - v) >= abs(r - v)


# ---------------------------------------------------------------- RMSNorm -----------

def test_rmsnorm_unit_rms_and_gain():
    x = rng.normal(0, 5, size=300)
    g = rand_bf16(300, 0.3)
    out = O64.rmsnorm(x, g, 0.0)
    assert abs(np.sqrt(np.mean((out / dec(g)) ** 2)) - 1.0) < 1e-12
    # eps enters under the square root
    eps = 0.7
    out = O64.rmsnorm(x, g, eps)
    ms = np.mean(x ** 2)
    assert abs(np.sqrt(np.mean((out / dec(g)) ** 2)) - math.sqrt(ms / (ms + eps))) < 1e-12
    # scale invariance with eps = 0
    np.testing.assert_allclose(O64.rmsnorm(3.5 * x, g, 0.0), O64.rmsnorm(x, g, 0.0), rtol=1e-12)


def test_rmsnorm_brute_force():
    x = [0.5, -1.25, 2.0, 3.0, -0.125, 7.0, 1.0]
    g = rand_bf16(7, 1.0)
    gd = dec(g)
    ms = sum(v * v for v in x) / 7 + 1e-5
    expect = [x[i] / math.sqrt(ms) * gd[i] for i in range(7)]
    np.testing.assert_allclose(O64.rmsnorm(x, g, 1e-5), expect, rtol=1e-14)


# ---------------------------------------------------------------- matrix-vector -----

@pytest.mark.parametrize("N,K", [(1, 8), (37, 51), (64, 256), (5, 1000)])
def test_gemv_matches_numpy_matmul(N, K):
    Wm = rand_bf16((N, K), 0.5)
    x = rng.normal(0, 1, size=K)
    ref = dec(Wm).reshape(N, K) @ x
    np.testing.assert_allclose(O64.gemv(Wm, x), ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(O32.gemv(Wm, x), ref, rtol=2e-4, atol=1e-4)


def test_gemv_transposed_operand_would_fail():
    # a non-square, non-symmetric case where W^T x has a different length: the
    # row-major [N][K] convention is the one that matches numpy's W @ x
    Wm = rand_bf16((3, 5), 1.0)
    x = rng.normal(0, 1, size=5)
    y = O64.gemv(Wm, x)
    assert y.shape == (3,)
    np.testing.assert_allclose(y, dec(Wm).reshape(3, 5) @ x, rtol=1e-13)


# ---------------------------------------------------------------- RoPE --------------

def test_rope_identity_at_pos0_and_norm_preserved():
    v = rng.normal(0, 1, size=128)
    np.testing.assert_array_equal(O64.rope(v, 0, 5e5), v)
    r = O64.rope(v, 777, 5e5)
    h = 64
    np.testing.assert_allclose(np.hypot(r[:h], r[h:]), np.hypot(v[:h], v[h:]), rtol=1e-13)


def test_rope_complex_form():
    # the pair (v_i, v_{i+D/2}) as the complex number v_i + j v_{i+D/2}, multiplied by
    # exp(j * pos * theta^(-2i/D))
    D, pos, theta = 64, 4099, 1e4
    v = rng.normal(0, 1, size=D)
    z = v[: D // 2] + 1j * v[D // 2:]
    i = np.arange(D // 2)
    z = z * np.exp(1j * pos * theta ** (-2.0 * i / D))
    np.testing.assert_allclose(O64.rope(v, pos, theta), np.concatenate([z.real, z.imag]),
                               rtol=1e-9, atol=1e-12)
    # D = 2: theta_0 = 1, so position p rotates (1, 0) by p radians
    np.testing.assert_allclose(O64.rope([1.0, 0.0], 1, 1e4), [math.cos(1), math.sin(1)],
                               rtol=1e-15)


def test_rope_scores_depend_on_relative_position_only():
    D, theta = 128, 5e5
    q, k = rng.normal(0, 1, size=D), rng.normal(0, 1, size=D)
    for m, n, s in ((10, 3, 100), (4096, 17, 5), (0, 0, 31)):
        a = O64.rope(q, m, theta) @ O64.rope(k, n, theta)
        b = O64.rope(q, m + s, theta) @ O64.rope(k, n + s, theta)
        assert abs(a - b) < 1e-9 * (1 + abs(a))


# ---------------------------------------------------------------- attention ---------

def naive_attention(q, kc, vc, P):
    """Pure-Python loops, fp64 (brute force)."""
    Hq, D = q.shape
    Hkv = kc.shape[0]
    G = Hq // Hkv
    K, V = dec(kc).reshape(kc.shape), dec(vc).reshape(vc.shape)
    out = np.zeros((Hq, D))
    for h in range(Hq):
        g = h // G
        s = [sum(q[h, d] * K[g, t, d] for d in range(D)) / math.sqrt(D) for t in range(P)]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        tot = sum(e)
        for d in range(D):
            out[h, d] = sum(e[t] / tot * V[g, t, d] for t in range(P))
    return out


def test_attention_brute_force():
    Hq, Hkv, D, cap, P = 4, 2, 8, 7, 5
    q = rng.normal(0, 1, size=(Hq, D))
    kc, vc = rand_bf16((Hkv, cap, D)), rand_bf16((Hkv, cap, D))
    np.testing.assert_allclose(O64.attention(q, kc, vc, P), naive_attention(q, kc, vc, P),
                               rtol=1e-12, atol=1e-13)


def test_attention_single_position_returns_v():
    Hq, Hkv, D, cap = 8, 2, 16, 4
    q = rng.normal(0, 3, size=(Hq, D))
    kc, vc = rand_bf16((Hkv, cap, D)), rand_bf16((Hkv, cap, D))
    out = O64.attention(q, kc, vc, 1)
    V = dec(vc).reshape(vc.shape)
    for h in range(Hq):
        np.testing.assert_array_equal(out[h], V[h // 4, 0])   # q head h reads kv head h/G


def test_attention_mha_head_mapping():
    Hq = Hkv = 3
    D, cap = 8, 2
    q = rng.normal(0, 1, size=(Hq, D))
    kc, vc = rand_bf16((Hkv, cap, D)), rand_bf16((Hkv, cap, D))
    out = O64.attention(q, kc, vc, 1)
    np.testing.assert_array_equal(out, dec(vc).reshape(vc.shape)[:, 0])


def test_attention_equal_keys_give_mean_of_v_and_probs_sum_to_one():
    Hq, Hkv, D, cap, P = 4, 1, 16, 9, 9
    q = rng.normal(0, 1, size=(Hq, D))
    krow = rand_bf16(D)
    kc = np.broadcast_to(krow, (Hkv, cap, D)).copy()
    vc = rand_bf16((Hkv, cap, D))
    out, p = O64.attention(q, kc, vc, P, want_probs=True)
    np.testing.assert_allclose(out, np.broadcast_to(dec(vc).reshape(vc.shape)[0].mean(0),
                                                    (Hq, D)), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(p, 1.0 / P, rtol=1e-12)
    kc = rand_bf16((Hkv, cap, D), 2.0)
    _, p = O64.attention(q, kc, vc, P, want_probs=True)
    assert (p >= 0).all()
    np.testing.assert_allclose(p.sum(1), 1.0, rtol=1e-14)


def test_attention_dominant_key_selects_its_value():
    Hq, Hkv, D, cap, P = 2, 1, 8, 6, 6
    q = np.zeros((Hq, D))
    q[:, 0] = 50.0
    kc = np.zeros((Hkv, cap, D), dtype=np.uint16)
    kc[0, 3, 0] = O64.round_bf16(8.0)          # score 50*8/sqrt(8) = 141 vs 0 elsewhere
    vc = rand_bf16((Hkv, cap, D))
    out = O64.attention(q, kc, vc, P)
    np.testing.assert_allclose(out[0], dec(vc).reshape(vc.shape)[0, 3], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- SiLU / argmax -----

def test_silu_special_values():
    assert O64.silu(0.0) == 0.0
    assert abs(O64.silu(40.0) - 40.0) < 1e-14
    assert abs(O64.silu(-40.0)) < 1e-15
    assert abs(O64.silu(1.0) - 0.7310585786300049) < 1e-15     # 1 / (1 + e^-1)
    assert abs(O64.silu(-1.0) + 0.2689414213699951) < 1e-15    # -1 / (1 + e)


def test_argmax_lowest_index_on_ties():
    assert O64.argmax([1.0, 3.0, 3.0, 2.0]) == 1
    assert O64.argmax([-1.0]) == 0
    assert O64.argmax([0.0, 0.0]) == 0


# ---------------------------------------------------------------- the decode step ---

SMALL = W.TINY.replace(name="pin", n_layers=2, hidden=64, n_q_heads=4, n_kv_heads=2,
                       head_dim=16, ffn=40, vocab=50, prefill=6, decode_steps=2, seed=77)


def np_rms(x, g, eps):
    return x / np.sqrt(np.mean(x * x) + eps) * dec(g)


def np_rope(v, pos, theta):
    D = v.size
    z = v[: D // 2] + 1j * v[D // 2:]
    z = z * np.exp(1j * pos * theta ** (-2.0 * np.arange(D // 2) / D))
    return np.concatenate([z.real, z.imag])


def mat(t):
    return dec(t).reshape(t.shape)


def fresh_model(wl=SMALL, **zero):
    m = W.gen_gqa_model(wl)
    for slot in zero.get("zero_slots", ()):
        for l in range(wl.n_layers):
            m["layers"][l][slot][...] = 0
    return m


def test_step_with_zero_wo_and_wdown_is_embedding_passthrough():
    wl = SMALL
    m = fresh_model(zero_slots=(4, 8))
    tok, pos = 13, wl.prefill
    logits, hidden = O64.decode_step(wl, m, tok, pos)
    x = mat(m["embed"])[tok]
    for l in range(wl.n_layers):
        np.testing.assert_array_equal(hidden[l], x)
    ref = mat(m["lm_head"]) @ np_rms(x, m["final_norm"], wl.norm_eps)
    np.testing.assert_allclose(logits, ref, rtol=1e-12, atol=1e-14)
    # the appended cache rows: bf16(RoPE(Wk xn)) and bf16(Wv xn), per kv head
    for l in range(wl.n_layers):
        Lw = m["layers"][l]
        xn = np_rms(x, Lw[0], wl.norm_eps)
        k = (mat(Lw[2]) @ xn).reshape(wl.n_kv_heads, wl.head_dim)
        v = (mat(Lw[3]) @ xn).reshape(wl.n_kv_heads, wl.head_dim)
        for g in range(wl.n_kv_heads):
            kr = np_rope(k[g], pos, wl.rope_theta)
            np.testing.assert_array_equal(m["k_cache"][l][g, pos], torch_bf16_words(kr))
            np.testing.assert_array_equal(m["v_cache"][l][g, pos], torch_bf16_words(v[g]))


def test_step_at_pos0_with_zero_wdown_is_closed_form():
    # one cached position: attention returns that position's v, so the layer is
    # h1 = x + Wo [v_{h/G} for each q head]
    wl = SMALL.replace(prefill=0)
    m = fresh_model(wl, zero_slots=(8,))
    tok = 7
    logits, hidden = O64.decode_step(wl, m, tok, 0)
    x = mat(m["embed"])[tok]
    G = wl.n_q_heads // wl.n_kv_heads
    for l in range(wl.n_layers):
        Lw = m["layers"][l]
        xn = np_rms(x, Lw[0], wl.norm_eps)
        v = dec(torch_bf16_words(mat(Lw[3]) @ xn)).reshape(wl.n_kv_heads, wl.head_dim)
        o = np.concatenate([v[h // G] for h in range(wl.n_q_heads)])
        x = x + mat(Lw[4]) @ o
        np.testing.assert_allclose(hidden[l], x, rtol=1e-12, atol=1e-13)
    ref = mat(m["lm_head"]) @ np_rms(x, m["final_norm"], wl.norm_eps)
    np.testing.assert_allclose(logits, ref, rtol=1e-11, atol=1e-13)


def test_step_with_zero_wo_is_swiglu_closed_form():
    wl = SMALL
    m = fresh_model(zero_slots=(4,))
    tok, pos = 3, wl.prefill
    _, hidden = O64.decode_step(wl, m, tok, pos)
    x = mat(m["embed"])[tok]
    for l in range(wl.n_layers):
        Lw = m["layers"][l]
        hn = np_rms(x, Lw[5], wl.norm_eps)
        gt, up = mat(Lw[6]) @ hn, mat(Lw[7]) @ hn
        x = x + mat(Lw[8]) @ (gt / (1 + np.exp(-gt)) * up)
        np.testing.assert_allclose(hidden[l], x, rtol=1e-12, atol=1e-13)


def test_step_invariant_under_mlp_hidden_unit_permutation():
    wl = SMALL
    m1, m2 = fresh_model(), fresh_model()
    for l in range(wl.n_layers):
        perm = rng.permutation(wl.ffn)
        L2 = m2["layers"][l]
        L2[6][...] = L2[6][perm]
        L2[7][...] = L2[7][perm]
        L2[8][...] = L2[8][:, perm]
    a, _ = O64.decode_step(wl, m1, 5, wl.prefill)
    b, _ = O64.decode_step(wl, m2, 5, wl.prefill)
    np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-13)


def test_step_invariant_under_kv_group_permutation():
    # relabel kv head g -> perm[g] together with its group of q heads (rows of Wq),
    # its Wk / Wv rows, its cache, and the matching columns of Wo
    wl = SMALL
    Hq, Hkv, D = wl.n_q_heads, wl.n_kv_heads, wl.head_dim
    G = Hq // Hkv
    m1, m2 = fresh_model(), fresh_model()
    for l in range(wl.n_layers):
        perm = rng.permutation(Hkv)
        qrows = np.concatenate([np.arange(perm[g] * G * D, (perm[g] + 1) * G * D)
                                for g in range(Hkv)])
        kvrows = np.concatenate([np.arange(perm[g] * D, (perm[g] + 1) * D) for g in range(Hkv)])
        L2 = m2["layers"][l]
        L2[1][...] = L2[1][qrows]
        L2[2][...] = L2[2][kvrows]
        L2[3][...] = L2[3][kvrows]
        L2[4][...] = L2[4][:, qrows]
        m2["k_cache"][l][...] = m2["k_cache"][l][perm]
        m2["v_cache"][l][...] = m2["v_cache"][l][perm]
    a, _ = O64.decode_step(wl, m1, 9, wl.prefill)
    b, _ = O64.decode_step(wl, m2, 9, wl.prefill)
    np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-13)


def test_step_writes_only_position_pos_of_the_caches():
    wl = SMALL
    m = fresh_model()
    before = [(k.copy(), v.copy()) for k, v in zip(m["k_cache"], m["v_cache"])]
    pos = wl.prefill
    O64.decode_step(wl, m, 11, pos)
    for l, (k0, v0) in enumerate(before):
        mask = np.ones(wl.kv_capacity, bool)
        mask[pos] = False
        np.testing.assert_array_equal(m["k_cache"][l][:, mask], k0[:, mask])
        np.testing.assert_array_equal(m["v_cache"][l][:, mask], v0[:, mask])
        assert (m["k_cache"][l][:, pos] != k0[:, pos]).any()


def test_fp32_stack_agrees_with_fp64_stack_on_tiny():
    wl = W.TINY
    m64, m32 = W.gen_gqa_model(wl), W.gen_gqa_model(wl)
    tok = W.first_token(wl)
    a, ha = O64.decode_step(wl, m64, tok, wl.prefill)
    b, hb = O32.decode_step(wl, m32, tok, wl.prefill)
    assert np.abs(a - b).max() <= 1e-5 * np.abs(a).max()
    assert np.abs(ha - hb).max() <= 1e-5 * np.abs(ha).max()
