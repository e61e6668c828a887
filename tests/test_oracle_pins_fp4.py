"""Pins of the oracle's FP4-expert path (MXFP4 rows: E2M1 codes, one E8M0 scale per 32
weights) against things other than itself: the OCP Microscaling formats' value tables,
a hand-made row whose every nibble and scale is known, a numpy matrix product on the
decoded matrix, and the bf16 MoE layer on weights equal to the decoded FP4 experts."""
import math

import numpy as np
import pytest

import oracle
from persistent_tile_pipelined_b200 import synth
from persistent_tile_pipelined_b200.synth import workloads as W

O64 = oracle.Oracle(64)
O32 = oracle.Oracle(32)

# The OCP Microscaling spec's FP4 E2M1 value table: codes 0-7 positive, 8-15 their negatives.
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_decoding_matches_the_format_table():
    for o in (O64, O32):
        for c in range(16):
            v = o.e2m1_to_real(c)
            assert v == (-1 if c >= 8 else 1) * E2M1_TABLE[c & 7]
            assert math.copysign(1.0, v) == (-1.0 if c >= 8 else 1.0)  # code 8 is -0
        # only the low nibble counts
        assert o.e2m1_to_real(0xF3) == o.e2m1_to_real(0x03) == 1.5


def test_e8m0_closed_values():
    for o in (O64,):
        assert o.e8m0_to_real(127) == 1.0 and o.e8m0_to_real(128) == 2.0
        assert o.e8m0_to_real(120) == 2.0 ** -7 and o.e8m0_to_real(254) == 2.0 ** 127
        assert o.e8m0_to_real(0) == 2.0 ** -127
        assert math.isnan(o.e8m0_to_real(255))


def test_pitch_covers_codes_and_scales():
    for K in (32, 64, 96, 512, 2048, 7168):
        p = O64.mxfp4_pitch(K)
        assert p == synth.mxfp4_pitch(K) and p % 16 == 0 and K // 2 + K // 32 <= p < K // 2 + K // 32 + 16
    assert O64.mxfp4_pitch(7168) == 3808 and O64.mxfp4_pitch(2048) == 1088


def test_hand_made_row_fixes_nibble_order_and_scale_blocks():
    """Row of K = 64: byte 0 = 0x21 holds element 0 (low nibble, code 1 = 0.5) and element 1
    (high nibble, code 2 = 1.0); byte 16 = 0xF7 holds element 32 (code 7 = 6) and element 33
    (code 15 = -6); scales: block 0 = 2^0, block 1 = 2^3."""
    K = 64
    row = np.zeros((1, O64.mxfp4_pitch(K)), dtype=np.uint8)
    row[0, 0] = 0x21
    row[0, 16] = 0xF7
    row[0, K // 2] = 127
    row[0, K // 2 + 1] = 130
    want = np.zeros(K)
    want[0], want[1], want[32], want[33] = 0.5, 1.0, 48.0, -48.0
    for k in range(K):
        x = np.zeros(K)
        x[k] = 1.0
        assert O64.gemv_mxfp4(row, K, x)[0] == want[k], k


def decode_rows(rows, K):
    """Dense [N][K] values of MXFP4 rows, from the table above (numpy, vectorised)."""
    codes = rows[:, : K // 2]
    nib = np.stack([codes & 15, codes >> 4], axis=-1).reshape(rows.shape[0], K)
    table = np.array(E2M1_TABLE + [-v for v in E2M1_TABLE])
    scale = np.ldexp(1.0, rows[:, K // 2: K // 2 + K // 32].astype(np.int64) - 127)
    return table[nib] * np.repeat(scale, 32, axis=1)


@pytest.mark.parametrize("N,K", [(5, 32), (17, 96), (40, 512)])
def test_gemv_mxfp4_matches_numpy_on_the_decoded_matrix(N, K):
    rng = np.random.default_rng(N * K)
    rows = synth.mxfp4_rows(7, 99, N, K)
    rows[:, K // 2: K // 2 + K // 32] = rng.integers(100, 140, size=(N, K // 32))
    x = rng.standard_normal(K)
    np.testing.assert_allclose(O64.gemv_mxfp4(rows, K, x), decode_rows(rows, K) @ x,
                               rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(O32.gemv_mxfp4(rows, K, x), decode_rows(rows, K) @ x,
                               rtol=1e-4, atol=1e-6)


def test_generator_rows_hold_random_codes_scales_and_zero_padding():
    K = 96
    rows = synth.mxfp4_rows(3, 5, 64, K)
    assert rows.shape == (64, synth.mxfp4_pitch(K))
    sc = rows[:, K // 2: K // 2 + K // 32]
    assert set(np.unique(sc).tolist()) == {119, 120}
    assert not rows[:, K // 2 + K // 32:].any()
    nib = np.concatenate([rows[:, : K // 2] & 15, rows[:, : K // 2] >> 4]).ravel()
    assert len(np.unique(nib)) == 16  # every code occurs
    np.testing.assert_array_equal(rows, synth.mxfp4_rows(3, 5, 64, K))  # seeded


def bf16_words(values):
    """bf16 words of values that bf16 holds exactly (asserted)."""
    f = np.asarray(values, dtype=np.float32)
    w = (f.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal((w.astype(np.uint32) << 16).view(np.float32), f)
    return w


def test_fp4_moe_layer_equals_the_bf16_layer_on_the_decoded_experts():
    """The MoE layer with FP4 routed experts gives the same bits as the bf16 MoE layer whose
    routed experts hold the decoded FP4 values (E2M1 x 2^-8 / 2^-7 is exact in bf16), so the
    FP4 composition (gate, up, down rows and their widths) is the pinned bf16 one."""
    wl4 = W.MOE4.replace(name="moe-fp4-pin", n_layers=1, hidden=256, n_q_heads=4, n_kv_heads=2,
                         head_dim=64, prefill=9, decode_steps=1, n_experts=6, top_k=2,
                         n_shared=1, expert_ffn=96, weight_format="fp4", seed=77)
    wlb = wl4.replace(weight_format="bf16")
    model = W.gen_moe_model(wl4)
    ex4 = {e: W.gen_expert(wl4, 0, e) for e in range(wl4.n_experts)}
    d, F = wl4.hidden, wl4.expert_ffn
    exb = {e: (bf16_words(decode_rows(g, d)), bf16_words(decode_rows(u, d)),
               bf16_words(decode_rows(dn, F))) for e, (g, u, dn) in ex4.items()}
    x = model["x_in"].astype(np.float64)
    outs = []
    for wl, ex in ((wl4, ex4), (wlb, exb)):
        kc, vc = model["k_cache"][0].copy(), model["v_cache"][0].copy()
        outs.append(O64.moe_layer_step(wl, model["layers"][0], kc, vc, lambda e: ex[e],
                                       wl.prefill, x))
    (y4, i4, w4), (yb, ib, wb) = outs
    np.testing.assert_array_equal(i4, ib)
    np.testing.assert_array_equal(y4, yb)
    # and the experts matter: another expert's rows change the output
    kc, vc = model["k_cache"][0].copy(), model["v_cache"][0].copy()
    y_other, _, _ = O64.moe_layer_step(wl4, model["layers"][0], kc, vc,
                                       lambda e: ex4[(e + 1) % wl4.n_experts], wl4.prefill, x)
    assert not np.array_equal(y_other, y4)
