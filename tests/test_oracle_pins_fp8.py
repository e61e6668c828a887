"""Pins of the oracle's FP8 (E4M3, 128 x 128 block scales) weight path, and of the
generator's block quantiser, against things other than themselves: torch's float8_e4m3fn
conversion, the format's closed values, a numpy matrix product on the decoded matrix, and
the bf16 decode step on a model whose bf16 weights equal the FP8 weights exactly."""
import math

import numpy as np
import pytest
import torch

import oracle
from persistent_tile_pipelined_b200 import synth
from persistent_tile_pipelined_b200.synth import workloads as W

O64 = oracle.Oracle(64)
O32 = oracle.Oracle(32)
rng = np.random.default_rng(8)


def torch_e4m3_values(codes):
    t = torch.from_numpy(np.asarray(codes, dtype=np.uint8).copy()).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def test_e4m3_decoding_of_every_byte_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch_e4m3_values(codes)
    for o in (O64, O32):
        got = np.array([o.e4m3_to_real(int(b)) for b in codes])
        nan = np.isnan(ref)
        assert (np.isnan(got) == nan).all() and nan.sum() == 2  # S.1111.111
        np.testing.assert_array_equal(got[~nan], ref[~nan])


def test_e4m3_closed_values():
    v = O64.e4m3_to_real
    assert v(0x38) == 1.0 and v(0x40) == 2.0 and v(0xB8) == -1.0
    assert v(0x7E) == 448.0 and v(0xFE) == -448.0        # largest finite
    assert v(0x01) == 2.0 ** -9 and v(0x07) == 7 * 2.0 ** -9  # subnormals
    assert v(0x08) == 2.0 ** -6                           # smallest normal
    assert v(0x3C) == 1.5 and v(0x00) == 0.0
    assert math.copysign(1.0, v(0x80)) == -1.0 and v(0x80) == 0.0


@pytest.mark.parametrize("N,K", [(1, 8), (130, 264), (256, 128), (77, 1000)])
def test_fp8_gemv_matches_numpy_on_the_decoded_matrix(N, K):
    codes = rng.integers(0, 256, size=(N, K), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3C  # no NaN codes
    S = rng.uniform(0.5, 2.0, size=((N + 127) // 128, (K + 127) // 128)).astype(np.float32)
    x = rng.normal(size=K)
    Wd = torch_e4m3_values(codes) * np.repeat(np.repeat(S.astype(np.float64), 128, 0), 128, 1)[:N, :K]
    ref = Wd @ x
    got = O64.gemv_fp8(codes, S, x)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(Wd).sum(axis=1).max())
    got32 = O32.gemv_fp8(codes, S, x)
    np.testing.assert_allclose(got32, ref, rtol=2e-5, atol=2e-5 * np.abs(ref).max())


def test_fp8_gemv_block_index():
    """One nonzero block scale at a time: the output moves with the ROW block and the
    input with the COLUMN block (a transposed scale index fails)."""
    N, K = 300, 260
    codes = np.full((N, K), 0x38, dtype=np.uint8)  # all 1.0
    x = np.zeros(K)
    x[200] = 1.0                                   # column block 1
    for nb, kb in ((2, 1), (0, 1), (1, 0)):
        S = np.zeros((3, 3), dtype=np.float32)
        S[nb, kb] = 4.0
        y = O64.gemv_fp8(codes, S, x)
        expect = np.zeros(N)
        if kb == 1:
            expect[nb * 128:min(N, nb * 128 + 128)] = 4.0
        np.testing.assert_array_equal(y, expect)


def test_generator_block_quantiser_matches_torch():
    """The FP8 workload's weights: per 128 x 128 block, scale = max |w| / 448 (fp32) and
    bytes = torch's E4M3 rounding of w / scale; every block's largest entry maps to 448."""
    N, K = 300, 260
    codes, S = synth.e4m3_blocks(5, 77, (N, K), 0.02)
    w = synth.normal_f64(5, 77, (N, K), 0.0, 0.02)
    for nb in range(3):
        for kb in range(3):
            blk = w[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            assert S[nb, kb] == np.float32(np.abs(blk).max() / 448.0)
    Sx = np.repeat(np.repeat(S.astype(np.float64), 128, 0), 128, 1)[:N, :K]
    ref = torch.from_numpy(np.clip(w / Sx, -448, 448)).to(torch.float8_e4m3fn)
    np.testing.assert_array_equal(codes, ref.view(torch.uint8).numpy())
    assert (np.abs(torch_e4m3_values(codes)).max() == 448.0)


def fp8_tiny_model(wl, scale_fn):
    """A tiny FP8 model with chosen block scales, and the bf16 model whose weights equal
    its dequantised weights exactly (E4M3 values times powers of two are bf16 numbers)."""
    m8 = W.gen_gqa_model(wl)
    mb = {k: v for k, v in m8.items()}
    mb["layers"] = []
    for layer in m8["layers"]:
        lb = dict(layer)
        for slot, sslot in W.FP8_SCALE_SLOT.items():
            codes = layer[slot]
            S = scale_fn(layer[sslot].shape, slot).astype(np.float32)
            layer[sslot] = S
            deq = torch_e4m3_values(codes) * np.repeat(np.repeat(S.astype(np.float64), 128, 0),
                                                       128, 1)[:codes.shape[0], :codes.shape[1]]
            t = torch.from_numpy(deq.astype(np.float32)).to(torch.bfloat16)
            assert (t.to(torch.float64).numpy() == deq).all()  # exactly representable
            lb[slot] = t.view(torch.int16).numpy().view(np.uint16)
            del lb[sslot]
        mb["layers"].append(lb)
    mb["k_cache"] = [c.copy() for c in m8["k_cache"]]
    mb["v_cache"] = [c.copy() for c in m8["v_cache"]]
    return m8, mb


@pytest.mark.parametrize("scales", ["ones", "pow2"])
def test_fp8_decode_step_equals_bf16_step_on_equal_weights(scales):
    """The FP8 decode step (every projection through the block-scaled path) gives the same
    logits, hidden states and appended K / V bits as the bf16 step on the exactly equal
    bf16 weights.  pow2: block (nb, kb) of projection slot s scaled by
    2^((3 nb + kb + s) % 5 - 2), so a wrong block index or another matrix's scales change
    the result."""
    wl = W.TINY.replace(weight_format="fp8", n_layers=2)
    if scales == "ones":
        fn = lambda shape, slot: np.ones(shape)  # noqa: E731
    else:
        def fn(shape, slot):
            nb, kb = np.arange(shape[0])[:, None], np.arange(shape[1])[None, :]
            return np.exp2((3 * nb + kb + slot) % 5 - 2)
    m8, mb = fp8_tiny_model(wl, fn)
    tok, pos = W.first_token(wl), wl.prefill
    l8, h8 = O64.decode_step(wl, m8, tok, pos)
    lb, hb = O64.decode_step(wl.replace(weight_format="bf16"), mb, tok, pos)
    np.testing.assert_array_equal(l8, lb)
    np.testing.assert_array_equal(h8, hb)
    for l in range(wl.n_layers):
        np.testing.assert_array_equal(m8["k_cache"][l], mb["k_cache"][l])
        np.testing.assert_array_equal(m8["v_cache"][l], mb["v_cache"][l])
