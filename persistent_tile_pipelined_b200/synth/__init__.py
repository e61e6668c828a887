"""Seeded synthetic inputs shared by the GPU engine's uploads and the CPU oracle.

The numbers come from one counter-based generator written in C (``gen.c``: SplitMix64
stream per (seed, tensor id) + Box-Muller, rounded to bf16 by round-to-nearest-even),
so both sides consume bit-identical bf16 words.  This module holds none of the decode
arithmetic.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libtre_synth.so")
_LIB = None


def _lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        if not os.path.exists(_LIB_PATH):
            from .. import build as _build  # compile on first use (gcc, seconds)

            _build.build_synth()
        lib = ctypes.CDLL(_LIB_PATH)
        u64, i64, dbl = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double
        for name in ("synth_normal_f64", "synth_normal_f32", "synth_normal_bf16"):
            fn = getattr(lib, name)
            fn.argtypes = [u64, u64, i64, dbl, dbl, ctypes.c_void_p]
            fn.restype = None
        lib.synth_u64.argtypes = [u64, u64, u64]
        lib.synth_u64.restype = u64
        lib.synth_e4m3_blocks.argtypes = [u64, u64, i64, i64, dbl, ctypes.c_void_p,
                                          ctypes.c_void_p]
        lib.synth_e4m3_blocks.restype = None
        lib.synth_mxfp4_rows.argtypes = [u64, u64, i64, i64, i64, ctypes.c_int32,
                                         ctypes.c_void_p]
        lib.synth_mxfp4_rows.restype = None
        _LIB = lib
    return _LIB


def _fill(name: str, dtype, seed: int, tensor_id: int, shape, mean: float, std: float,
          out: np.ndarray | None = None) -> np.ndarray:
    shape = tuple(int(s) for s in (shape if isinstance(shape, (tuple, list)) else (shape,)))
    n = int(np.prod(shape)) if shape else 1
    if out is None:
        out = np.empty(shape, dtype=dtype)
    else:
        assert out.dtype == dtype and out.size == n and out.flags.c_contiguous
    if n:
        getattr(_lib(), name)(seed, tensor_id, n, float(mean), float(std),
                              out.ctypes.data_as(ctypes.c_void_p))
    return out


def normal_bf16(seed: int, tensor_id: int, shape, mean: float = 0.0, std: float = 1.0,
                out: np.ndarray | None = None) -> np.ndarray:
    """bf16 words (uint16) of mean + std * N(0,1), rounded to nearest even."""
    return _fill("synth_normal_bf16", np.uint16, seed, tensor_id, shape, mean, std, out)


def normal_f32(seed: int, tensor_id: int, shape, mean: float = 0.0, std: float = 1.0,
               out: np.ndarray | None = None) -> np.ndarray:
    return _fill("synth_normal_f32", np.float32, seed, tensor_id, shape, mean, std, out)


def normal_f64(seed: int, tensor_id: int, shape, mean: float = 0.0, std: float = 1.0,
               out: np.ndarray | None = None) -> np.ndarray:
    return _fill("synth_normal_f64", np.float64, seed, tensor_id, shape, mean, std, out)


def e4m3_blocks(seed: int, tensor_id: int, shape, std: float):
    """A block-scaled FP8 matrix [N][K] of values std * N(0,1) (the same stream as
    normal_f64 with mean 0): E4M3 bytes (uint8) and fp32 scales [ceil(N/128)][ceil(K/128)],
    each scale = block max |value| / 448, each byte the nearest E4M3 of value / scale."""
    N, K = (int(s) for s in shape)
    codes = np.empty((N, K), dtype=np.uint8)
    scales = np.empty(((N + 127) // 128, (K + 127) // 128), dtype=np.float32)
    if N and K:
        _lib().synth_e4m3_blocks(seed, tensor_id, N, K, float(std),
                                 codes.ctypes.data_as(ctypes.c_void_p),
                                 scales.ctypes.data_as(ctypes.c_void_p))
    return codes, scales


def mxfp4_pitch(K: int) -> int:
    """Bytes per stored MXFP4 row of K elements: K/2 code bytes and K/32 scale bytes,
    padded to a multiple of 16."""
    return (K // 2 + K // 32 + 15) // 16 * 16


def mxfp4_rows(seed: int, tensor_id: int, N: int, K: int, scale_lo: int = 119) -> np.ndarray:
    """[N][mxfp4_pitch(K)] bytes of random MXFP4 rows (K a multiple of 32): uniform random
    E2M1 code bytes, then K/32 scale exponents scale_lo or scale_lo + 1, then zero padding."""
    N, K = int(N), int(K)
    assert K % 32 == 0
    out = np.empty((N, mxfp4_pitch(K)), dtype=np.uint8)
    if N and K:
        _lib().synth_mxfp4_rows(seed, tensor_id, N, K, out.shape[1], int(scale_lo),
                                out.ctypes.data_as(ctypes.c_void_p))
    return out


def u64(seed: int, tensor_id: int, index: int) -> int:
    return int(_lib().synth_u64(seed, tensor_id, index))


def token_id(seed: int, vocab: int, index: int = 0) -> int:
    """A seed-fixed token id in [0, vocab)."""
    return u64(seed, TID_TOKEN, index) % int(vocab)


# Tensor ids: fixed, so every tensor of every workload has its own stream.
TID_EMBED, TID_FINAL_NORM, TID_LM_HEAD, TID_X_IN, TID_TOKEN = 1, 2, 3, 4, 5


def tid_layer(layer: int, slot: int) -> int:
    return (int(layer) + 1) * 256 + int(slot)


def tid_kcache(layer: int) -> int:
    return tid_layer(layer, 200)


def tid_vcache(layer: int) -> int:
    return tid_layer(layer, 201)


def bf16_to_f32(words: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 words to float32 (a bit shift)."""
    return (words.astype(np.uint32) << 16).view(np.float32)
