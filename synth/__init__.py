"""Seeded synthetic inputs for the GQA forward (Python side of ``synth.c``).

This module is the only code shared by the fp64 oracle's tests and the CUDA
path's tests and benchmark.  It draws numbers and rounds them; it computes no
part of attention.  Every tensor is a pure function of (seed, stream, flat
index), so a slice of a very large tensor (one batch entry, one kv head) can be
generated on its own and matches the same slice of the full tensor bit for bit.

Streams: 0 = Q, 1 = K, 2 = V, 3 = mask lengths / random mask.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")

STREAM_Q, STREAM_K, STREAM_V, STREAM_MASK = 0, 1, 2, 3

_lib = None


def build(force: bool = False) -> str:
    """Compile ``synth.c`` into ``libsynth.so`` next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        u64, i64 = ctypes.c_uint64, ctypes.c_int64
        vp = ctypes.c_void_p
        lib.synth_stream_key.argtypes = [u64, u64]
        lib.synth_stream_key.restype = u64
        lib.synth_u64.argtypes = [u64, u64]
        lib.synth_u64.restype = u64
        lib.synth_normal_f32.argtypes = [u64, u64, u64, i64, vp]
        lib.synth_normal_bf16.argtypes = [u64, u64, u64, i64, vp]
        lib.synth_round_bf16.argtypes = [vp, i64, vp]
        lib.synth_bf16_to_f64.argtypes = [vp, i64, vp]
        lib.synth_uniform_int.argtypes = [u64, u64, i64, i64, i64, vp]
        lib.synth_mask_lengths.argtypes = [vp, i64, i64, i64, vp]
        lib.synth_mask_random.argtypes = [u64, u64, i64, i64, i64, ctypes.c_double, vp]
        for f in ("synth_normal_f32", "synth_normal_bf16", "synth_round_bf16",
                  "synth_bf16_to_f64", "synth_uniform_int", "synth_mask_lengths",
                  "synth_mask_random"):
            getattr(lib, f).restype = None
        _lib = lib
    return _lib


def splitmix64_at(key: int, i: int) -> int:
    """i-th output of the SplitMix64 stream seeded with ``key``."""
    return int(_load().synth_u64(key, i))


def stream_key(seed: int, stream: int) -> int:
    return int(_load().synth_stream_key(seed, stream))


def normal_f32(seed: int, stream: int, count: int, offset: int = 0) -> np.ndarray:
    """N(0,1) float32 values, elements [offset, offset+count) of the stream."""
    out = np.empty(count, dtype=np.float32)
    _load().synth_normal_f32(seed, stream, offset, count, out.ctypes.data)
    return out


def normal_bf16_bits(seed: int, stream: int, count: int, offset: int = 0) -> np.ndarray:
    """N(0,1) values rounded to bf16, as uint16 bit patterns."""
    out = np.empty(count, dtype=np.uint16)
    _load().synth_normal_bf16(seed, stream, offset, count, out.ctypes.data)
    return out


def normal_bf16_into(seed: int, stream: int, ptr: int, count: int, offset: int = 0) -> None:
    """Write N(0,1) bf16 bit patterns straight into host memory at ``ptr``."""
    _load().synth_normal_bf16(seed, stream, offset, count, ptr)


def round_bf16_bits(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().synth_round_bf16(x.ctypes.data, x.size, out.ctypes.data)
    return out


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, dtype=np.float64)
    _load().synth_bf16_to_f64(bits.ctypes.data, bits.size, out.ctypes.data)
    return out


def uniform_int(seed: int, stream: int, n: int, lo: int, hi: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int64)
    _load().synth_uniform_int(seed, stream, n, lo, hi, out.ctypes.data)
    return out


def mask_from_lengths(lengths: np.ndarray, Sq: int, Sk: int) -> np.ndarray:
    """Right-padding mask ``mask[b, i, j] = j < len[b]`` as uint8 [B, Sq, Sk]."""
    lengths = np.ascontiguousarray(lengths, dtype=np.int64)
    B = lengths.shape[0]
    out = np.empty((B, Sq, Sk), dtype=np.uint8)
    _load().synth_mask_lengths(lengths.ctypes.data, B, Sq, Sk, out.ctypes.data)
    return out


def mask_random(seed: int, B: int, Sq: int, Sk: int, p_true: float,
                stream: int = STREAM_MASK) -> np.ndarray:
    """Bernoulli(p_true) uint8 mask [B, Sq, Sk] with at least one true per row."""
    out = np.empty((B, Sq, Sk), dtype=np.uint8)
    _load().synth_mask_random(seed, stream, B, Sq, Sk, p_true, out.ctypes.data)
    return out


def qkv_bf16_bits(seed: int, B: int, Hq: int, Hkv: int, Sq: int, Sk: int, D: int):
    """Q [B,Hq,Sq,D], K and V [B,Hkv,Sk,D] as bf16 bit patterns (uint16)."""
    q = normal_bf16_bits(seed, STREAM_Q, B * Hq * Sq * D).reshape(B, Hq, Sq, D)
    k = normal_bf16_bits(seed, STREAM_K, B * Hkv * Sk * D).reshape(B, Hkv, Sk, D)
    v = normal_bf16_bits(seed, STREAM_V, B * Hkv * Sk * D).reshape(B, Hkv, Sk, D)
    return q, k, v


def qkv_f32(seed: int, B: int, Hq: int, Hkv: int, Sq: int, Sk: int, D: int):
    """Q, K, V as float32 N(0,1) values (same streams as the bf16 variant)."""
    q = normal_f32(seed, STREAM_Q, B * Hq * Sq * D).reshape(B, Hq, Sq, D)
    k = normal_f32(seed, STREAM_K, B * Hkv * Sk * D).reshape(B, Hkv, Sk, D)
    v = normal_f32(seed, STREAM_V, B * Hkv * Sk * D).reshape(B, Hkv, Sk, D)
    return q, k, v


def kv_slice_bf16_bits(seed: int, stream: int, B: int, H: int, S: int, D: int,
                       b: int, h: int) -> np.ndarray:
    """Rows [b, h, :, :] of a [B, H, S, D] bf16 tensor, generated on their own."""
    assert 0 <= b < B and 0 <= h < H
    off = ((b * H + h) * S) * D
    return normal_bf16_bits(seed, stream, S * D, offset=off).reshape(S, D)
