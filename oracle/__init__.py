"""fp64 CPU oracle for the grouped-query attention forward (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the benchmark's ``cpu_baseline`` / ``--impl reference`` leg, never by the
product package.  The arithmetic lives in ``gqa_oracle.cpp`` (single-threaded,
double precision, the plain definition with a two-pass softmax); this file only
compiles it, converts arrays to contiguous float64 and calls it.

Pins: every function here is checked by ``tests/test_oracle_pins.py`` against
the pages' printed figures, closed forms, invariants and PyTorch's own fp64
attention routine, and planted mistakes in the C++ source are shown to fail
those pins.  No function is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gqa_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle (g++ -O2, strict IEEE: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + ".tmp%d" % os.getpid()
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared",
                               "-fno-fast-math", "-ffp-contract=off", src, "-o", tmp])
        os.replace(tmp, out)
    return out


def _bind(lib):
    i64, vp, dbl, cint = ctypes.c_int64, ctypes.c_void_p, ctypes.c_double, ctypes.c_int
    lib.oracle_gqa_probs.argtypes = [vp, vp, vp] + [i64] * 6 + [cint, dbl, vp]
    lib.oracle_gqa_probs.restype = cint
    lib.oracle_gqa_forward.argtypes = [vp, vp, vp, vp] + [i64] * 6 + [cint, dbl, vp]
    lib.oracle_gqa_forward.restype = cint
    lib.oracle_gqa_forward_rows.argtypes = ([vp, vp, vp, vp] + [i64] * 6 +
                                            [cint, dbl, vp, i64, vp])
    lib.oracle_gqa_forward_rows.restype = cint
    lib.oracle_kv_cache_bytes.argtypes = [i64] * 6
    lib.oracle_kv_cache_bytes.restype = i64
    lib.oracle_gqa_forward_ex.argtypes = ([vp, vp, vp, vp, vp] + [i64] * 6 +
                                          [cint, i64, i64, dbl, vp])
    lib.oracle_gqa_forward_ex.restype = cint
    lib.oracle_gqa_forward_rows_ex.argtypes = ([vp, vp, vp, vp, vp] + [i64] * 6 +
                                               [cint, i64, i64, dbl, vp, i64, vp])
    lib.oracle_gqa_forward_rows_ex.restype = cint
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _bind(ctypes.CDLL(_LIB))
    return _lib


def load_library(path: str):
    """Bind another build of the oracle source (the pin tests use this to show
    that a mistake planted in the C++ makes them fail)."""
    return _bind(ctypes.CDLL(path))


class OracleError(ValueError):
    pass


def _f64(x):
    return np.ascontiguousarray(x, dtype=np.float64)


def _shapes(q, k, v, mask):
    if q.ndim != 4 or k.ndim != 4:
        raise OracleError("q and k must be 4-D [B, H, S, D]")
    B, Hq, Sq, D = q.shape
    Bk, Hkv, Sk, Dk = k.shape
    if Bk != B or Dk != D:
        raise OracleError("q and k disagree on batch or head dim")
    if v is not None and tuple(v.shape) != tuple(k.shape):
        raise OracleError("v must have k's shape")
    if mask is not None and tuple(np.shape(mask)) != (B, Sq, Sk):
        raise OracleError("mask must be [B, Sq, Sk]")
    return B, Hq, Hkv, Sq, Sk, D


def _mask_arg(mask):
    if mask is None:
        return None, None
    m = np.ascontiguousarray(np.asarray(mask).astype(np.uint8))
    return m, m.ctypes.data


def forward(q, k, v, mask=None, causal=False, scale=None, lib=None, causal_offset=None,
            window=0, kv_lens=None) -> np.ndarray:
    """out [B, Hq, Sq, D] in float64.  ``scale`` defaults to 1/sqrt(D).

    ``causal_offset`` (with ``causal``): key j is visible to query i iff
    j <= i + causal_offset; None keeps the pages' form (offset 0, Sq == Sk).
    ``window`` > 0 (with ``causal``) also hides keys j <= i + offset - window.
    ``kv_lens`` (int per batch entry): keys j >= kv_lens[b] are hidden and the
    causal offset moves by kv_lens[b] - Sk."""
    if causal_offset is not None or window or kv_lens is not None:
        return _forward_ex(q, k, v, mask, causal, 0 if causal_offset is None else causal_offset,
                           window, scale, lib, kv_lens)
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Hkv, Sq, Sk, D = _shapes(q, k, v, mask)
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    m, mp = _mask_arg(mask)
    out = np.empty((B, Hq, Sq, D), dtype=np.float64)
    rc = (lib or _load()).oracle_gqa_forward(q.ctypes.data, k.ctypes.data, v.ctypes.data, mp,
                                             B, Hq, Hkv, Sq, Sk, D, int(bool(causal)),
                                             float(scale), out.ctypes.data)
    if rc != 0:
        raise OracleError("invalid problem for the oracle")
    return out


def probs(q, k, mask=None, causal=False, scale=None, lib=None) -> np.ndarray:
    """Attention weights [B, Hq, Sq, Sk] in float64."""
    q, k = _f64(q), _f64(k)
    B, Hq, Hkv, Sq, Sk, D = _shapes(q, k, None, mask)
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    m, mp = _mask_arg(mask)
    out = np.empty((B, Hq, Sq, Sk), dtype=np.float64)
    rc = (lib or _load()).oracle_gqa_probs(q.ctypes.data, k.ctypes.data, mp, B, Hq, Hkv, Sq,
                                           Sk, D, int(bool(causal)), float(scale),
                                           out.ctypes.data)
    if rc != 0:
        raise OracleError("invalid problem for the oracle")
    return out


def _lens_arg(kv_lens, B):
    if kv_lens is None:
        return None, None
    a = np.ascontiguousarray(np.asarray(kv_lens, dtype=np.int32).reshape(-1))
    if a.shape[0] != B:
        raise OracleError("kv_lens must have one entry per batch entry")
    return a, a.ctypes.data


def _forward_ex(q, k, v, mask, causal, causal_offset, window, scale, lib, kv_lens=None):
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Hkv, Sq, Sk, D = _shapes(q, k, v, mask)
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    m, mp = _mask_arg(mask)
    la, lp = _lens_arg(kv_lens, B)
    out = np.empty((B, Hq, Sq, D), dtype=np.float64)
    rc = (lib or _load()).oracle_gqa_forward_ex(q.ctypes.data, k.ctypes.data, v.ctypes.data, mp,
                                                lp, B, Hq, Hkv, Sq, Sk, D, int(bool(causal)),
                                                int(causal_offset), int(window), float(scale),
                                                out.ctypes.data)
    if rc != 0:
        raise OracleError("invalid problem for the oracle")
    return out


def forward_rows(q, k, v, rows, mask=None, causal=False, scale=None, lib=None,
                 causal_offset=None, window=0, kv_lens=None) -> np.ndarray:
    """Only the rows ``rows`` = [(b, h, i), ...]; returns [n, D] float64."""
    if causal_offset is not None or window or kv_lens is not None:
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, Hq, Hkv, Sq, Sk, D = _shapes(q, k, v, mask)
        if scale is None:
            scale = 1.0 / np.sqrt(D)
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
        m, mp = _mask_arg(mask)
        la, lp = _lens_arg(kv_lens, B)
        out = np.empty((r.shape[0], D), dtype=np.float64)
        rc = (lib or _load()).oracle_gqa_forward_rows_ex(
            q.ctypes.data, k.ctypes.data, v.ctypes.data, mp, lp, B, Hq, Hkv, Sq, Sk, D,
            int(bool(causal)), int(0 if causal_offset is None else causal_offset), int(window),
            float(scale), r.ctypes.data, r.shape[0], out.ctypes.data)
        if rc != 0:
            raise OracleError("invalid problem or row index for the oracle")
        return out
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Hkv, Sq, Sk, D = _shapes(q, k, v, mask)
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    m, mp = _mask_arg(mask)
    out = np.empty((r.shape[0], D), dtype=np.float64)
    rc = (lib or _load()).oracle_gqa_forward_rows(q.ctypes.data, k.ctypes.data, v.ctypes.data,
                                                  mp, B, Hq, Hkv, Sq, Sk, D, int(bool(causal)),
                                                  float(scale), r.ctypes.data, r.shape[0],
                                                  out.ctypes.data)
    if rc != 0:
        raise OracleError("invalid problem or row index for the oracle")
    return out


def kv_cache_bytes(layers: int, tokens: int, h_kv: int, d_head: int, batch: int,
                   elem_bytes: int, lib=None) -> int:
    """bytes_KV = 2 * L * n * h_kv * d_head * b * sizeof(dtype)."""
    return int((lib or _load()).oracle_kv_cache_bytes(layers, tokens, h_kv, d_head, batch,
                                                      elem_bytes))
