"""Helpers shared by the GPU parity tests: seeded inputs on the device, the
oracle on the same (bf16-rounded) values, and the parity bar."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

# Parity bar: fp32 max |err| <= 1e-5; bf16 max |err| <= 2e-2 and
# ||gpu - ref||_2 / ||ref||_2 <= 1e-2 against the oracle on the same
# bf16-rounded inputs.
F32_ABS = 1e-5
BF16_ABS = 2e-2
BF16_REL_RMS = 1e-2


def bits_to_dev(bits: np.ndarray, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def bf16_inputs(seed, B, Hq, Hkv, Sq, Sk, D, device="cuda"):
    qb, kb, vb = synth.qkv_bf16_bits(seed, B, Hq, Hkv, Sq, Sk, D)
    return (qb, kb, vb), tuple(bits_to_dev(x, device) for x in (qb, kb, vb))


def f64(bits: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f64(bits)


def rel_rms(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def assert_bf16_parity(got: np.ndarray, ref: np.ndarray, what: str = ""):
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), what
    max_abs = float(np.abs(got - ref).max()) if got.size else 0.0
    rr = rel_rms(got, ref) if got.size else 0.0
    assert max_abs <= BF16_ABS and rr <= BF16_REL_RMS, (what, max_abs, rr)
    return max_abs, rr


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def oracle_bf16(bits_q, bits_k, bits_v, mask=None, causal=False, scale=None):
    return oracle.forward(f64(bits_q), f64(bits_k), f64(bits_v), mask=mask, causal=causal,
                          scale=scale)


def f16_inputs(seed, B, Hq, Hkv, Sq, Sk, D, device="cuda"):
    """Seeded N(0,1) q, k, v rounded to fp16: (float64 copies for the oracle,
    fp16 device tensors)."""
    q, k, v = synth.qkv_f32(seed, B, Hq, Hkv, Sq, Sk, D)
    h = [x.astype(np.float16) for x in (q, k, v)]
    return tuple(x.astype(np.float64) for x in h), tuple(torch.from_numpy(x).to(device) for x in h)


def oracle_rows_threaded(q, k, v, rows, mask=None, causal=False, threads=None):
    """oracle.forward_rows over chunks of ``rows`` on several host threads
    (the oracle's ctypes calls release the GIL); the per-row arithmetic is the
    oracle's own, unchanged.  Returns [len(rows), D] float64 in row order."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    rows = list(rows)
    n = max(1, min(threads or os.cpu_count() or 1, 64, len(rows)))
    chunks = [rows[i::n] for i in range(n)]
    with ThreadPoolExecutor(max_workers=n) as ex:
        parts = list(ex.map(lambda c: oracle.forward_rows(q, k, v, c, mask=mask, causal=causal),
                            chunks))
    out = np.empty((len(rows), q.shape[-1]))
    for i, part in enumerate(parts):
        out[i::n] = part
    return out


def bf16_round(x: np.ndarray) -> np.ndarray:
    """x rounded to the nearest bf16 (ties to even), as float64."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).bfloat16()
    return t.float().numpy().astype(np.float64)
