"""The FMA-pipe exponential used by the prefill softmax (exp2_poly in
csrc/epilogue.cuh), compiled for the host from the same header and checked
against the bound its derivation states (7.5e-5 relative, Remez degree 3 on
[-1/2, 1/2], see csrc/exp2_poly_fit.py) over the range the softmax uses."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "grouped_query_attention_fwd_b200", "csrc")

SRC = r'''
#include "epilogue.cuh"
extern "C" void exp2_poly_batch(const float* x, float* y, int n) {
  for (int i = 0; i < n; ++i) y[i] = gqa::exp2_poly(x[i]);
}
'''


@pytest.fixture(scope="module")
def lib(tmp_path_factory):
    d = tmp_path_factory.mktemp("exp2")
    src = d / "exp2_host.cu"
    src.write_text(SRC)
    so = str(d / "libexp2_host.so")
    subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-O2", "-std=c++17", "-shared",
                           "-Xcompiler", "-fPIC", "-I" + CSRC, str(src), "-o", so])
    L = ctypes.CDLL(so)
    L.exp2_poly_batch.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    return L


def _run(lib, x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    y = np.empty_like(x)
    lib.exp2_poly_batch(x.ctypes.data, y.ctypes.data, x.size)
    return y


def test_relative_error_bound(lib):
    x = np.linspace(-125.0, 9.0, 2_000_001, dtype=np.float32)
    y = _run(lib, x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() <= 7.5e-5 * 1.01 + 1e-6, rel.max()


def test_fine_grid_near_zero(lib):
    x = (np.arange(-2 ** 16, 2 ** 16) / 2 ** 14).astype(np.float32)  # [-4, 4) step 2^-14
    y = _run(lib, x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() <= 7.6e-5


def test_hidden_keys_vanish(lib):
    """Hidden keys (-inf) and anything below -126 weigh exactly 0."""
    y = _run(lib, np.array([-np.inf, -1e30, -200.0, -126.5], dtype=np.float32))
    assert np.all(y == 0.0)
    y = _run(lib, np.array([-126.0], dtype=np.float32))
    assert 0 < y[0] < 2.0 ** -124
