"""gqa_forward_decode_noalloc: the decode path for callers that cannot
allocate device memory (they are only handed the q/k/v/out buffers, or must
not call cudaMalloc in a steady-state loop).  Its scratch is the library's
static device array, so it takes no workspace.  Checked against gqa_forward
on the same inputs, on two calls in a row (the second call finds the first
call's leftovers in the shared array)."""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gqa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import grouped_query_attention_fwd_b200 as m
    return m


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _noalloc(gqa, q, k, v, out, mask=None):
    p = gqa.problem_for(q, k, v, mask=mask, out=out)
    stream = torch.cuda.current_stream().cuda_stream
    return gqa._lib.gqa_forward_decode_noalloc(
        ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(),
        mask.data_ptr() if mask is not None else None, out.data_ptr(), stream)


def _close(a, b):
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(a)) and np.all(np.isfinite(b))
    max_abs = np.abs(a - b).max()
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert max_abs <= 2e-2 and rel <= 1e-2, (max_abs, rel)


@pytest.mark.parametrize("shape", [(16, 32, 8, 4096, 128), (3, 24, 2, 777, 64)])
def test_noalloc_matches_workspace_entry_point_twice(gqa, shape):
    B, Hq, Hkv, Sk, D = shape
    for call, seed in enumerate((41, 42)):  # two calls in a row, different inputs
        qb, kb, vb = synth.qkv_bf16_bits(seed + Sk, B, Hq, Hkv, 1, Sk, D)
        q, k, v = _dev_bf16(qb), _dev_bf16(kb), _dev_bf16(vb)
        ref = gqa.forward(q, k, v)
        out = torch.full_like(ref, float("nan"))
        rc = _noalloc(gqa, q, k, v, out)
        assert rc == gqa.GQA_OK, gqa.status_string(rc)
        torch.cuda.synchronize()
        _close(out, ref)


def test_noalloc_rejects_what_it_cannot_hold(gqa):
    # More scratch than the static array holds: one ticket counter per kv
    # head, 2.2 M heads.  Zero-stride views: the call is refused before it
    # reads or writes any of them.
    H = 2200000
    one = torch.zeros(1, 1, 1, 64, dtype=torch.bfloat16, device="cuda")
    big_q = one.expand(1, H, 1, 64)
    big_k = one.expand(1, H, 1, 64)
    big_out = torch.zeros(1, 1, 1, 64, dtype=torch.bfloat16, device="cuda").expand(1, H, 1, 64)
    plan = gqa.query(big_q, big_k, big_k)
    assert plan["workspace_bytes"] > gqa.STATIC_SCRATCH_BYTES
    assert _noalloc(gqa, big_q, big_k, big_k, big_out) == gqa.GQA_ERR_SCRATCH_LIMIT
    # Not the decode path.
    q2 = torch.zeros(1, 16, 4, 128, dtype=torch.bfloat16, device="cuda")
    k2 = torch.zeros(1, 1, 4, 128, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(gqa, q2, k2, k2, torch.empty_like(q2)) == gqa.GQA_ERR_UNSUPPORTED
