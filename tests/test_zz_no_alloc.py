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


def _noalloc(gqa, q, k, v, out, mask=None, **kw):
    p = gqa.problem_for(q, k, v, mask=mask, out=out, **kw)
    stream = torch.cuda.current_stream().cuda_stream
    return gqa._lib.gqa_forward_decode_noalloc(
        ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(),
        mask.data_ptr() if mask is not None else None, out.data_ptr(), stream)


def _close(a, b):
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(a)) and np.all(np.isfinite(b))
    if not np.any(b):
        assert not np.any(a)
        return
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


def _variant_inputs(kind, seed):
    """Inputs of one decode-path variant: (q, k, v, forward kwargs)."""
    B, Hq, Hkv, Sk, D = 3, 16, 4, 700, 128
    Sq = 2 if kind == "short_query_block" else 1
    qb, kb, vb = synth.qkv_bf16_bits(seed, B, Hq, Hkv, Sq, Sk, D)
    q, k, v = _dev_bf16(qb), _dev_bf16(kb), _dev_bf16(vb)
    kw = {}
    if kind == "fp16":
        q, k, v = q.half(), k.half(), v.half()
    elif kind == "short_query_block":
        kw = dict(causal=True, causal_offset="bottom_right", window=300)
    elif kind == "mask":
        kw = dict(mask=torch.from_numpy(synth.mask_random(seed, B, Sq, Sk, 0.7)).cuda())
    elif kind in ("kv_lens", "paged"):
        kw = dict(kv_lens=torch.tensor([700, 1, 333], dtype=torch.int32, device="cuda"))
        if kind == "paged":
            ps, per = 128, 6  # 768-key capacity in 128-key pages, scattered over a pool
            pool_k = torch.full((B * per + 2, Hkv, ps, D), float("nan"), dtype=k.dtype, device="cuda")
            pool_v = pool_k.clone()
            perm = torch.randperm(B * per, generator=torch.Generator().manual_seed(seed)) + 2
            kp = torch.nn.functional.pad(k, (0, 0, 0, per * ps - Sk))
            vp = torch.nn.functional.pad(v, (0, 0, 0, per * ps - Sk))
            for b in range(B):
                for j in range(per):
                    slot = int(perm[b * per + j])
                    pool_k[slot] = kp[b, :, j * ps:(j + 1) * ps]
                    pool_v[slot] = vp[b, :, j * ps:(j + 1) * ps]
            k, v = pool_k, pool_v
            kw["block_table"] = perm.view(B, per).to(torch.int32).cuda()
    return q, k, v, kw


@pytest.mark.parametrize("kind", ["fp16", "short_query_block", "mask", "kv_lens", "paged"])
def test_noalloc_decode_variants_match_twice(gqa, kind):
    """Every kind of problem the decode kernel takes: the allocation-free call
    gives gqa_forward's result, on two calls in a row with different inputs."""
    for seed in (51, 52):
        q, k, v, kw = _variant_inputs(kind, seed)
        assert gqa.query(q, k, v, **kw)["kernel_name"] == "decode"
        ref = gqa.forward(q, k, v, **kw)
        assert gqa.device_status() == 0
        out = torch.full_like(ref, float("nan"))
        mask = kw.pop("mask", None)
        rc = _noalloc(gqa, q, k, v, out, mask=mask, **kw)
        assert rc == gqa.GQA_OK, gqa.status_string(rc)
        torch.cuda.synchronize()
        _close(out, ref)


def test_noalloc_fills_empty_and_hidden_problems(gqa):
    """seq_k == 0 gives zeros and a problem with no visible key gives NaN, as
    gqa_forward gives them; fp32 and long query blocks are refused."""
    q = torch.randn(2, 8, 1, 64, device="cuda").bfloat16()
    k0 = torch.zeros(2, 2, 0, 64, dtype=torch.bfloat16, device="cuda")
    out = torch.full_like(q, float("nan"))
    assert _noalloc(gqa, q, k0, k0, out) == gqa.GQA_OK
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0
    k = torch.randn(2, 2, 50, 64, device="cuda").bfloat16()
    out = torch.zeros_like(q)
    assert _noalloc(gqa, q, k, k, out, causal=True, causal_offset=-1) == gqa.GQA_OK
    torch.cuda.synchronize()
    assert torch.isnan(out.float()).all()
    q32, k32 = q.float(), k.float()
    assert _noalloc(gqa, q32, k32, k32, torch.empty_like(q32)) == gqa.GQA_ERR_UNSUPPORTED
