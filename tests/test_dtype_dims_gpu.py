"""fp16 operands and head dims other than 64 / 128 on the tensor-core paths,
through the C ABI, against the fp64 oracle on the same rounded inputs."""
import numpy as np
import pytest
import torch

import oracle
import synth

from gpu_util import assert_bf16_parity, bf16_inputs, f16_inputs, f64, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gqa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import grouped_query_attention_fwd_b200 as m
    return m


def _inputs(dtype, seed, B, Hq, Hkv, Sq, Sk, D):
    if dtype == "f16":
        return f16_inputs(seed, B, Hq, Hkv, Sq, Sk, D)
    bits, dev = bf16_inputs(seed, B, Hq, Hkv, Sq, Sk, D)
    return tuple(f64(b) for b in bits), dev


def _check(gqa, out, ref, what):
    assert gqa.device_status() == 0
    nan_ref = np.isnan(ref).all(axis=-1)
    assert np.array_equal(np.isnan(out).all(axis=-1), nan_ref), what
    assert_bf16_parity(out[~nan_ref], ref[~nan_ref], what)


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D", [
    (3, 32, 8, 1, 1000, 128),    # decode, g = 4
    (2, 12, 2, 1, 700, 64),      # decode, g = 6, D = 64
    (2, 32, 2, 1, 513, 128),     # decode, g = 16: Q fragments from shared memory
    (2, 8, 2, 3, 600, 128),      # short multi-query decode, non-causal
    (2, 8, 2, 300, 300, 128),    # prefill, causal below
    (1, 12, 2, 200, 500, 64),    # prefill, g = 6, D = 64
])
def test_f16_parity(gqa, B, Hq, Hkv, Sq, Sk, D):
    causal = Sq == Sk
    (q, k, v), (qd, kd, vd) = _inputs("f16", 5000 + Sq + Sk, B, Hq, Hkv, Sq, Sk, D)
    off = None if Sq == Sk or not causal else Sk - Sq
    out = to_np(gqa.forward(qd, kd, vd, causal=causal, causal_offset=off))
    assert out.dtype == np.float64 and qd.dtype == torch.float16
    _check(gqa, out, oracle.forward(q, k, v, causal=causal, causal_offset=off),
           "f16 %s" % ((B, Hq, Hkv, Sq, Sk, D),))


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("D", [8, 24, 40, 72, 96, 120])
def test_head_dims_decode(gqa, dtype, D):
    B, Hq, Hkv, Sk = 2, 16, 4, 333
    (q, k, v), (qd, kd, vd) = _inputs(dtype, 5100 + D, B, Hq, Hkv, 1, Sk, D)
    out = to_np(gqa.forward(qd, kd, vd))
    assert out.shape == (B, Hq, 1, D)
    _check(gqa, out, oracle.forward(q, k, v), "decode %s D=%d" % (dtype, D))


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("D", [8, 24, 72, 96])
def test_head_dims_prefill(gqa, dtype, D):
    B, Hq, Hkv, S = 2, 8, 2, 260
    (q, k, v), (qd, kd, vd) = _inputs(dtype, 5200 + D, B, Hq, Hkv, S, S, D)
    out = to_np(gqa.forward(qd, kd, vd, causal=True))
    _check(gqa, out, oracle.forward(q, k, v, causal=True), "prefill %s D=%d" % (dtype, D))


def test_head_dim_24_page_example(gqa):
    """The usage example's shape: 32 query heads of dimension 768 / 32 = 24 over
    4 kv heads (8 per group), masked and causal prefill plus a decode step."""
    B, Hq, Hkv, S, D = 2, 32, 4, 96, 24
    (q, k, v), (qd, kd, vd) = _inputs("bf16", 5300, B, Hq, Hkv, S, S, D)
    out = to_np(gqa.forward(qd, kd, vd, causal=True))
    _check(gqa, out, oracle.forward(q, k, v, causal=True), "D=24 prefill")
    mask = synth.mask_random(5301, B, S, S, 0.7)
    for i in range(S):
        mask[:, i, 0] = 1
    out = to_np(gqa.forward(qd, kd, vd, mask=torch.from_numpy(mask).cuda()))
    _check(gqa, out, oracle.forward(q, k, v, mask=mask), "D=24 masked")


def test_odd_head_dim_ragged_and_strided(gqa):
    """D = 96 with per-sequence lengths, a [B, S, H, D] cache viewed as
    [B, H, S, D], and a short bottom-right query block."""
    B, Hq, Hkv, Sq, Sk, D = 3, 8, 2, 2, 400, 96
    q, k, v = synth.qkv_f32(5400, B, Hq, Hkv, Sq, Sk, D)
    qh, kh, vh = (x.astype(np.float16) for x in (q, k, v))
    kd = torch.from_numpy(np.ascontiguousarray(kh.transpose(0, 2, 1, 3))).cuda().transpose(1, 2)
    vd = torch.from_numpy(np.ascontiguousarray(vh.transpose(0, 2, 1, 3))).cuda().transpose(1, 2)
    lens = np.array([400, 37, 2], dtype=np.int32)
    out = to_np(gqa.forward(torch.from_numpy(qh).cuda(), kd, vd, causal=True,
                            causal_offset="bottom_right", kv_lens=torch.from_numpy(lens).cuda()))
    ref = oracle.forward(qh.astype(np.float64), kh.astype(np.float64), vh.astype(np.float64),
                         causal=True, causal_offset=Sk - Sq, kv_lens=lens)
    _check(gqa, out, ref, "D=96 ragged strided f16")


def test_kv_append_f16_bitwise(gqa):
    B, Hkv, cap, D, n = 2, 4, 100, 40, 3
    rng = np.random.default_rng(5500)
    kc = rng.standard_normal((B, Hkv, cap, D)).astype(np.float16)
    kn = rng.standard_normal((B, Hkv, n, D)).astype(np.float16)
    ck, cv = torch.from_numpy(kc).cuda(), torch.from_numpy(kc.copy()).cuda()
    lens = torch.tensor([0, 97], dtype=torch.int32, device="cuda")
    gqa.kv_append(ck, cv, torch.from_numpy(kn).cuda(), torch.from_numpy(kn).cuda(), lens)
    assert gqa.device_status() == 0
    exp = kc.copy()
    exp[0, :, 0:3] = kn[0]
    exp[1, :, 97:100] = kn[1]
    assert np.array_equal(ck.cpu().numpy(), exp) and np.array_equal(cv.cpu().numpy(), exp)
    assert lens.cpu().tolist() == [3, 100]
