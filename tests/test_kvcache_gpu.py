"""Ragged KV caches (per-sequence lengths) and the KV-cache append, through
the C ABI, against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth

from gpu_util import F32_ABS, assert_bf16_parity, bf16_inputs, bits_to_dev, f64, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gqa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import grouped_query_attention_fwd_b200 as m
    return m


def _status(gqa):
    return gqa.device_status()


def _lens(seed, B, lo, hi, pinned=()):
    lens = synth.uniform_int(seed, synth.STREAM_MASK, B, lo, hi).astype(np.int32)
    for i, x in pinned:
        lens[i] = x
    return lens


def _check(out, ref, what):
    """NaN exactly where the oracle has a fully hidden row; parity elsewhere."""
    nan_ref = np.isnan(ref).all(axis=-1)
    assert np.array_equal(np.isnan(out).all(axis=-1), nan_ref), what
    assert_bf16_parity(out[~nan_ref], ref[~nan_ref], what)


# ------------------------------------------------------------ ragged decode

@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D,causal,window,pinned", [
    # one query per sequence: every length class, an empty cache (NaN rows)
    (6, 8, 2, 1, 1000, 128, False, 0, ((0, 1000), (1, 1), (2, 64), (3, 0), (4, 65))),
    (4, 32, 8, 1, 4096, 128, True, 0, ((0, 4096), (1, 4095))),
    (3, 16, 2, 1, 700, 64, True, 100, ((0, 700), (1, 99), (2, 101))),
    # short query blocks after a cache: (head, query) rows, bottom-right causal
    (5, 8, 2, 3, 600, 128, True, 0, ((0, 3), (1, 600), (2, 2))),
    (3, 4, 1, 4, 900, 128, True, 50, ((0, 900), (1, 4))),
    # few units: most CTAs get no range
    (2, 8, 2, 1, 2000, 128, False, 0, ((0, 1), (1, 2))),
])
def test_ragged_decode(gqa, B, Hq, Hkv, Sq, Sk, D, causal, window, pinned):
    seed = 3000 + B + Sk + Sq
    bits, (q, k, v) = bf16_inputs(seed, B, Hq, Hkv, Sq, Sk, D)
    lens = _lens(seed, B, 0, Sk, pinned)
    off = Sk - Sq if causal else None
    out = to_np(gqa.forward(q, k, v, causal=causal, causal_offset=off, window=window,
                            kv_lens=torch.from_numpy(lens).cuda()))
    assert _status(gqa) == 0
    assert gqa.query(q, k, v, causal=causal, causal_offset=off, window=window,
                     kv_lens=torch.from_numpy(lens).cuda())["kernel_name"] == "decode"
    ref = oracle.forward(f64(bits[0]), f64(bits[1]), f64(bits[2]), causal=causal,
                         causal_offset=off, window=window, kv_lens=lens)
    _check(out, ref, "ragged decode %s" % ((B, Hq, Hkv, Sq, Sk, D, causal, window),))


def test_ragged_decode_many_sequences_sampled(gqa):
    """B=48 sequences of 0..4096 keys in a 4096-key cache, Hq=32, Hkv=8, D=128:
    the device-side schedule with split groups of every size."""
    B, Hq, Hkv, Sk, D = 48, 32, 8, 4096, 128
    bits, (q, k, v) = bf16_inputs(3100, B, Hq, Hkv, 1, Sk, D)
    lens = _lens(3100, B, 1, Sk, ((0, 0), (1, 4096), (2, 1), (3, 63), (4, 64), (5, 65)))
    out = to_np(gqa.forward(q, k, v, kv_lens=torch.from_numpy(lens).cuda()))
    assert _status(gqa) == 0
    picks = list(range(0, B, 5)) + [1, 2, 3, 4, 5]
    for b in picks:
        n = int(lens[b])
        if n == 0:
            assert np.all(np.isnan(out[b]))
            continue
        ref = oracle.forward(f64(bits[0][b:b + 1]), f64(bits[1][b:b + 1, :, :n]),
                             f64(bits[2][b:b + 1, :, :n]))
        assert_bf16_parity(out[b:b + 1], ref, "ragged decode b=%d len=%d" % (b, n))


def test_ragged_decode_mask_and_lengths(gqa):
    B, Hq, Hkv, Sk, D = 3, 12, 2, 500, 64
    bits, (q, k, v) = bf16_inputs(3200, B, Hq, Hkv, 1, Sk, D)
    lens = np.array([500, 130, 7], dtype=np.int32)
    mask = synth.mask_random(3200, B, 1, Sk, 0.5)
    mask[:, 0, 0] = 1
    out = to_np(gqa.forward(q, k, v, mask=torch.from_numpy(mask).cuda(),
                            kv_lens=torch.from_numpy(lens).cuda()))
    assert _status(gqa) == 0
    ref = oracle.forward(f64(bits[0]), f64(bits[1]), f64(bits[2]), mask=mask, kv_lens=lens)
    _check(out, ref, "ragged decode with mask")


# ------------------------------------------------------------ ragged prefill / fp32

@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D,window,pinned", [
    (3, 8, 2, 200, 1000, 128, 0, ((0, 1000), (1, 200), (2, 450))),
    (2, 12, 2, 150, 700, 64, 0, ((0, 160), (1, 700))),
    (2, 8, 2, 256, 1024, 128, 300, ((0, 1024), (1, 700))),
    (2, 8, 2, 130, 600, 128, 0, ((0, 100), (1, 0))),  # shorter than the block: NaN rows
])
def test_ragged_prefill(gqa, B, Hq, Hkv, Sq, Sk, D, window, pinned):
    """A chunk of Sq new queries at the end of each sequence (bottom-right)."""
    seed = 3300 + Sq + Sk
    bits, (q, k, v) = bf16_inputs(seed, B, Hq, Hkv, Sq, Sk, D)
    lens = _lens(seed, B, Sq, Sk, pinned)
    out = to_np(gqa.forward(q, k, v, causal=True, causal_offset="bottom_right", window=window,
                            kv_lens=torch.from_numpy(lens).cuda()))
    assert _status(gqa) == 0
    ref = oracle.forward(f64(bits[0]), f64(bits[1]), f64(bits[2]), causal=True,
                         causal_offset=Sk - Sq, window=window, kv_lens=lens)
    _check(out, ref, "ragged prefill %s" % ((B, Hq, Hkv, Sq, Sk, D, window),))


@pytest.mark.parametrize("dtype,D,causal", [("bf16", 128, True), ("bf16", 64, False),
                                             ("f16", 128, False)])
def test_ragged_prefill_nan_tail(gqa, dtype, D, causal):
    """A contiguous cache whose rows past each length are NaN (K and V), on the
    prefill path: the result must not see them."""
    B, Hq, Hkv, Sq, Sk = 3, 8, 2, 100, 700
    seed = 3500 + D
    if dtype == "bf16":
        bits = synth.qkv_bf16_bits(seed, B, Hq, Hkv, Sq, Sk, D)
        qc, kc, vc = (f64(x) for x in bits)
        tdt = torch.bfloat16
    else:
        qc, kc, vc = (x.astype(np.float16).astype(np.float64)
                      for x in synth.qkv_f32(seed, B, Hq, Hkv, Sq, Sk, D))
        tdt = torch.float16
    lens = np.array([700, 333, 129], dtype=np.int32)
    kn, vn = kc.copy(), vc.copy()
    for b in range(B):
        kn[b, :, lens[b]:] = np.nan
        vn[b, :, lens[b]:] = np.nan
        kc[b, :, lens[b]:] = 0.0
        vc[b, :, lens[b]:] = 0.0
    q, k, v = (torch.from_numpy(x).to(tdt).cuda() for x in (qc, kn, vn))
    kw = dict(causal=True, causal_offset="bottom_right") if causal else {}
    out = to_np(gqa.forward(q, k, v, kv_lens=torch.from_numpy(lens).cuda(), **kw))
    assert _status(gqa) == 0
    ref = oracle.forward(qc, kc, vc, kv_lens=lens,
                         **(dict(causal=True, causal_offset=Sk - Sq) if causal else {}))
    _check(out, ref, "ragged prefill NaN tail %s D=%d causal=%s" % (dtype, D, causal))


def test_ragged_prefill_non_causal(gqa):
    B, Hq, Hkv, Sq, Sk, D = 2, 8, 2, 100, 800, 128
    bits, (q, k, v) = bf16_inputs(3400, B, Hq, Hkv, Sq, Sk, D)
    lens = np.array([333, 800], dtype=np.int32)
    out = to_np(gqa.forward(q, k, v, kv_lens=torch.from_numpy(lens).cuda()))
    assert _status(gqa) == 0
    ref = oracle.forward(f64(bits[0]), f64(bits[1]), f64(bits[2]), kv_lens=lens)
    _check(out, ref, "ragged prefill non-causal")


def test_ragged_f32(gqa):
    B, Hq, Hkv, Sq, Sk, D = 3, 6, 2, 4, 90, 40
    q, k, v = synth.qkv_f32(3500, B, Hq, Hkv, Sq, Sk, D)
    lens = np.array([90, 3, 0], dtype=np.int32)
    out = gqa.forward(torch.from_numpy(q).cuda(), torch.from_numpy(k).cuda(),
                      torch.from_numpy(v).cuda(), causal=True, causal_offset="bottom_right",
                      kv_lens=torch.from_numpy(lens).cuda()).cpu().numpy()
    assert _status(gqa) == 0
    ref = oracle.forward(q, k, v, causal=True, causal_offset=Sk - Sq, kv_lens=lens)
    nan_ref = np.isnan(ref).all(axis=-1)
    assert np.array_equal(np.isnan(out).all(axis=-1), nan_ref)
    assert np.abs(out[~nan_ref] - ref[~nan_ref]).max() <= F32_ABS


def test_length_out_of_range_is_reported(gqa):
    bits, (q, k, v) = bf16_inputs(3600, 2, 8, 2, 1, 300, 128)
    lens = torch.tensor([300, 301], dtype=torch.int32, device="cuda")
    gqa.forward(q, k, v, kv_lens=lens)
    assert _status(gqa) == gqa.GQA_ERR_KV_LENGTH
    assert _status(gqa) == 0  # the error word was cleared
    gqa.forward(q, k, v, kv_lens=torch.tensor([300, 5], dtype=torch.int32, device="cuda"))
    assert _status(gqa) == 0


# ------------------------------------------------------------ append

def _rows_bits(seed, B, H, S, D):
    return synth.qkv_bf16_bits(seed, B, H, H, S, S, D)[1:]


@pytest.mark.parametrize("B,Hkv,cap,D,n_new,pinned", [
    (4, 8, 300, 128, 1, ((0, 0), (1, 299), (2, 17))),
    (3, 2, 1000, 64, 37, ((0, 963), (1, 0))),
    (2, 4, 64, 128, 64, ((0, 0), (1, 0))),
])
def test_kv_append_bitwise(gqa, B, Hkv, cap, D, n_new, pinned):
    kc, vc = _rows_bits(3700 + cap, B, Hkv, cap, D)
    kn, vn = _rows_bits(3800 + n_new, B, Hkv, n_new, D)
    lens = _lens(3700 + cap, B, 0, cap - n_new, pinned)
    ck, cv = bits_to_dev(kc), bits_to_dev(vc)
    dl = torch.from_numpy(lens.copy()).cuda()
    gqa.kv_append(ck, cv, bits_to_dev(kn), bits_to_dev(vn), dl)
    assert _status(gqa) == 0
    ek, ev = kc.copy(), vc.copy()
    for b in range(B):
        ek[b, :, lens[b]:lens[b] + n_new] = kn[b]
        ev[b, :, lens[b]:lens[b] + n_new] = vn[b]
    assert np.array_equal(ck.cpu().view(torch.int16).numpy().view(np.uint16), ek)
    assert np.array_equal(cv.cpu().view(torch.int16).numpy().view(np.uint16), ev)
    assert np.array_equal(dl.cpu().numpy(), lens + n_new)


def test_kv_append_overflow_leaves_entry(gqa):
    B, Hkv, cap, D, n_new = 3, 2, 100, 128, 10
    kc, vc = _rows_bits(3900, B, Hkv, cap, D)
    kn, vn = _rows_bits(3901, B, Hkv, n_new, D)
    lens = np.array([90, 91, -1], dtype=np.int32)  # 91 + 10 > 100; -1 invalid
    ck, cv = bits_to_dev(kc), bits_to_dev(vc)
    dl = torch.from_numpy(lens.copy()).cuda()
    gqa.kv_append(ck, cv, bits_to_dev(kn), bits_to_dev(vn), dl)
    assert _status(gqa) == gqa.GQA_ERR_KV_LENGTH
    ek = kc.copy()
    ek[0, :, 90:100] = kn[0]
    assert np.array_equal(ck.cpu().view(torch.int16).numpy().view(np.uint16), ek)
    assert np.array_equal(dl.cpu().numpy(), np.array([100, 91, -1], dtype=np.int32))


def test_kv_append_strided_and_f32(gqa):
    """New rows as a [B, n, H, D] buffer viewed as [B, H, n, D]; an fp32 cache."""
    B, Hkv, cap, D, n_new = 2, 4, 50, 24, 3
    rng = np.random.default_rng(4000)
    kc = rng.standard_normal((B, Hkv, cap, D)).astype(np.float32)
    vc = rng.standard_normal((B, Hkv, cap, D)).astype(np.float32)
    kn = rng.standard_normal((B, n_new, Hkv, D)).astype(np.float32)
    vn = rng.standard_normal((B, n_new, Hkv, D)).astype(np.float32)
    ck, cv = torch.from_numpy(kc).cuda(), torch.from_numpy(vc).cuda()
    kn_d = torch.from_numpy(kn).cuda().transpose(1, 2)
    vn_d = torch.from_numpy(vn).cuda().transpose(1, 2)
    lens = np.array([5, 47], dtype=np.int32)
    dl = torch.from_numpy(lens.copy()).cuda()
    gqa.kv_append(ck, cv, kn_d, vn_d, dl)
    assert _status(gqa) == 0
    for b in range(B):
        kc[b, :, lens[b]:lens[b] + n_new] = kn[b].transpose(1, 0, 2)
        vc[b, :, lens[b]:lens[b] + n_new] = vn[b].transpose(1, 0, 2)
    assert np.array_equal(ck.cpu().numpy(), kc) and np.array_equal(cv.cpu().numpy(), vc)


def test_append_then_decode_steps(gqa):
    """Three generation steps: append one token per sequence, then attend over
    the grown cache with the bottom-right diagonal."""
    B, Hq, Hkv, cap, D = 3, 16, 4, 400, 128
    kc, vc = _rows_bits(4100, B, Hkv, cap, D)
    ck, cv = bits_to_dev(kc), bits_to_dev(vc)
    lens = np.array([10, 0, 200], dtype=np.int32)
    dl = torch.from_numpy(lens.copy()).cuda()
    for step in range(3):
        qb = synth.qkv_bf16_bits(4200 + step, B, Hq, Hkv, 1, 1, D)[0]
        kn, vn = _rows_bits(4300 + step, B, Hkv, 1, D)
        gqa.kv_append(ck, cv, bits_to_dev(kn), bits_to_dev(vn), dl)
        out = to_np(gqa.forward(bits_to_dev(qb), ck, cv, causal=True,
                                causal_offset="bottom_right", kv_lens=dl))
        assert _status(gqa) == 0
        for b in range(B):
            kc[b, :, lens[b]] = kn[b, :, 0]
            vc[b, :, lens[b]] = vn[b, :, 0]
        lens += 1
        assert np.array_equal(dl.cpu().numpy(), lens)
        ref = oracle.forward(f64(qb), f64(kc), f64(vc), causal=True, causal_offset=cap - 1,
                             kv_lens=lens)
        assert_bf16_parity(out, ref, "append + decode step %d" % step)
