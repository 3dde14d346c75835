"""CUDA path vs the fp64 oracle, element by element, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import synth

from gpu_util import (BF16_ABS, BF16_REL_RMS, F32_ABS, assert_bf16_parity, bf16_inputs, bits_to_dev,
                      f64, oracle_bf16, rel_rms, to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gqa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import grouped_query_attention_fwd_b200 as m
    return m


def _status_ok(gqa):
    st = gqa.device_status()
    assert st == 0, gqa.status_string(st)


# ------------------------------------------------------------------ fp32

def test_f32_page_toy(gqa):
    """q (1,4,5,4), k, v (1,2,5,4): the page-1 example, fp32, scale 1/sqrt(4)."""
    q, k, v = synth.qkv_f32(1, 1, 4, 2, 5, 5, 4)
    out = gqa.forward(torch.from_numpy(q).cuda(), torch.from_numpy(k).cuda(),
                      torch.from_numpy(v).cuda(), scale=0.5)
    assert tuple(out.shape) == (1, 4, 5, 4)
    ref = oracle.forward(q, k, v, scale=0.5)
    assert np.abs(out.cpu().numpy() - ref).max() <= F32_ABS


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D,causal,masked", [
    (2, 6, 3, 7, 9, 8, False, False),
    (2, 8, 2, 33, 33, 64, True, False),
    (3, 12, 2, 5, 70, 37, False, True),
    (1, 4, 1, 1, 300, 128, False, False),
    (2, 4, 4, 16, 16, 256, True, True),
])
def test_f32_shapes(gqa, B, Hq, Hkv, Sq, Sk, D, causal, masked):
    q, k, v = synth.qkv_f32(B + Sk, B, Hq, Hkv, Sq, Sk, D)
    mask = synth.mask_random(5, B, Sq, Sk, 0.5) if masked else None
    if masked and causal:  # keep the diagonal so that no row is fully hidden
        for i in range(min(Sq, Sk)):
            mask[:, i, i] = 1
    out = gqa.forward(torch.from_numpy(q).cuda(), torch.from_numpy(k).cuda(),
                      torch.from_numpy(v).cuda(),
                      mask=torch.from_numpy(mask).cuda() if masked else None, causal=causal)
    ref = oracle.forward(q, k, v, mask=mask, causal=causal)
    assert np.abs(out.cpu().numpy() - ref).max() <= F32_ABS


# ------------------------------------------------------------------ decode

DECODE_CASES = [
    # B, Hq, Hkv, Sk, D
    (1, 4, 2, 1, 128),
    (2, 8, 2, 63, 128),
    (2, 8, 2, 64, 128),
    (2, 8, 2, 65, 128),
    (3, 32, 8, 333, 128),
    (2, 12, 2, 1000, 64),
    (1, 8, 8, 200, 128),      # g = 1 (MHA)
    (2, 8, 1, 517, 128),      # g = 8, one kv head (MQA)
    (2, 6, 2, 129, 64),       # g = 3
    (1, 24, 2, 700, 128),     # g = 12: two 8-wide column tiles
    (1, 40, 1, 300, 64),      # g = 40: three 16-head passes
    (5, 32, 8, 4096, 128),
    (2, 8, 2, 127, 128),      # one key short of a 128-key tile
    (2, 8, 2, 128, 128),      # exactly one tile
    (2, 8, 2, 129, 128),      # one key into the second tile
    (2, 32, 2, 1025, 128),    # g = 16: Q fragments from shared memory
    (3, 64, 4, 2000, 64),     # g = 16, D = 64
]


@pytest.mark.parametrize("B,Hq,Hkv,Sk,D", DECODE_CASES)
def test_decode_parity(gqa, B, Hq, Hkv, Sk, D):
    bits, (q, k, v) = bf16_inputs(100 + Sk, B, Hq, Hkv, 1, Sk, D)
    out = gqa.forward(q, k, v)
    _status_ok(gqa)
    assert_bf16_parity(to_np(out), oracle_bf16(*bits), "decode %s" % ((B, Hq, Hkv, Sk, D),))


@pytest.mark.parametrize("Sk", [77, 1500])
def test_decode_masked(gqa, Sk):
    B, Hq, Hkv, D = 3, 16, 4, 128
    bits, (q, k, v) = bf16_inputs(7, B, Hq, Hkv, 1, Sk, D)
    mask = synth.mask_random(8, B, 1, Sk, 0.3)
    out = gqa.forward(q, k, v, mask=torch.from_numpy(mask).cuda())
    _status_ok(gqa)
    assert_bf16_parity(to_np(out), oracle_bf16(*bits, mask=mask), "decode masked")


def test_decode_strided_bshd_views(gqa):
    """K/V cache stored [B, Sk, Hkv, D] and viewed as [B, Hkv, Sk, D]; q and out too."""
    B, Hq, Hkv, Sk, D = 2, 16, 4, 300, 128
    qb, kb, vb = synth.qkv_bf16_bits(9, B, Hq, Hkv, 1, Sk, D)
    q = bits_to_dev(qb.transpose(0, 2, 1, 3).copy()).transpose(1, 2)
    k = bits_to_dev(kb.transpose(0, 2, 1, 3).copy()).transpose(1, 2)
    v = bits_to_dev(vb.transpose(0, 2, 1, 3).copy()).transpose(1, 2)
    assert not k.is_contiguous()
    out = torch.empty(B, 1, Hq, D, dtype=torch.bfloat16, device="cuda").transpose(1, 2)
    gqa.forward(q, k, v, out=out)
    _status_ok(gqa)
    assert_bf16_parity(to_np(out), oracle_bf16(qb, kb, vb), "decode strided")


def test_decode_scale_and_determinism(gqa):
    bits, (q, k, v) = bf16_inputs(10, 4, 32, 8, 1, 2000, 128)
    a = gqa.forward(q, k, v, scale=0.3)
    b = gqa.forward(q, k, v, scale=0.3)
    _status_ok(gqa)
    assert torch.equal(a, b)
    assert_bf16_parity(to_np(a), oracle_bf16(*bits, scale=0.3), "decode scale")


def test_decode_fully_hidden_row_is_nan(gqa):
    bits, (q, k, v) = bf16_inputs(11, 2, 8, 2, 1, 100, 128)
    mask = np.ones((2, 1, 100), dtype=np.uint8)
    mask[1] = 0
    out = to_np(gqa.forward(q, k, v, mask=torch.from_numpy(mask).cuda()))
    _status_ok(gqa)
    assert np.all(np.isnan(out[1])) and np.all(np.isfinite(out[0]))


def test_empty_and_zero_length(gqa):
    q = torch.zeros(0, 4, 1, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(0, 2, 10, 128, dtype=torch.bfloat16, device="cuda")
    assert gqa.forward(q, k, k).shape == (0, 4, 1, 128)
    q = torch.randn(2, 4, 3, 64, device="cuda").bfloat16()
    k = torch.zeros(2, 2, 0, 64, dtype=torch.bfloat16, device="cuda")
    out = torch.full((2, 4, 3, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    gqa.forward(q, k, k, out=out)
    assert torch.count_nonzero(out).item() == 0  # empty weighted sum


def test_bad_alignment_rejected(gqa):
    base = torch.zeros(1 + 8 * 64, dtype=torch.bfloat16, device="cuda")
    q = base[1:].view(1, 8, 1, 64)  # 2-byte offset: not 16-byte aligned
    k = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gqa.GQAError) as ei:
        gqa.forward(q, k, k)
    assert ei.value.status == gqa.GQA_ERR_LAYOUT


# ------------------------------------------------------ full-size decode

def _full_decode(gqa, seed, B, Hq, Hkv, Sk, D, groups):
    """Full-size decode on the GPU; the oracle recomputes the given (b, kv)
    groups from their own slices of the seeded inputs."""
    bits, (q, k, v) = bf16_inputs(seed, B, Hq, Hkv, 1, Sk, D)
    out = to_np(gqa.forward(q, k, v))
    _status_ok(gqa)
    g = Hq // Hkv
    qb = bits[0]
    del bits
    for (b, kv) in groups:
        ks = synth.kv_slice_bf16_bits(seed, synth.STREAM_K, B, Hkv, Sk, D, b, kv)
        vs = synth.kv_slice_bf16_bits(seed, synth.STREAM_V, B, Hkv, Sk, D, b, kv)
        ref = oracle.forward(f64(qb[b:b + 1, kv * g:(kv + 1) * g]), f64(ks)[None, None],
                             f64(vs)[None, None])
        assert_bf16_parity(out[b:b + 1, kv * g:(kv + 1) * g], ref, "group %s" % ((b, kv),))
    return out


def test_decode_mistral7b_layer_full(gqa):
    """B=16, Hq=32, Hkv=8, Sk=4096, D=128: the whole output against the oracle."""
    bits, (q, k, v) = bf16_inputs(2, 16, 32, 8, 1, 4096, 128)
    out = to_np(gqa.forward(q, k, v))
    _status_ok(gqa)
    ma, rr = assert_bf16_parity(out, oracle_bf16(*bits), "mistral-7b decode")
    print("decode B16 Hq32 Hkv8 Sk4096: max_abs=%.3e rel_rms=%.3e" % (ma, rr))


def test_decode_llama70b_layer_sampled(gqa):
    """B=16, Hq=64, Hkv=8, Sk=32768, D=128 (2 GiB of K+V): sampled groups."""
    _full_decode(gqa, 3, 16, 64, 8, 32768, 128, [(0, 0), (7, 3), (15, 7), (9, 5)])


def test_decode_after_other_calls_on_one_workspace(gqa):
    """One workspace shared by a masked prefill, a small decode and a large
    decode, in that order: leftovers of earlier calls must not leak into the
    decode's split-merge counters."""
    shapes = [(3, 12, 2, 300, 300, 64, True), (1, 4, 2, 1, 700, 128, False),
              (16, 32, 8, 1, 4096, 128, False), (2, 8, 2, 1, 333, 128, False)]
    cases = []
    need = 256
    for i, (B, Hq, Hkv, Sq, Sk, D, masked) in enumerate(shapes):
        bits, (q, k, v) = bf16_inputs(300 + i, B, Hq, Hkv, Sq, Sk, D)
        mask = synth.mask_random(301 + i, B, Sq, Sk, 0.4) if masked else None
        md = torch.from_numpy(mask).cuda() if masked else None
        need = max(need, gqa.query(q, k, v, mask=md)["workspace_bytes"])
        cases.append((bits, q, k, v, mask, md))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for rep in range(2):
        for bits, q, k, v, mask, md in cases:
            out = gqa.forward(q, k, v, mask=md, workspace=ws)
            st = gqa.device_status(ws)
            assert st == 0, gqa.status_string(st)
            assert_bf16_parity(to_np(out), oracle_bf16(*bits, mask=mask),
                               "shared workspace %s" % (tuple(q.shape),))


# ----------------------------------------------- causal offset and sliding window

def _nan_rows_match(got, ref):
    """Rows the oracle leaves NaN (no visible key) must be NaN on the GPU too;
    returns the boolean array of the other rows."""
    nan_ref = np.isnan(ref).all(axis=-1)
    assert np.array_equal(np.isnan(got).all(axis=-1), nan_ref)
    return ~nan_ref


@pytest.mark.parametrize("Sq,Sk,off,window", [(5, 40, 35, 0), (5, 40, 35, 7), (6, 6, -2, 0),
                                              (4, 30, 10, 3)])
def test_f32_offset_window(gqa, Sq, Sk, off, window):
    q, k, v = synth.qkv_f32(Sq * 7 + Sk, 2, 8, 2, Sq, Sk, 32)
    out = gqa.forward(torch.from_numpy(q).cuda(), torch.from_numpy(k).cuda(),
                      torch.from_numpy(v).cuda(), causal=True, causal_offset=off, window=window)
    ref = oracle.forward(q, k, v, causal=True, causal_offset=off, window=window)
    got = out.cpu().numpy().astype(np.float64)
    ok = _nan_rows_match(got, ref)
    assert np.abs(got[ok] - ref[ok]).max() <= F32_ABS


@pytest.mark.parametrize("Sk,off,window,masked", [
    (1000, 999, 0, False),     # bottom-right: the one query sees every key
    (4096, 4095, 256, False),  # sliding window over the last 256 keys
    (1000, 500, 200, True),    # keys 301..500, with a mask
    (777, 700, 65, False),     # window straddling tile edges
])
def test_decode_offset_window(gqa, Sk, off, window, masked):
    B, Hq, Hkv, D = 3, 16, 4, 128
    bits, (q, k, v) = bf16_inputs(Sk + window, B, Hq, Hkv, 1, Sk, D)
    mask = synth.mask_random(9, B, 1, Sk, 0.5) if masked else None
    if masked:  # keep a visible key inside the window
        mask[:, :, off] = 1
    out = gqa.forward(q, k, v, mask=torch.from_numpy(mask).cuda() if masked else None,
                      causal=True, causal_offset=off, window=window)
    _status_ok(gqa)
    ref = oracle.forward(f64(bits[0]), f64(bits[1]), f64(bits[2]), mask=mask, causal=True,
                         causal_offset=off, window=window)
    assert_bf16_parity(to_np(out), ref, "decode offset/window")


def test_nothing_visible_is_nan(gqa):
    bits, (q, k, v) = bf16_inputs(12, 2, 8, 2, 4, 64, 128)
    out = to_np(gqa.forward(q, k, v, causal=True, causal_offset=-4))
    assert np.all(np.isnan(out))


# ------------------------------------------------ short multi-query decode

@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D,off,window,masked", [
    (2, 8, 2, 4, 1000, 128, "br", 0, False),   # 4 heads x 4 queries = 16 rows, bottom-right
    (3, 8, 1, 2, 517, 64, None, 0, False),     # 8 heads x 2 queries, no causal
    (1, 4, 4, 16, 300, 128, "br", 50, False),  # MHA, 16 queries, sliding window
    (2, 8, 2, 3, 400, 128, "br", 0, True),     # 12 rows with a mask
    (2, 6, 2, 5, 129, 64, "br", 0, False),     # g = 3: 15 rows
])
def test_short_query_block_decode(gqa, B, Hq, Hkv, Sq, Sk, D, off, window, masked):
    bits, (q, k, v) = bf16_inputs(Sq * 100 + Sk, B, Hq, Hkv, Sq, Sk, D)
    plan = gqa.query(q, k, v, causal=off is not None,
                     causal_offset="bottom_right" if off else None, window=window)
    assert plan["kernel_name"] == "decode"
    mask = synth.mask_random(31, B, Sq, Sk, 0.5) if masked else None
    if masked:
        for i in range(Sq):
            mask[:, i, Sk - Sq + i] = 1
    out = gqa.forward(q, k, v, mask=torch.from_numpy(mask).cuda() if masked else None,
                      causal=off is not None, causal_offset="bottom_right" if off else None,
                      window=window)
    _status_ok(gqa)
    ref = oracle.forward(f64(bits[0]), f64(bits[1]), f64(bits[2]), mask=mask,
                         causal=off is not None, causal_offset=(Sk - Sq) if off else None,
                         window=window)
    assert_bf16_parity(to_np(out), ref, "short query decode")


def test_decode_many_groups_zeroes_its_counters(gqa):
    """16800 (batch, kv head) groups: more ticket counters than the workspace's
    counter region holds, so the call zeroes its own; sampled rows checked."""
    B, Hq, Hkv, Sk, D = 2100, 32, 8, 100, 128
    assert gqa.query(*(torch.empty(s, dtype=torch.bfloat16, device="cuda") for s in
                       ((B, Hq, 1, D), (B, Hkv, Sk, D), (B, Hkv, Sk, D))))["launches"] == 2
    bits, (q, k, v) = bf16_inputs(4400, B, Hq, Hkv, 1, Sk, D)
    for _ in range(2):  # twice: the counters must be clean for the second call too
        out = to_np(gqa.forward(q, k, v))
        _status_ok(gqa)
    for b in (0, 777, 2099):
        ref = oracle_bf16(bits[0][b:b + 1], bits[1][b:b + 1], bits[2][b:b + 1])
        assert_bf16_parity(out[b:b + 1], ref, "many groups b=%d" % b)


def test_default_workspaces_on_two_streams(gqa):
    """Decodes issued on two streams with the default arguments each get the
    workspace of their own stream: split groups merge correctly on both even
    when the launches overlap on the GPU."""
    dev = torch.device("cuda")
    cases = []
    for seed in (41, 42):
        (qb, kb, vb), (q, k, v) = bf16_inputs(seed, 2, 8, 2, 1, 8192, 128)
        cases.append(((qb, kb, vb), (q, k, v)))
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for s in streams:
        s.wait_stream(torch.cuda.current_stream())
    outs = [[], []]
    for _ in range(6):
        for i, s in enumerate(streams):
            with torch.cuda.stream(s):
                outs[i].append(gqa.forward(*cases[i][1]))
    torch.cuda.synchronize()
    ws = [gqa.workspace_for(dev, 256, s.cuda_stream) for s in streams]
    assert ws[0].data_ptr() != ws[1].data_ptr()
    for i, s in enumerate(streams):
        assert gqa.device_status(stream=s.cuda_stream) == 0
        ref = oracle_bf16(*cases[i][0])
        for o in outs[i]:
            assert_bf16_parity(to_np(o), ref, "stream %d" % i)
