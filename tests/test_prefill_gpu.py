"""tcgen05 prefill kernel vs the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import synth

from gpu_util import (assert_bf16_parity, bf16_inputs, bf16_round, bits_to_dev, f64, oracle_bf16,
                      oracle_rows_threaded, rel_rms, to_np)

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


def _mask(kind, seed, B, Sq, Sk, causal):
    if kind is None:
        return None
    if kind == "random":
        m = synth.mask_random(seed, B, Sq, Sk, 0.5)
    else:
        lens = synth.uniform_int(seed, synth.STREAM_MASK, B, 1, Sk)
        m = synth.mask_from_lengths(lens, Sq, Sk)
    if causal:  # keep the diagonal so that no row is fully hidden
        for i in range(min(Sq, Sk)):
            m[:, i, i] = 1
    return m


PREFILL_CASES = [
    # B, Hq, Hkv, Sq, Sk, D, causal, mask
    (1, 8, 2, 200, 200, 128, True, None),        # g=4: 32 queries x 4 heads per tile
    (1, 8, 2, 200, 200, 128, False, None),
    (2, 12, 2, 150, 300, 64, False, "random"),   # g=6: 21 x 6 = 126 rows + 2 pad
    (1, 4, 4, 130, 130, 128, False, None),       # g=1 (MHA): 128 queries per tile
    (2, 8, 1, 64, 64, 128, True, None),          # g=8 (MQA-like): 16 queries per tile
    (1, 6, 2, 77, 513, 64, False, None),         # g=3: 42 x 3 = 126 rows
    (1, 16, 1, 9, 257, 128, False, None),        # g=16: 8 queries per tile
    (1, 128, 1, 5, 100, 64, False, None),        # g=128: one query per tile
    (2, 8, 2, 256, 256, 128, True, "random"),    # causal and mask together
    (1, 4, 2, 3, 1, 64, False, None),            # one key
    (1, 4, 2, 2, 2, 128, True, None),            # smallest causal prefill
    (3, 12, 2, 300, 300, 64, False, "lengths"),  # right-padded batch
    (2, 32, 8, 384, 384, 128, True, None),       # several 128-key tiles, exact multiple
    (1, 8, 2, 129, 1000, 128, False, "lengths"),
]


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D,causal,mask_kind", PREFILL_CASES)
def test_prefill_parity(gqa, B, Hq, Hkv, Sq, Sk, D, causal, mask_kind):
    seed = 1000 + Sq + Sk + Hq
    bits, (q, k, v) = bf16_inputs(seed, B, Hq, Hkv, Sq, Sk, D)
    mask = _mask(mask_kind, seed, B, Sq, Sk, causal)
    out = gqa.forward(q, k, v, mask=torch.from_numpy(mask).cuda() if mask is not None else None,
                      causal=causal)
    _status_ok(gqa)
    ref = oracle_bf16(*bits, mask=mask, causal=causal)
    assert_bf16_parity(to_np(out), ref, "prefill %s" % ((B, Hq, Hkv, Sq, Sk, D, causal, mask_kind),))


def test_prefill_strided_bshd(gqa):
    B, Hq, Hkv, S, D = 2, 8, 2, 160, 128
    qb, kb, vb = synth.qkv_bf16_bits(21, B, Hq, Hkv, S, S, D)
    q = bits_to_dev(qb.transpose(0, 2, 1, 3).copy()).transpose(1, 2)
    k = bits_to_dev(kb.transpose(0, 2, 1, 3).copy()).transpose(1, 2)
    v = bits_to_dev(vb.transpose(0, 2, 1, 3).copy()).transpose(1, 2)
    out = torch.empty(B, S, Hq, D, dtype=torch.bfloat16, device="cuda").transpose(1, 2)
    gqa.forward(q, k, v, out=out, causal=True)
    _status_ok(gqa)
    assert_bf16_parity(to_np(out), oracle_bf16(qb, kb, vb, causal=True), "prefill strided")


def test_prefill_determinism_and_scale(gqa):
    bits, (q, k, v) = bf16_inputs(22, 2, 8, 2, 300, 300, 128)
    a = gqa.forward(q, k, v, causal=True, scale=0.05)
    b = gqa.forward(q, k, v, causal=True, scale=0.05)
    _status_ok(gqa)
    assert torch.equal(a, b)
    assert_bf16_parity(to_np(a), oracle_bf16(*bits, causal=True, scale=0.05), "prefill scale")


def test_prefill_large_scores_rescale(gqa):
    """Scores that grow along the keys force the lazy O rescale path."""
    B, Hq, Hkv, S, D = 1, 8, 2, 512, 64
    qb, kb, vb = synth.qkv_bf16_bits(23, B, Hq, Hkv, S, S, D)
    ramp = np.linspace(0.0, 6.0, S, dtype=np.float32)[None, None, :, None]
    kf = (synth.bf16_bits_to_f64(kb).astype(np.float32) + ramp).astype(np.float32)
    kb2 = synth.round_bf16_bits(kf)
    q, k, v = bits_to_dev(qb), bits_to_dev(kb2), bits_to_dev(vb)
    out = gqa.forward(q, k, v, scale=1.0)
    _status_ok(gqa)
    assert_bf16_parity(to_np(out), oracle_bf16(qb, kb2, vb, scale=1.0), "prefill rescale")


@pytest.mark.parametrize("D", [128, 64])
def test_prefill_fully_hidden_rows_are_nan(gqa, D):
    """Rows with no visible key come out NaN, the others match the oracle.  At
    head dim 64 part of the exponentials run as a polynomial that gives 2^-126,
    not 0, for a hidden key, so this also checks that an empty row is told by
    its running maximum."""
    bits, (q, k, v) = bf16_inputs(24 + D, 2, 8, 2, 70, 300, D)
    mask = np.ones((2, 70, 300), dtype=np.uint8)
    mask[1, 5, :] = 0          # one hidden row
    mask[0, 40:70, :] = 0      # a whole query tile hidden (no key tile visited)
    out = to_np(gqa.forward(q, k, v, mask=torch.from_numpy(mask).cuda()))
    _status_ok(gqa)
    assert np.all(np.isnan(out[1, :, 5])) and np.all(np.isnan(out[0, :, 40:70]))
    ok = np.ones(out.shape[:3], dtype=bool)
    ok[1, :, 5] = False
    ok[0, :, 40:70] = False
    ref = oracle_bf16(*bits, mask=mask)
    assert np.all(np.isfinite(out[ok]))
    assert_bf16_parity(out[ok], ref[ok], "prefill visible rows")


# ------------------------------------------------------------ full size

def _full_size(gqa, seed, B, Hq, Hkv, S, D, causal, mask_lens, whole):
    """One full-size workload: every output row of the (b, kv) group `whole`,
    and from every other (b, kv) group one row of every query tile of the
    kernel (qpt = 128 // g query positions per tile), against the oracle."""
    bits, (q, k, v) = bf16_inputs(seed, B, Hq, Hkv, S, S, D)
    mask = None
    if mask_lens:
        lens = synth.uniform_int(seed, synth.STREAM_MASK, B, 256, S)
        mask = synth.mask_from_lengths(lens, S, S)
    out = to_np(gqa.forward(q, k, v, causal=causal,
                            mask=torch.from_numpy(mask).cuda() if mask is not None else None))
    _status_ok(gqa)
    qb, kb, vb = bits
    g = Hq // Hkv
    qpt = 128 // g
    m_tiles = -(-S // qpt)
    got, ref, tiles_seen = [], [], set()
    for b in range(B):
        for kv in range(Hkv):
            if (b, kv) == whole:
                rows = [(hh, i) for hh in range(g) for i in range(S)]
            else:
                rows = []
                for mt in range(m_tiles):
                    hh = (mt + 3 * b + kv) % g
                    i = min(S - 1, mt * qpt + (7 * mt + b + 5 * kv) % qpt)
                    rows.append((hh, i))
                    tiles_seen.add((b, kv, i // qpt))
            qs = f64(qb[b:b + 1, kv * g:(kv + 1) * g])
            ks, vs = f64(kb[b:b + 1, kv:kv + 1]), f64(vb[b:b + 1, kv:kv + 1])
            ms = mask[b:b + 1] if mask is not None else None
            ref.append(oracle_rows_threaded(qs, ks, vs, [(0, hh, i) for (hh, i) in rows],
                                            mask=ms, causal=causal))
            got.append(np.stack([out[b, kv * g + hh, i] for (hh, i) in rows]))
    assert len(tiles_seen) == (B * Hkv - 1) * m_tiles
    return np.concatenate(got), np.concatenate(ref)


def _report(name, got, ref):
    """The parity bar, plus the diagnostic split of the error: against the
    unrounded oracle (what the bar checks) and against the oracle rounded to
    bf16 (the error left once the output rounding is taken out)."""
    max_abs, rr = assert_bf16_parity(got, ref, name)
    rr_rounded = rel_rms(got, bf16_round(ref))
    print("%s: rows %d, max_abs %.3e, rel_rms %.3e (vs oracle rounded to bf16: %.3e)"
          % (name, got.shape[0], max_abs, rr, rr_rounded))


def test_prefill_causal_full_size(gqa):
    """B=4, Hq=32, Hkv=8, S=4096, D=128, causal: one whole (b, kv) group (4 heads
    x 4096 rows) element by element, and a row of every query tile of every
    other group."""
    got, ref = _full_size(gqa, 4, 4, 32, 8, 4096, 128, True, False, whole=(1, 3))
    _report("causal prefill full size", got, ref)


def test_prefill_masked_full_size(gqa):
    """B=8, Hq=12, Hkv=2, S=2048, D=64, padding mask len_b ~ U[256, 2048]: one
    whole (b, kv) group (6 heads x 2048 rows) and a row of every query tile of
    every other group."""
    got, ref = _full_size(gqa, 5, 8, 12, 2, 2048, 64, False, True, whole=(5, 1))
    _report("masked prefill full size", got, ref)


# ----------------------------------------------- causal offset and sliding window

@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D,off,window,mask_kind", [
    (1, 8, 2, 200, 700, 128, 500, 0, None),       # bottom-right causal, query block at the end
    (2, 8, 2, 600, 600, 128, 0, 256, None),       # sliding window of 256 keys
    (1, 12, 2, 300, 900, 64, 600, 130, "random"), # bottom-right + window + mask, g = 6
    (1, 8, 2, 130, 130, 128, -3, 0, None),        # first three rows see nothing: NaN
    (2, 32, 8, 256, 2048, 128, 1792, 1000, None), # several key tiles, window > tile
])
def test_prefill_offset_window(gqa, B, Hq, Hkv, Sq, Sk, D, off, window, mask_kind):
    seed = 2000 + Sq + Sk + window
    bits, (q, k, v) = bf16_inputs(seed, B, Hq, Hkv, Sq, Sk, D)
    mask = synth.mask_random(seed, B, Sq, Sk, 0.6) if mask_kind else None
    if mask is not None:  # keep the diagonal key visible
        for i in range(Sq):
            if 0 <= i + off < Sk:
                mask[:, i, i + off] = 1
    out = to_np(gqa.forward(q, k, v, mask=torch.from_numpy(mask).cuda() if mask is not None else None,
                            causal=True, causal_offset=off, window=window))
    _status_ok(gqa)
    ref = oracle.forward(f64(bits[0]), f64(bits[1]), f64(bits[2]), mask=mask, causal=True,
                         causal_offset=off, window=window)
    nan_ref = np.isnan(ref).all(axis=-1)
    assert np.array_equal(np.isnan(out).all(axis=-1), nan_ref)
    assert_bf16_parity(out[~nan_ref], ref[~nan_ref], "prefill offset/window")


def test_prefill_long_keys_one_tile(gqa):
    """Keys past 1024 tiles (131072) per item: plans take the one-query-tile
    kernel (its work units are single query tiles).  Contiguous cache with a
    bottom-right causal block, then a ragged batch in 64-key pages of a pool
    that is NaN outside the valid rows."""
    import test_paged_gpu as pg
    # contiguous, bottom-right causal (g = 4: 32 queries per tile)
    B, Hq, Hkv, Sq, Sk, D = 1, 4, 1, 40, 132000, 64
    bits, (q, k, v) = bf16_inputs(7100, B, Hq, Hkv, Sq, Sk, D)
    plan = gqa.query(q, k, v, causal=True, causal_offset="bottom_right")
    m_tiles = -(-Sq // 32)
    assert plan["kernel_name"] == "prefill" and plan["work_units"] == B * Hkv * m_tiles
    out = to_np(gqa.forward(q, k, v, causal=True, causal_offset="bottom_right"))
    _status_ok(gqa)
    ref = oracle.forward(f64(bits[0]), f64(bits[1]), f64(bits[2]), causal=True,
                         causal_offset=Sk - Sq)
    assert_bf16_parity(out, ref, "prefill, 132000 keys, one query tile per SM")
    # ragged and paged: capacity 2100 pages of 64 keys, lengths 134000 and 5000
    B, Hq, Hkv, Sq, D, ps, per_seq = 2, 4, 1, 64, 64, 64, 2100
    lens = np.array([134000, 5000], dtype=np.int32)
    kc, vc, kd, vd, table = pg._paged(7200, B, Hkv, D, ps, per_seq, lens, "bf16")
    qh, qd = pg._q(7200, B, Hq, Sq, D, "bf16")
    cap = ps * per_seq
    plan = gqa.query(qd, kd, vd, causal=True, causal_offset="bottom_right",
                     kv_lens=torch.from_numpy(lens).cuda(), block_table=table)
    assert plan["work_units"] == B * Hkv * 2  # two query tiles of 32 positions
    out = to_np(gqa.forward(qd, kd, vd, causal=True, causal_offset="bottom_right",
                            kv_lens=torch.from_numpy(lens).cuda(), block_table=table))
    _status_ok(gqa)
    ref = oracle.forward(qh, kc, vc, causal=True, causal_offset=cap - Sq, kv_lens=lens)
    pg._check_nan_rows(out, ref, "paged prefill, 134000 keys, one query tile per SM")
