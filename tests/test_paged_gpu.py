"""Paged KV caches (a page pool and a block table per sequence), through the
C ABI, against the fp64 oracle on the same values gathered into a contiguous
cache.  The pools start as NaN everywhere except the rows of valid keys, so
any read of a row past a sequence's length that reached the result would show."""
import numpy as np
import pytest
import torch

import oracle
import synth

from gpu_util import assert_bf16_parity, bits_to_dev, f64, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gqa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import grouped_query_attention_fwd_b200 as m
    return m


def _paged(seed, B, Hkv, D, page_size, per_seq, lens, dtype, spare=7):
    """Contiguous K/V [B, Hkv, cap, D] (finite, zero past each length), a pool
    [num_pages, Hkv, page_size, D] holding the valid rows in shuffled pages and
    NaN elsewhere, and the block table (-1 for pages no key uses)."""
    cap = per_seq * page_size
    if dtype == "bf16":
        kb, vb = synth.qkv_bf16_bits(seed, B, Hkv, Hkv, cap, cap, D)[1:]
        kc, vc = f64(kb), f64(vb)
    else:
        k32, v32 = synth.qkv_f32(seed, B, Hkv, Hkv, cap, cap, D)[1:]
        np_t = np.float16 if dtype == "f16" else np.float32
        kc, vc = k32.astype(np_t).astype(np.float64), v32.astype(np_t).astype(np.float64)
    for b in range(B):
        kc[b, :, lens[b]:] = 0.0
        vc[b, :, lens[b]:] = 0.0
    used = [(b, i) for b in range(B) for i in range(-(-int(lens[b]) // page_size))]
    num_pages = len(used) + spare
    rng = np.random.default_rng(seed)
    perm = rng.permutation(num_pages)
    table = np.full((B, per_seq), -1, dtype=np.int32)
    kp = np.full((num_pages, Hkv, page_size, D), np.nan)
    vp = np.full((num_pages, Hkv, page_size, D), np.nan)
    for n, (b, i) in enumerate(used):
        page = int(perm[n])
        table[b, i] = page
        hi = min(page_size, int(lens[b]) - i * page_size)
        kp[page, :, :hi] = kc[b, :, i * page_size:i * page_size + hi]
        vp[page, :, :hi] = vc[b, :, i * page_size:i * page_size + hi]
    tdt = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[dtype]
    kd = torch.from_numpy(kp).to(tdt).cuda()
    vd = torch.from_numpy(vp).to(tdt).cuda()
    return kc, vc, kd, vd, torch.from_numpy(table).cuda()


def _q(seed, B, Hq, Sq, D, dtype):
    q32 = synth.qkv_f32(seed + 1, B, Hq, Hq, Sq, 1, D)[0]
    tdt = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[dtype]
    qd = torch.from_numpy(q32).to(tdt).cuda()
    return qd.double().cpu().numpy(), qd


@pytest.mark.parametrize("page_size", [64, 128, 256])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_paged_decode(gqa, page_size, dtype):
    B, Hq, Hkv, D, per_seq = 6, 32, 8, 128, 4096 // page_size
    lens = np.array([4096, 1, 63, 64, 65, 0], dtype=np.int32)
    lens[1:] = np.minimum(lens[1:], per_seq * page_size)
    kc, vc, kd, vd, table = _paged(6000 + page_size, B, Hkv, D, page_size, per_seq, lens, dtype)
    q, qd = _q(6000, B, Hq, 1, D, dtype)
    dl = torch.from_numpy(lens).cuda()
    out = to_np(gqa.forward(qd, kd, vd, kv_lens=dl, block_table=table))
    assert gqa.device_status() == 0
    ref = oracle.forward(q, kc, vc, kv_lens=lens)
    nan_ref = np.isnan(ref).all(axis=-1)
    assert np.array_equal(np.isnan(out).all(axis=-1), nan_ref)   # only the empty sequence
    assert_bf16_parity(out[~nan_ref], ref[~nan_ref], "paged decode ps=%d %s" % (page_size, dtype))


def test_paged_short_query_block(gqa):
    """Three new queries per sequence at the end of each (bottom-right causal),
    g = 4: (head, query) rows, D = 96, fp16."""
    B, Hq, Hkv, Sq, D, ps, per_seq = 3, 16, 4, 3, 96, 64, 12
    lens = np.array([700, 3, 130], dtype=np.int32)
    kc, vc, kd, vd, table = _paged(6100, B, Hkv, D, ps, per_seq, lens, "f16")
    q, qd = _q(6100, B, Hq, Sq, D, "f16")
    dl = torch.from_numpy(lens).cuda()
    cap = per_seq * ps
    out = to_np(gqa.forward(qd, kd, vd, causal=True, causal_offset="bottom_right", kv_lens=dl,
                            block_table=table))
    assert gqa.device_status() == 0
    ref = oracle.forward(q, kc, vc, causal=True, causal_offset=cap - Sq, kv_lens=lens)
    assert_bf16_parity(out, ref, "paged short query block")


def _check_nan_rows(out, ref, what):
    nan_ref = np.isnan(ref).all(axis=-1)
    assert np.array_equal(np.isnan(out).all(axis=-1), nan_ref), what
    assert_bf16_parity(out[~nan_ref], ref[~nan_ref], what)


@pytest.mark.parametrize("page_size,dtype,D", [(64, "bf16", 128), (128, "f16", 128),
                                               (256, "bf16", 64), (64, "f16", 96)])
def test_paged_prefill(gqa, page_size, dtype, D):
    """A block of new queries at the end of each sequence (bottom-right
    causal) on the prefill path, the cache in shuffled pages of a pool that is
    NaN outside the valid rows."""
    B, Hq, Hkv, Sq = 3, 16, 4, 100
    per_seq = 1024 // page_size
    lens = np.array([1024, 333, 129], dtype=np.int32)
    kc, vc, kd, vd, table = _paged(6800 + page_size + D, B, Hkv, D, page_size, per_seq, lens,
                                   dtype)
    q, qd = _q(6800 + D, B, Hq, Sq, D, dtype)
    cap = per_seq * page_size
    out = to_np(gqa.forward(qd, kd, vd, causal=True, causal_offset="bottom_right",
                            kv_lens=torch.from_numpy(lens).cuda(), block_table=table))
    assert gqa.device_status() == 0
    ref = oracle.forward(q, kc, vc, causal=True, causal_offset=cap - Sq, kv_lens=lens)
    _check_nan_rows(out, ref, "paged prefill ps=%d %s D=%d" % (page_size, dtype, D))


def test_paged_prefill_full_cache_non_causal(gqa):
    """No lengths: every key of the capacity is in use, non-causal, g = 6."""
    B, Hq, Hkv, Sq, D, ps, per_seq = 2, 12, 2, 150, 128, 128, 5
    cap = ps * per_seq
    lens = np.full(B, cap, dtype=np.int32)
    kc, vc, kd, vd, table = _paged(6900, B, Hkv, D, ps, per_seq, lens, "bf16")
    q, qd = _q(6900, B, Hq, Sq, D, "bf16")
    out = to_np(gqa.forward(qd, kd, vd, block_table=table))
    assert gqa.device_status() == 0
    assert_bf16_parity(out, oracle.forward(q, kc, vc), "paged prefill, full cache")


@pytest.mark.parametrize("Sq,causal", [(150, False), (150, True), (1, False), (3, True)])
def test_paged_capacity_not_a_page_multiple(gqa, Sq, causal):
    """A block table without lengths and seq_k = 600 (not a multiple of the
    128-key page or tile): keys 600..639 of the last page hold NaN in the pool
    and must not reach the result, causal (bottom-right) or not."""
    B, Hq, Hkv, D, ps, per_seq, Sk = 2, 12, 2, 128, 128, 5, 600
    lens = np.full(B, Sk, dtype=np.int32)
    kc, vc, kd, vd, table = _paged(7100 + Sq, B, Hkv, D, ps, per_seq, lens, "bf16")
    q, qd = _q(7100 + Sq, B, Hq, Sq, D, "bf16")
    out = torch.empty_like(qd)
    p = gqa.problem_for(qd, kd, vd, causal=causal, out=out,
                        causal_offset=(Sk - Sq) if causal else None, block_table=table)
    p.seq_k = Sk
    plan = gqa.query_problem(p)
    ws = gqa.workspace_for(qd.device, plan.workspace_bytes)
    gqa.forward_ptrs(p, qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), None, out.data_ptr(),
                     ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
    assert gqa.device_status() == 0
    ref = oracle.forward(q, kc[:, :, :Sk], vc[:, :, :Sk], causal=causal,
                         causal_offset=(Sk - Sq) if causal else None)
    assert_bf16_parity(to_np(out), ref, "paged, seq_k %d, Sq %d, causal %s" % (Sk, Sq, causal))


def test_paged_prefill_bad_page_is_reported(gqa):
    B, Hq, Hkv, Sq, D, ps, per_seq = 2, 8, 2, 64, 64, 64, 4
    lens = np.array([200, 150], dtype=np.int32)
    kc, vc, kd, vd, table = _paged(7000, B, Hkv, D, ps, per_seq, lens, "bf16")
    bad = table.clone()
    bad[1, 1] = -5                      # keys 64..127 of entry 1 are in use
    q, qd = _q(7000, B, Hq, Sq, D, "bf16")
    dl = torch.from_numpy(lens).cuda()
    gqa.forward(qd, kd, vd, causal=True, causal_offset="bottom_right", kv_lens=dl,
                block_table=bad)
    assert gqa.device_status() == gqa.GQA_ERR_PAGE
    gqa.forward(qd, kd, vd, causal=True, causal_offset="bottom_right", kv_lens=dl,
                block_table=table)
    assert gqa.device_status() == 0


def test_paged_f32(gqa):
    B, Hq, Hkv, D, ps, per_seq = 3, 8, 2, 40, 64, 5
    lens = np.array([320, 1, 100], dtype=np.int32)
    kc, vc, kd, vd, table = _paged(6200, B, Hkv, D, ps, per_seq, lens, "f32")
    q, qd = _q(6200, B, Hq, 2, D, "f32")
    out = gqa.forward(qd, kd, vd, kv_lens=torch.from_numpy(lens).cuda(),
                      block_table=table).cpu().numpy()
    assert gqa.device_status() == 0
    ref = oracle.forward(q, kc, vc, kv_lens=lens)
    assert np.abs(out - ref).max() <= 1e-5


def test_ragged_contiguous_nan_tail(gqa):
    """A contiguous cache whose rows past each length are NaN: the decode
    result must not see them."""
    B, Hq, Hkv, Sk, D = 3, 16, 4, 700, 128
    kb, vb = synth.qkv_bf16_bits(6300, B, Hkv, Hkv, Sk, Sk, D)[1:]
    kc, vc = f64(kb), f64(vb)
    lens = np.array([700, 129, 5], dtype=np.int32)
    kn, vn = kc.copy(), vc.copy()
    for b in range(B):
        kn[b, :, lens[b]:] = np.nan
        vn[b, :, lens[b]:] = np.nan
        kc[b, :, lens[b]:] = 0.0
        vc[b, :, lens[b]:] = 0.0
    q, qd = _q(6300, B, Hq, 1, D, "bf16")
    kd = torch.from_numpy(kn).to(torch.bfloat16).cuda()
    vd = torch.from_numpy(vn).to(torch.bfloat16).cuda()
    out = to_np(gqa.forward(qd, kd, vd, kv_lens=torch.from_numpy(lens).cuda()))
    assert gqa.device_status() == 0
    assert_bf16_parity(out, oracle.forward(q, kc, vc, kv_lens=lens), "NaN tail")


def test_paged_bad_page_is_reported(gqa):
    B, Hq, Hkv, D, ps, per_seq = 2, 8, 2, 64, 64, 4
    lens = np.array([200, 50], dtype=np.int32)
    kc, vc, kd, vd, table = _paged(6400, B, Hkv, D, ps, per_seq, lens, "bf16")
    bad = table.clone()
    bad[1, 0] = 10 ** 6                 # a page the pool does not have, for keys in use
    q, qd = _q(6400, B, Hq, 1, D, "bf16")
    gqa.forward(qd, kd, vd, kv_lens=torch.from_numpy(lens).cuda(), block_table=bad)
    assert gqa.device_status() == gqa.GQA_ERR_PAGE
    gqa.forward(qd, kd, vd, kv_lens=torch.from_numpy(lens).cuda(), block_table=table)
    assert gqa.device_status() == 0


def test_paged_append_then_decode(gqa):
    """Generation steps on a paged cache: append one token per sequence through
    the block table, then decode over the grown cache."""
    B, Hq, Hkv, D, ps, per_seq = 3, 16, 4, 128, 64, 4
    lens = np.array([63, 0, 128], dtype=np.int32)
    cap = ps * per_seq
    kc, vc, kd, vd, table = _paged(6500, B, Hkv, D, ps, per_seq, lens, "bf16", spare=0)
    # give every sequence all its pages up front (fresh ones start as NaN)
    tab = table.cpu().numpy()
    pool_pages = kd.shape[0]
    extra = []
    for b in range(B):
        for i in range(per_seq):
            if tab[b, i] < 0:
                tab[b, i] = pool_pages + len(extra)
                extra.append((b, i))
    nan_pages = torch.full((len(extra), Hkv, ps, D), float("nan"), dtype=torch.bfloat16,
                           device="cuda")
    kd = torch.cat([kd, nan_pages])
    vd = torch.cat([vd, nan_pages.clone()])
    table = torch.from_numpy(tab).cuda()
    dl = torch.from_numpy(lens.copy()).cuda()
    for step in range(3):
        knb, vnb = synth.qkv_bf16_bits(6600 + step, B, Hkv, Hkv, 1, 1, D)[1:]
        gqa.kv_append(kd, vd, bits_to_dev(knb), bits_to_dev(vnb), dl, block_table=table)
        for b in range(B):
            kc[b, :, lens[b]] = f64(knb)[b, :, 0]
            vc[b, :, lens[b]] = f64(vnb)[b, :, 0]
        lens += 1
        q, qd = _q(6700 + step, B, Hq, 1, D, "bf16")
        out = to_np(gqa.forward(qd, kd, vd, causal=True, causal_offset="bottom_right",
                                kv_lens=dl, block_table=table))
        assert gqa.device_status() == 0
        assert np.array_equal(dl.cpu().numpy(), lens)
        ref = oracle.forward(q, kc, vc, causal=True, causal_offset=cap - 1, kv_lens=lens)
        assert_bf16_parity(out, ref, "paged append step %d" % step)
