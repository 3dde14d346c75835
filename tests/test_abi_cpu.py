"""The C-ABI library on a machine without a GPU: it loads, exports what
``include/gqa.h`` declares, validates arguments and plans without a device."""
import math
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def gqa():
    import grouped_query_attention_fwd_b200 as m
    return m


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "gqa.h")).read()
    return sorted(set(re.findall(r"GQA_API\s+[\w\s\*]+?\b(gqa_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(gqa):
    syms = _declared_symbols()
    assert set(syms) == set(gqa.EXPORTS)
    for s in syms:
        assert hasattr(gqa._lib, s), s


def test_status_strings(gqa):
    for code in range(0, 13):
        s = gqa.status_string(code)
        assert s and s != "unknown status"
    assert gqa.status_string(1234) == "unknown status"
    assert gqa.version() >= 10000


def _contig(B, H, S, D):
    return (H * S * D, S * D, D, 1)


def _p(gqa, B=2, Hq=8, Hkv=2, Sq=1, Sk=100, D=128, dtype=0, causal=False, mask=False,
       scale=None, **over):
    qs, ks, os_ = _contig(B, Hq, Sq, D), _contig(B, Hkv, Sk, D), _contig(B, Hq, Sq, D)
    ms = (Sq * Sk, Sk, 1) if mask else None
    p = gqa.make_problem(dtype, B, Hq, Hkv, Sq, Sk, D, over.pop("q_stride", qs),
                         over.pop("k_stride", ks), over.pop("v_stride", ks),
                         over.pop("o_stride", os_), over.pop("mask_stride", ms),
                         causal=causal, scale=scale)
    for k, v in over.items():
        setattr(p, k, v)
    return p


def _rc(gqa, p, sms=148):
    plan = gqa.Plan()
    import ctypes
    return gqa._lib.gqa_query(ctypes.byref(p), sms, ctypes.byref(plan)), plan


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=6, Hkv=4), 2),                       # Hq not a multiple of Hkv
    (dict(B=-1), 2),
    (dict(D=0), 2),
    (dict(Hkv=0), 2),
    (dict(D=100), 4),                             # bf16 / fp16: a multiple of 8
    (dict(D=136), 4),                             # bf16 / fp16: at most 128
    (dict(D=136, dtype=2), 4),
    (dict(D=300, dtype=1), 4),                    # fp32 path: D <= 256
    (dict(window=4), 8),                          # a window needs causal
    (dict(causal=True, window=-1), 8),
    (dict(scale=float("nan")), 8),
    (dict(scale=float("inf")), 8),
    (dict(dtype=7), 8),
    (dict(q_stride=(1024, 128, 128, 2)), 3),      # innermost stride != 1
    (dict(k_stride=(25600, 12804, 128, 1)), 3),   # bf16 stride not a multiple of 16 bytes
    (dict(mask=True, mask_stride=(100, 100, 2)), 3),
    (dict(Sq=4, Sk=4, Hq=129 * 2, Hkv=2), 4),     # prefill packs at most 128 heads per tile
])
def test_validation_errors(gqa, kw, code):
    rc, _ = _rc(gqa, _p(gqa, **kw))
    assert rc == code, (kw, rc, gqa.status_string(rc))


def test_null_arguments(gqa):
    import ctypes
    plan = gqa.Plan()
    assert gqa._lib.gqa_query(None, 148, ctypes.byref(plan)) == gqa.GQA_ERR_NULL
    assert gqa._lib.gqa_query(ctypes.byref(_p(gqa)), 148, None) == gqa.GQA_ERR_NULL
    assert gqa._lib.gqa_device_status(None, 0, None) == gqa.GQA_ERR_NULL


def test_plans_for_the_five_workloads(gqa):
    # page-1 toy, fp32
    rc, pl = _rc(gqa, _p(gqa, B=1, Hq=4, Hkv=2, Sq=5, Sk=5, D=4, dtype=1, scale=0.5))
    assert rc == 0 and gqa.KERNEL_NAMES[pl.kernel] == "f32"
    # decode, Mistral-7B-shaped layer
    rc, pl = _rc(gqa, _p(gqa, B=16, Hq=32, Hkv=8, Sq=1, Sk=4096, D=128))
    assert rc == 0 and gqa.KERNEL_NAMES[pl.kernel] == "decode"
    assert pl.algorithmic_bytes == 268697600
    assert pl.grid == 148 and pl.work_units == 16 * 8 * 32 and pl.launches == 1
    assert pl.workspace_bytes > 256 and pl.workspace_bytes % 256 == 0
    assert pl.smem_bytes <= 227 * 1024
    # long-context decode, Llama-2-70B-shaped layer
    rc, pl = _rc(gqa, _p(gqa, B=16, Hq=64, Hkv=8, Sq=1, Sk=32768, D=128))
    assert rc == 0 and pl.algorithmic_bytes == 2148007936
    assert math.isclose(pl.algorithmic_flops, 4 * 16 * 64 * 32768 * 128)
    # causal prefill
    rc, pl = _rc(gqa, _p(gqa, B=4, Hq=32, Hkv=8, Sq=4096, Sk=4096, D=128, causal=True))
    assert rc == 0 and gqa.KERNEL_NAMES[pl.kernel] == "prefill"
    assert math.isclose(pl.algorithmic_flops, 4 * 4 * 32 * 4096 * 4096 * 128 / 2)
    # padded-batch prefill with an explicit mask
    rc, pl = _rc(gqa, _p(gqa, B=8, Hq=12, Hkv=2, Sq=2048, Sk=2048, D=64, mask=True))
    assert rc == 0 and gqa.KERNEL_NAMES[pl.kernel] == "prefill"
    assert pl.algorithmic_bytes == 2 * 8 * 12 * 2048 * 64 * 2 + 2 * 8 * 2 * 2048 * 64 * 2 + 8 * 2048 * 2048


def test_short_query_blocks_decode(gqa):
    # g * Sq rows per kv head: up to 16 run on the decode stream in one pass.
    for (Hq, Hkv, Sq, kind) in ((8, 2, 4, "decode"), (8, 1, 2, "decode"), (4, 4, 16, "decode"),
                                (8, 2, 5, "prefill"), (16, 1, 2, "prefill")):
        rc, pl = _rc(gqa, _p(gqa, Hq=Hq, Hkv=Hkv, Sq=Sq, Sk=300))
        assert rc == 0 and gqa.KERNEL_NAMES[pl.kernel] == kind, (Hq, Hkv, Sq)


def test_decode_grid_small_problem(gqa):
    # Fewer 128-key tiles than SMs: one tile per CTA.
    rc, pl = _rc(gqa, _p(gqa, B=1, Hq=4, Hkv=1, Sq=1, Sk=300, D=64))
    assert rc == 0 and pl.work_units == 3 and pl.grid == 3
    # g > 8 uses 16-head passes.
    rc, pl = _rc(gqa, _p(gqa, B=1, Hq=40, Hkv=1, Sq=1, Sk=64, D=128))
    assert rc == 0 and pl.work_units == 3  # ceil(40 / 16) passes x 1 tile


def test_causal_offset_and_window_plans(gqa):
    # Causal with Sq != Sk is defined by the offset (bottom-right here); a short
    # query block (g * Sq <= 16 rows) stays on the decode stream.
    rc, pl = _rc(gqa, _p(gqa, Sq=3, Sk=5, causal=True, causal_offset=2))
    assert rc == 0 and gqa.KERNEL_NAMES[pl.kernel] == "decode"
    rc, pl = _rc(gqa, _p(gqa, Sq=5, Sk=9, causal=True, causal_offset=4))
    assert rc == 0 and gqa.KERNEL_NAMES[pl.kernel] == "prefill"
    # No query sees any key: NaN fill, no attention kernel.
    rc, pl = _rc(gqa, _p(gqa, Sq=4, Sk=8, causal=True, causal_offset=-4))
    assert rc == 0 and gqa.KERNEL_NAMES[pl.kernel] == "nan"
    rc, pl = _rc(gqa, _p(gqa, Sq=1, Sk=8, causal=True, causal_offset=20, window=4))
    assert rc == 0 and gqa.KERNEL_NAMES[pl.kernel] == "nan"
    # Decode with a sliding window streams only the window's tiles.
    rc, full = _rc(gqa, _p(gqa, B=1, Hq=8, Hkv=2, Sq=1, Sk=4096, causal=True, causal_offset=4095))
    rc2, win = _rc(gqa, _p(gqa, B=1, Hq=8, Hkv=2, Sq=1, Sk=4096, causal=True, causal_offset=4095,
                           window=256))
    assert rc == rc2 == 0 and full.work_units == 2 * 32 and win.work_units == 2 * 2


def test_binding_offset_rules(gqa):
    assert gqa._offset(False, None, 3, 5) == 0
    assert gqa._offset(True, None, 4, 4) == 0
    assert gqa._offset(True, "bottom_right", 3, 5) == 2
    assert gqa._offset(True, "top_left", 3, 5) == 0
    with pytest.raises(ValueError):
        gqa._offset(True, None, 3, 5)


def test_empty_problems(gqa):
    rc, pl = _rc(gqa, _p(gqa, B=0))
    assert rc == 0 and gqa.KERNEL_NAMES[pl.kernel] == "none"
    rc, pl = _rc(gqa, _p(gqa, Sq=0, Sk=10))
    assert rc == 0 and gqa.KERNEL_NAMES[pl.kernel] == "none"
    rc, pl = _rc(gqa, _p(gqa, Sq=3, Sk=0))
    assert rc == 0 and gqa.KERNEL_NAMES[pl.kernel] == "zero"


def test_no_device_is_an_error_not_a_fallback(gqa):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    rc, _ = _rc(gqa, _p(gqa), sms=0)
    assert rc == gqa.GQA_ERR_DEVICE
    with pytest.raises(gqa.GQAError) as ei:
        gqa.forward_ptrs(_p(gqa), 16, 16, 16, None, 16, 256, 1 << 20, 0)
    assert ei.value.status == gqa.GQA_ERR_DEVICE
    with pytest.raises(ValueError):
        gqa.forward(torch.zeros(1, 2, 1, 64), torch.zeros(1, 1, 3, 64), torch.zeros(1, 1, 3, 64))


# ------------------------------------------------------------ ragged caches and append

def test_ragged_plans(gqa):
    """With kv_lens the decode plan covers the whole capacity (the kernel cuts
    the real units on the device) and reserves shared memory for the lengths."""
    fake = 1 << 20  # never dereferenced by gqa_query
    rc, uni = _rc(gqa, _p(gqa, B=16, Hq=32, Hkv=8, Sq=1, Sk=4096))
    rc2, rag = _rc(gqa, _p(gqa, B=16, Hq=32, Hkv=8, Sq=1, Sk=4096, kv_lens=fake))
    assert rc == rc2 == 0
    assert gqa.KERNEL_NAMES[rag.kernel] == "decode"
    assert rag.work_units == uni.work_units == 16 * 8 * 32
    assert rag.smem_bytes >= uni.smem_bytes + 8 * 16
    assert rag.smem_bytes <= 227 * 1024
    # Many sequences: the ring gives up stages to keep the lengths resident.
    rc, big = _rc(gqa, _p(gqa, B=8000, Hq=8, Hkv=1, Sq=1, Sk=256, kv_lens=fake))
    assert rc == 0 and big.smem_bytes <= 227 * 1024
    rc, _ = _rc(gqa, _p(gqa, B=20000, Hq=8, Hkv=1, Sq=1, Sk=256, kv_lens=fake))
    assert rc == gqa.GQA_ERR_UNSUPPORTED
    # Prefill and fp32 take lengths too.
    rc, pf = _rc(gqa, _p(gqa, B=2, Hq=8, Hkv=2, Sq=300, Sk=1000, causal=True,
                         causal_offset=700, kv_lens=fake))
    assert rc == 0 and gqa.KERNEL_NAMES[pf.kernel] == "prefill"
    rc, f = _rc(gqa, _p(gqa, dtype=1, D=40, kv_lens=fake))
    assert rc == 0 and gqa.KERNEL_NAMES[f.kernel] == "f32"


def _append(gqa, B=2, H=2, cap=100, D=128, n=1, dtype=0, **over):
    c = (H * cap * D, cap * D, D, 1)
    nw = (H * n * D, n * D, D, 1)
    d = gqa.append_desc(dtype, B, H, cap, D, n, over.pop("ck", c), over.pop("cv", c),
                        over.pop("kn", nw), over.pop("vn", nw))
    for k, v in over.items():
        setattr(d, k, v)
    return d


def _append_rc(gqa, d, ptr=256, lens=256, ws=256, wsb=256):
    import ctypes
    return gqa._lib.gqa_kv_append(ctypes.byref(d), ptr, ptr, ptr, ptr, lens, ws, wsb, None)


@pytest.mark.parametrize("over,code", [
    (dict(dtype=7), 8),
    (dict(reserved=1), 8),
    (dict(batch=-1), 2),
    (dict(heads_kv=0), 2),
    (dict(head_dim=0), 2),
    (dict(n_new=-1), 2),
    (dict(n_new=101), 2),
    (dict(ck=(100 * 2 * 128, 100 * 128, 128, 2)), 3),
    (dict(vn=(-1, 128, 128, 1)), 3),
])
def test_append_validation(gqa, over, code):
    assert _append_rc(gqa, _append(gqa, **over)) == code


def test_append_nulls_and_workspace(gqa):
    d = _append(gqa)
    assert _append_rc(gqa, d, lens=None) == gqa.GQA_ERR_NULL
    assert _append_rc(gqa, d, ptr=None) == gqa.GQA_ERR_NULL
    assert _append_rc(gqa, d, ws=None) == gqa.GQA_ERR_WORKSPACE
    assert _append_rc(gqa, d, ws=128) == gqa.GQA_ERR_WORKSPACE
    assert _append_rc(gqa, d, wsb=64) == gqa.GQA_ERR_WORKSPACE
    assert _append_rc(gqa, d, ptr=257) == gqa.GQA_ERR_LAYOUT  # bf16 rows need 2-byte alignment
    assert _append_rc(gqa, _append(gqa, dtype=1), ptr=258) == gqa.GQA_ERR_LAYOUT
    # Nothing to append: OK without touching the device.
    assert _append_rc(gqa, _append(gqa, B=0)) == gqa.GQA_OK
    assert _append_rc(gqa, _append(gqa, n=0)) == gqa.GQA_OK


def test_workspace_layout_keeps_counters_apart(gqa):
    """Decode counters live in a fixed region after the 256-byte head; every
    other scratch starts past it, so a workspace shared by calls of any shape
    never needs clearing.  Huge decode problems keep their counters past the
    region and zero them per call (one extra launch)."""
    region = 256 + 64 * 1024
    rc, dec = _rc(gqa, _p(gqa, B=16, Hq=32, Hkv=8, Sq=1, Sk=4096))
    assert rc == 0 and dec.workspace_bytes > region and dec.launches == 1
    rc, pre = _rc(gqa, _p(gqa, B=2, Hq=8, Hkv=2, Sq=300, Sk=300, mask=True))
    # after it: the tile classes [B][m_tiles][n_tiles], then (256-aligned) the
    # key-tile bounds of every query tile (two int32), then the item order of
    # the two-tile kernel, one int32 per pair of query tiles
    # (g = 4: 32 query positions per tile, 10 query tiles, 3 key tiles)
    classes_end = (region + 2 * 10 * 3 + 255) // 256 * 256
    bounds_end = (classes_end + 2 * 10 * 8 + 255) // 256 * 256
    assert rc == 0 and pre.launches == 3
    assert pre.workspace_bytes == (bounds_end + 2 * 2 * 5 * 4 + 255) // 256 * 256
    rc, huge = _rc(gqa, _p(gqa, B=2100, Hq=32, Hkv=8, Sq=1, Sk=100))
    assert rc == 0 and huge.launches == 2 and huge.workspace_bytes > region + 2100 * 8 * 4


def test_half_dtypes_and_head_dims(gqa):
    """fp16 takes the bf16 kernels; any multiple of 8 up to 128 is accepted and
    planned at the padded width (64 or 128)."""
    for dtype in (0, 2):
        for D in (8, 24, 64, 72, 96, 128):
            rc, pl = _rc(gqa, _p(gqa, D=D, dtype=dtype))
            assert rc == 0 and gqa.KERNEL_NAMES[pl.kernel] == "decode", (dtype, D)
            rc, pl = _rc(gqa, _p(gqa, D=D, dtype=dtype, Sq=300, Sk=300, causal=True))
            assert rc == 0 and gqa.KERNEL_NAMES[pl.kernel] == "prefill", (dtype, D)
            # algorithmic bytes count the real head dim
            rc, pl = _rc(gqa, _p(gqa, B=1, Hq=2, Hkv=1, Sq=1, Sk=10, D=D, dtype=dtype))
            assert pl.algorithmic_bytes == 2 * (2 * D * 2) + 2 * (10 * D * 2)


def test_paged_validation(gqa):
    fake = 1 << 20
    base = dict(B=4, Hq=32, Hkv=8, Sq=1, Sk=1024, block_table=fake, block_table_stride=8,
                num_pages=100, kv_lens=fake)
    # pool strides over (page, kv head, key in page, d)
    pool = (8 * 128 * 128, 128 * 128, 128, 1)
    rc, pl = _rc(gqa, _p(gqa, **base, page_size=128, k_stride=pool, v_stride=pool))
    assert rc == 0 and gqa.KERNEL_NAMES[pl.kernel] == "decode"
    assert _rc(gqa, _p(gqa, **base, page_size=96, k_stride=pool, v_stride=pool))[0] == 2
    assert _rc(gqa, _p(gqa, **dict(base, Sk=1025), page_size=128, k_stride=pool,
                       v_stride=pool))[0] == 2        # more keys than the table can address
    assert _rc(gqa, _p(gqa, **dict(base, num_pages=0), page_size=128, k_stride=pool,
                       v_stride=pool))[0] == 2
    # the prefill path reads pages too
    rc, pl = _rc(gqa, _p(gqa, **dict(base, Sq=300, causal=True, causal_offset=724),
                         page_size=128, k_stride=pool, v_stride=pool))
    assert rc == 0 and gqa.KERNEL_NAMES[pl.kernel] == "prefill"
    # fp32 gathers through the table too
    rc, pl = _rc(gqa, _p(gqa, **base, page_size=128, dtype=1, k_stride=pool, v_stride=pool))
    assert rc == 0 and gqa.KERNEL_NAMES[pl.kernel] == "f32"


def test_paged_append_validation(gqa):
    d = _append(gqa, cap=1024)
    d.block_table, d.block_table_stride, d.page_size, d.num_pages = 256, 4, 128, 16
    assert _append_rc(gqa, d) == gqa.GQA_ERR_SHAPE   # 4 pages of 128 < capacity 1024


@pytest.mark.parametrize("Sq,lens,causal", [(5, [7, 3, 5, 0], True), (4, [6, 2], False),
                                            (1, [9], True), (8, [8, 20], True)])
def test_bench_visible_pairs_brute_force(Sq, lens, causal):
    """The bench's FLOP count for prefill over per-sequence lengths counts the
    (query, key) pairs the oracle's bottom-right causal rule leaves visible."""
    import bench
    brute = 0
    for n in lens:
        for i in range(Sq):
            for j in range(n):
                brute += (not causal) or (j <= i + n - Sq)
    assert bench.visible_pairs(Sq, lens, causal) == brute
    if causal and all(n >= Sq for n in lens):  # the closed form used in the docs
        assert brute == sum(Sq * n - Sq * (Sq - 1) // 2 for n in lens)
