"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each check ties the oracle to something it does not contain: the shapes and
KV-cache figures the pages print, closed forms of softmax attention, exact
invariants, and PyTorch's own fp64 ``scaled_dot_product_attention`` (a library
routine whose ``enable_gqa`` mode implements the contiguous head grouping of
"28. Grouped-Query Attention (GQA)", "Step-by-Step Approach" step 2).  The last
test plants plausible mistakes in a copy of the oracle's C++ and checks that
some pin catches each one.
"""
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _sdpa(q, k, v, mask=None, causal=False, scale=None, gqa=True):
    """PyTorch's fp64 CPU attention; ``mask`` True = attend, broadcast over heads."""
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(x)) for x in (q, k, v))
    am = None
    if mask is not None:
        am = torch.from_numpy(np.array(mask, dtype=bool))[:, None, :, :]
    if causal:
        Sq, Sk = q.shape[2], k.shape[2]
        cm = torch.ones(Sq, Sk, dtype=torch.bool).tril()
        am = cm[None, None] if am is None else (am & cm[None, None])
    out = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=am, scale=scale,
                                         enable_gqa=gqa)
    return out.numpy()


# ---------------------------------------------------------------- page figures

def test_worked_example_shape(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "worked_example_shape.json")))
    rng = np.random.default_rng(0)
    q = _rand(rng, *g["q_shape"])
    kv = _rand(rng, *g["kv_shape"])
    out = oracle_mod.forward(q, kv, kv)
    assert list(out.shape) == g["out_shape"]
    assert np.all(np.isfinite(out))


def test_kv_cache_bytes_page_figures(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "kv_cache_figures.json")))
    for case in g["cases"]:
        b = oracle_mod.kv_cache_bytes(**case["args"])
        val = b / case["unit_bytes"]
        tol = case["tolerance_units"]
        if tol == 0.0:
            assert val == case["page_value"], case
        else:
            assert abs(val - case["page_value"]) <= tol, (case, val)


def test_kv_cache_bytes_ratios_and_configs(oracle_mod):
    kb = oracle_mod.kv_cache_bytes
    mha = kb(1, 32768, 64, 128, 16, 2)
    assert mha == 8 * kb(1, 32768, 8, 128, 16, 2) == 64 * kb(1, 32768, 1, 128, 16, 2)
    # One Llama-2-70B-shaped layer, 32k context, batch 16, bf16: 2 GiB of K+V.
    assert kb(1, 32768, 8, 128, 16, 2) == 2 * 1024 ** 3
    # Mistral-7B-shaped layer, 4096 tokens, batch 16, bf16.
    assert kb(1, 4096, 8, 128, 16, 2) == 268435456
    # Linear in every factor.
    assert kb(3, 5, 7, 11, 13, 2) == 2 * 3 * 5 * 7 * 11 * 13 * 2


# ---------------------------------------------------------- library routine

CASES = [
    # B, Hq, Hkv, Sq, Sk, D, mask_kind, causal
    (1, 4, 2, 5, 5, 4, None, False),
    (2, 6, 3, 7, 9, 8, None, False),
    (2, 8, 2, 6, 6, 16, None, True),
    (2, 6, 1, 4, 11, 8, "random", False),
    (1, 12, 2, 9, 9, 8, "random", True),
    (3, 4, 4, 3, 17, 5, "lengths", False),
    (1, 3, 1, 1, 13, 7, "random", False),
]


def _mask(kind, rng, B, Sq, Sk):
    if kind is None:
        return None
    if kind == "random":
        m = rng.random((B, Sq, Sk)) < 0.6
        m[np.arange(B)[:, None], np.arange(Sq)[None, :], 0] = True  # never a fully hidden row
        return m
    lens = rng.integers(1, Sk + 1, size=B)
    return np.arange(Sk)[None, None, :] < lens[:, None, None] + np.zeros((B, Sq, 1), dtype=int)


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D,mask_kind,causal", CASES)
def test_matches_torch_sdpa_fp64(oracle_mod, B, Hq, Hkv, Sq, Sk, D, mask_kind, causal):
    rng = np.random.default_rng(B * 1000 + Hq * 100 + Sk)
    q, k, v = _rand(rng, B, Hq, Sq, D), _rand(rng, B, Hkv, Sk, D), _rand(rng, B, Hkv, Sk, D)
    mask = _mask(mask_kind, rng, B, Sq, Sk)
    for scale in (None, 0.37):
        ours = oracle_mod.forward(q, k, v, mask=mask, causal=causal, scale=scale)
        ref = _sdpa(q, k, v, mask=mask, causal=causal,
                    scale=(1.0 / np.sqrt(D)) if scale is None else scale)
        np.testing.assert_allclose(ours, ref, rtol=1e-11, atol=1e-12)


def test_large_scores_stay_finite(oracle_mod):
    """Scores of order 1e3 (exp overflows in double) still give PyTorch's result."""
    rng = np.random.default_rng(4)
    q, k, v = _rand(rng, 1, 4, 5, 8) * 60.0, _rand(rng, 1, 2, 7, 8) * 60.0, _rand(rng, 1, 2, 7, 8)
    ours = oracle_mod.forward(q, k, v, scale=1.0)
    assert np.all(np.isfinite(ours))
    np.testing.assert_allclose(ours, _sdpa(q, k, v, scale=1.0), rtol=1e-11, atol=1e-12)


def test_mha_special_case_is_plain_mha(oracle_mod):
    """g = 1: the result is ordinary multi-head attention."""
    rng = np.random.default_rng(5)
    q, k, v = _rand(rng, 2, 4, 6, 8), _rand(rng, 2, 4, 9, 8), _rand(rng, 2, 4, 9, 8)
    ours = oracle_mod.forward(q, k, v)
    ref = _sdpa(q, k, v, gqa=False)
    np.testing.assert_allclose(ours, ref, rtol=1e-11, atol=1e-12)


def test_mqa_special_case(oracle_mod):
    """Hkv = 1: every query head attends over the single kv head."""
    rng = np.random.default_rng(6)
    q, k, v = _rand(rng, 2, 5, 4, 8), _rand(rng, 2, 1, 7, 8), _rand(rng, 2, 1, 7, 8)
    ours = oracle_mod.forward(q, k, v)
    ke, ve = np.broadcast_to(k, (2, 5, 7, 8)), np.broadcast_to(v, (2, 5, 7, 8))
    np.testing.assert_allclose(ours, _sdpa(q, ke, ve, gqa=False), rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- head map

def test_head_map_is_repeat_interleave_bitwise(oracle_mod):
    rng = np.random.default_rng(7)
    for (Hq, Hkv) in ((4, 2), (6, 2), (6, 3), (8, 1), (12, 2)):
        g = Hq // Hkv
        q, k, v = _rand(rng, 2, Hq, 5, 8), _rand(rng, 2, Hkv, 6, 8), _rand(rng, 2, Hkv, 6, 8)
        ours = oracle_mod.forward(q, k, v)
        expanded = oracle_mod.forward(q, np.repeat(k, g, axis=1), np.repeat(v, g, axis=1))
        assert np.array_equal(ours, expanded)


def test_head_map_is_not_tiling(oracle_mod):
    """The tiling variant (head h -> kv head h % Hkv) gives a different result."""
    rng = np.random.default_rng(8)
    q, k, v = _rand(rng, 1, 4, 5, 4), _rand(rng, 1, 2, 5, 4), _rand(rng, 1, 2, 5, 4)
    ours = oracle_mod.forward(q, k, v)
    tiled = oracle_mod.forward(q, np.tile(k, (1, 2, 1, 1)), np.tile(v, (1, 2, 1, 1)))
    assert np.abs(ours - tiled).max() > 1e-3
    # Heads 0 and 3 use the same kv head under both maps; heads 1 and 2 do not.
    assert np.array_equal(ours[:, 0], tiled[:, 0]) and np.array_equal(ours[:, 3], tiled[:, 3])


# ---------------------------------------------------------------- closed forms

def test_single_key_returns_that_value_row(oracle_mod):
    rng = np.random.default_rng(9)
    q, k, v = _rand(rng, 2, 4, 3, 8), _rand(rng, 2, 2, 1, 8), _rand(rng, 2, 2, 1, 8)
    out = oracle_mod.forward(q, k, v)
    for h in range(4):
        assert np.array_equal(out[:, h], np.broadcast_to(v[:, h // 2, 0][:, None, :], (2, 3, 8)))


def test_one_hot_mask_selects_value_row(oracle_mod):
    rng = np.random.default_rng(10)
    B, Hq, Hkv, Sq, Sk, D = 2, 6, 2, 4, 9, 8
    q, k, v = _rand(rng, B, Hq, Sq, D), _rand(rng, B, Hkv, Sk, D), _rand(rng, B, Hkv, Sk, D)
    pick = rng.integers(0, Sk, size=(B, Sq))
    mask = np.zeros((B, Sq, Sk), dtype=bool)
    for b in range(B):
        for i in range(Sq):
            mask[b, i, pick[b, i]] = True
    out = oracle_mod.forward(q, k, v, mask=mask)
    for b in range(B):
        for h in range(Hq):
            for i in range(Sq):
                assert np.array_equal(out[b, h, i], v[b, h // 3, pick[b, i]])


def test_zero_scale_gives_mean_of_visible_rows(oracle_mod):
    rng = np.random.default_rng(11)
    B, Hq, Hkv, Sq, Sk, D = 2, 4, 2, 3, 10, 6
    q, k, v = _rand(rng, B, Hq, Sq, D), _rand(rng, B, Hkv, Sk, D), _rand(rng, B, Hkv, Sk, D)
    mask = _mask("random", rng, B, Sq, Sk)
    out = oracle_mod.forward(q, k, v, mask=mask, scale=0.0)
    for b in range(B):
        for h in range(Hq):
            for i in range(Sq):
                vis = v[b, h // 2][mask[b, i]]
                np.testing.assert_allclose(out[b, h, i], vis.mean(axis=0), rtol=0, atol=1e-14)


def test_causal_rows(oracle_mod):
    rng = np.random.default_rng(12)
    B, Hq, Hkv, S, D = 2, 4, 2, 7, 5
    q, k, v = _rand(rng, B, Hq, S, D), _rand(rng, B, Hkv, S, D), _rand(rng, B, Hkv, S, D)
    out = oracle_mod.forward(q, k, v, causal=True)
    for h in range(Hq):
        assert np.array_equal(out[:, h, 0], v[:, h // 2, 0])  # row 0 sees key 0 only
    flat = oracle_mod.forward(q, k, v, causal=True, scale=0.0)
    for i in range(S):
        np.testing.assert_allclose(flat[:, :, i], np.repeat(v[:, :, : i + 1].mean(axis=2), 2, axis=1),
                                   rtol=0, atol=1e-14)
    # The last row of a causal problem sees every key.
    np.testing.assert_array_equal(out[:, :, -1], oracle_mod.forward(q, k, v)[:, :, -1])


def test_constant_values_give_constant_output(oracle_mod):
    rng = np.random.default_rng(13)
    q, k = _rand(rng, 2, 6, 5, 8), _rand(rng, 2, 3, 12, 8)
    c = rng.standard_normal(8)
    v = np.broadcast_to(c, (2, 3, 12, 8)).copy()
    out = oracle_mod.forward(q, k, v, mask=_mask("random", rng, 2, 5, 12))
    np.testing.assert_allclose(out, np.broadcast_to(c, out.shape), rtol=0, atol=1e-14)


# ---------------------------------------------------------------- invariants

def test_weights_are_a_distribution(oracle_mod):
    rng = np.random.default_rng(14)
    B, Hq, Hkv, S, D = 2, 6, 2, 8, 8
    q, k = _rand(rng, B, Hq, S, D), _rand(rng, B, Hkv, S, D)
    mask = _mask("random", rng, B, S, S)
    w = oracle_mod.probs(q, k, mask=mask, causal=True)
    assert np.all(w >= 0)
    np.testing.assert_allclose(w.sum(axis=-1), 1.0, rtol=0, atol=1e-12)
    hidden = ~(mask[:, None] & np.tril(np.ones((S, S), dtype=bool))[None, None])
    assert np.all(w[np.broadcast_to(hidden, w.shape)] == 0.0)


def test_output_in_value_hull(oracle_mod):
    rng = np.random.default_rng(15)
    q, k, v = _rand(rng, 2, 4, 6, 8) * 3, _rand(rng, 2, 2, 11, 8), _rand(rng, 2, 2, 11, 8)
    out = oracle_mod.forward(q, k, v)
    for h in range(4):
        lo = v[:, h // 2].min(axis=1)[:, None, :]
        hi = v[:, h // 2].max(axis=1)[:, None, :]
        assert np.all(out[:, h] >= lo - 1e-14) and np.all(out[:, h] <= hi + 1e-14)


def test_key_shift_invariance(oracle_mod):
    rng = np.random.default_rng(16)
    q, k, v = _rand(rng, 2, 4, 5, 8), _rand(rng, 2, 2, 9, 8), _rand(rng, 2, 2, 9, 8)
    u = rng.standard_normal((2, 2, 1, 8))
    np.testing.assert_allclose(oracle_mod.forward(q, k + u, v), oracle_mod.forward(q, k, v),
                               rtol=1e-12, atol=1e-13)


def test_key_permutation_invariance(oracle_mod):
    rng = np.random.default_rng(17)
    B, Sq, Sk = 2, 5, 13
    q, k, v = _rand(rng, B, 6, Sq, 8), _rand(rng, B, 3, Sk, 8), _rand(rng, B, 3, Sk, 8)
    mask = _mask("random", rng, B, Sq, Sk)
    perm = rng.permutation(Sk)
    a = oracle_mod.forward(q, k, v, mask=mask)
    b = oracle_mod.forward(q, k[:, :, perm], v[:, :, perm], mask=mask[:, :, perm])
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


def test_scale_multiplies_scores(oracle_mod):
    rng = np.random.default_rng(18)
    q, k, v = _rand(rng, 1, 4, 3, 8), _rand(rng, 1, 2, 7, 8), _rand(rng, 1, 2, 7, 8)
    np.testing.assert_allclose(oracle_mod.forward(q, k, v, scale=0.25),
                               oracle_mod.forward(q * 0.25, k, v, scale=1.0), rtol=1e-12, atol=1e-13)


def test_rows_match_full(oracle_mod):
    rng = np.random.default_rng(19)
    B, Hq, Hkv, S, D = 2, 6, 2, 9, 8
    q, k, v = _rand(rng, B, Hq, S, D), _rand(rng, B, Hkv, S, D), _rand(rng, B, Hkv, S, D)
    mask = _mask("random", rng, B, S, S)
    full = oracle_mod.forward(q, k, v, mask=mask, causal=True)
    rows = [(1, 5, 8), (0, 0, 0), (1, 2, 3)]
    got = oracle_mod.forward_rows(q, k, v, rows, mask=mask, causal=True)
    for r, (b, h, i) in enumerate(rows):
        assert np.array_equal(got[r], full[b, h, i])


def test_fully_hidden_row_is_nan(oracle_mod):
    """A row with no visible key: the reference solution's softmax over an
    all -inf row is NaN, and the oracle keeps that."""
    assert torch.isnan(torch.softmax(torch.full((4,), float("-inf"), dtype=torch.float64), -1)).all()
    rng = np.random.default_rng(20)
    q, k, v = _rand(rng, 1, 2, 2, 4), _rand(rng, 1, 1, 3, 4), _rand(rng, 1, 1, 3, 4)
    mask = np.ones((1, 2, 3), dtype=bool)
    mask[0, 1, :] = False
    out = oracle_mod.forward(q, k, v, mask=mask)
    assert np.all(np.isnan(out[0, :, 1])) and np.all(np.isfinite(out[0, :, 0]))


def test_invalid_shapes_rejected(oracle_mod):
    rng = np.random.default_rng(21)
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.forward(_rand(rng, 1, 5, 2, 4), _rand(rng, 1, 2, 2, 4), _rand(rng, 1, 2, 2, 4))
    with pytest.raises(oracle_mod.OracleError):  # causal needs Sq == Sk
        oracle_mod.forward(_rand(rng, 1, 2, 2, 4), _rand(rng, 1, 1, 3, 4), _rand(rng, 1, 1, 3, 4),
                           causal=True)


# ------------------------------------------- causal offset and sliding window

def _offset_window_mask(Sq, Sk, off, window):
    i = np.arange(Sq)[:, None]
    j = np.arange(Sk)[None, :]
    vis = j <= i + off
    if window:
        vis &= j > i + off - window
    return vis


OFFSET_CASES = [
    # B, Hq, Hkv, Sq, Sk, D, offset, window
    (2, 8, 2, 5, 12, 8, 7, 0),      # bottom-right causal, Sq < Sk
    (1, 6, 3, 9, 9, 4, 0, 3),       # sliding window of 3 keys
    (2, 4, 1, 4, 20, 8, 16, 5),     # bottom-right + window
    (1, 4, 2, 6, 6, 8, -2, 0),      # diagonal shifted down: first rows fully hidden
]


def _offset_window_ref(q, k, v, off, window, mask=None):
    B, Sq, Sk = q.shape[0], q.shape[2], k.shape[2]
    vis = np.broadcast_to(_offset_window_mask(Sq, Sk, off, window), (B, Sq, Sk))
    if mask is not None:
        vis = vis & mask
    return _sdpa(q, k, v, mask=vis, scale=1.0 / np.sqrt(q.shape[-1])), vis


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D,off,window", OFFSET_CASES)
def test_causal_offset_and_window_match_torch(oracle_mod, B, Hq, Hkv, Sq, Sk, D, off, window):
    rng = np.random.default_rng(Sq * 31 + Sk)
    q, k, v = _rand(rng, B, Hq, Sq, D), _rand(rng, B, Hkv, Sk, D), _rand(rng, B, Hkv, Sk, D)
    ours = oracle_mod.forward(q, k, v, causal=True, causal_offset=off, window=window)
    ref, vis = _offset_window_ref(q, k, v, off, window)
    hidden_rows = ~vis.any(axis=-1)  # [B, Sq]
    for b in range(B):
        for i in range(Sq):
            if hidden_rows[b, i]:
                assert np.all(np.isnan(ours[b, :, i]))
            else:
                np.testing.assert_allclose(ours[b, :, i], ref[b, :, i], rtol=1e-11, atol=1e-12)


def test_offset_zero_is_the_pages_causal(oracle_mod):
    rng = np.random.default_rng(41)
    q, k, v = _rand(rng, 2, 4, 7, 8), _rand(rng, 2, 2, 7, 8), _rand(rng, 2, 2, 7, 8)
    assert np.array_equal(oracle_mod.forward(q, k, v, causal=True),
                          oracle_mod.forward(q, k, v, causal=True, causal_offset=0))
    # A window covering every visible key changes nothing.
    assert np.array_equal(oracle_mod.forward(q, k, v, causal=True),
                          oracle_mod.forward(q, k, v, causal=True, causal_offset=0, window=7))


def test_window_of_one_selects_the_diagonal_value(oracle_mod):
    rng = np.random.default_rng(42)
    q, k, v = _rand(rng, 1, 4, 5, 8), _rand(rng, 1, 2, 9, 8), _rand(rng, 1, 2, 9, 8)
    out = oracle_mod.forward(q, k, v, causal=True, causal_offset=4, window=1)
    for h in range(4):
        for i in range(5):
            assert np.array_equal(out[0, h, i], v[0, h // 2, i + 4])


def test_bottom_right_decode_sees_everything(oracle_mod):
    rng = np.random.default_rng(43)
    q, k, v = _rand(rng, 2, 8, 1, 8), _rand(rng, 2, 2, 33, 8), _rand(rng, 2, 2, 33, 8)
    np.testing.assert_array_equal(oracle_mod.forward(q, k, v, causal=True, causal_offset=32),
                                  oracle_mod.forward(q, k, v))


def test_window_needs_causal(oracle_mod):
    rng = np.random.default_rng(44)
    q, k = _rand(rng, 1, 2, 3, 4), _rand(rng, 1, 1, 3, 4)
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.forward(q, k, k, causal=False, causal_offset=0, window=2)


# ---------------------------------------------------------- ragged KV cache

def test_kv_lens_equal_truncated_cache(oracle_mod):
    """Batch entry b with kv_lens[b] = n gives what the pages' function gives on
    the first n keys alone (bottom-right causal included)."""
    rng = np.random.default_rng(45)
    B, Hq, Hkv, Sq, Sk, D = 3, 8, 2, 3, 20, 8
    q, k, v = _rand(rng, B, Hq, Sq, D), _rand(rng, B, Hkv, Sk, D), _rand(rng, B, Hkv, Sk, D)
    lens = np.array([20, 7, 12], dtype=np.int32)
    for causal in (False, True):
        out = oracle_mod.forward(q, k, v, causal=causal,
                                 causal_offset=(Sk - Sq) if causal else None, kv_lens=lens)
        for b in range(B):
            n = int(lens[b])
            ref, _ = _offset_window_ref(q[b:b + 1], k[b:b + 1, :, :n], v[b:b + 1, :, :n],
                                        n - Sq if causal else n, 0)
            np.testing.assert_allclose(out[b:b + 1], ref, rtol=1e-11, atol=1e-12)


def test_rows_ex_match_torch_and_full(oracle_mod):
    """forward_rows with a causal offset, a window and per-sequence lengths
    (lengths 0 and full included): each requested row equals PyTorch's fp64
    attention on that entry's first len_b keys under the same visibility
    rule, and equals the same row of the full-output function bitwise; the
    rows come back in the order asked for, duplicates included."""
    rng = np.random.default_rng(47)
    B, Hq, Hkv, Sq, Sk, D = 3, 6, 2, 4, 15, 8
    q, k, v = _rand(rng, B, Hq, Sq, D), _rand(rng, B, Hkv, Sk, D), _rand(rng, B, Hkv, Sk, D)
    lens = np.array([15, 0, 9], dtype=np.int32)
    rows = [(2, 5, 3), (0, 0, 0), (1, 3, 2), (2, 1, 0), (0, 4, 3), (2, 5, 3), (0, 2, 1)]
    for causal, off, window in ((False, None, 0), (True, Sk - Sq, 0), (True, Sk - Sq, 5),
                                (True, 3, 2)):
        full = oracle_mod.forward(q, k, v, causal=causal, causal_offset=off, window=window,
                                  kv_lens=lens)
        got = oracle_mod.forward_rows(q, k, v, rows, causal=causal, causal_offset=off,
                                      window=window, kv_lens=lens)
        for r, (b, h, i) in enumerate(rows):
            assert np.array_equal(got[r], full[b, h, i], equal_nan=True), (causal, off, window, r)
            n = int(lens[b])
            vis = np.arange(Sk) < n
            if causal:
                j = np.arange(Sk)
                lim = i + off + (n - Sk)
                vis &= j <= lim
                if window:
                    vis &= j > lim - window
            if not vis.any():
                assert np.all(np.isnan(got[r]))
                continue
            ref = _sdpa(q[b:b + 1, h:h + 1, i:i + 1], k[b:b + 1, h // 3:h // 3 + 1],
                        v[b:b + 1, h // 3:h // 3 + 1], mask=vis[None, None, :],
                        scale=1.0 / np.sqrt(D))
            np.testing.assert_allclose(got[r], ref[0, 0, 0], rtol=1e-11, atol=1e-12)


def test_kv_lens_bounds(oracle_mod):
    rng = np.random.default_rng(46)
    q, k = _rand(rng, 2, 2, 1, 4), _rand(rng, 2, 1, 5, 4)
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.forward(q, k, k, kv_lens=[5, 6])
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.forward(q, k, k, kv_lens=[5])


# ---------------------------------------------------------- planted mistakes

MUTANTS = {
    "tiling head map": ("const int64_t kv = h / g;", "const int64_t kv = h % p.Hkv;"),
    "scale dropped": ("double s = p.scale * dot;", "double s = dot;"),
    "causal off by one": ("if (p.causal && j > i + off)", "if (p.causal && j >= i + off)"),
    "causal offset ignored": ("if (p.causal && j > i + off)", "if (p.causal && j > i)"),
    "window off by one": ("j <= i + off - p.window", "j < i + off - p.window"),
    "kv length off by one": ("if (j >= len) s = neg_inf;", "if (j > len) s = neg_inf;"),
    "kv length ignored by causal": ("const int64_t off = p.causal_offset + (len - p.Sk);",
                                    "const int64_t off = p.causal_offset;"),
    "mask polarity": ("p.mask[(b * p.Sq + i) * p.Sk + j] == 0", "p.mask[(b * p.Sq + i) * p.Sk + j] != 0"),
    "max not subtracted": ("w[j] = std::exp(w[j] - m);", "w[j] = std::exp(w[j]);"),
    "no normalisation": ("for (int64_t j = 0; j < p.Sk; ++j) w[j] = w[j] / l;", ""),
    "q/k transposed index": ("const double* krow = kbase + j * p.D;", "const double* krow = kbase + (j % p.D) * p.D;"),
    "v from q head": ("const double* vbase = p.v + ((b * p.Hkv + kv) * p.Sk) * p.D;",
                      "const double* vbase = p.v + ((b * p.Hkv + (h % p.Hkv)) * p.Sk) * p.D;"),
    "kv bytes factor": ("return 2 * layers * tokens", "return layers * tokens"),
    # Mistakes confined to the selected-rows entry point with lengths, offset
    # and window: (function, text, replacement) plants them in that function only.
    "rows_ex rows written out of order": ("oracle_gqa_forward_rows_ex",
                                          "row_output(p, b, h, i, w.data(), out + r * D);",
                                          "row_output(p, b, h, i, w.data(), out + (n - 1 - r) * D);"),
    "rows_ex ignores the lengths": ("oracle_gqa_forward_rows_ex", "true,\n            kv_lens};",
                                    "true,\n            nullptr};"),
    "rows_ex ignores the window": ("oracle_gqa_forward_rows_ex", "causal_offset, window, true",
                                   "causal_offset, 0, true"),
}


def _pins_hold(oracle_mod, lib):
    """A compact re-run of the pins above against another oracle build."""
    rng = np.random.default_rng(99)
    ok = True
    for (B, Hq, Hkv, Sq, Sk, D, mk, causal) in CASES:
        q, k, v = _rand(rng, B, Hq, Sq, D), _rand(rng, B, Hkv, Sk, D), _rand(rng, B, Hkv, Sk, D)
        mask = _mask(mk, rng, B, Sq, Sk)
        try:
            ours = oracle_mod.forward(q, k, v, mask=mask, causal=causal, lib=lib)
        except oracle_mod.OracleError:
            return False
        ref = _sdpa(q, k, v, mask=mask, causal=causal, scale=1.0 / np.sqrt(D))
        ok &= bool(np.allclose(ours, ref, rtol=1e-11, atol=1e-12))
    for (B, Hq, Hkv, Sq, Sk, D, off, window) in OFFSET_CASES[:3]:
        q, k, v = _rand(rng, B, Hq, Sq, D), _rand(rng, B, Hkv, Sk, D), _rand(rng, B, Hkv, Sk, D)
        try:
            ours = oracle_mod.forward(q, k, v, causal=True, causal_offset=off, window=window, lib=lib)
        except oracle_mod.OracleError:
            return False
        ref, _ = _offset_window_ref(q, k, v, off, window)
        ok &= bool(np.allclose(ours, ref, rtol=1e-11, atol=1e-12))
    q, k, v = _rand(rng, 2, 4, 2, 8), _rand(rng, 2, 2, 9, 8), _rand(rng, 2, 2, 9, 8)
    try:
        ragged = oracle_mod.forward(q, k, v, causal=True, causal_offset=7, kv_lens=[9, 5], lib=lib)
    except oracle_mod.OracleError:
        return False
    plain = oracle_mod.forward(q, k, v, kv_lens=[9, 5], lib=lib)
    for b, n in ((0, 9), (1, 5)):
        ref, _ = _offset_window_ref(q[b:b + 1], k[b:b + 1, :, :n], v[b:b + 1, :, :n], n - 2, 0)
        ok &= bool(np.allclose(ragged[b:b + 1], ref, rtol=1e-11, atol=1e-12))
        ref, _ = _offset_window_ref(q[b:b + 1], k[b:b + 1, :, :n], v[b:b + 1, :, :n], n, 0)
        ok &= bool(np.allclose(plain[b:b + 1], ref, rtol=1e-11, atol=1e-12))
    # Selected rows, plain and with offset / window / lengths, against the
    # full-output functions pinned above (rows in a scrambled order).
    q, k, v = _rand(rng, 2, 4, 3, 8), _rand(rng, 2, 2, 11, 8), _rand(rng, 2, 2, 11, 8)
    rows = [(1, 3, 2), (0, 0, 0), (1, 0, 1), (0, 2, 2)]
    try:
        for kw in ({}, dict(causal=True, causal_offset=8, window=4, kv_lens=[11, 6])):
            full = oracle_mod.forward(q, k, v, lib=lib, **kw)
            sel = oracle_mod.forward_rows(q, k, v, rows, lib=lib, **kw)
            ok &= all(np.allclose(sel[r], full[b, h, i], rtol=1e-13, atol=1e-14)
                      for r, (b, h, i) in enumerate(rows))
            ref, _ = _offset_window_ref(q[:1], k[:1], v[:1], 8, 4) if kw else (None, None)
            if kw:
                ok &= bool(np.allclose(sel[1], ref[0, 0, 0], rtol=1e-11, atol=1e-12))
                ok &= bool(np.allclose(sel[3], ref[0, 2, 2], rtol=1e-11, atol=1e-12))
    except oracle_mod.OracleError:
        return False
    q, k, v = _rand(rng, 1, 4, 5, 8) * 60.0, _rand(rng, 1, 2, 7, 8) * 60.0, _rand(rng, 1, 2, 7, 8)
    big = oracle_mod.forward(q, k, v, scale=1.0, lib=lib)
    ok &= bool(np.allclose(big, _sdpa(q, k, v, scale=1.0), rtol=1e-11, atol=1e-12))
    g = json.load(open(os.path.join(GOLDEN, "kv_cache_figures.json")))
    for case in g["cases"]:
        val = oracle_mod.kv_cache_bytes(**case["args"], lib=lib) / case["unit_bytes"]
        ok &= abs(val - case["page_value"]) <= case["tolerance_units"]
    return ok


def test_pins_hold_for_the_real_oracle(oracle_mod):
    assert _pins_hold(oracle_mod, None)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(oracle_mod, tmp_path, name):
    spec = MUTANTS[name]
    src = open(os.path.join(ROOT, "oracle", "gqa_oracle.cpp")).read()
    if len(spec) == 3:  # only inside the named function (its definition onwards)
        func, old, new = spec
        start = src.index("int %s(" % func)
        at = src.index(old, start)
        mutated = src[:at] + new + src[at + len(old):]
    else:
        old, new = spec
        assert src.count(old) >= 1, name
        mutated = src.replace(old, new)
    assert mutated != src, name
    mutant_src = tmp_path / "mutant.cpp"
    mutant_src.write_text(mutated)
    so = str(tmp_path / "libmutant.so")
    oracle_mod.build(force=True, src=str(mutant_src), out=so)
    lib = oracle_mod.load_library(so)
    assert not _pins_hold(oracle_mod, lib), name
