"""The seeded input generator shared by the oracle tests and the CUDA path."""
import numpy as np
import torch


def test_splitmix64_published_outputs(synth_mod):
    # First outputs of SplitMix64 seeded with 0 (Steele, Lea, Flood 2014; the
    # values printed alongside Vigna's reference implementation).
    assert synth_mod.splitmix64_at(0, 0) == 0xE220A8397B1DCDAF
    assert synth_mod.splitmix64_at(0, 1) == 0x6E789E6AA1B965F4
    assert synth_mod.splitmix64_at(0, 2) == 0x06C45D188009454F


def test_normal_moments(synth_mod):
    x = synth_mod.normal_f32(3, 1, 1 << 20).astype(np.float64)
    assert abs(x.mean()) < 5e-3 and abs(x.var() - 1.0) < 1e-2
    assert abs((x ** 3).mean()) < 2e-2 and abs((x ** 4).mean() - 3.0) < 5e-2


def test_bf16_rounding_matches_torch(synth_mod):
    x = synth_mod.normal_f32(4, 0, 100000) * np.float32(37.0)
    ours = synth_mod.round_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = synth_mod.bf16_bits_to_f64(ours)
    assert np.array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_bf16_stream_is_rounded_f32_stream(synth_mod):
    f = synth_mod.normal_f32(5, 2, 4097)
    assert np.array_equal(synth_mod.normal_bf16_bits(5, 2, 4097), synth_mod.round_bf16_bits(f))


def test_slices_match_full_tensor(synth_mod):
    B, H, S, D = 3, 4, 33, 8
    full = synth_mod.normal_bf16_bits(7, 1, B * H * S * D).reshape(B, H, S, D)
    for b, h in ((0, 0), (2, 3), (1, 2)):
        assert np.array_equal(synth_mod.kv_slice_bf16_bits(7, 1, B, H, S, D, b, h), full[b, h])
    assert np.array_equal(synth_mod.normal_bf16_bits(7, 1, 5, offset=11), full.reshape(-1)[11:16])


def test_masks(synth_mod):
    lens = synth_mod.uniform_int(5, 3, 1000, 256, 2048)
    assert lens.min() >= 256 and lens.max() <= 2048 and len(set(lens.tolist())) > 500
    m = synth_mod.mask_from_lengths(np.array([1, 3]), 2, 4)
    assert m.tolist() == [[[1, 0, 0, 0]] * 2, [[1, 1, 1, 0]] * 2]
    r = synth_mod.mask_random(1, 2, 5, 64, 0.1)
    assert r.shape == (2, 5, 64) and r.sum(axis=-1).min() >= 1
    assert 0.05 < r.mean() < 0.2
