"""The seeded input generators (shared by both sides): determinism, bf16
rounding against torch's float32 -> bfloat16 conversion, split recipes."""
import numpy as np
import torch

from context_attention_long_b200 import inputs


def test_bf16_rounding_matches_torch():
    rng = np.random.Generator(np.random.PCG64(5))
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10 ** rng.uniform(-6, 6, 100000).astype(np.float32),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38, -2.5e-39], dtype=np.float32)])
    ours = inputs.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_widening_is_exact():
    bits = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]          # finite values only
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(inputs.bf16_bits_to_f64(bits), ref)


def test_generator_is_deterministic_and_seeded():
    a = inputs.make_qkv(1, 8, 2, 16, 7, True)
    b = inputs.make_qkv(1, 8, 2, 16, 7, True)
    c = inputs.make_qkv(1, 8, 2, 16, 8, True)
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
    assert not np.array_equal(a[0], c[0])


def test_rms_normalised_rows_have_unit_rms():
    q, k, v = inputs.make_qkv(1, 64, 3, 128, 9, True)
    for t in (q, k):
        x = inputs.bf16_bits_to_f64(t)
        rms = np.sqrt(np.mean(x * x, axis=-1))
        assert np.max(np.abs(rms - 1.0)) < 1e-2
    xv = inputs.bf16_bits_to_f64(v)
    assert abs(np.std(xv) - 1.0) < 0.05


def test_split_recipes():
    assert inputs.front_loaded_splits(30, 4) == [8, 8, 7, 7]
    assert inputs.front_loaded_splits(10007, 4) == [2502, 2502, 2502, 2501]
    assert inputs.front_loaded_splits(4095, 2) == [2048, 2047]
    lens = inputs.ring_anything_lens(10007, 6, 1237)
    assert sorted(lens) == [1667] + [1668] * 5 and sum(lens) == 10007
    assert lens[1237 % 6] == 1667
    assert inputs.ring_anything_lens(4608, 4, 3) == [1152] * 4
    for seed in range(20):
        s = inputs.random_splits(37, 5, seed)
        assert len(s) == 5 and sum(s) == 37 and min(s) >= 0
        s = inputs.random_splits(37, 5, seed, allow_zero=False)
        assert min(s) >= 1 and sum(s) == 37
