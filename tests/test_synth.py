"""Host side of the seeded input generator: determinism, distribution, rounding."""
import numpy as np
import torch

import synth


def test_deterministic_and_index_addressed():
    idx = np.arange(1000, dtype=np.uint64)
    a = synth.bf16_values(7, synth.tensor_id(3, synth.ROLE_K), idx)
    b = synth.bf16_values(7, synth.tensor_id(3, synth.ROLE_K), idx[::-1].copy())[::-1]
    np.testing.assert_array_equal(a, b)
    c = synth.bf16_values(8, synth.tensor_id(3, synth.ROLE_K), idx)
    d = synth.bf16_values(7, synth.tensor_id(3, synth.ROLE_V), idx)
    assert np.mean(a == c) < 0.05 and np.mean(a == d) < 0.05


def test_distribution_is_close_to_unit_normal():
    x = synth.values_f32(1, 5, np.arange(400_000, dtype=np.uint64)).astype(np.float64)
    assert abs(x.mean()) < 0.01
    assert abs(x.std() - 1.0) < 0.01
    assert np.abs(x).max() <= 6.0
    y = synth.values_f32(1, 5, np.arange(1000, dtype=np.uint64), sigma=0.5)
    np.testing.assert_array_equal(y, 0.5 * synth.values_f32(1, 5, np.arange(1000, dtype=np.uint64)))


def test_bf16_rounding_matches_torch_round_to_nearest_even():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100_000).astype(np.float32),
                        np.array([1.00390625, 1.01171875, -1.00390625, 0.0, -0.0, 3.0e-39], np.float32)])
    ours = synth.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)


def test_token_tensor_layout():
    pos = np.arange(5, 9)
    t = synth.token_tensor(0, 11, 2, 3, 4, pos)
    assert t.shape == (2, 4, 3, 4)
    # element (b=1, t=2, h=0, d=3) is the value at position 7
    idx = ((1 * 3 + 0) * (1 << 20) + 7) * 4 + 3
    assert t[1, 2, 0, 3] == synth.bf16_values(0, 11, np.array([idx], np.uint64))[0]
    s = synth.head_slice(0, 11, 1, 0, 3, 4, np.array([7]))
    assert s[0, 3] == t[1, 2, 0, 3]
    g = synth.token_tensor(0, 12, 2, 3, 1, pos)
    assert g.shape == (2, 4, 3)
