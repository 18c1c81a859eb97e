"""The seeded input generator: bf16 rounding is round-to-nearest-even (checked against torch's
own float32 -> bfloat16 conversion) and draws are reproducible."""

import numpy as np
import torch

from block_causal_linear_relu_b200.inputs import bf16_bits_to_f32, draw_qkv, f32_to_bf16_bits


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100_000).astype(np.float32) * 10,
                        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, 1e-40, np.inf, -np.inf], np.float32)])
    ours = f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(bf16_bits_to_f32(ours), torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_draw_is_seeded_and_ordered():
    a = draw_qkv((1, 2, 5, 4), 7, "bf16")
    b = draw_qkv((1, 2, 5, 4), 7, "bf16")
    c = draw_qkv((1, 2, 5, 4), 8, "bf16")
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
    assert not np.array_equal(a[0], c[0])
    assert not np.array_equal(a[0], a[1]) and not np.array_equal(a[1], a[2])
    f = draw_qkv((1, 2, 5, 4), 7, "f32")
    assert f[0].dtype == np.float32 and np.array_equal(f32_to_bf16_bits(f[0]), a[0])
