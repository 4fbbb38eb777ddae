"""The seeded input generator shared by the oracle and the CUDA path (CPU):
its bf16 rounding equals torch's float32 -> bfloat16 conversion (round to
nearest even), and every (tensor, batch, head) slice is its own stream, so a
slice drawn alone equals the same slice drawn with the others."""
import numpy as np
import torch

from synth import inputs as S


def test_bf16_rounding_equals_torch_conversion():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(100_000).astype(np.float32),
        (rng.standard_normal(10_000) * 1e30).astype(np.float32),
        (rng.standard_normal(10_000) * 1e-30).astype(np.float32),
        # exact ties: the low 16 bits 0x8000, with even and odd kept mantissas
        (rng.integers(0, 1 << 15, 10_000, dtype=np.uint32) << np.uint32(16) | np.uint32(0x8000)).view(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 3.4e38, -3.4e38, 1e-45, np.inf, -np.inf], dtype=np.float32),
    ])
    x = x[np.isfinite(x) | np.isinf(x)]
    ours = S.bf16_round_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    # and the decode is exact
    assert np.array_equal(S.bf16_bits_to_f64(ours), torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16)
                          .double().numpy())


def test_slices_are_independent_streams():
    w = S.small_workload("gen", 5, 2, 3, 64, (2, 4, 4), (1, 2, 2), (1, 1, 1), (1, 1, 1))
    full = S.draw(w, S.Q_ID)
    assert full.shape == (2, 3, 32, 64)
    assert np.array_equal(S.draw(w, S.Q_ID, heads=[2], batches=[1])[0, 0], full[1, 2])
    assert np.array_equal(S.draw_head(w, S.Q_ID, 0, 1), full[0, 1])
    # other tensors and other slices differ
    assert not np.array_equal(S.draw_head(w, S.K_ID, 0, 1), full[0, 1])
    assert not np.array_equal(full[0, 0], full[0, 1])
    # and the same seed gives the same bytes
    assert np.array_equal(S.draw(w, S.Q_ID), full)


def test_head_scale_and_blend_factor_ranges():
    w = S.WORKLOADS["720p"]
    s = S.head_scales(w)
    assert s.shape == (w.heads,) and s.min() >= 0.5 and s.max() <= 2.0
    g = S.blend_g(S.WORKLOADS["1080p"])
    assert g.shape == (24,) and g.min() >= 0.0 and g.max() <= 1.0
