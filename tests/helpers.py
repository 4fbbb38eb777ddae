"""Shared test plumbing: seeded inputs on the GPU, sampled query tiles, and the
parity bars.  No attention arithmetic lives here (the oracle computes the
expected values, the library the actual ones)."""
from __future__ import annotations

import math

import numpy as np

from synth import inputs as S

# Parity bars for bf16 outputs against the fp64 oracle.
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3


def geom_for(V, w):
    return V.make_geom(w.batch, w.heads, w.head_dim, w.grid, w.tile, w.window, w.pool)


def bits_to_gpu(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def gpu_tensor(w, tensor_id: int, check: list):
    """[B, heads, N, d] bf16 raster on the GPU.  The (b, h) slices in `check`
    come from the shared seeded generator (and are what the oracle sees); the
    rest are filled from a seeded torch generator with the same distribution,
    so the launch has the full workload's shape."""
    import torch
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1000 * w.seed + tensor_id)
    std = 0.1 if tensor_id == S.DO_ID else 1.0
    t = torch.empty((w.batch, w.heads, w.n_tokens, w.head_dim), dtype=torch.bfloat16, device="cuda")
    scales = S.head_scales(w)
    for b in range(w.batch):
        for h in range(w.heads):
            if (b, h) in check:
                t[b, h] = bits_to_gpu(S.draw_head(w, tensor_id, b, h))
            else:
                x = torch.randn((w.n_tokens, w.head_dim), generator=gen, device="cuda") * std
                if w.head_scale and tensor_id != S.DO_ID:
                    x *= float(scales[h])
                t[b, h] = x.to(torch.bfloat16)
    return t


def host_f64(w, tensor_id: int, b: int, h: int) -> np.ndarray:
    return S.bf16_bits_to_f64(S.draw_head(w, tensor_id, b, h))


def to_f64(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def sample_tiles(tiles_per_dim, n_random: int = 12, seed: int = 0) -> list:
    """Query tiles covering every boundary class per dim (first, second,
    middle, second-last, last) at the corners, plus a seeded random subset of
    the full product of classes."""
    per = []
    for n in tiles_per_dim:
        c = sorted({0, min(1, n - 1), n // 2, max(n - 2, 0), n - 1})
        per.append(c)
    nt, nh, nw = tiles_per_dim
    prod = [(a, b, c) for a in per[0] for b in per[1] for c in per[2]]
    corners = [(a, b, c) for a in (per[0][0], per[0][-1]) for b in (per[1][0], per[1][-1])
               for c in (per[2][0], per[2][-1])]
    rng = np.random.default_rng(seed)
    pick = [prod[i] for i in rng.choice(len(prod), size=min(n_random, len(prod)), replace=False)]
    out = []
    for a, b, c in corners + pick:
        tid = (a * nh + b) * nw + c
        if tid not in out:
            out.append(tid)
    return out


def assert_close(actual: np.ndarray, expected: np.ndarray, max_abs: float, mean_abs: float = math.inf, what=""):
    err = np.abs(actual - expected)
    assert np.isfinite(actual).all(), f"{what}: non-finite values"
    assert err.max() <= max_abs, f"{what}: max abs err {err.max():.3e} > {max_abs}"
    assert err.mean() <= mean_abs, f"{what}: mean abs err {err.mean():.3e} > {mean_abs}"
