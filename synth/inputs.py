"""Seeded synthetic inputs shared by the oracle tests, the GPU parity tests and
the benchmark.

This module holds no attention arithmetic: it only draws random numbers and
rounds them to bfloat16.  Every tensor is drawn in RASTER token order
(token n = (t*H + y)*W + x), shaped [B, heads, N, head_dim].

Recipe (each (tensor, batch, head) slice has its own PCG64 stream so that any
head can be regenerated alone, e.g. for the oracle's sampled checks):

  stream(seed, tensor_id, b, h) = Generator(PCG64(SeedSequence(seed,
                                       spawn_key=(tensor_id, b, h))))
  tensor_id: 0 = Q, 1 = K, 2 = V, 3 = dO
  Q, K, V ~ N(0, 1) float32; dO ~ N(0, 0.1^2) float32
  per-head scale s_h ~ U(0.5, 2) from stream (seed, spawn_key=(10,)), multiplied
      into that head's Q, K and V before rounding (the 720p workload)
  per-head blend g_h ~ U(0, 1) from stream (seed, spawn_key=(11,))
  every value is rounded once to bfloat16, round-to-nearest-even, by bit
  arithmetic on the float32 pattern.

The workloads are the shapes of the video latents of the 720P/1080P/4K
generators the pages discuss (UltraGen §5 and App. C; Sliding Tile Attention
abstract); the real latents are not available and these draws stand in for
them.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

Q_ID, K_ID, V_ID, DO_ID = 0, 1, 2, 3
SCALE_STREAM, G_STREAM, CONV_STREAM = 10, 11, 12


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    batch: int
    heads: int
    head_dim: int
    grid: tuple            # (T, H, W)
    tile: tuple            # (t_t, t_h, t_w)
    window: tuple          # (w_t, w_h, w_w), in tiles
    pool: tuple            # (p_t, p_h, p_w)
    head_scale: bool = False   # per-head U(0.5, 2) scale on Q, K, V
    dual: bool = False         # has a global branch and a blend factor g
    backward: bool = False     # has an upstream gradient dO

    @property
    def n_tokens(self) -> int:
        T, H, W = self.grid
        return T * H * W


WORKLOADS = {
    "tiny": Workload("tiny", 0, 1, 2, 64, (4, 8, 8), (2, 4, 4), (1, 2, 2), (1, 1, 1)),
    "720p": Workload("720p", 1, 1, 24, 128, (30, 48, 80), (6, 8, 8), (3, 3, 3), (1, 1, 1),
                     head_scale=True),
    "1080p": Workload("1080p", 2, 1, 24, 128, (21, 72, 120), (3, 8, 8), (3, 3, 3), (1, 4, 4),
                      dual=True),
    "4k": Workload("4k", 3, 1, 24, 128, (21, 144, 240), (3, 8, 8), (3, 3, 5), (1, 8, 8),
                   dual=True),
    "train": Workload("train", 4, 2, 24, 128, (21, 72, 120), (3, 8, 8), (3, 3, 3), (1, 4, 4),
                      dual=True, backward=True),
}


def bf16_round_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> exact float64 values."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _stream(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=tuple(key))))


def head_scales(w: Workload) -> np.ndarray:
    if not w.head_scale:
        return np.ones(w.heads, dtype=np.float32)
    return _stream(w.seed, SCALE_STREAM).uniform(0.5, 2.0, size=w.heads).astype(np.float32)


def blend_g(w: Workload) -> np.ndarray:
    """Per-head blend factor g in [0, 1], float32 [heads]."""
    return _stream(w.seed, G_STREAM).uniform(0.0, 1.0, size=w.heads).astype(np.float32)


def learned_weights(w: Workload) -> dict:
    """Random weights of the learned compression / restoration convolutions
    (the method's trained values are not available), float32, taps-major:
      wq, wk, wv  [heads, p_t*p_h*p_w, d]  compression taps in (dt, dy, dx)
                  raster order, 1/P * (1 + 0.25 z): average pooling with a
                  perturbation, so the pooled tokens keep unit scale;
      w3          [heads, 27, d]  restoring 3x3x3 taps in (a, b, e) raster
                  order over {-1, 0, 1}^3: the identity tap 1 at the centre
                  plus 0.05 z everywhere."""
    P = w.pool[0] * w.pool[1] * w.pool[2]
    rng = _stream(w.seed, CONV_STREAM)
    out = {}
    for name in ("wq", "wk", "wv"):
        z = rng.standard_normal((w.heads, P, w.head_dim), dtype=np.float32)
        out[name] = ((1.0 + 0.25 * z) / np.float32(P)).astype(np.float32)
    w3 = 0.05 * rng.standard_normal((w.heads, 27, w.head_dim), dtype=np.float32)
    w3[:, 13, :] += 1.0
    out["w3"] = w3.astype(np.float32)
    return out


def draw_head(w: Workload, tensor_id: int, b: int, h: int) -> np.ndarray:
    """One [N, head_dim] slice as bfloat16 bits (uint16), raster order."""
    std = 0.1 if tensor_id == DO_ID else 1.0
    x = _stream(w.seed, tensor_id, b, h).standard_normal((w.n_tokens, w.head_dim), dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    if w.head_scale and tensor_id in (Q_ID, K_ID, V_ID):
        x *= head_scales(w)[h]
    return bf16_round_bits(x)


def draw(w: Workload, tensor_id: int, heads: Optional[list] = None,
         batches: Optional[list] = None) -> np.ndarray:
    """[len(batches), len(heads), N, head_dim] bfloat16 bits, raster order."""
    heads = list(range(w.heads)) if heads is None else list(heads)
    batches = list(range(w.batch)) if batches is None else list(batches)
    out = np.empty((len(batches), len(heads), w.n_tokens, w.head_dim), dtype=np.uint16)
    for i, b in enumerate(batches):
        for j, h in enumerate(heads):
            out[i, j] = draw_head(w, tensor_id, b, h)
    return out


def small_workload(name: str, seed: int, batch: int, heads: int, head_dim: int, grid, tile,
                   window, pool, dual: bool = True, backward: bool = True) -> Workload:
    """A workload outside the fixed table (parity and edge-case tests)."""
    return Workload(name, seed, batch, heads, head_dim, tuple(grid), tuple(tile), tuple(window),
                    tuple(pool), dual=dual, backward=backward)
