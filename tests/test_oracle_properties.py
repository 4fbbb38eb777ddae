"""Property-based pins of the oracle (CPU): random small geometries drawn by
hypothesis, each oracle function against an independent token-level masked
softmax built in the test (library SDPA in float64), and the kept-tile count
against its closed form.  The masks come from token coordinates only; the
oracle's tile-iteration code is not used to build them."""
import math

import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from oracle import vattn_oracle as O

SETTINGS = settings(max_examples=25, deadline=None, suppress_health_check=[HealthCheck.too_slow])


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa(q, k, v, scale, mask):
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(a)) for a in (q, k, v))
    return torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.from_numpy(mask),
                                                            scale=scale).numpy()


def _window_set(a, w, n):
    """The clamped window by its characterisation: the interval of length
    min(w, n) inside [0, n) whose start is nearest to a - floor(w/2)."""
    e = min(w, n)
    start = min(range(0, n - e + 1), key=lambda s: abs(s - (a - w // 2)))
    return set(range(start, start + e))


def _coords(T, H, W):
    return [(t, y, x) for t in range(T) for y in range(H) for x in range(W)]


@st.composite
def geoms(draw, max_tokens=320):
    tile = tuple(draw(st.integers(1, 3)) for _ in range(3))
    tiles = tuple(draw(st.integers(1, 4)) for _ in range(3))
    window = tuple(draw(st.integers(1, 5)) for _ in range(3))
    T, H, W = (a * b for a, b in zip(tile, tiles))
    if T * H * W > max_tokens:
        tiles = (1, tiles[1], tiles[2])
        T = tile[0]
    return O.Geom(T, H, W, tile, window)


@SETTINGS
@given(g=geoms(), seed=st.integers(0, 10_000))
def test_sta_matches_coordinate_mask(g, seed):
    cs = _coords(g.T, g.H, g.W)
    dims = g.tiles_per_dim
    wins = [[_window_set(a, g.window[ax], dims[ax]) for a in range(dims[ax])] for ax in range(3)]
    tile_of = [tuple(c[ax] // g.tile[ax] for ax in range(3)) for c in cs]
    mask = np.array([[all(tj[ax] in wins[ax][ti[ax]] for ax in range(3)) for tj in tile_of] for ti in tile_of])
    q, k, v = (_rand((1, 1, g.n, 4), seed + i) for i in range(3))
    o, _ = O.sta_attention(q, k, v, g, 0.5)
    np.testing.assert_allclose(o, _sdpa(q, k, v, 0.5, mask), rtol=0, atol=1e-12)
    # kept tiles per query tile: the closed form
    assert all(len(O.kept_tiles(g)[t]) == O.kept_count_closed_form(g) for t in range(math.prod(dims)))


@SETTINGS
@given(g=geoms(), shifted=st.booleans(), seed=st.integers(0, 10_000))
def test_xwin_matches_coordinate_blocks(g, shifted, seed):
    cs = _coords(g.T, g.H, g.W)

    def block(a, w, n):
        size, off = (w + 1, (w + 1) // 2) if shifted else (w, 0)
        return (a + off) // size

    tile_of = [tuple(c[ax] // g.tile[ax] for ax in range(3)) for c in cs]
    lab = [tuple(block(t[ax], g.window[ax], g.tiles_per_dim[ax]) for ax in range(3)) for t in tile_of]
    mask = np.array([[li == lj for lj in lab] for li in lab])
    q, k, v = (_rand((1, 1, g.n, 4), seed + i) for i in range(3))
    o, _ = O.xwin_attention(q, k, v, g, 0.5, shifted)
    np.testing.assert_allclose(o, _sdpa(q, k, v, 0.5, mask), rtol=0, atol=1e-12)


@st.composite
def hier_geoms(draw):
    tile = tuple(draw(st.integers(1, 2)) for _ in range(3))
    hp = tuple(draw(st.integers(1, 2)) for _ in range(3))
    coarse = tuple(draw(st.integers(1, 3)) for _ in range(3))
    window = tuple(draw(st.integers(1, 4)) for _ in range(3))
    T, H, W = (t * p * c for t, p, c in zip(tile, hp, coarse))
    return O.Geom(T, H, W, tile, window), hp


@SETTINGS
@given(gh=hier_geoms(), seed=st.integers(0, 10_000))
def test_hier_matches_coordinate_mask(gh, seed):
    g, hp = gh
    cs = _coords(g.T, g.H, g.W)
    P = (g.T // hp[0], g.H // hp[1], g.W // hp[2])
    pcs = _coords(*P)
    nc = tuple(P[ax] // g.tile[ax] for ax in range(3))
    dims = g.tiles_per_dim
    fw = [[_window_set(a, g.window[ax], dims[ax]) for a in range(dims[ax])] for ax in range(3)]
    cw = [[_window_set(a, g.window[ax], nc[ax]) for a in range(nc[ax])] for ax in range(3)]
    tile_of = [tuple(c[ax] // g.tile[ax] for ax in range(3)) for c in cs]
    fine = np.array([[all(tj[ax] in fw[ax][ti[ax]] for ax in range(3)) for tj in tile_of] for ti in tile_of])
    ctile = [tuple(c[ax] // g.tile[ax] for ax in range(3)) for c in pcs]
    coarse = np.array([[all(ck[ax] in cw[ax][ti[ax] // hp[ax]] for ax in range(3)) for ck in ctile]
                       for ti in tile_of])
    q, k, v = (_rand((1, 1, g.n, 4), seed + i) for i in range(3))

    def pool(x):   # block mean by reshape
        y = x.reshape(1, 1, P[0], hp[0], P[1], hp[1], P[2], hp[2], 4)
        return y.mean(axis=(3, 5, 7)).reshape(1, 1, -1, 4)

    keys = np.concatenate([k, pool(k)], axis=2)
    vals = np.concatenate([v, pool(v)], axis=2)
    o, _ = O.hier_attention(q, k, v, g, hp, 0.5)
    np.testing.assert_allclose(o, _sdpa(q, keys, vals, 0.5, np.concatenate([fine, coarse], axis=1)), rtol=0,
                               atol=1e-12)
