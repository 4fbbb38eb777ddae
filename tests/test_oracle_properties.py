"""Property-based pins of the oracle (CPU): random small geometries drawn by
hypothesis, each oracle function against an independent token-level masked
softmax built in the test (library SDPA in float64 for O, torch logsumexp of
the masked scores for LSE), and the kept-tile count
against its closed form.  The masks come from token coordinates only; the
oracle's tile-iteration code is not used to build them.  Every backward
oracle is also held to four identities of normalised softmax attention
(below), on random geometries, pools and blend factors."""
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


def _masked_lse(q, k, scale, mask):
    """ln sum_j exp(scale q_i . k_j) over the mask's keys (torch logsumexp, float64)."""
    s = torch.from_numpy(np.ascontiguousarray(q)) @ torch.from_numpy(np.ascontiguousarray(k)).transpose(-1, -2)
    s = (scale * s).masked_fill(~torch.from_numpy(mask), float("-inf"))
    return torch.logsumexp(s, dim=-1).numpy()


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
    o, lse = O.sta_attention(q, k, v, g, 0.5)
    np.testing.assert_allclose(o, _sdpa(q, k, v, 0.5, mask), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, _masked_lse(q, k, 0.5, mask), rtol=0, atol=1e-12)
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
    o, lse = O.xwin_attention(q, k, v, g, 0.5, shifted)
    np.testing.assert_allclose(o, _sdpa(q, k, v, 0.5, mask), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, _masked_lse(q, k, 0.5, mask), rtol=0, atol=1e-12)


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
    o, lse = O.hier_attention(q, k, v, g, hp, 0.5)
    joint = np.concatenate([fine, coarse], axis=1)
    np.testing.assert_allclose(o, _sdpa(q, keys, vals, 0.5, joint), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, _masked_lse(q, keys, 0.5, joint), rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# Backward identities that hold for any softmax attention whose rows are
# normalised over their key set, whatever the mask, pooling or blend:
#   sum_tokens dK = 0          (every row of dS sums to zero; pool^T keeps sums)
#   sum_tokens dV = sum dO     (rows of P sum to one; g + (1 - g) = 1; the
#                               upsampling weights of an output row sum to one)
#   <Q, dQ> = <K, dK>          (both equal scale * sum_ij dS_ij (q_i . k_j);
#                               pooling is linear, so it holds through it)
#   <V, dV> = <O, dO>          (both equal sum_ij P_ij (v_j . dO_i), per branch
#                               weight, with O the blended output)
# all per (batch, head).  They come from the mathematics, not from the
# oracle's code, and a dropped pool^T term, a missing branch weight, a
# transposed operand or a wrong sign in the softmax Jacobian breaks one.
# ---------------------------------------------------------------------------

def _identity_residuals(q, k, v, do, o, dq, dk, dv):
    sk = np.abs(dk.sum(axis=2)).max()
    sv = np.abs(dv.sum(axis=2) - do.sum(axis=2)).max()
    qk = np.abs((q * dq).sum(axis=(2, 3)) - (k * dk).sum(axis=(2, 3))).max()
    vo = np.abs((v * dv).sum(axis=(2, 3)) - (o * do).sum(axis=(2, 3))).max()
    return sk, sv, qk, vo


def _assert_identities(*a, atol=1e-9):
    sk, sv, qk, vo = _identity_residuals(*a)
    assert sk < atol, f"sum dK = {sk}"
    assert sv < atol, f"sum dV - sum dO = {sv}"
    assert qk < atol, f"<Q,dQ> - <K,dK> = {qk}"
    assert vo < atol, f"<V,dV> - <O,dO> = {vo}"


def _divisors(n):
    return [p for p in range(1, n + 1) if n % p == 0]


@st.composite
def pooled_geoms(draw):
    g = draw(geoms(max_tokens=192))
    pool = tuple(draw(st.sampled_from(_divisors(n))) for n in (g.T, g.H, g.W))
    return g._replace(pool=pool)


def _qkvdo(n, seed, heads=2, d=4):
    q, k, v = (_rand((1, heads, n, d), seed + i) for i in range(3))
    return q, k, v, 0.3 * _rand((1, heads, n, d), seed + 3)


@SETTINGS
@given(g=geoms(max_tokens=192), seed=st.integers(0, 10_000))
def test_sta_backward_identities(g, seed):
    q, k, v, do = _qkvdo(g.n, seed)
    o, _ = O.sta_attention(q, k, v, g, 0.5)
    _assert_identities(q, k, v, do, o, *O.sta_backward(q, k, v, do, g, 0.5))


@SETTINGS
@given(g=geoms(max_tokens=192), shifted=st.booleans(), seed=st.integers(0, 10_000))
def test_xwin_backward_identities(g, shifted, seed):
    q, k, v, do = _qkvdo(g.n, seed)
    o, _ = O.xwin_attention(q, k, v, g, 0.5, shifted)
    _assert_identities(q, k, v, do, o, *O.xwin_backward(q, k, v, do, g, 0.5, shifted))


@SETTINGS
@given(g=pooled_geoms(), seed=st.integers(0, 10_000))
def test_dual_backward_identities(g, seed):
    q, k, v, do = _qkvdo(g.n, seed)
    gvec = np.random.default_rng(seed).uniform(0, 1, 2)
    o = O.dual_forward(q, k, v, gvec, g, 0.5)["O"]
    r = O.dual_backward(q, k, v, gvec, do, g, 0.5)
    _assert_identities(q, k, v, do, o, r["dQ"], r["dK"], r["dV"])


@SETTINGS
@given(g=pooled_geoms(), seed=st.integers(0, 10_000))
def test_dual_sym_backward_identities(g, seed):
    q, k, v, do = _qkvdo(g.n, seed)
    gvec = np.random.default_rng(seed).uniform(0, 1, 2)
    o = O.dual_sym_forward(q, k, v, gvec, g, 0.5)["O"]
    r = O.dual_sym_backward(q, k, v, gvec, do, g, 0.5)
    _assert_identities(q, k, v, do, o, r["dQ"], r["dK"], r["dV"])


@SETTINGS
@given(gh=hier_geoms(), seed=st.integers(0, 10_000))
def test_hier_backward_identities(gh, seed):
    g, hp = gh
    q, k, v, do = _qkvdo(g.n, seed)
    o, _ = O.hier_attention(q, k, v, g, hp, 0.5)
    _assert_identities(q, k, v, do, o, *O.hier_backward(q, k, v, do, g, hp, 0.5))


def test_identities_catch_planted_mistakes(monkeypatch):
    """Mistakes planted in the oracle (on the CPU) break an identity."""
    g = O.Geom(2, 4, 4, (1, 2, 2), (1, 1, 1), (1, 2, 2))
    q, k, v, do = _qkvdo(g.n, 7)
    gvec = np.array([0.3, 0.8])
    o = O.dual_forward(q, k, v, gvec, g, 0.5)["O"]

    def residuals():
        r = O.dual_backward(q, k, v, gvec, do, g, 0.5)
        return _identity_residuals(q, k, v, do, o, r["dQ"], r["dK"], r["dV"])

    assert max(residuals()) < 1e-9
    with monkeypatch.context() as m:   # the pooled branch's gradients not sent back through the pooling
        m.setattr(O, "pool_transpose", lambda y, g: np.zeros(y.shape[:2] + (g.n, y.shape[3])))
        assert max(residuals()) > 1e-3
    true_bwd = O._softmax_attend_bwd

    def no_rowsum(q_, k_, v_, do_, scale):   # dS = P * dP: the Jacobian's rank-one term dropped
        _, _, p = O._softmax_attend(q_, k_, v_, scale)
        ds = p * (do_ @ v_.T)
        return scale * (ds @ k_), scale * (ds.T @ q_), p.T @ do_
    with monkeypatch.context() as m:
        m.setattr(O, "_softmax_attend_bwd", no_rowsum)
        assert residuals()[0] > 1e-3

    def dk_without_scale(q_, k_, v_, do_, scale):   # scale applied to dQ but not to dK
        a, b, c = true_bwd(q_, k_, v_, do_, scale)
        return a, b / scale, c
    with monkeypatch.context() as m:
        m.setattr(O, "_softmax_attend_bwd", dk_without_scale)
        assert residuals()[2] > 1e-3


def _avg_pool(x, g):
    """Raster [B, h, n, d] -> pooled raster [B, h, n_p, d] by torch avg_pool3d."""
    B, h, _, d = x.shape
    t = torch.from_numpy(np.ascontiguousarray(x)).reshape(B * h, g.T, g.H, g.W, d).permute(0, 4, 1, 2, 3)
    p = torch.nn.functional.avg_pool3d(t, kernel_size=g.pool, stride=g.pool)
    return p.permute(0, 2, 3, 4, 1).reshape(B, h, -1, d).numpy()


def _trilinear(x, g):
    """Pooled raster -> full grid by torch trilinear interpolation (half-pixel centres)."""
    B, h, _, d = x.shape
    PT, PH, PW = g.pooled_dims
    t = torch.from_numpy(np.ascontiguousarray(x)).reshape(B * h, PT, PH, PW, d).permute(0, 4, 1, 2, 3)
    u = torch.nn.functional.interpolate(t, size=(g.T, g.H, g.W), mode="trilinear", align_corners=False)
    return u.permute(0, 2, 3, 4, 1).reshape(B, h, -1, d).numpy()


def _sta_mask(g):
    cs = _coords(g.T, g.H, g.W)
    dims = g.tiles_per_dim
    wins = [[_window_set(a, g.window[ax], dims[ax]) for a in range(dims[ax])] for ax in range(3)]
    tile_of = [tuple(c[ax] // g.tile[ax] for ax in range(3)) for c in cs]
    return np.array([[all(tj[ax] in wins[ax][ti[ax]] for ax in range(3)) for tj in tile_of] for ti in tile_of])


@SETTINGS
@given(g=pooled_geoms(), seed=st.integers(0, 10_000))
def test_dual_forward_matches_library_pooling(g, seed):
    q, k, v, _ = _qkvdo(g.n, seed)
    gvec = np.random.default_rng(seed).uniform(0, 1, 2)
    r = O.dual_forward(q, k, v, gvec, g, 0.5)
    kp, vp = _avg_pool(k, g), _avg_pool(v, g)
    np.testing.assert_allclose(r["K_p"], kp, rtol=0, atol=1e-13)
    o_l = _sdpa(q, k, v, 0.5, _sta_mask(g))
    o_g = _sdpa(q, kp, vp, 0.5, np.ones((g.n, g.n_pooled), dtype=bool))
    gb = gvec[None, :, None, None]
    np.testing.assert_allclose(r["O"], gb * o_l + (1 - gb) * o_g, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["LSE_g"], _masked_lse(q, kp, 0.5, np.ones((g.n, g.n_pooled), dtype=bool)),
                               rtol=0, atol=1e-12)


@SETTINGS
@given(g=pooled_geoms(), seed=st.integers(0, 10_000))
def test_dual_sym_forward_matches_library_pool_and_trilinear(g, seed):
    q, k, v, _ = _qkvdo(g.n, seed)
    gvec = np.random.default_rng(seed).uniform(0, 1, 2)
    r = O.dual_sym_forward(q, k, v, gvec, g, 0.5)
    qp, kp, vp = (_avg_pool(x, g) for x in (q, k, v))
    o_p = _sdpa(qp, kp, vp, 0.5, np.ones((g.n_pooled, g.n_pooled), dtype=bool))
    np.testing.assert_allclose(r["O_p"], o_p, rtol=0, atol=1e-12)
    o_l = _sdpa(q, k, v, 0.5, _sta_mask(g))
    gb = gvec[None, :, None, None]
    np.testing.assert_allclose(r["O"], gb * o_l + (1 - gb) * _trilinear(o_p, g), rtol=0, atol=1e-12)
