"""Pins of the fp64 oracle against facts the definition fixes (CPU only).

The pages print no worked numeric example, so every pin here is one of:
invariants of the definition, reductions to a textbook or library routine
(torch scaled_dot_product_attention in float64), brute force on tiny grids
written independently of the oracle's own index code, or fp64 central finite
differences for the backward.  The mutation tests at the end plant a plausible
mistake in the oracle and check that some pin catches it.
"""
import itertools
import math

import numpy as np
import pytest
import torch

from oracle import vattn_oracle as O
from synth import inputs as S


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa(q, k, v, scale, mask=None):
    """Library softmax attention in float64 (the textbook definition's routine)."""
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(a)) for a in (q, k, v))
    m = None if mask is None else torch.from_numpy(mask)
    return torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=m, scale=scale).numpy()


def _brute_window(a, w, n):
    """Independent characterisation of the clamped window: among all intervals
    of length min(w, n) inside [0, n), the one whose start is nearest to
    a - floor(w/2)."""
    e = min(w, n)
    best = min(range(0, n - e + 1), key=lambda s: abs(s - (a - w // 2)))
    return set(range(best, best + e))


def _brute_mask(g):
    """Token-by-token visibility mask from token coordinates (no oracle code)."""
    T, H, W = g.T, g.H, g.W
    coords = [(t, y, x) for t in range(T) for y in range(H) for x in range(W)]
    dims = (T // g.tile[0], H // g.tile[1], W // g.tile[2])
    win = [[_brute_window(a, g.window[ax], dims[ax]) for a in range(dims[ax])] for ax in range(3)]
    n = len(coords)
    mask = np.zeros((n, n), dtype=bool)
    for i, ci in enumerate(coords):
        ti = [ci[ax] // g.tile[ax] for ax in range(3)]
        for j, cj in enumerate(coords):
            tj = [cj[ax] // g.tile[ax] for ax in range(3)]
            mask[i, j] = all(tj[ax] in win[ax][ti[ax]] for ax in range(3))
    return mask


TINY = O.Geom(4, 8, 8, (2, 4, 4), (1, 2, 2), (1, 1, 1))
TINY_POOLED = O.Geom(4, 8, 8, (2, 4, 4), (1, 2, 2), (1, 2, 2))
ODD = O.Geom(6, 12, 20, (2, 4, 4), (3, 3, 3), (1, 2, 2))   # 3x3x5 tile grid, clamped interior+edges

ALL_GEOMS = [O.geom_of(w) for w in S.WORKLOADS.values()]


# ---------------------------------------------------------------- permutation

@pytest.mark.parametrize("g", ALL_GEOMS + [TINY, ODD], ids=lambda g: f"{g.T}x{g.H}x{g.W}")
def test_permutation_matches_reshape_formulation(g):
    # raster [T,H,W] -> [Nt,tt,Nh,th,Nw,tw] -> [Nt,Nh,Nw,tt,th,tw]: tile-major by construction
    nt, nh, nw = g.tiles_per_dim
    tt, th, tw = g.tile
    raster_ids = np.arange(g.n).reshape(nt, tt, nh, th, nw, tw).transpose(0, 2, 4, 1, 3, 5).reshape(-1)
    m = O.tile_major_index(g)
    # tiled position p holds raster token raster_ids[p]  <=>  m[raster_ids[p]] == p
    assert np.array_equal(m[raster_ids], np.arange(g.n))


@pytest.mark.parametrize("g", [TINY, ODD])
def test_permute_roundtrip_and_bijection(g):
    x = _rand((2, 3, g.n, 8), 1)
    assert np.array_equal(O.unpermute(O.permute(x, g), g), x)
    m = O.tile_major_index(g)
    assert np.array_equal(np.sort(m), np.arange(g.n))
    # each tile is contiguous and holds only tokens of that tile
    xt = O.permute(O.token_coords(g).astype(np.float64), g)
    s = g.tile_volume
    for tid in range(g.n // s):
        tc = xt[tid * s:(tid + 1) * s] // np.asarray(g.tile)
        assert (tc == tc[0]).all()


# ---------------------------------------------------------------- kept tiles

@pytest.mark.parametrize("g", ALL_GEOMS + [TINY, ODD], ids=lambda g: f"{g.T}x{g.H}x{g.W}")
def test_kept_count_closed_form_every_tile(g):
    kt = O.kept_tiles(g)
    assert kt.shape == (math.prod(g.tiles_per_dim), O.kept_count_closed_form(g))
    for row in kt:
        assert len(set(row.tolist())) == kt.shape[1]


@pytest.mark.parametrize("g", ALL_GEOMS + [ODD], ids=lambda g: f"{g.T}x{g.H}x{g.W}")
def test_kept_window_matches_bruteforce_window(g):
    dims = g.tiles_per_dim
    for ax in range(3):
        for a in range(dims[ax]):
            assert set(O.window_range(a, g.window[ax], dims[ax])) == _brute_window(a, g.window[ax], dims[ax])


def test_inverse_counts():
    # 1080p grid, w dim: N=15 tiles, w=3; t dim: N=7, w=3; 720p t dim: N=5, w=3.
    def inverse(n, w):
        cnt = [0] * n
        for a in range(n):
            for kk in _brute_window(a, w, n):
                cnt[kk] += 1
        return cnt
    assert inverse(7, 3) == [2, 3, 4, 3, 4, 3, 2]
    assert inverse(5, 3) == [2, 3, 5, 3, 2]
    for w in S.WORKLOADS.values():
        g = O.geom_of(w)
        kt = O.kept_tiles(g)
        inv = np.bincount(kt.reshape(-1), minlength=kt.shape[0])
        assert inv.sum() == kt.shape[0] * kt.shape[1]
        # per-dim factorisation of the inverse count
        dims = g.tiles_per_dim
        per = [inverse(dims[ax], g.window[ax]) for ax in range(3)]
        expect = np.array([per[0][a] * per[1][b] * per[2][c]
                           for a in range(dims[0]) for b in range(dims[1]) for c in range(dims[2])])
        assert np.array_equal(inv, expect)


# ---------------------------------------------------------------- local branch

def test_tiny_tiled_equals_independent_masked_softmax():
    w = S.WORKLOADS["tiny"]
    g = O.geom_of(w)
    q, k, v = (S.bf16_bits_to_f64(S.draw(w, i)) for i in range(3))
    scale = 1 / math.sqrt(w.head_dim)
    mask = _brute_mask(g)
    assert np.array_equal(mask, O.sta_mask_bruteforce(g))
    o, lse = O.sta_attention(q, k, v, g, scale)
    ref = _sdpa(q, k, v, scale, mask)
    assert np.abs(o - ref).max() < 1e-12
    s = np.einsum("bhid,bhjd->bhij", q, k) * scale
    s = np.where(mask, s, -np.inf)
    from scipy.special import logsumexp
    assert np.abs(lse - logsumexp(s, axis=-1)).max() < 1e-12
    o2, lse2 = O.sta_attention_bruteforce(q, k, v, g, scale)
    assert np.abs(o - o2).max() < 1e-12 and np.abs(lse - lse2).max() < 1e-12


@pytest.mark.parametrize("g", [O.Geom(4, 8, 8, (2, 4, 4), (2, 2, 2)), O.Geom(6, 12, 20, (2, 4, 4), (9, 9, 9))])
def test_window_covering_grid_equals_full_attention(g):
    q, k, v = (_rand((1, 2, g.n, 16), s) for s in (3, 4, 5))
    o, lse = O.sta_attention(q, k, v, g, 0.25)
    assert np.abs(o - _sdpa(q, k, v, 0.25)).max() < 1e-12
    from scipy.special import logsumexp
    assert np.abs(lse - logsumexp(np.einsum("bhid,bhjd->bhij", q, k) * 0.25, axis=-1)).max() < 1e-12


def test_odd_grid_against_independent_mask():
    g = ODD
    q, k, v = (_rand((1, 1, g.n, 8), s) for s in (6, 7, 8))
    mask = _brute_mask(g)
    o, _ = O.sta_attention(q, k, v, g, 0.3)
    assert np.abs(o - _sdpa(q, k, v, 0.3, mask)).max() < 1e-12


# ---------------------------------------------------------------- pooling / global branch

@pytest.mark.parametrize("g", [TINY_POOLED, ODD, O.Geom(3, 8, 8, (3, 8, 8), (1, 1, 1), (1, 8, 8))])
def test_pool_reshape_constant_adjoint(g):
    x = _rand((2, g.n, 5), 9)
    pt, ph, pw = g.pool
    T, H, W = g.T, g.H, g.W
    ref = x.reshape(2, T // pt, pt, H // ph, ph, W // pw, pw, 5).mean(axis=(2, 4, 6)).reshape(2, -1, 5)
    assert np.abs(O.pool(x, g) - ref).max() < 1e-13
    c = np.full((g.n, 3), 0.3125)
    assert np.abs(O.pool(c, g) - 0.3125).max() == 0.0
    y = _rand((2, g.n_pooled, 5), 10)
    assert abs((O.pool(x, g) * y).sum() - (x * O.pool_transpose(y, g)).sum()) < 1e-10


def test_pool_one_global_equals_full_attention():
    g = O.Geom(4, 8, 8, (2, 4, 4), (1, 2, 2), (1, 1, 1))
    q, k, v = (_rand((1, 2, g.n, 16), s) for s in (11, 12, 13))
    kp, vp = O.pool(k, g), O.pool(v, g)
    assert np.array_equal(kp, k) and np.array_equal(vp, v)
    o, _ = O.global_attention(q, kp, vp, 0.25)
    assert np.abs(o - _sdpa(q, k, v, 0.25)).max() < 1e-12


def test_constant_values_give_constant_output():
    g = TINY_POOLED
    q, k = (_rand((1, 2, g.n, 8), s) for s in (14, 15))
    v = np.broadcast_to(np.linspace(-1, 1, 8), (1, 2, g.n, 8)).copy()
    r = O.dual_forward(q, k, v, [0.3, 0.8], g, 0.35)
    for key in ("O", "O_l", "O_g"):
        assert np.abs(r[key] - v).max() < 1e-12


def test_blend_endpoints():
    g = TINY_POOLED
    q, k, v = (_rand((1, 2, g.n, 8), s) for s in (16, 17, 18))
    r = O.dual_forward(q, k, v, [1.0, 0.0], g, 0.35)
    assert np.array_equal(r["O"][:, 0], r["O_l"][:, 0])
    assert np.array_equal(r["O"][:, 1], r["O_g"][:, 1])


# ---------------------------------------------------------------- backward

def _dual_loss(q, k, v, gvec, do, g, scale):
    return float((O.dual_forward(q, k, v, gvec, g, scale)["O"] * do).sum())


@pytest.mark.parametrize("g", [TINY, TINY_POOLED, ODD], ids=["tiny", "tiny_pooled", "odd"])
def test_dual_backward_finite_differences(g):
    rng = np.random.default_rng(20)
    B, nh, d = 1, 2, 8
    q, k, v = (rng.standard_normal((B, nh, g.n, d)) for _ in range(3))
    do = 0.1 * rng.standard_normal((B, nh, g.n, d))
    gvec = np.array([0.3, 0.7])
    scale = 0.4
    grads = O.dual_backward(q, k, v, gvec, do, g, scale)
    eps = 1e-5
    for name, arr, key in (("q", q, "dQ"), ("k", k, "dK"), ("v", v, "dV")):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, s)) for s in arr.shape)
            old = arr[idx]
            arr[idx] = old + eps
            lp = _dual_loss(q, k, v, gvec, do, g, scale)
            arr[idx] = old - eps
            lm = _dual_loss(q, k, v, gvec, do, g, scale)
            arr[idx] = old
            fd = (lp - lm) / (2 * eps)
            an = grads[key][idx]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, an)
    for h in range(nh):
        gp, gm = gvec.copy(), gvec.copy()
        gp[h] += eps
        gm[h] -= eps
        fd = (_dual_loss(q, k, v, gp, do, g, scale) - _dual_loss(q, k, v, gm, do, g, scale)) / (2 * eps)
        assert abs(fd - grads["dg"][h]) <= 1e-6 * max(1.0, abs(fd))


def test_backward_matches_autograd_masked_reference():
    g = TINY_POOLED
    rng = np.random.default_rng(21)
    q, k, v = (rng.standard_normal((1, 2, g.n, 8)) for _ in range(3))
    do = rng.standard_normal((1, 2, g.n, 8))
    gvec = np.array([0.25, 0.6])
    scale = 0.3
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    mask = torch.from_numpy(_brute_mask(g))
    o_l = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=scale)
    T, H, W = g.T, g.H, g.W
    pt, ph, pw = g.pool

    def tpool(x):
        return x.reshape(1, 2, T // pt, pt, H // ph, ph, W // pw, pw, 8).mean(dim=(3, 5, 7)).reshape(1, 2, -1, 8)
    o_g = torch.nn.functional.scaled_dot_product_attention(tq, tpool(tk), tpool(tv), scale=scale)
    gb = torch.tensor(gvec)[None, :, None, None]
    (gb * o_l + (1 - gb) * o_g).backward(torch.from_numpy(do))
    r = O.dual_backward(q, k, v, gvec, do, g, scale)
    assert np.abs(r["dQ"] - tq.grad.numpy()).max() < 1e-12
    assert np.abs(r["dK"] - tk.grad.numpy()).max() < 1e-12
    assert np.abs(r["dV"] - tv.grad.numpy()).max() < 1e-12


# ---------------------------------------------------------------- accounting

def test_ultragen_complexity_closed_form():
    # "UltraGen ..." App. B: about a 12-fold reduction at K = 4
    r = O.ultragen_cost_ratio(4)
    assert abs(r - (5 / 64 + 1 / 256)) < 1e-15
    assert round(1 / r) == 12


def test_pair_counts():
    g = O.geom_of(S.WORKLOADS["720p"])
    assert O.kept_pairs_local(g, 1, 24) == 24 * 115200 * 27 * 384
    g = O.geom_of(S.WORKLOADS["1080p"])
    assert g.n_pooled == 11340 and O.pairs_global(g, 1, 24) == 24 * 181440 * 11340
    assert O.geom_of(S.WORKLOADS["4k"]).n_pooled == 11340


# ---------------------------------------------------------------- planted mistakes (oracle only)

def test_pins_catch_unclamped_window(monkeypatch):
    def bad(a, w, n):
        lo = max(a - w // 2, 0)
        return range(lo, min(lo + w, n))     # truncates instead of shifting inward
    monkeypatch.setattr(O, "window_range", bad)
    g = ODD
    with pytest.raises(AssertionError):
        test_kept_window_matches_bruteforce_window(g)
    with pytest.raises(AssertionError):
        test_odd_grid_against_independent_mask()


def test_pins_catch_wrong_jacobian_sign(monkeypatch):
    orig = O._softmax_attend_bwd

    def bad(q, k, v, do, scale):
        dq, dk, dv = orig(q, k, v, do, scale)
        return dq, -dk, dv
    monkeypatch.setattr(O, "_softmax_attend_bwd", bad)
    with pytest.raises(AssertionError):
        test_dual_backward_finite_differences(TINY_POOLED)


def test_pins_catch_wrong_pool_count(monkeypatch):
    orig = O.pool
    monkeypatch.setattr(O, "pool", lambda x, g: orig(x, g) * 1.0001)
    with pytest.raises(AssertionError):
        test_pool_reshape_constant_adjoint(TINY_POOLED)


def test_pins_catch_transposed_tile_order(monkeypatch):
    orig = O.tile_major_index

    def bad(g):
        tt, th, tw = g.tile
        nt, nh, nw = g.tiles_per_dim
        c = O.token_coords(g)
        t, y, x = c[:, 0], c[:, 1], c[:, 2]
        tile_id = ((x // tw) * nh + y // th) * nt + t // tt     # w outermost: wrong
        local = ((t % tt) * th + y % th) * tw + x % tw
        return tile_id * g.tile_volume + local
    monkeypatch.setattr(O, "tile_major_index", bad)
    with pytest.raises(AssertionError):
        test_permutation_matches_reshape_formulation(ODD)
    monkeypatch.setattr(O, "tile_major_index", orig)


def test_sampled_evaluators_equal_full_definitions():
    """The row-restricted helpers used for large grids agree with the full
    definitions on a grid where both run."""
    g = ODD
    rng = np.random.default_rng(33)
    q, k, v = (rng.standard_normal((1, 1, g.n, 8)) for _ in range(3))
    do = rng.standard_normal((1, 1, g.n, 8))
    full = O.dual_backward(q, k, v, [0.35], do, g, 0.4)
    s = O.dual_backward_sampled(q[0, 0], k[0, 0], v[0, 0], 0.35, do[0, 0], g, 0.4, [0, 7, 44], [0, 13, 44], chunk=97)
    assert np.abs(s["dQ"] - full["dQ"][0, 0][s["q_ids"]]).max() < 1e-12
    assert np.abs(s["dK"] - full["dK"][0, 0][s["k_ids"]]).max() < 1e-12
    assert np.abs(s["dV"] - full["dV"][0, 0][s["k_ids"]]).max() < 1e-12
    fwd = O.dual_forward(q, k, v, [0.35], g, 0.4)
    ids, ol, lsel = O.sta_attention_tiles(q[0, 0], k[0, 0], v[0, 0], g, 0.4, [3, 20])
    assert np.abs(ol - fwd["O_l"][0, 0][ids]).max() < 1e-12 and np.abs(lsel - fwd["LSE_l"][0, 0][ids]).max() < 1e-12
    og, lseg = O.global_attention_rows(q[0, 0], fwd["K_p"][0, 0], fwd["V_p"][0, 0], 0.4, ids)
    assert np.abs(og - fwd["O_g"][0, 0][ids]).max() < 1e-12


# ---------------------------------------------------------------- cross-window local attention

def _brute_blocks(n, w, shifted):
    """Independent construction of the partition: walk the dim and start a new
    block at every cut (cuts at positions p with (p + off) % size == 0)."""
    size = w + 1 if shifted else w
    off = (w + 1) // 2 if shifted else 0
    blocks, cur = [], []
    for p in range(n):
        if cur and (p + off) % size == 0:
            blocks.append(cur)
            cur = []
        cur.append(p)
    blocks.append(cur)
    return blocks


@pytest.mark.parametrize("shifted", [False, True])
def test_partition_blocks_tile_the_dim_and_match_walk(shifted):
    for n in range(1, 17):
        for w in range(1, 9):
            blocks = _brute_blocks(n, w, shifted)
            assert sorted(x for b in blocks for x in b) == list(range(n))
            for b in blocks:
                for a in b:
                    assert list(O.partition_range(a, w, n, shifted)) == b


def test_shifted_blocks_straddle_unshifted_cuts():
    # every interior cut of the K-partition lies strictly inside a shifted block
    for n in (9, 15, 30):
        for w in (2, 3, 4):
            cuts = [b[0] for b in _brute_blocks(n, w, False)][1:]
            for c in cuts:
                r = O.partition_range(c, w, n, True)
                if r.start != c:
                    continue
                # a cut shared by both partitions is allowed only where the periods realign
                assert (c + (w + 1) // 2) % (w + 1) == 0 and c % w == 0


def _xwin_mask(g, shifted):
    c = O.token_coords(g)
    tc = c // np.asarray(g.tile)
    dims = g.tiles_per_dim
    lab = []
    for ax in range(3):
        blocks = _brute_blocks(dims[ax], g.window[ax], shifted)
        label = np.empty(dims[ax], dtype=int)
        for i, b in enumerate(blocks):
            label[b] = i
        lab.append(label[tc[:, ax]])
    same = np.ones((g.n, g.n), dtype=bool)
    for ax in range(3):
        same &= lab[ax][:, None] == lab[ax][None, :]
    return same


@pytest.mark.parametrize("shifted", [False, True])
def test_xwin_equals_masked_softmax(shifted):
    g = O.Geom(4, 16, 24, (2, 4, 4), (1, 2, 3))
    q, k, v = (_rand((1, 2, g.n, 8), s) for s in (40, 41, 42))
    mask = _xwin_mask(g, shifted)
    assert np.array_equal(mask, mask.T)        # symmetric relation
    o, _ = O.xwin_attention(q, k, v, g, 0.3, shifted)
    assert np.abs(o - _sdpa(q, k, v, 0.3, mask)).max() < 1e-12


def test_xwin_window_covering_grid_is_full_attention():
    g = O.Geom(4, 8, 8, (2, 4, 4), (2, 2, 2))
    q, k, v = (_rand((1, 1, g.n, 8), s) for s in (43, 44, 45))
    o, _ = O.xwin_attention(q, k, v, g, 0.3, False)
    assert np.abs(o - _sdpa(q, k, v, 0.3)).max() < 1e-12


@pytest.mark.parametrize("shifted", [False, True])
def test_xwin_backward_finite_differences(shifted):
    g = O.Geom(4, 16, 24, (2, 4, 4), (1, 2, 3))
    rng = np.random.default_rng(46)
    q, k, v = (rng.standard_normal((1, 1, g.n, 4)) for _ in range(3))
    do = rng.standard_normal((1, 1, g.n, 4))
    dq, dk, dv = O.xwin_backward(q, k, v, do, g, 0.4, shifted)

    def loss():
        return float((O.xwin_attention(q, k, v, g, 0.4, shifted)[0] * do).sum())
    eps = 1e-5
    for arr, grad in ((q, dq), (k, dk), (v, dv)):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, s)) for s in arr.shape)
            old = arr[idx]
            arr[idx] = old + eps
            lp = loss()
            arr[idx] = old - eps
            lm = loss()
            arr[idx] = old
            assert abs((lp - lm) / (2 * eps) - grad[idx]) <= 1e-6 * max(1.0, abs(grad[idx]))


# ---------------------------------------------------------------- symmetric global branch

@pytest.mark.parametrize("g", [O.Geom(4, 8, 12, (2, 4, 4), (1, 1, 1), (2, 4, 4)),
                               O.Geom(3, 16, 8, (1, 8, 8), (1, 1, 1), (1, 2, 4))],
                         ids=["pool244", "pool124"])
def test_upsample_matches_torch_trilinear(g):
    x = _rand((2, g.n_pooled, 3), 50)
    PT, PH, PW = g.pooled_dims
    t = torch.from_numpy(x).reshape(2, PT, PH, PW, 3).permute(0, 4, 1, 2, 3)
    ref = torch.nn.functional.interpolate(t, size=(g.T, g.H, g.W), mode="trilinear", align_corners=False)
    ref = ref.permute(0, 2, 3, 4, 1).reshape(2, g.n, 3).numpy()
    assert np.abs(O.upsample(x, g) - ref).max() < 1e-12


def test_upsample_adjoint_and_constants():
    g = O.Geom(4, 8, 12, (2, 4, 4), (1, 1, 1), (2, 4, 4))
    x = _rand((2, g.n_pooled, 3), 51)
    y = _rand((2, g.n, 3), 52)
    assert abs((O.upsample(x, g) * y).sum() - (x * O.upsample_transpose(y, g)).sum()) < 1e-10
    c = np.full((g.n_pooled, 2), -0.75)
    assert np.abs(O.upsample(c, g) + 0.75).max() < 1e-15        # partition of unity
    g1 = O.Geom(4, 8, 12, (2, 4, 4), (1, 1, 1), (1, 1, 1))   # pool 1: upsampling is the identity
    assert np.array_equal(O.upsample(y, g1), y)


def test_symmetric_global_pool_one_is_full_attention():
    g = O.Geom(4, 8, 8, (2, 4, 4), (1, 2, 2), (1, 1, 1))
    q, k, v = (_rand((1, 2, g.n, 8), s) for s in (53, 54, 55))
    o_g, _, _ = O.global_sym_forward(q, k, v, g, 0.3)
    assert np.abs(o_g - _sdpa(q, k, v, 0.3)).max() < 1e-12


def test_dual_sym_backward_finite_differences():
    g = O.Geom(4, 8, 8, (2, 4, 4), (1, 2, 2), (2, 2, 4))
    rng = np.random.default_rng(56)
    q, k, v = (rng.standard_normal((1, 2, g.n, 4)) for _ in range(3))
    do = 0.1 * rng.standard_normal((1, 2, g.n, 4))
    gvec = np.array([0.35, 0.8])
    r = O.dual_sym_backward(q, k, v, gvec, do, g, 0.4)

    def loss():
        return float((O.dual_sym_forward(q, k, v, gvec, g, 0.4)["O"] * do).sum())
    eps = 1e-5
    for arr, key in ((q, "dQ"), (k, "dK"), (v, "dV")):
        for _ in range(8):
            idx = tuple(int(rng.integers(0, s)) for s in arr.shape)
            old = arr[idx]
            arr[idx] = old + eps
            lp = loss()
            arr[idx] = old - eps
            lm = loss()
            arr[idx] = old
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - r[key][idx]) <= 1e-6 * max(1.0, abs(fd)), (key, fd, r[key][idx])


def test_sampled_symmetric_backward_equals_full():
    g = ODD
    rng = np.random.default_rng(57)
    q, k, v = (rng.standard_normal((1, 1, g.n, 8)) for _ in range(3))
    do = rng.standard_normal((1, 1, g.n, 8))
    full = O.dual_sym_backward(q, k, v, [0.4], do, g, 0.4)
    s = O.dual_backward_sampled(q[0, 0], k[0, 0], v[0, 0], 0.4, do[0, 0], g, 0.4, [0, 7, 44], [0, 13, 44],
                                symmetric=True)
    for key, ids in (("dQ", "q_ids"), ("dK", "k_ids"), ("dV", "k_ids")):
        assert np.abs(s[key] - full[key][0, 0][s[ids]]).max() < 1e-12


# ---------------------------------------------------------------- hierarchical local attention (NEXT-2)

def _pool_reshape(x, g, hp):
    """Independent block mean by reshape: [..., N, d] raster -> [..., N_h, d]."""
    lead, d = x.shape[:-2], x.shape[-1]
    y = x.reshape(lead + (g.T // hp[0], hp[0], g.H // hp[1], hp[1], g.W // hp[2], hp[2], d))
    return y.mean(axis=(-6, -4, -2)).reshape(lead + (-1, d))


def _hier_brute_mask(g, hp):
    """[N, N + N_h] visibility built token by token from coordinates: the fine
    part is the sliding-tile mask; pooled key j is visible to query i iff j's
    coarse tile (its pooled coordinates // tile) lies in the clamped window of
    the coarse tile holding i's fine tile (fine tile coordinates // h_pool)."""
    fine = _brute_mask(g)
    dims_p = (g.T // hp[0], g.H // hp[1], g.W // hp[2])
    nc = tuple(dp // t for dp, t in zip(dims_p, g.tile))
    cq = []
    for n in range(g.n):
        t, rem = divmod(n, g.H * g.W)
        y, x = divmod(rem, g.W)
        cq.append((t // g.tile[0] // hp[0], y // g.tile[1] // hp[1], x // g.tile[2] // hp[2]))
    ck = []
    for j in range(math.prod(dims_p)):
        t, rem = divmod(j, dims_p[1] * dims_p[2])
        y, x = divmod(rem, dims_p[2])
        ck.append((t // g.tile[0], y // g.tile[1], x // g.tile[2]))
    wins = [[_brute_window(a, g.window[ax], nc[ax]) for a in range(nc[ax])] for ax in range(3)]
    coarse = np.zeros((g.n, len(ck)), dtype=bool)
    for i, c in enumerate(cq):
        for j, e in enumerate(ck):
            coarse[i, j] = all(e[ax] in wins[ax][c[ax]] for ax in range(3))
    return np.concatenate([fine, coarse], axis=1)


HIER_CASES = [
    (O.Geom(4, 16, 32, (2, 4, 4), (1, 3, 3)), (1, 2, 2)),   # coarse window clamps along W only
    (O.Geom(4, 16, 16, (1, 4, 4), (3, 1, 1)), (2, 2, 2)),   # pooled in time as well
]


@pytest.mark.parametrize("g,hp", HIER_CASES)
def test_hier_equals_independent_masked_softmax(g, hp):
    q, k, v = (_rand((1, 2, g.n, 16), s) for s in (41, 42, 43))
    o, lse = O.hier_attention(q, k, v, g, hp, 0.3)
    keys = np.concatenate([k, _pool_reshape(k, g, hp)], axis=2)
    vals = np.concatenate([v, _pool_reshape(v, g, hp)], axis=2)
    mask = _hier_brute_mask(g, hp)
    np.testing.assert_allclose(o, _sdpa(q, keys, vals, 0.3, mask), rtol=0, atol=1e-12)
    s = np.einsum("bhnd,bhmd->bhnm", q, keys) * 0.3
    ref_lse = np.log(np.where(mask, np.exp(s), 0.0).sum(-1))
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_hier_pool_one_duplicates_every_local_key():
    """With h_pool = 1 the coarse keys are the fine keys again: each key counts
    twice, so O is the sliding-tile O and the LSE grows by exactly ln 2."""
    g = O.Geom(4, 8, 16, (2, 4, 4), (1, 1, 3))
    q, k, v = (_rand((2, 1, g.n, 8), s) for s in (44, 45, 46))
    o, lse = O.hier_attention(q, k, v, g, (1, 1, 1), 0.5)
    o_l, lse_l = O.sta_attention(q, k, v, g, 0.5)
    np.testing.assert_allclose(o, o_l, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lse_l + math.log(2.0), rtol=0, atol=1e-13)


def test_hier_windows_covering_everything_is_full_attention_over_both_sets():
    g = O.Geom(2, 8, 16, (1, 4, 4), (5, 5, 5))
    hp = (1, 2, 2)
    q, k, v = (_rand((1, 1, g.n, 8), s) for s in (47, 48, 49))
    o, lse = O.hier_attention(q, k, v, g, hp, 0.4)
    keys = np.concatenate([k, _pool_reshape(k, g, hp)], axis=2)
    vals = np.concatenate([v, _pool_reshape(v, g, hp)], axis=2)
    np.testing.assert_allclose(o, _sdpa(q, keys, vals, 0.4), rtol=0, atol=1e-12)


def test_hier_backward_finite_differences():
    g = O.Geom(2, 8, 16, (1, 4, 4), (1, 1, 3))
    hp = (1, 2, 2)
    q, k, v, do = (_rand((1, 1, g.n, 4), s) for s in (50, 51, 52, 53))
    dq, dk, dv = O.hier_backward(q, k, v, do, g, hp, 0.7)

    def loss(q_, k_, v_):
        return float((O.hier_attention(q_, k_, v_, g, hp, 0.7)[0] * do).sum())

    rng = np.random.default_rng(54)
    eps = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(6):
            idx = (0, 0, int(rng.integers(g.n)), int(rng.integers(4)))
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - grad[idx]) < 1e-7, (name, idx, fd, grad[idx])


def test_hier_sampled_evaluator_equals_full_definition():
    g, hp = HIER_CASES[0]
    q, k, v = (_rand((1, 1, g.n, 8), s) for s in (55, 56, 57))
    o, lse = O.hier_attention(q, k, v, g, hp, 0.3)
    tiles = [0, 5, 17, 63]
    ids, o_s, l_s = O.hier_attention_tiles(q[0, 0], k[0, 0], v[0, 0], g, hp, 0.3, tiles)
    np.testing.assert_allclose(o_s, o[0, 0][ids], rtol=0, atol=1e-13)
    np.testing.assert_allclose(l_s, lse[0, 0][ids], rtol=0, atol=1e-13)


def test_pins_catch_coarse_tile_without_division(monkeypatch):
    """Planted mistake: the coarse window centred on the fine tile index."""
    monkeypatch.setattr(O, "coarse_tile_of", lambda a, hp: tuple(a))
    g, hp = HIER_CASES[0]
    with pytest.raises(AssertionError):
        test_hier_equals_independent_masked_softmax(g, hp)


def test_hier_sampled_dq_equals_full_backward():
    g, hp = HIER_CASES[0]
    q, k, v, do = (_rand((1, 1, g.n, 8), s) for s in (58, 59, 60, 61))
    dq, _, _ = O.hier_backward(q, k, v, do, g, hp, 0.3)
    tiles = [0, 7, 19, 63]
    ids, rows = O.hier_backward_dq_tiles(q[0, 0], k[0, 0], v[0, 0], do[0, 0], g, hp, 0.3, tiles)
    np.testing.assert_allclose(rows, dq[0, 0][ids], rtol=0, atol=1e-13)


def test_hier_sampled_dkdv_equals_full_backward():
    """The key-tile restriction of the hierarchical backward returns exactly
    the rows of the full definition, for tiles at the grid's corners and in
    its interior (so both the fine and the pooled contributions are met)."""
    for g, hp in HIER_CASES:
        q, k, v, do = (_rand((1, 1, g.n, 8), s) for s in (62, 63, 64, 65))
        _, dk, dv = O.hier_backward(q, k, v, do, g, hp, 0.3)
        n_tiles = math.prod(g.tiles_per_dim)
        tiles = sorted({0, 3, n_tiles // 2, n_tiles - 1})
        ids, rk, rv = O.hier_backward_dkdv_tiles(q[0, 0], k[0, 0], v[0, 0], do[0, 0], g, hp, 0.3, tiles)
        np.testing.assert_allclose(rk, dk[0, 0][ids], rtol=0, atol=1e-13)
        np.testing.assert_allclose(rv, dv[0, 0][ids], rtol=0, atol=1e-13)
