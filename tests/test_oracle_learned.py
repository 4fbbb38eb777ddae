"""Pins of the oracle's learned compressed global branch (CPU): the depthwise
strided compression against explicit per-tap loops, against torch's strided
grouped conv3d and, with uniform taps, against average pooling; the 3x3x3 restoring convolution against torch's
grouped conv3d (cross-correlation, zero padding), the identity tap and a
one-voxel shift; and the whole learned dual forward, with uniform
compression and the identity restoration, against the average-pooling form."""
import math

import numpy as np
import pytest
import torch

from oracle import vattn_oracle as O


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


GEOMS = [
    O.Geom(2, 8, 12, (1, 4, 4), (1, 1, 3), (1, 2, 2)),
    O.Geom(4, 8, 8, (2, 4, 4), (2, 2, 2), (2, 2, 4)),
    O.Geom(3, 6, 9, (3, 2, 3), (1, 3, 3), (3, 3, 3)),
]


@pytest.mark.parametrize("g", GEOMS)
def test_conv_compress_matches_per_tap_loops(g):
    B, nh, d = 2, 2, 3
    P = g.pool[0] * g.pool[1] * g.pool[2]
    x = _rand((B, nh, g.n, d), 1)
    w = _rand((nh, P, d), 2)
    got = O.conv_compress(x, g, w)
    PT, PH, PW = g.pooled_dims
    pt, ph, pw = g.pool
    xg = x.reshape(B, nh, g.T, g.H, g.W, d)
    for b in range(B):
        for h in range(nh):
            for t in range(PT):
                for y in range(PH):
                    for xx in range(PW):
                        acc = np.zeros(d)
                        tap = 0
                        for dt in range(pt):
                            for dy in range(ph):
                                for dx in range(pw):
                                    acc += w[h, tap] * xg[b, h, t * pt + dt, y * ph + dy, xx * pw + dx]
                                    tap += 1
                        np.testing.assert_allclose(got[b, h, (t * PH + y) * PW + xx], acc, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("g", GEOMS)
def test_conv_compress_uniform_taps_is_average_pooling(g):
    P = g.pool[0] * g.pool[1] * g.pool[2]
    x = _rand((1, 3, g.n, 4), 3)
    w = np.full((3, P, 4), 1.0 / P)
    np.testing.assert_allclose(O.conv_compress(x, g, w), O.pool(x, g), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("g", GEOMS)
def test_conv_compress_matches_torch_strided_grouped_conv3d(g):
    """Depthwise convolution with stride equal to its kernel ("UltraGen ..."
    §4.2): torch's grouped conv3d with kernel = stride = the pool size."""
    B, nh, d = 2, 2, 3
    P = g.pool[0] * g.pool[1] * g.pool[2]
    x = _rand((B, nh, g.n, d), 6)
    w = _rand((nh, P, d), 7)
    got = O.conv_compress(x, g, w)
    for h in range(nh):
        xt = torch.from_numpy(x[:, h].reshape(B, g.T, g.H, g.W, d)).permute(0, 4, 1, 2, 3).contiguous()
        wt = torch.from_numpy(np.ascontiguousarray(w[h].T.reshape(d, 1, *g.pool)))   # taps (dt, dy, dx)
        ref = torch.nn.functional.conv3d(xt, wt, stride=tuple(g.pool), groups=d)
        ref = ref.permute(0, 2, 3, 4, 1).reshape(B, g.n_pooled, d).numpy()
        np.testing.assert_allclose(got[:, h], ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("g", GEOMS)
def test_conv3d_depthwise_matches_torch_grouped_conv3d(g):
    B, nh, d = 2, 3, 4
    x = _rand((B, nh, g.n, d), 4)
    w3 = _rand((nh, 27, d), 5)
    got = O.conv3d_depthwise(x, g, w3)
    for h in range(nh):
        xt = torch.from_numpy(x[:, h].reshape(B, g.T, g.H, g.W, d)).permute(0, 4, 1, 2, 3).contiguous()
        wt = torch.from_numpy(np.ascontiguousarray(w3[h].T.reshape(d, 1, 3, 3, 3)))
        ref = torch.nn.functional.conv3d(xt, wt, padding=1, groups=d)   # cross-correlation, zero padding
        ref = ref.permute(0, 2, 3, 4, 1).reshape(B, g.n, d).numpy()
        np.testing.assert_allclose(got[:, h], ref, rtol=1e-12, atol=1e-12)


def test_conv3d_depthwise_identity_and_shift_taps():
    g = GEOMS[1]
    x = _rand((1, 2, g.n, 3), 6)
    w3 = np.zeros((2, 27, 3))
    w3[:, 13] = 1.0                      # (0, 0, 0): identity
    np.testing.assert_array_equal(O.conv3d_depthwise(x, g, w3), x)
    w3 = np.zeros((2, 27, 3))
    w3[:, 14] = 1.0                      # (0, 0, +1): y[t, y, x] = x[t, y, x + 1], zero past the edge
    got = O.conv3d_depthwise(x, g, w3).reshape(1, 2, g.T, g.H, g.W, 3)
    xg = x.reshape(1, 2, g.T, g.H, g.W, 3)
    np.testing.assert_array_equal(got[..., :-1, :], xg[..., 1:, :])
    np.testing.assert_array_equal(got[..., -1, :], 0.0)
    w3 = np.zeros((2, 27, 3))
    w3[:, 4] = 1.0                       # (-1, 0, 0): y[t] = x[t - 1], zero at t = 0
    got = O.conv3d_depthwise(x, g, w3).reshape(1, 2, g.T, g.H, g.W, 3)
    np.testing.assert_array_equal(got[:, :, 1:], xg[:, :, :-1])
    np.testing.assert_array_equal(got[:, :, 0], 0.0)


def test_learned_dual_forward_reduces_to_average_pooling_form():
    g = O.Geom(4, 8, 8, (2, 4, 4), (1, 2, 2), (2, 2, 2))
    nh, d = 2, 8
    q, k, v = (_rand((1, nh, g.n, d), s) for s in (7, 8, 9))
    gvec = np.array([0.3, 0.8])
    P = 8
    wu = np.full((nh, P, d), 1.0 / P)
    w3 = np.zeros((nh, 27, d))
    w3[:, 13] = 1.0
    scale = 1 / math.sqrt(d)
    ref = O.dual_sym_forward(q, k, v, gvec, g, scale)
    got = O.dual_sym_learned_forward(q, k, v, gvec, wu, wu, wu, w3, g, scale)
    np.testing.assert_allclose(got["O"], ref["O"], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(got["O_p"], ref["O_p"], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(got["LSE_p"], ref["LSE_p"], rtol=1e-11, atol=1e-12)


def test_learned_dual_forward_global_part_is_linear_in_the_restoring_taps():
    """O_g = conv3d(upsample(O_p)) is linear in w3 for fixed inputs: doubling
    the taps doubles O_g, and the sum of two tap sets gives the sum."""
    g = O.Geom(2, 8, 8, (1, 4, 4), (1, 2, 2), (1, 2, 2))
    nh, d = 1, 4
    q, k, v = (_rand((1, nh, g.n, d), s) for s in (10, 11, 12))
    wq, wk, wv = (_rand((nh, 4, d), s) * 0.25 + 0.25 for s in (13, 14, 15))
    wa, wb = _rand((nh, 27, d), 16), _rand((nh, 27, d), 17)
    f = lambda w3: O.dual_sym_learned_forward(q, k, v, [0.5], wq, wk, wv, w3, g, 0.5)["O_g"]
    np.testing.assert_allclose(f(wa + wb), f(wa) + f(wb), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(f(2 * wa), 2 * f(wa), rtol=1e-10, atol=1e-12)
