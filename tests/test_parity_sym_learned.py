"""GPU parity of the dual forward with the learned compressed global branch
(vattn_dual_sym_learned_fwd: depthwise strided compression of Q, K, V, pooled
attention, upsampling, 3x3x3 depthwise restoration, blend) against the fp64
oracle, on seeded random weights."""
import math

import numpy as np
import pytest

from helpers import O_MAX_ABS, O_MEAN_ABS, assert_close, geom_for, gpu_tensor, host_f64, sample_tiles, to_f64
from oracle import vattn_oracle as O
from synth import inputs as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def V():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import video_dit_local_b200 as V
    return V


def _perm(V, geom, x):
    import torch
    out = torch.empty_like(x)
    V.vattn_tile_permute(geom, x, out)
    return out


def _unperm(V, geom, x):
    import torch
    out = torch.empty_like(x)
    V.vattn_tile_unpermute(geom, x, out)
    return out


def _run(V, w, check, weights=None):
    """Learned forward on the GPU; returns raster O and the weights used."""
    import torch
    geom = geom_for(V, w)
    q, k, v = (_perm(V, geom, gpu_tensor(w, i, check)) for i in (S.Q_ID, S.K_ID, S.V_ID))
    gvec = torch.from_numpy(S.blend_g(w)).cuda()
    wts = S.learned_weights(w) if weights is None else weights
    dw = {n: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda() for n, a in wts.items()}
    o = torch.full_like(q, float("nan"))
    ws = torch.empty(V.vattn_workspace_size(V.VATTN_OP_DUAL_SYM_LEARNED_FWD, geom), dtype=torch.uint8,
                     device="cuda")
    V.vattn_dual_sym_learned_fwd(geom, q, k, v, gvec, dw["wq"], dw["wk"], dw["wv"], dw["w3"],
                                 1 / math.sqrt(w.head_dim), o, ws)
    out = _unperm(V, geom, o)
    torch.cuda.synchronize()
    assert V.vattn_get_status() == 0, V.vattn_last_error()
    return out, wts


@pytest.mark.parametrize("grid,tile,window,pool,d,batch,heads", [
    ((4, 8, 8), (2, 4, 4), (1, 2, 2), (2, 2, 4), 64, 1, 2),       # temporal compression too
    ((3, 16, 24), (3, 8, 8), (1, 1, 3), (1, 4, 4), 128, 2, 1),    # frame-wise 4x4 compression, batch 2
    ((6, 24, 40), (3, 8, 8), (3, 3, 3), (3, 8, 8), 128, 1, 2),    # pooled grid 2x3x5 (restoration at every edge)
    # 6 rows: the restoration's last 4-row band is half empty; 12 columns: one partial 32-column band
    ((4, 6, 12), (2, 2, 4), (1, 2, 3), (1, 3, 4), 64, 1, 2),
    # pool widths 2 and 3: the compression's 2-wide load rows and its one-at-a-time loop
    ((2, 8, 12), (1, 4, 4), (1, 2, 3), (1, 2, 2), 64, 1, 1),
    ((2, 8, 12), (1, 4, 4), (1, 2, 3), (1, 2, 3), 64, 1, 1),
])
def test_dual_sym_learned_small_full(V, grid, tile, window, pool, d, batch, heads):
    w = S.small_workload("symlearn", 37, batch, heads, d, grid, tile, window, pool)
    g = O.geom_of(w)
    check = [(b, h) for b in range(batch) for h in range(heads)]
    out, wts = _run(V, w, check)
    hq, hk, hv = (np.stack([np.stack([host_f64(w, i, b, h) for h in range(heads)]) for b in range(batch)])
                  for i in (S.Q_ID, S.K_ID, S.V_ID))
    gv = S.blend_g(w).astype(np.float64)
    f64 = {n: a.astype(np.float64) for n, a in wts.items()}
    ref = O.dual_sym_learned_forward(hq, hk, hv, gv, f64["wq"], f64["wk"], f64["wv"], f64["w3"], g,
                                     1 / math.sqrt(d))
    assert_close(to_f64(out), ref["O"], O_MAX_ABS, O_MEAN_ABS, "O")


def test_dual_sym_learned_uniform_identity_matches_average_pooling_path(V):
    """Uniform compression taps and the identity restoring tap make the learned
    branch the average-pooling one: the two entry points agree within the
    rounding of their different kernels."""
    import torch
    w = S.small_workload("symlearn", 41, 1, 2, 128, (3, 16, 24), (3, 8, 8), (1, 3, 3), (1, 4, 4))
    P = 16
    wts = {n: np.full((w.heads, P, w.head_dim), 1.0 / P, dtype=np.float32) for n in ("wq", "wk", "wv")}
    w3 = np.zeros((w.heads, 27, w.head_dim), dtype=np.float32)
    w3[:, 13] = 1.0
    wts["w3"] = w3
    check = [(0, 0), (0, 1)]
    out, _ = _run(V, w, check, wts)
    geom = geom_for(V, w)
    q, k, v = (_perm(V, geom, gpu_tensor(w, i, check)) for i in (S.Q_ID, S.K_ID, S.V_ID))
    gvec = torch.from_numpy(S.blend_g(w)).cuda()
    o = torch.empty_like(q)
    ws = torch.empty(V.vattn_workspace_size(V.VATTN_OP_DUAL_SYM_FWD, geom), dtype=torch.uint8, device="cuda")
    V.vattn_dual_sym_fwd(geom, q, k, v, gvec, 1 / math.sqrt(128), o, workspace=ws)
    ref = to_f64(_unperm(V, geom, o))
    assert_close(to_f64(out), ref, O_MAX_ABS, O_MEAN_ABS, "learned (uniform, identity) vs average pooling")


def test_dual_sym_learned_1080p_shape_sampled(V):
    """The 1080p dual workload's shape (B1 h24 d128, pool 1x4x4) through the
    learned branch; head 23 compared on sampled query tiles (the global part
    on the whole grid: the restoring convolution needs every neighbour)."""
    w = S.WORKLOADS["1080p"]
    h = w.heads - 1
    out, wts = _run(V, w, [(0, h)])
    g = O.geom_of(w)
    scale = 1 / math.sqrt(w.head_dim)
    q, k, v = (host_f64(w, i, 0, h) for i in (S.Q_ID, S.K_ID, S.V_ID))
    f64 = {n: a[h:h + 1].astype(np.float64) for n, a in wts.items()}
    tiles = sample_tiles(g.tiles_per_dim, 4)
    ids, o_l, _ = O.sta_attention_tiles(q, k, v, g, scale, tiles)
    qp, kp, vp = (O.conv_compress(x[None, None], g, f64[n])[0, 0] for x, n in ((q, "wq"), (k, "wk"), (v, "wv")))
    o_p, _ = O.full_attention(qp[None, None], kp[None, None], vp[None, None], scale)
    o_g = O.conv3d_depthwise(O.upsample(o_p, g), g, f64["w3"])[0, 0]
    gval = float(S.blend_g(w)[h])
    ref = gval * o_l + (1.0 - gval) * o_g[ids]
    assert_close(to_f64(out[0, h])[ids], ref, O_MAX_ABS, O_MEAN_ABS, "O h23")
