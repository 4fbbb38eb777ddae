"""GPU parity of hierarchical local attention (vattn_hier_fwd) against the fp64
oracle: fine sliding-tile keys and medium-pooled keys of a coarse-tile window
in one softmax ("UltraGen ..." §4.3).

Bars as for the other forward paths: O within max-abs 2e-2 and mean-abs 2e-3,
LSE within 1e-3 (natural log).  Small grids compare every query tile; the
720p-shaped workload compares the seeded heads on query tiles that cover every
boundary class of the coarse window.
"""
import math

import numpy as np
import pytest

from helpers import (LSE_MAX_ABS, O_MAX_ABS, O_MEAN_ABS, assert_close, geom_for, gpu_tensor, host_f64,
                     sample_tiles, to_f64)
from oracle import vattn_oracle as O
from synth import inputs as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def V():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import video_dit_local_b200 as V
    return V


def _hier_gpu(V, w, check):
    """Runs vattn_hier_fwd on tile-major copies; returns raster O, LSE."""
    import torch
    geom = geom_for(V, w)   # pool = the medium pool factor
    tiled = []
    for tid in (S.Q_ID, S.K_ID, S.V_ID):
        x = gpu_tensor(w, tid, check)
        t = torch.empty_like(x)
        V.vattn_tile_permute(geom, x, t)
        tiled.append(t)
    q, k, v = tiled
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    ws = torch.empty(V.vattn_workspace_size(V.VATTN_OP_HIER_FWD, geom), dtype=torch.uint8, device="cuda")
    V.vattn_hier_fwd(geom, q, k, v, 1 / math.sqrt(w.head_dim), o, lse, ws)
    o_r, lse_r = torch.empty_like(o), torch.empty_like(lse)
    V.vattn_tile_unpermute(geom, o, o_r)
    V.vattn_tile_unpermute(geom, lse, lse_r, 4)
    torch.cuda.synchronize()
    assert V.vattn_get_status() == 0, V.vattn_last_error()
    return o_r, lse_r


def _check(w, o_r, lse_r, check, tiles):
    g = O.geom_of(w)._replace(pool=(1, 1, 1))
    hp = tuple(w.pool)
    scale = 1 / math.sqrt(w.head_dim)
    for b, h in check:
        q, k, v = (host_f64(w, i, b, h) for i in (S.Q_ID, S.K_ID, S.V_ID))
        ids, o_ref, lse_ref = O.hier_attention_tiles(q, k, v, g, hp, scale, tiles)
        assert_close(to_f64(o_r[b, h])[ids], o_ref, O_MAX_ABS, O_MEAN_ABS, f"O b{b} h{h}")
        assert_close(lse_r[b, h].cpu().numpy().astype(np.float64)[ids], lse_ref, LSE_MAX_ABS, what=f"LSE b{b} h{h}")


@pytest.mark.parametrize("grid,tile,window,hpool,d,batch,heads", [
    ((6, 16, 32), (3, 8, 8), (1, 3, 3), (1, 2, 2), 128, 1, 2),   # coarse window clamps along W
    ((4, 16, 16), (1, 4, 4), (3, 1, 1), (2, 2, 2), 64, 2, 1),    # pooled in time too, d = 64, batch 2
    ((4, 8, 16), (2, 4, 4), (1, 1, 3), (1, 1, 1), 128, 1, 1),    # h_pool 1: every local key twice
    ((2, 16, 48), (2, 8, 8), (1, 1, 1), (1, 2, 3), 128, 1, 2),   # window of one tile, uneven factors
    ((3, 8, 144), (3, 8, 8), (1, 1, 3), (1, 1, 3), 128, 1, 1),   # 192-row tiles paired; coarse windows a tile apart
])
def test_hier_fwd_small_full(V, grid, tile, window, hpool, d, batch, heads):
    w = S.small_workload("hier", 61, batch, heads, d, grid, tile, window, hpool)
    check = [(b, h) for b in range(batch) for h in range(heads)]
    o_r, lse_r = _hier_gpu(V, w, check)
    g = O.geom_of(w)
    _check(w, o_r, lse_r, check, range(math.prod(g.tiles_per_dim)))


def test_hier_fwd_720p_sampled(V):
    """The 720p-shaped workload (24 heads, tile 6x8x8, window 3x3x3) with
    h_pool 1x2x2: coarse tiles 5x3x5."""
    w = S.small_workload("hier_720p", 62, 1, 24, 128, (30, 48, 80), (6, 8, 8), (3, 3, 3), (1, 2, 2))
    check = [(0, 0), (0, 23)]
    o_r, lse_r = _hier_gpu(V, w, check)
    _check(w, o_r, lse_r, check, sample_tiles(O.geom_of(w).tiles_per_dim, 10))


def test_hier_fwd_rejects_tiles_not_divisible_by_pool(V):
    import torch
    geom = V.make_geom(1, 1, 128, (3, 24, 40), (3, 8, 8), (1, 3, 3), (1, 2, 2))   # 3 x 5 tiles
    t = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(V.VattnError) as e:
        V.vattn_hier_fwd(geom, t, t, t, 0.1, t, None, t, 1 << 30)
    assert e.value.code == V.binding.VATTN_ERR_SHAPE


# ---------------------------------------------------------------- backward

def _hier_fwd_bwd(V, w, check):
    """GPU forward (o, lse saved) then backward; returns raster dQ, dK, dV."""
    import torch
    geom = geom_for(V, w)
    tiled = []
    for tid in (S.Q_ID, S.K_ID, S.V_ID, S.DO_ID):
        x = gpu_tensor(w, tid, check)
        t = torch.empty_like(x)
        V.vattn_tile_permute(geom, x, t)
        tiled.append(t)
    q, k, v, do = tiled
    scale = 1 / math.sqrt(w.head_dim)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    ws = torch.empty(V.vattn_workspace_size(V.VATTN_OP_HIER_FWD, geom), dtype=torch.uint8, device="cuda")
    V.vattn_hier_fwd(geom, q, k, v, scale, o, lse, ws)
    dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
    wsb = torch.empty(V.vattn_workspace_size(V.VATTN_OP_HIER_BWD, geom), dtype=torch.uint8, device="cuda")
    V.vattn_hier_bwd(geom, q, k, v, o, lse, do, scale, dq, dk, dv, wsb)
    torch.cuda.synchronize()
    assert V.vattn_get_status() == 0, V.vattn_last_error()
    out = []
    for t in (dq, dk, dv):
        r = torch.empty_like(t)
        V.vattn_tile_unpermute(geom, t, r)
        out.append(r)
    return out


@pytest.mark.parametrize("grid,tile,window,hpool,d,batch,heads", [
    ((6, 16, 32), (3, 8, 8), (1, 3, 3), (1, 2, 2), 128, 1, 2),
    ((4, 16, 16), (1, 4, 4), (3, 1, 1), (2, 2, 2), 64, 2, 1),
    ((2, 16, 48), (2, 8, 8), (1, 1, 1), (1, 2, 3), 128, 1, 1),
    ((6, 32, 48), (3, 8, 8), (1, 3, 3), (1, 2, 3), 128, 1, 1),   # fine windows clamp in H and W
    ((3, 8, 144), (3, 8, 8), (1, 1, 3), (1, 1, 3), 128, 1, 1),   # paired dQ query blocks over coarse windows
])
def test_hier_bwd_small_full(V, grid, tile, window, hpool, d, batch, heads):
    w = S.small_workload("hier_bwd", 63, batch, heads, d, grid, tile, window, hpool)
    check = [(b, h) for b in range(batch) for h in range(heads)]
    dq, dk, dv = _hier_fwd_bwd(V, w, check)
    g = O.geom_of(w)._replace(pool=(1, 1, 1))
    scale = 1 / math.sqrt(d)
    q, k, v, do = (np.stack([np.stack([host_f64(w, i, b, h) for h in range(heads)]) for b in range(batch)])
                   for i in (S.Q_ID, S.K_ID, S.V_ID, S.DO_ID))
    rq, rk, rv = O.hier_backward(q, k, v, do, g, tuple(hpool), scale)
    for name, got, ref in (("dQ", dq, rq), ("dK", dk, rk), ("dV", dv, rv)):
        for b, h in check:
            assert_close(to_f64(got[b, h]), ref[b, h], O_MAX_ABS, O_MEAN_ABS, f"{name} b{b} h{h}")


def test_hier_bwd_720p_sampled(V):
    """The 720p shape (24 heads, h_pool 1x2x2) through forward and backward:
    dQ of heads 0 and 23 on query tiles covering every boundary class, and
    dK, dV of head 0 on a corner and an interior key tile.  A key's
    gradient has a fine part (query tiles whose sliding window holds its tile)
    and a coarse part through the medium pooling (query tiles whose coarse
    window holds its pooled key), which the coarse-key pass computes."""
    w = S.small_workload("hier_720p_bwd", 64, 1, 24, 128, (30, 48, 80), (6, 8, 8), (3, 3, 3), (1, 2, 2))
    check = [(0, 0), (0, 23)]
    dq, dk, dv = _hier_fwd_bwd(V, w, check)
    g = O.geom_of(w)._replace(pool=(1, 1, 1))
    scale = 1 / math.sqrt(w.head_dim)
    tiles = sample_tiles(g.tiles_per_dim, 8)
    nt, nh, nw = g.tiles_per_dim
    k_tiles = [0, ((nt // 2) * nh + nh // 2) * nw + nw // 2]
    for b, h in check:
        q, k, v, do = (host_f64(w, i, b, h) for i in (S.Q_ID, S.K_ID, S.V_ID, S.DO_ID))
        ids, ref = O.hier_backward_dq_tiles(q, k, v, do, g, (1, 2, 2), scale, tiles)
        assert_close(to_f64(dq[b, h])[ids], ref, O_MAX_ABS, O_MEAN_ABS, f"dQ b{b} h{h}")
        if h == 0:  # each key tile takes the oracle about a hundred query tiles of the joint softmax
            kid, rk, rv = O.hier_backward_dkdv_tiles(q, k, v, do, g, (1, 2, 2), scale, k_tiles)
            assert_close(to_f64(dk[b, h])[kid], rk, O_MAX_ABS, O_MEAN_ABS, f"dK b{b} h{h}")
            assert_close(to_f64(dv[b, h])[kid], rv, O_MAX_ABS, O_MEAN_ABS, f"dV b{b} h{h}")
