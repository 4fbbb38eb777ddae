"""GPU parity of cross-window local attention (vattn_xwin_fwd / _bwd, both the
partition and the shifted partition) against the fp64 oracle."""
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


def _perm(V, geom, x):
    import torch
    out = torch.empty_like(x)
    V.vattn_tile_permute(geom, x, out)
    return out


def _unperm(V, geom, x, row_bytes=None):
    import torch
    out = torch.empty_like(x)
    V.vattn_tile_unpermute(geom, x, out, row_bytes)
    return out


def _xwin_tiles(q, k, v, g, scale, shifted, tiles):
    """Oracle restricted to the listed query tiles."""
    sel = set(int(t) for t in tiles)
    ids, outs, lses = [], [], []
    for tid, (qi, kj) in enumerate(O.xwin_query_tiles(g, shifted)):
        if tid in sel:
            o, lse, _ = O._softmax_attend(q[qi], k[kj], v[kj], scale)
            ids.append(qi)
            outs.append(o)
            lses.append(lse)
    return np.concatenate(ids), np.concatenate(outs), np.concatenate(lses)


@pytest.mark.parametrize("shifted", [0, 1])
@pytest.mark.parametrize("grid,tile,window,d,batch,heads", [
    ((4, 16, 24), (2, 4, 4), (1, 2, 3), 64, 1, 2),
    ((6, 24, 40), (3, 8, 8), (2, 2, 2), 128, 2, 1),     # tile 192, truncated edge blocks
    # tile 192, 9 tiles along w: partitions of 3 pair tiles 0-1, 3-4, 6-7 (a unit table), shifted blocks of 4
    # (cuts at 2 and 6) pair every even tile with the next (uniform pairs)
    ((3, 16, 72), (3, 8, 8), (1, 2, 3), 128, 1, 2),
])
def test_xwin_fwd_bwd_small_full(V, shifted, grid, tile, window, d, batch, heads):
    import torch
    w = S.small_workload("xwin", 23, batch, heads, d, grid, tile, window, (1, 1, 1))
    g = O.geom_of(w)
    geom = geom_for(V, w)
    check = [(b, h) for b in range(batch) for h in range(heads)]
    q, k, v, do = (_perm(V, geom, gpu_tensor(w, i, check)) for i in (S.Q_ID, S.K_ID, S.V_ID, S.DO_ID))
    scale = 1 / math.sqrt(d)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    V.vattn_xwin_fwd(geom, shifted, q, k, v, scale, o, lse)
    dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
    ws = torch.empty(V.vattn_workspace_size(V.VATTN_OP_STA_BWD, geom), dtype=torch.uint8, device="cuda")
    V.vattn_xwin_bwd(geom, shifted, q, k, v, o, lse, do, scale, dq, dk, dv, ws)
    torch.cuda.synchronize()
    assert V.vattn_get_status() == 0, V.vattn_last_error()
    hq, hk, hv, hdo = (np.stack([np.stack([host_f64(w, i, b, h) for h in range(heads)]) for b in range(batch)])
                       for i in (S.Q_ID, S.K_ID, S.V_ID, S.DO_ID))
    ro, rl = O.xwin_attention(hq, hk, hv, g, scale, bool(shifted))
    assert_close(to_f64(_unperm(V, geom, o)), ro, O_MAX_ABS, O_MEAN_ABS, "O")
    assert_close(_unperm(V, geom, lse, 4).cpu().numpy().astype(np.float64), rl, LSE_MAX_ABS, what="LSE")
    rq, rk, rv = O.xwin_backward(hq, hk, hv, hdo, g, scale, bool(shifted))
    for name, got, ref in (("dQ", dq, rq), ("dK", dk, rk), ("dV", dv, rv)):
        assert_close(to_f64(_unperm(V, geom, got)), ref, O_MAX_ABS, O_MEAN_ABS, name)


@pytest.mark.parametrize("shifted", [0, 1])
def test_xwin_fwd_1080p_grid_sampled(V, shifted):
    import torch
    w = S.WORKLOADS["1080p"]
    g = O.geom_of(w)
    geom = geom_for(V, w)
    check = [(0, 0), (0, w.heads - 1)]
    q, k, v = (_perm(V, geom, gpu_tensor(w, i, check)) for i in (S.Q_ID, S.K_ID, S.V_ID))
    scale = 1 / math.sqrt(w.head_dim)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    V.vattn_xwin_fwd(geom, shifted, q, k, v, scale, o, lse)
    o_r, l_r = _unperm(V, geom, o), _unperm(V, geom, lse, 4)
    torch.cuda.synchronize()
    assert V.vattn_get_status() == 0
    tiles = sample_tiles(g.tiles_per_dim, 6)
    for b, h in check:
        hq, hk, hv = (host_f64(w, i, b, h) for i in (S.Q_ID, S.K_ID, S.V_ID))
        ids, ro, rl = _xwin_tiles(hq, hk, hv, g, scale, bool(shifted), tiles)
        assert_close(to_f64(o_r[b, h])[ids], ro, O_MAX_ABS, O_MEAN_ABS, "O")
        assert_close(l_r[b, h].cpu().numpy().astype(np.float64)[ids], rl, LSE_MAX_ABS, what="LSE")
