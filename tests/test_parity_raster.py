"""GPU parity of the raster-order sliding-tile forward (vattn_sta_fwd_raster):
the raster <-> tile-major reorder is done by the kernel's 5-D tensor-map
boxes and raster-addressed epilogue stores, so its O and LSE must equal
vattn_tile_permute + vattn_sta_fwd + vattn_tile_unpermute bit for bit; the
seeded heads are also compared with the fp64 oracle on every query tile of
the small grids."""
import math

import numpy as np
import pytest

from helpers import (LSE_MAX_ABS, O_MAX_ABS, O_MEAN_ABS, assert_close, geom_for, gpu_tensor, host_f64,
                     to_f64)
from oracle import vattn_oracle as O
from synth import inputs as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def V():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import video_dit_local_b200 as V
    return V


def _both(V, w, check):
    import torch
    geom = geom_for(V, w)
    qr, kr, vr = (gpu_tensor(w, i, check) for i in (S.Q_ID, S.K_ID, S.V_ID))
    scale = 1 / math.sqrt(w.head_dim)
    # the permute path
    q, k, v = (torch.empty_like(qr) for _ in range(3))
    for src, dst in ((qr, q), (kr, k), (vr, v)):
        V.vattn_tile_permute(geom, src, dst)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    V.vattn_sta_fwd(geom, q, k, v, scale, o, lse)
    o_ref, lse_ref = torch.empty_like(o), torch.empty_like(lse)
    V.vattn_tile_unpermute(geom, o, o_ref)
    V.vattn_tile_unpermute(geom, lse, lse_ref, 4)
    # the fused raster path
    o_r = torch.full_like(qr, float("nan"))
    lse_r = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device="cuda")
    V.vattn_sta_fwd_raster(geom, qr, kr, vr, scale, o_r, lse_r)
    torch.cuda.synchronize()
    assert V.vattn_get_status() == 0, V.vattn_last_error()
    return o_r, lse_r, o_ref, lse_ref


def _same(a, b):
    import torch
    if a.dtype == torch.bfloat16:
        return torch.equal(a.view(torch.int16), b.view(torch.int16))
    return torch.equal(a.view(torch.int32), b.view(torch.int32))


@pytest.mark.parametrize("grid,tile,window,d,batch,heads", [
    ((4, 8, 8), (2, 4, 4), (1, 2, 2), 64, 1, 2),        # the tiny workload's shape
    ((6, 16, 24), (3, 8, 8), (1, 1, 3), 128, 1, 2),     # tile 192: a ragged second query block
    ((6, 16, 32), (6, 8, 8), (1, 3, 3), 64, 2, 1),      # tile 384, d = 64, batch 2
    ((4, 8, 16), (2, 4, 4), (1, 1, 1), 128, 1, 3),      # window of one tile
    ((2, 8, 8), (2, 4, 4), (3, 5, 7), 128, 1, 1),       # window wider than the grid in every dim
])
def test_raster_fwd_equals_permute_path_and_oracle(V, grid, tile, window, d, batch, heads):
    w = S.small_workload("raster", 81, batch, heads, d, grid, tile, window, (1, 1, 1))
    check = [(b, h) for b in range(batch) for h in range(heads)]
    o_r, lse_r, o_ref, lse_ref = _both(V, w, check)
    assert _same(o_r, o_ref) and _same(lse_r, lse_ref)
    g = O.geom_of(w)
    scale = 1 / math.sqrt(d)
    for b, h in check:
        q, k, v = (host_f64(w, i, b, h) for i in (S.Q_ID, S.K_ID, S.V_ID))
        ids, o_or, lse_or = O.sta_attention_tiles(q, k, v, g, scale, range(math.prod(g.tiles_per_dim)))
        assert_close(to_f64(o_r[b, h])[ids], o_or, O_MAX_ABS, O_MEAN_ABS, f"O b{b} h{h}")
        assert_close(lse_r[b, h].cpu().numpy().astype(np.float64)[ids], lse_or, LSE_MAX_ABS, what=f"LSE b{b} h{h}")


def test_raster_fwd_720p_equals_permute_path(V):
    """The benchmarked launch: all 24 heads, every output bit."""
    w = S.WORKLOADS["720p"]
    o_r, lse_r, o_ref, lse_ref = _both(V, w, [(0, 0), (0, w.heads - 1)])
    assert _same(o_r, o_ref) and _same(lse_r, lse_ref)
