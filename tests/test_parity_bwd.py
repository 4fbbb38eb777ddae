"""GPU parity of the backward path (vattn_sta_bwd, vattn_dual_bwd) against
the fp64 oracle, through the C ABI.  The GPU forward's saved outputs feed the
GPU backward; the oracle recomputes everything from the inputs.
Bars: dQ, dK, dV within max-abs 2e-2 and mean-abs 2e-3; dg within 2e-2
relative to its magnitude."""
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


def _run_dual(V, w, check):
    """Forward (saving what the backward needs) and backward on the GPU; returns
    raster dQ, dK, dV and dg."""
    import torch
    g = O.geom_of(w)
    geom = geom_for(V, w)
    q, k, v, do = (_perm(V, geom, gpu_tensor(w, i, check)) for i in (S.Q_ID, S.K_ID, S.V_ID, S.DO_ID))
    gvec = torch.from_numpy(S.blend_g(w)).cuda()
    scale = 1 / math.sqrt(w.head_dim)
    o, o_l, o_g = (torch.empty_like(q) for _ in range(3))
    lse_l = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    lse_g = torch.empty_like(lse_l)
    kp = torch.empty((w.batch, w.heads, g.n_pooled, w.head_dim), dtype=torch.bfloat16, device="cuda")
    vp = torch.empty_like(kp)
    V.vattn_dual_fwd(geom, q, k, v, gvec, scale, o, o_l, lse_l, o_g, lse_g, kp, vp)
    dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
    dg = torch.empty(w.heads, dtype=torch.float32, device="cuda")
    ws = torch.empty(V.vattn_workspace_size(V.VATTN_OP_DUAL_BWD, geom), dtype=torch.uint8, device="cuda")
    V.vattn_dual_bwd(geom, q, k, v, gvec, o_l, lse_l, o_g, lse_g, kp, vp, do, scale, dq, dk, dv, dg, ws)
    torch.cuda.synchronize()
    assert V.vattn_get_status() == 0, V.vattn_last_error()
    return [_unperm(V, geom, t) for t in (dq, dk, dv)] + [dg]


@pytest.mark.parametrize("grid,tile,window,pool,d,batch,heads", [
    ((4, 8, 8), (2, 4, 4), (1, 2, 2), (1, 2, 2), 64, 1, 2),
    ((3, 20, 24), (3, 4, 4), (1, 3, 3), (1, 2, 2), 128, 2, 3),    # ragged N, N_p; tile 48
    ((6, 16, 24), (3, 8, 8), (1, 1, 3), (1, 4, 4), 128, 1, 2),     # tile 192: half-empty second block
    ((6, 16, 32), (6, 8, 8), (1, 3, 3), (3, 4, 4), 64, 1, 1),      # tile 384, temporal pooling
    ((3, 16, 40), (3, 8, 8), (1, 3, 3), (1, 2, 2), 128, 1, 2),     # tile 192, 5 along w: paired dQ query blocks
    ((3, 16, 48), (3, 8, 8), (1, 2, 3), (1, 2, 2), 64, 2, 1),      # paired, d = 64, batch 2, even window along h
])
def test_dual_bwd_small_full(V, grid, tile, window, pool, d, batch, heads):
    w = S.small_workload("dbwd", 17, batch, heads, d, grid, tile, window, pool)
    check = [(b, h) for b in range(batch) for h in range(heads)]
    dq, dk, dv, dg = _run_dual(V, w, check)
    g = O.geom_of(w)
    q, k, v, do = (np.stack([np.stack([host_f64(w, i, b, h) for h in range(heads)]) for b in range(batch)])
                   for i in (S.Q_ID, S.K_ID, S.V_ID, S.DO_ID))
    ref = O.dual_backward(q, k, v, S.blend_g(w).astype(np.float64), do, g, 1 / math.sqrt(d))
    for name, got in (("dQ", dq), ("dK", dk), ("dV", dv)):
        assert_close(to_f64(got), ref[name], O_MAX_ABS, O_MEAN_ABS, name)
    dg_ref = ref["dg"]
    assert np.abs(dg.cpu().numpy() - dg_ref).max() <= 2e-2 * max(1.0, np.abs(dg_ref).max())


@pytest.mark.parametrize("grid,tile,window,d", [
    ((4, 8, 8), (2, 4, 4), (1, 2, 2), 64),
    ((6, 16, 24), (3, 8, 8), (3, 1, 3), 128),
    ((2, 16, 48), (1, 8, 8), (1, 1, 3), 64),      # tile 64: every dQ query block straddles two tiles
    ((3, 8, 64), (3, 8, 8), (1, 1, 5), 128),      # window of 5 along w: interior pairs a tile apart
])
def test_sta_bwd_small_full(V, grid, tile, window, d):
    import torch
    w = S.small_workload("sbwd", 19, 1, 2, d, grid, tile, window, (1, 1, 1))
    g = O.geom_of(w)
    geom = geom_for(V, w)
    check = [(0, 0), (0, 1)]
    q, k, v, do = (_perm(V, geom, gpu_tensor(w, i, check)) for i in (S.Q_ID, S.K_ID, S.V_ID, S.DO_ID))
    scale = 1 / math.sqrt(d)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    V.vattn_sta_fwd(geom, q, k, v, scale, o, lse)
    dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
    ws = torch.empty(V.vattn_workspace_size(V.VATTN_OP_STA_BWD, geom), dtype=torch.uint8, device="cuda")
    V.vattn_sta_bwd(geom, q, k, v, o, lse, do, scale, dq, dk, dv, ws)
    torch.cuda.synchronize()
    assert V.vattn_get_status() == 0, V.vattn_last_error()
    hq, hk, hv, hdo = (np.stack([host_f64(w, i, 0, h) for h in range(2)])[None] for i in
                       (S.Q_ID, S.K_ID, S.V_ID, S.DO_ID))
    rq, rk, rv = O.sta_backward(hq, hk, hv, hdo, g, scale)
    for name, got, ref in (("dQ", dq, rq), ("dK", dk, rk), ("dV", dv, rv)):
        assert_close(to_f64(_unperm(V, geom, got)), ref, O_MAX_ABS, O_MEAN_ABS, name)


def test_dual_bwd_train_sampled(V):
    """The training workload (B2 h24 d128, 1080p grid, pool 1x4x4) at full
    size; the last (batch, head) slice is compared on sampled query tiles (dQ)
    and sampled key tiles (dK, dV, through the pooling)."""
    w = S.WORKLOADS["train"]
    b, h = w.batch - 1, w.heads - 1
    dq, dk, dv, _ = _run_dual(V, w, [(b, h)])
    g = O.geom_of(w)
    q, k, v, do = (host_f64(w, i, b, h) for i in (S.Q_ID, S.K_ID, S.V_ID, S.DO_ID))
    qt = sample_tiles(g.tiles_per_dim, 4, seed=1)
    kt = sample_tiles(g.tiles_per_dim, 2, seed=2)
    ref = O.dual_backward_sampled(q, k, v, float(S.blend_g(w)[h]), do, g, 1 / math.sqrt(w.head_dim), qt, kt)
    assert_close(to_f64(dq[b, h])[ref["q_ids"]], ref["dQ"], O_MAX_ABS, O_MEAN_ABS, "dQ")
    assert_close(to_f64(dk[b, h])[ref["k_ids"]], ref["dK"], O_MAX_ABS, O_MEAN_ABS, "dK")
    assert_close(to_f64(dv[b, h])[ref["k_ids"]], ref["dV"], O_MAX_ABS, O_MEAN_ABS, "dV")
