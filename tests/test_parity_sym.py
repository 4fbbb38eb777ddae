"""GPU parity of the dual forward/backward with the symmetric compressed
global branch (vattn_dual_sym_fwd / _bwd) against the fp64 oracle."""
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


def _run(V, w, check, backward=True):
    import torch
    g = O.geom_of(w)
    geom = geom_for(V, w)
    q, k, v, do = (_perm(V, geom, gpu_tensor(w, i, check)) for i in (S.Q_ID, S.K_ID, S.V_ID, S.DO_ID))
    gvec = torch.from_numpy(S.blend_g(w)).cuda()
    scale = 1 / math.sqrt(w.head_dim)
    B, h, d, npool = w.batch, w.heads, w.head_dim, g.n_pooled
    o, o_l = torch.empty_like(q), torch.empty_like(q)
    lse_l = torch.empty((B, h, g.n), dtype=torch.float32, device="cuda")
    qp, kp, vp, o_p = (torch.empty((B, h, npool, d), dtype=torch.bfloat16, device="cuda") for _ in range(4))
    lse_p = torch.empty((B, h, npool), dtype=torch.float32, device="cuda")
    V.vattn_dual_sym_fwd(geom, q, k, v, gvec, scale, o, o_l, lse_l, qp, kp, vp, o_p, lse_p)
    out = dict(O=_unperm(V, geom, o), O_p=o_p, LSE_p=lse_p)
    ws = torch.empty(V.vattn_workspace_size(V.VATTN_OP_DUAL_SYM_FWD, geom), dtype=torch.uint8, device="cuda")
    o2 = torch.empty_like(q)
    V.vattn_dual_sym_fwd(geom, q, k, v, gvec, scale, o2, workspace=ws)
    out["O_inf"] = _unperm(V, geom, o2)
    if backward:
        dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
        wsb = torch.empty(V.vattn_workspace_size(V.VATTN_OP_DUAL_SYM_BWD, geom), dtype=torch.uint8, device="cuda")
        V.vattn_dual_sym_bwd(geom, q, k, v, gvec, o_l, lse_l, qp, kp, vp, o_p, lse_p, do, scale, dq, dk, dv, wsb)
        out.update(dQ=_unperm(V, geom, dq), dK=_unperm(V, geom, dk), dV=_unperm(V, geom, dv))
    torch.cuda.synchronize()
    assert V.vattn_get_status() == 0, V.vattn_last_error()
    return out


@pytest.mark.parametrize("grid,tile,window,pool,d,batch,heads", [
    ((4, 8, 8), (2, 4, 4), (1, 2, 2), (2, 2, 4), 64, 1, 2),
    ((3, 16, 24), (3, 8, 8), (1, 1, 3), (1, 4, 4), 128, 2, 1),
    ((6, 24, 40), (3, 8, 8), (3, 3, 3), (3, 8, 8), 128, 1, 2),
])
def test_dual_sym_small_full(V, grid, tile, window, pool, d, batch, heads):
    w = S.small_workload("sym", 29, batch, heads, d, grid, tile, window, pool)
    g = O.geom_of(w)
    check = [(b, h) for b in range(batch) for h in range(heads)]
    out = _run(V, w, check)
    hq, hk, hv, hdo = (np.stack([np.stack([host_f64(w, i, b, h) for h in range(heads)]) for b in range(batch)])
                       for i in (S.Q_ID, S.K_ID, S.V_ID, S.DO_ID))
    gv = S.blend_g(w).astype(np.float64)
    scale = 1 / math.sqrt(d)
    ref = O.dual_sym_forward(hq, hk, hv, gv, g, scale)
    assert_close(to_f64(out["O"]), ref["O"], O_MAX_ABS, O_MEAN_ABS, "O")
    assert_close(to_f64(out["O_inf"]), ref["O"], O_MAX_ABS, O_MEAN_ABS, "O (inference)")
    assert_close(to_f64(out["O_p"]), ref["O_p"], O_MAX_ABS, O_MEAN_ABS, "O_p")
    assert_close(out["LSE_p"].cpu().numpy().astype(np.float64), ref["LSE_p"], LSE_MAX_ABS, what="LSE_p")
    rb = O.dual_sym_backward(hq, hk, hv, gv, hdo, g, scale)
    for name in ("dQ", "dK", "dV"):
        assert_close(to_f64(out[name]), rb[name], O_MAX_ABS, O_MEAN_ABS, name)


def test_dual_sym_train_shape_sampled(V):
    """The training workload's shape (B2 h24 d128, 1080p grid, pool 1x4x4)
    through the symmetric branch; the last (batch, head) slice is compared on
    sampled tiles."""
    w = S.WORKLOADS["train"]
    b, h = w.batch - 1, w.heads - 1
    out = _run(V, w, [(b, h)])
    g = O.geom_of(w)
    scale = 1 / math.sqrt(w.head_dim)
    q, k, v, do = (host_f64(w, i, b, h) for i in (S.Q_ID, S.K_ID, S.V_ID, S.DO_ID))
    gval = float(S.blend_g(w)[h])
    tiles = sample_tiles(g.tiles_per_dim, 4, seed=3)
    ids, ol, _ = O.sta_attention_tiles(q, k, v, g, scale, tiles)
    og_full, _, _ = O.global_sym_forward(q[None, None], k[None, None], v[None, None], g, scale)
    o_ref = gval * ol + (1 - gval) * og_full[0, 0][ids]
    assert_close(to_f64(out["O"][b, h])[ids], o_ref, O_MAX_ABS, O_MEAN_ABS, "O")
    kt = sample_tiles(g.tiles_per_dim, 2, seed=4)
    ref = O.dual_backward_sampled(q, k, v, gval, do, g, scale, tiles, kt, symmetric=True)
    assert_close(to_f64(out["dQ"][b, h])[ref["q_ids"]], ref["dQ"], O_MAX_ABS, O_MEAN_ABS, "dQ")
    assert_close(to_f64(out["dK"][b, h])[ref["k_ids"]], ref["dK"], O_MAX_ABS, O_MEAN_ABS, "dK")
    assert_close(to_f64(out["dV"][b, h])[ref["k_ids"]], ref["dV"], O_MAX_ABS, O_MEAN_ABS, "dV")
