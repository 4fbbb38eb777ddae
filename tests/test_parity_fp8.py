"""GPU parity of the FP8 Q*K^T sliding-tile forward (vattn_sta_fwd_fp8).

Three checks:
  * the quantisation: the e4m3 bytes of Q and K equal torch's float8_e4m3fn
    conversion (round to nearest even) of x * (448 / absmax) computed in fp32,
    and the absmax words equal the inputs' absmax -- bit-exact;
  * the attention on the quantised values: the fp64 oracle run on the
    dequantised Q, K (bytes * absmax / 448) and the exact V, with the bf16
    bars of the other forward paths (O 2e-2 / 2e-3, LSE 1e-3);
  * against the exact (unquantised) oracle, a bar derived from e4m3 rounding:
    relative error <= 2^-4 per operand, so with q, k ~ N(0, 1) and
    scale = d^-1/2 each logit moves by about sqrt(2/3) * 2^-4 ~ 0.05 (std);
    five standard deviations give 0.25 for LSE and O (max-abs), and the O
    mean-abs bar 0.02 sits above the ~0.05 / sqrt(effective keys) average.
"""
import math

import numpy as np
import pytest

from helpers import (LSE_MAX_ABS, O_MAX_ABS, O_MEAN_ABS, assert_close, geom_for, gpu_tensor, host_f64, to_f64)
from oracle import vattn_oracle as O
from synth import inputs as S

pytestmark = pytest.mark.gpu

FP8_O_MAX_ABS, FP8_O_MEAN_ABS, FP8_LSE_MAX_ABS = 0.25, 0.02, 0.25


@pytest.fixture(scope="module")
def V():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import video_dit_local_b200 as V
    return V


def _run(V, w, check):
    import torch
    geom = geom_for(V, w)
    tiled = []
    for tid in (S.Q_ID, S.K_ID, S.V_ID):
        x = gpu_tensor(w, tid, check)
        t = torch.empty_like(x)
        V.vattn_tile_permute(geom, x, t)
        tiled.append(t)
    q, k, v = tiled
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    need = V.vattn_workspace_size(V.VATTN_OP_STA_FWD_FP8, geom)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    V.vattn_sta_fwd_fp8(geom, q, k, v, 1 / math.sqrt(w.head_dim), o, lse, ws)
    torch.cuda.synchronize()
    assert V.vattn_get_status() == 0, V.vattn_last_error()
    n = q.numel()
    t = (n + 255) // 256 * 256
    q8 = ws[:n].view(q.shape).cpu()
    k8 = ws[t:t + n].view(q.shape).cpu()
    amax = ws[2 * t:2 * t + 8 * w.batch * w.heads].view(torch.int32).view(torch.float32).cpu().numpy().reshape(-1, 2)
    o_r, lse_r = torch.empty_like(o), torch.empty_like(lse)
    V.vattn_tile_unpermute(geom, o, o_r)
    V.vattn_tile_unpermute(geom, lse, lse_r, 4)
    torch.cuda.synchronize()
    return q.cpu(), k.cpu(), q8, k8, amax, o_r, lse_r


def _e4m3_bytes(x_bf16, amax):
    """torch's e4m3 conversion of x * (448 / absmax), the product in fp32."""
    import torch
    inv = np.float32(448.0) / np.float32(amax) if amax > 0 else np.float32(1.0)
    x32 = x_bf16.float().numpy().astype(np.float32) * inv
    return torch.from_numpy(x32).clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)


def _dequant(bytes_u8, amax):
    import torch
    s = amax / 448.0 if amax > 0 else 1.0
    return bytes_u8.view(torch.float8_e4m3fn).float().numpy().astype(np.float64) * s


CASES = [
    ((6, 16, 24), (3, 8, 8), (1, 3, 3), 1, 2),     # tile 192: a ragged second query block
    ((6, 16, 32), (6, 8, 8), (1, 3, 3), 2, 1),     # tile 384, batch 2
    ((4, 8, 16), (2, 4, 4), (1, 1, 3), 1, 3),      # tile 32
]


@pytest.mark.parametrize("grid,tile,window,batch,heads", CASES)
def test_fp8_quantisation_bit_exact(V, grid, tile, window, batch, heads):
    import torch
    w = S.small_workload("fp8", 71, batch, heads, 128, grid, tile, window, (1, 1, 1))
    check = [(b, h) for b in range(batch) for h in range(heads)]
    q, k, q8, k8, amax, _, _ = _run(V, w, check)
    for b in range(batch):
        for h in range(heads):
            i = b * heads + h
            for x, x8, a in ((q, q8, amax[i, 0]), (k, k8, amax[i, 1])):
                assert a == float(x[b, h].float().abs().max()), "absmax"
                assert torch.equal(x8[b, h], _e4m3_bytes(x[b, h], a)), "e4m3 bytes"


@pytest.mark.parametrize("grid,tile,window,batch,heads", CASES)
def test_fp8_fwd_equals_oracle_on_dequantised_inputs(V, grid, tile, window, batch, heads):
    w = S.small_workload("fp8", 72, batch, heads, 128, grid, tile, window, (1, 1, 1))
    check = [(b, h) for b in range(batch) for h in range(heads)]
    _, _, q8, k8, amax, o_r, lse_r = _run(V, w, check)
    g = O.geom_of(w)
    scale = 1 / math.sqrt(128)
    for b, h in check:
        i = b * heads + h
        # the workspace bytes are tile-major: back to raster for the oracle
        qd = O.unpermute(_dequant(q8[b, h], amax[i, 0]), g)
        kd = O.unpermute(_dequant(k8[b, h], amax[i, 1]), g)
        v = host_f64(w, S.V_ID, b, h)
        o_ref, lse_ref = O.sta_attention(qd[None, None], kd[None, None], v[None, None], g, scale)
        assert_close(to_f64(o_r[b, h]), o_ref[0, 0], O_MAX_ABS, O_MEAN_ABS, f"O b{b} h{h}")
        assert_close(lse_r[b, h].cpu().numpy().astype(np.float64), lse_ref[0, 0], LSE_MAX_ABS, what=f"LSE b{b} h{h}")
        # against the exact oracle: the e4m3-derived bar
        q, k = host_f64(w, S.Q_ID, b, h), host_f64(w, S.K_ID, b, h)
        o_ex, lse_ex = O.sta_attention(q[None, None], k[None, None], v[None, None], g, scale)
        assert_close(to_f64(o_r[b, h]), o_ex[0, 0], FP8_O_MAX_ABS, FP8_O_MEAN_ABS, f"O vs exact b{b} h{h}")
        assert_close(lse_r[b, h].cpu().numpy().astype(np.float64), lse_ex[0, 0], FP8_LSE_MAX_ABS,
                     what=f"LSE vs exact b{b} h{h}")


def test_fp8_fwd_720p_sampled(V):
    """The benchmarked 720p workload, all 24 heads in one launch; heads 0 and
    23 compared on query tiles covering every boundary class, against the
    oracle on their dequantised Q and K."""
    from helpers import sample_tiles
    w = S.WORKLOADS["720p"]
    check = [(0, 0), (0, w.heads - 1)]
    _, _, q8, k8, amax, o_r, lse_r = _run(V, w, check)
    g = O.geom_of(w)
    scale = 1 / math.sqrt(w.head_dim)
    tiles = sample_tiles(g.tiles_per_dim, 10)
    for b, h in check:
        i = b * w.heads + h
        qd = O.unpermute(_dequant(q8[b, h], amax[i, 0]), g)
        kd = O.unpermute(_dequant(k8[b, h], amax[i, 1]), g)
        v = host_f64(w, S.V_ID, b, h)
        ids, o_ref, lse_ref = O.sta_attention_tiles(qd, kd, v, g, scale, tiles)
        assert_close(to_f64(o_r[b, h])[ids], o_ref, O_MAX_ABS, O_MEAN_ABS, f"O b{b} h{h}")
        assert_close(lse_r[b, h].cpu().numpy().astype(np.float64)[ids], lse_ref, LSE_MAX_ABS, what=f"LSE b{b} h{h}")


def _a256(x):
    return (x + 255) // 256 * 256


@pytest.mark.parametrize("grid,tile,window,pool,batch,heads", [
    ((6, 16, 24), (3, 8, 8), (1, 3, 3), (1, 4, 4), 1, 2),   # tile 192, N_p = 144
    ((6, 16, 32), (6, 8, 8), (1, 3, 3), (2, 2, 2), 2, 1),   # temporal pooling, batch 2
])
def test_dual_fp8_fwd(V, grid, tile, window, pool, batch, heads):
    """vattn_dual_fwd_fp8: the K_p bytes and the shared Q scale bit-exact; the
    blended output against the oracle on the dequantised operands (bf16 bars)
    and against the exact dual oracle (e4m3 bars)."""
    import torch
    w = S.small_workload("fp8dual", 73, batch, heads, 128, grid, tile, window, pool)
    check = [(b, h) for b in range(batch) for h in range(heads)]
    g = O.geom_of(w)
    geom = geom_for(V, w)
    tiled = []
    for tid in (S.Q_ID, S.K_ID, S.V_ID):
        x = gpu_tensor(w, tid, check)
        t = torch.empty_like(x)
        V.vattn_tile_permute(geom, x, t)
        tiled.append(t)
    q, k, v = tiled
    gvec = torch.from_numpy(S.blend_g(w)).cuda()
    o = torch.empty_like(q)
    ws = torch.zeros(V.vattn_workspace_size(V.VATTN_OP_DUAL_FWD_FP8, geom), dtype=torch.uint8, device="cuda")
    scale = 1 / math.sqrt(128)
    V.vattn_dual_fwd_fp8(geom, q, k, v, gvec, scale, o, ws)
    o_r = torch.empty_like(o)
    V.vattn_tile_unpermute(geom, o, o_r)
    torch.cuda.synchronize()
    assert V.vattn_get_status() == 0, V.vattn_last_error()
    bh, n, npl = batch * heads, g.n, g.n_pooled
    t8, p8, am = _a256(bh * n * 128), _a256(bh * npl * 128), _a256(bh * 8)
    off_kp8, off_al = 2 * t8, 2 * t8 + p8
    off_ag, off_ol = off_al + am, off_al + 2 * am
    off_kp = off_ol + _a256(bh * n * 128 * 2)
    off_vp = off_kp + _a256(bh * npl * 128 * 2)
    wsc = ws.cpu()
    q8 = wsc[:bh * n * 128].view(batch, heads, n, 128)
    k8 = wsc[t8:t8 + bh * n * 128].view(batch, heads, n, 128)
    kp8 = wsc[off_kp8:off_kp8 + bh * npl * 128].view(batch, heads, npl, 128)
    amax_l = wsc[off_al:off_al + 8 * bh].view(torch.int32).view(torch.float32).numpy().reshape(-1, 2)
    amax_g = wsc[off_ag:off_ag + 8 * bh].view(torch.int32).view(torch.float32).numpy().reshape(-1, 2)
    kp = wsc[off_kp:off_kp + bh * npl * 256].view(torch.bfloat16).view(batch, heads, npl, 128)
    vp = wsc[off_vp:off_vp + bh * npl * 256].view(torch.bfloat16).view(batch, heads, npl, 128)
    assert np.array_equal(amax_g[:, 0], amax_l[:, 0])
    gv = S.blend_g(w)
    for b, h in check:
        i = b * heads + h
        assert amax_g[i, 1] == float(kp[b, h].float().abs().max())
        assert torch.equal(kp8[b, h], _e4m3_bytes(kp[b, h], amax_g[i, 1])), "K_p e4m3 bytes"
        qd = O.unpermute(_dequant(q8[b, h], amax_l[i, 0]), g)
        kd = O.unpermute(_dequant(k8[b, h], amax_l[i, 1]), g)
        kpd = _dequant(kp8[b, h], amax_g[i, 1])
        vv = host_f64(w, S.V_ID, b, h)
        o_l, _ = O.sta_attention(qd[None, None], kd[None, None], vv[None, None], g, scale)
        o_g, _ = O.global_attention(qd[None, None], kpd[None, None], vp[b, h].double().numpy()[None, None], scale)
        ref = gv[h] * o_l[0, 0] + (1 - gv[h]) * o_g[0, 0]
        assert_close(to_f64(o_r[b, h]), ref, O_MAX_ABS, O_MEAN_ABS, f"O b{b} h{h}")
        qx, kx = host_f64(w, S.Q_ID, b, h), host_f64(w, S.K_ID, b, h)
        ex = O.dual_forward(qx[None, None], kx[None, None], vv[None, None], gv[h:h + 1], g, scale)["O"]
        assert_close(to_f64(o_r[b, h]), ex[0, 0], FP8_O_MAX_ABS, FP8_O_MEAN_ABS, f"O vs exact b{b} h{h}")
