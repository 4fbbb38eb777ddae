"""GPU parity of the FP8 (e4m3) forwards (vattn_sta_fwd_fp8, vattn_dual_fwd_fp8):
Q*K^T and P*V both on e4m3 operands.

Four checks:
  * the quantisation: the e4m3 bytes of Q, K and V equal torch's
    float8_e4m3fn conversion (round to nearest even) of x * (448 / absmax)
    computed in fp32 on the host inputs, and the absmax words equal the host
    inputs' absmax -- bit-exact;
  * LSE on the quantised operands: the fp64 oracle run on the dequantised Q, K
    (bytes * absmax / 448), bar 1e-3 as for the bf16 paths (the row sum is
    accumulated from unrounded probabilities);
  * O on the quantised operands: the oracle on the dequantised Q, K, V.  The
    kernel also rounds P to e4m3, relative error <= 2^-4 per probability, so
    per element |err| <= 2e-2 + 2^-4 * sum_j p_ij |v_jc| (every rounding at
    its worst) and, for independent roundings, mean |err| <= 2e-3 + 2^-4 *
    mean sqrt(sum_j p_ij^2 v_jc^2) (the rms bound); both sums are oracle
    attentions of |V| and of V^2 (the latter at twice the scale, rescaled by
    exp(LSE_2s - 2 LSE_s));
  * against the exact (unquantised) oracle, by the triangle inequality: the
    oracle's own change when Q, K are replaced by their dequantised values
    (|O(Q', K', V) - O(Q, K, V)| per element, |LSE(Q', K') - LSE(Q, K)| per
    row), plus the bars above with V's rounding added (another 2^-4 relative
    per value: 2^-3 times the two sums).
"""
import math

import numpy as np
import pytest

from helpers import (LSE_MAX_ABS, O_MAX_ABS, O_MEAN_ABS, geom_for, gpu_tensor, host_f64, sample_tiles, to_f64)
from oracle import vattn_oracle as O
from synth import inputs as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def V():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import video_dit_local_b200 as V
    return V


def _a256(x):
    return (x + 255) // 256 * 256


def _bf16_ulp(x):
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


def _e4m3_bytes(x, amax):
    """torch's e4m3 conversion of x * (448 / absmax), the product in fp32."""
    import torch
    inv = np.float32(448.0) / np.float32(amax) if amax > 0 else np.float32(1.0)
    x32 = x.float().numpy().astype(np.float32) * inv
    return torch.from_numpy(x32).clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)


def _dequant(bytes_u8, amax):
    import torch
    s = amax / 448.0 if amax > 0 else 1.0
    return bytes_u8.view(torch.float8_e4m3fn).float().numpy().astype(np.float64) * s


def _host_e4m3(x64):
    """Host-side e4m3 quantisation of one head ([N, d] float64 holding bf16 or
    pooled values): absmax, bytes and the dequantised values."""
    import torch
    t = torch.from_numpy(x64.astype(np.float32))
    a = float(t.abs().max())
    b = _e4m3_bytes(t, a)
    return a, b, _dequant(b, a)


def _sums(attn, q, k, v, scale):
    """sum_j p_ij |v_jc| and sqrt(sum_j p_ij^2 v_jc^2) for the rows attn
    compares, from oracle attentions: attn(q, k, values, scale) -> (O, LSE)."""
    a, _ = attn(q, k, np.abs(v), scale)
    _, lse1 = attn(q, k, v, scale)
    o2, lse2 = attn(q, k, v * v, 2 * scale)
    return a, np.sqrt(o2 * np.exp(lse2 - 2 * lse1)[:, None])


def _assert_bounded(got, ref, max_abs, mean_abs, what):
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    bad = err > max_abs
    assert not bad.any(), f"{what}: {int(bad.sum())} elements above their bar, worst excess {(err - max_abs).max():.3e}"
    assert err.mean() <= mean_abs, f"{what}: mean abs err {err.mean():.3e} > {mean_abs:.3e}"


def _run(V, w, check):
    """vattn_sta_fwd_fp8 on tile-major copies; returns raster O, LSE and, for
    the checked heads, the workspace's e4m3 Q, K, V bytes and absmax words."""
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
    ws = torch.zeros(V.vattn_workspace_size(V.VATTN_OP_STA_FWD_FP8, geom), dtype=torch.uint8, device="cuda")
    V.vattn_sta_fwd_fp8(geom, q, k, v, 1 / math.sqrt(w.head_dim), o, lse, ws)
    torch.cuda.synchronize()
    assert V.vattn_get_status() == 0, V.vattn_last_error()
    n = q.numel()
    t = _a256(n)
    bh = w.batch * w.heads
    x8 = [ws[i * t:i * t + n].view(q.shape) for i in range(3)]
    amax = ws[3 * t:3 * t + 8 * bh].view(torch.int32).view(torch.float32).cpu().numpy().reshape(-1, 2)
    off_v = 3 * t + _a256(8 * bh)
    vamax = ws[off_v:off_v + 4 * bh].view(torch.int32).view(torch.float32).cpu().numpy()
    o_r, lse_r = torch.empty_like(o), torch.empty_like(lse)
    V.vattn_tile_unpermute(geom, o, o_r)
    V.vattn_tile_unpermute(geom, lse, lse_r, 4)
    torch.cuda.synchronize()
    heads = {(b, h): [x[b, h].cpu() for x in x8] for b, h in check}
    return heads, amax, vamax, o_r, lse_r


def _check_sta_fp8(w, heads, amax, vamax, o_r, lse_r, tiles=None):
    """Every expected value from the host inputs alone (see the module
    docstring); tiles = None compares every query."""
    import torch
    g = O.geom_of(w)
    scale = 1 / math.sqrt(w.head_dim)
    if tiles is None:
        def attn(q, k, v, sc):
            o, l = O.sta_attention(q[None, None], k[None, None], v[None, None], g, sc)
            return o[0, 0], l[0, 0]
        rows = slice(None)
    else:
        def attn(q, k, v, sc):
            return O.sta_attention_tiles(q, k, v, g, sc, tiles)[1:]
        rows = O.sta_attention_tiles(np.zeros((g.n, 1)), np.zeros((g.n, 1)), np.zeros((g.n, 1)), g, 1.0, tiles)[0]
    for (b, h), (q8, k8, v8) in heads.items():
        i = b * w.heads + h
        q, k, v = (host_f64(w, t, b, h) for t in (S.Q_ID, S.K_ID, S.V_ID))
        aq, q8h, qd = _host_e4m3(q)
        ak, k8h, kd = _host_e4m3(k)
        av, v8h, vd = _host_e4m3(v)
        assert amax[i, 0] == aq and amax[i, 1] == ak and vamax[i] == av, f"absmax b{b} h{h}"
        for got, host, name in ((q8, q8h, "Q"), (k8, k8h, "K"), (v8, v8h, "V")):
            assert torch.equal(got, torch.from_numpy(O.permute(host.numpy(), g))), f"{name} e4m3 bytes b{b} h{h}"
        got_o = to_f64(o_r[b, h])[rows]
        got_l = lse_r[b, h].cpu().numpy().astype(np.float64)[rows]
        # on the quantised operands
        o_ref, lse_ref = attn(qd, kd, vd, scale)
        a, rms = _sums(attn, qd, kd, vd, scale)
        _assert_bounded(got_o, o_ref, O_MAX_ABS + 2.0 ** -4 * a, O_MEAN_ABS + 2.0 ** -4 * rms.mean(),
                        f"O on dequantised operands b{b} h{h}")
        _assert_bounded(got_l, lse_ref, LSE_MAX_ABS, math.inf, f"LSE on dequantised operands b{b} h{h}")
        # against the exact oracle: the oracle's own change under the Q, K
        # quantisation, plus the P and V roundings
        o_ex, lse_ex = attn(q, k, v, scale)
        o_qk, lse_qk = attn(qd, kd, v, scale)
        a, rms = _sums(attn, qd, kd, v, scale)
        dq_o = np.abs(o_qk - o_ex)
        _assert_bounded(got_o, o_ex, dq_o + O_MAX_ABS + 2.0 ** -3 * a,
                        dq_o.mean() + O_MEAN_ABS + 2.0 ** -3 * rms.mean(), f"O vs exact b{b} h{h}")
        _assert_bounded(got_l, lse_ex, np.abs(lse_qk - lse_ex) + LSE_MAX_ABS, math.inf, f"LSE vs exact b{b} h{h}")


CASES = [
    ((6, 16, 24), (3, 8, 8), (1, 3, 3), 1, 2),     # tile 192: a ragged second query block
    ((6, 16, 32), (6, 8, 8), (1, 3, 3), 2, 1),     # tile 384, batch 2
    ((4, 8, 16), (2, 4, 4), (1, 1, 3), 1, 3),      # tile 32
    ((3, 16, 40), (3, 8, 8), (1, 3, 3), 1, 2),     # tile 192, 5 tiles along w, interior windows a tile apart
]


@pytest.mark.parametrize("grid,tile,window,batch,heads", CASES)
def test_fp8_fwd_small_full(V, grid, tile, window, batch, heads):
    w = S.small_workload("fp8", 72, batch, heads, 128, grid, tile, window, (1, 1, 1))
    check = [(b, h) for b in range(batch) for h in range(heads)]
    _check_sta_fp8(w, *_run(V, w, check))


def test_fp8_fwd_720p_sampled(V):
    """The benchmarked 720p workload, all 24 heads in one launch; heads 0 and
    23 compared on query tiles covering every boundary class."""
    w = S.WORKLOADS["720p"]
    check = [(0, 0), (0, w.heads - 1)]
    _check_sta_fp8(w, *_run(V, w, check), tiles=sample_tiles(O.geom_of(w).tiles_per_dim, 10))


def _dual_fp8_run(V, w, check):
    """vattn_dual_fwd_fp8 on tile-major copies; returns raster O and, for the
    checked heads only, the workspace's e4m3 Q, K, V, K_p, V_p bytes, the
    absmax words and bf16 K_p, V_p (copied from the device slice by slice)."""
    import torch
    g = O.geom_of(w)
    geom = geom_for(V, w)
    tiled = []
    for tid in (S.Q_ID, S.K_ID, S.V_ID):
        x = gpu_tensor(w, tid, check)
        t = torch.empty_like(x)
        V.vattn_tile_permute(geom, x, t)
        tiled.append(t)
        del x
    q, k, v = tiled
    gvec = torch.from_numpy(S.blend_g(w)).cuda()
    o = torch.empty_like(q)
    ws = torch.zeros(V.vattn_workspace_size(V.VATTN_OP_DUAL_FWD_FP8, geom), dtype=torch.uint8, device="cuda")
    V.vattn_dual_fwd_fp8(geom, q, k, v, gvec, 1 / math.sqrt(w.head_dim), o, ws)
    o_r = torch.empty_like(o)
    V.vattn_tile_unpermute(geom, o, o_r)
    torch.cuda.synchronize()
    assert V.vattn_get_status() == 0, V.vattn_last_error()
    B, H, d = w.batch, w.heads, w.head_dim
    bh, n, npl = B * H, g.n, g.n_pooled
    t8, p8, am, av = _a256(bh * n * d), _a256(bh * npl * d), _a256(bh * 8), _a256(bh * 4)
    off_kp8 = 3 * t8
    off_vp8 = off_kp8 + p8
    off_al = off_vp8 + p8
    off_ag = off_al + am
    off_vl = off_ag + am
    off_vg = off_vl + av
    off_ol = off_vg + av
    off_kp = off_ol + _a256(bh * n * d * 2)
    off_vp = off_kp + _a256(bh * npl * d * 2)

    def f32(off, cnt):
        return ws[off:off + 4 * cnt].view(torch.int32).view(torch.float32).cpu().numpy()
    amax_l, amax_g = f32(off_al, 2 * bh).reshape(-1, 2), f32(off_ag, 2 * bh).reshape(-1, 2)
    vamax_l, vamax_g = f32(off_vl, bh), f32(off_vg, bh)
    x8 = [ws[i * t8:i * t8 + bh * n * d].view(B, H, n, d) for i in range(3)]
    kp8 = ws[off_kp8:off_kp8 + bh * npl * d].view(B, H, npl, d)
    vp8 = ws[off_vp8:off_vp8 + bh * npl * d].view(B, H, npl, d)
    kp = ws[off_kp:off_kp + bh * npl * d * 2].view(torch.bfloat16).view(B, H, npl, d)
    vp = ws[off_vp:off_vp + bh * npl * d * 2].view(torch.bfloat16).view(B, H, npl, d)
    heads = {(b, h): dict(q8=x8[0][b, h].cpu(), k8=x8[1][b, h].cpu(), v8=x8[2][b, h].cpu(), kp8=kp8[b, h].cpu(),
                          vp8=vp8[b, h].cpu(), kp=to_f64(kp[b, h]), vp=to_f64(vp[b, h])) for b, h in check}
    return o_r, (amax_l, amax_g, vamax_l, vamax_g), heads


def _check_dual_fp8(w, o_r, amaxes, heads, tiles=None):
    """Every expected value is built from the host inputs alone:
      * the workspace's e4m3 Q, K, V bytes equal the host quantisation of the
        host Q, K, V (bit-exact); its K_p and V_p lie within one bf16 ulp of
        the oracle's exact pooling, and its K_p, V_p bytes equal the host
        quantisation of that pooling rounded to bf16;
      * O against the dual oracle run on the host-dequantised Q, K, V, K_p, V_p
        with the P-rounding bars of the module docstring, blended;
      * O against the exact dual oracle: the oracle's own change under the
        Q, K, K_p quantisation plus the P and V / V_p roundings."""
    import torch
    g = O.geom_of(w)
    gv = S.blend_g(w).astype(np.float64)
    scale = 1 / math.sqrt(w.head_dim)
    amax_l, amax_g, vamax_l, vamax_g = amaxes
    assert np.array_equal(amax_g[:, 0], amax_l[:, 0]), "shared Q scale"
    if tiles is None:
        def local(q, k, v, sc):
            o, l = O.sta_attention(q[None, None], k[None, None], v[None, None], g, sc)
            return o[0, 0], l[0, 0]

        def glob(q, k, v, sc):
            o, l = O.global_attention(q[None, None], k[None, None], v[None, None], sc)
            return o[0, 0], l[0, 0]
        rows = slice(None)
    else:
        rows = O.sta_attention_tiles(np.zeros((g.n, 1)), np.zeros((g.n, 1)), np.zeros((g.n, 1)), g, 1.0, tiles)[0]

        def local(q, k, v, sc):
            return O.sta_attention_tiles(q, k, v, g, sc, tiles)[1:]

        def glob(q, k, v, sc):
            return O.global_attention_rows(q, k, v, sc, rows)
    for (b, h), got in heads.items():
        i = b * w.heads + h
        q, k, v = (host_f64(w, t, b, h) for t in (S.Q_ID, S.K_ID, S.V_ID))
        aq, q8, qd = _host_e4m3(q)
        ak, k8, kd = _host_e4m3(k)
        av, v8, vd = _host_e4m3(v)
        assert amax_l[i, 0] == aq and amax_l[i, 1] == ak and vamax_l[i] == av, "absmax of Q, K, V"
        for name, hb in (("q8", q8), ("k8", k8), ("v8", v8)):
            assert torch.equal(got[name], torch.from_numpy(O.permute(hb.numpy(), g))), f"{name} bytes b{b} h{h}"
        kp_ex, vp_ex = O.pool(k, g), O.pool(v, g)
        assert (np.abs(got["kp"] - kp_ex) <= _bf16_ulp(kp_ex)).all(), "K_p vs the exact pooling"
        assert (np.abs(got["vp"] - vp_ex) <= _bf16_ulp(vp_ex)).all(), "V_p vs the exact pooling"
        pooled = []
        for name, ex, amax_dev in (("kp8", kp_ex, amax_g[i, 1]), ("vp8", vp_ex, vamax_g[i])):
            xb = S.bf16_bits_to_f64(S.bf16_round_bits(ex.astype(np.float32)))
            a, hb, xd = _host_e4m3(xb)
            # the device quantises its own bf16 pooling, which may sit one bf16
            # ulp from the host rounding of the exact mean (fp32 summation
            # order); the host reference below does not depend on its bytes
            assert abs(amax_dev - a) <= _bf16_ulp(a), f"absmax of {name}"
            if amax_dev == a:
                n_diff = int((got[name] != hb).sum())
                assert n_diff <= max(1, hb.numel() // 10000), f"{name} bytes: {n_diff} differ"
            pooled.append(xd)
        kpd, vpd = pooled
        got_o = to_f64(o_r[b, h])[rows]
        gl, gg = gv[h], 1 - gv[h]
        o_l, _ = local(qd, kd, vd, scale)
        o_g, _ = glob(qd, kpd, vpd, scale)
        a_l, r_l = _sums(local, qd, kd, vd, scale)
        a_g, r_g = _sums(glob, qd, kpd, vpd, scale)
        _assert_bounded(got_o, gl * o_l + gg * o_g, O_MAX_ABS + 2.0 ** -4 * (gl * a_l + gg * a_g),
                        O_MEAN_ABS + 2.0 ** -4 * (gl * r_l + gg * r_g).mean(), f"O b{b} h{h}")
        e_l, _ = local(q, k, v, scale)
        e_g, _ = glob(q, kp_ex, vp_ex, scale)
        ex = gl * e_l + gg * e_g
        d_qk = np.abs(gl * local(qd, kd, v, scale)[0] + gg * glob(qd, kpd, vp_ex, scale)[0] - ex)
        a_l, r_l = _sums(local, qd, kd, v, scale)
        a_g, r_g = _sums(glob, qd, kpd, vp_ex, scale)
        _assert_bounded(got_o, ex, d_qk + O_MAX_ABS + 2.0 ** -3 * (gl * a_l + gg * a_g),
                        d_qk.mean() + O_MEAN_ABS + 2.0 ** -3 * (gl * r_l + gg * r_g).mean(), f"O vs exact b{b} h{h}")


@pytest.mark.parametrize("grid,tile,window,pool,batch,heads", [
    ((6, 16, 24), (3, 8, 8), (1, 3, 3), (1, 4, 4), 1, 2),   # tile 192, N_p = 144
    ((6, 16, 32), (6, 8, 8), (1, 3, 3), (2, 2, 2), 2, 1),   # temporal pooling, batch 2
])
def test_dual_fp8_fwd(V, grid, tile, window, pool, batch, heads):
    """vattn_dual_fwd_fp8 on small grids, every head and query compared."""
    w = S.small_workload("fp8dual", 73, batch, heads, 128, grid, tile, window, pool)
    check = [(b, h) for b in range(batch) for h in range(heads)]
    _check_dual_fp8(w, *_dual_fp8_run(V, w, check))


def test_dual_fp8_fwd_1080p_sampled(V):
    """The benchmarked 1080p-shaped FP8 dual launch (all 24 heads); heads 0 and
    23 compared on query tiles covering every boundary class."""
    w = S.WORKLOADS["1080p"]
    check = [(0, 0), (0, w.heads - 1)]
    _check_dual_fp8(w, *_dual_fp8_run(V, w, check), tiles=sample_tiles(O.geom_of(w).tiles_per_dim, 4))
