"""GPU parity of the forward path against the fp64 oracle (through the C ABI).

Bars: tile mask and permutation bit-exact; pooled K/V within one bf16 ulp of
the exact mean; O within max-abs 2e-2 and mean-abs 2e-3; LSE within 1e-3.
Large workloads run the full launch (all heads) and compare the seeded heads
on query tiles that cover every boundary class.
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


def _permute(V, geom, x):
    import torch
    out = torch.empty_like(x)
    V.vattn_tile_permute(geom, x, out)
    return out


def _unpermute(V, geom, x):
    import torch
    out = torch.empty_like(x)
    V.vattn_tile_unpermute(geom, x, out)
    return out


# ------------------------------------------------------------------ permutation / kept tiles / pooling

@pytest.mark.parametrize("name", ["tiny", "720p"])
def test_permute_bit_exact(V, name):
    import torch
    w = S.WORKLOADS[name]
    g = O.geom_of(w)
    geom = geom_for(V, w)
    check = [(0, 0), (0, w.heads - 1)]
    x = gpu_tensor(w, S.Q_ID, check)
    xt = _permute(V, geom, x)
    for b, h in check:
        expect = O.permute(S.draw_head(w, S.Q_ID, b, h), g)
        got = xt[b, h].cpu().view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(got, expect)
    assert torch.equal(_unpermute(V, geom, xt).view(torch.int16), x.view(torch.int16))
    # 4-byte rows (LSE layout)
    l = torch.arange(w.batch * w.heads * w.n_tokens, dtype=torch.float32, device="cuda").view(
        w.batch, w.heads, w.n_tokens)
    lt = torch.empty_like(l)
    V.vattn_tile_permute(geom, l, lt, 4)
    expect = O.permute(l[0, 0].cpu().numpy()[:, None], g)[:, 0]
    assert np.array_equal(lt[0, 0].cpu().numpy(), expect)
    back = torch.empty_like(l)
    V.vattn_tile_unpermute(geom, lt, back, 4)
    assert torch.equal(back, l)


@pytest.mark.parametrize("name", list(S.WORKLOADS))
def test_kept_tiles_bit_exact(V, name):
    import torch
    w = S.WORKLOADS[name]
    g = O.geom_of(w)
    expect = O.kept_tiles(g)
    out = torch.full(expect.shape, -1, dtype=torch.int32, device="cuda")
    V.vattn_kept_tiles(geom_for(V, w), out)
    assert np.array_equal(out.cpu().numpy(), expect)


def test_kept_tiles_odd_grid(V):
    import torch
    g = O.Geom(6, 12, 20, (2, 4, 4), (3, 2, 4))
    expect = O.kept_tiles(g)
    out = torch.full(expect.shape, -1, dtype=torch.int32, device="cuda")
    V.vattn_kept_tiles(V.make_geom(1, 1, 64, (6, 12, 20), (2, 4, 4), (3, 2, 4)), out)
    assert np.array_equal(out.cpu().numpy(), expect)


def _bf16_ulp(x):
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


@pytest.mark.parametrize("name", ["1080p", "4k"])
def test_pool_within_one_ulp(V, name):
    import torch
    w = S.WORKLOADS[name]
    g = O.geom_of(w)
    geom = geom_for(V, w)
    check = [(0, 0)] if name == "4k" else [(0, 0), (0, w.heads - 1)]
    k = _permute(V, geom, gpu_tensor(w, S.K_ID, check))
    v = _permute(V, geom, gpu_tensor(w, S.V_ID, check))
    kp = torch.empty((w.batch, w.heads, g.n_pooled, w.head_dim), dtype=torch.bfloat16, device="cuda")
    vp = torch.empty_like(kp)
    V.vattn_pool_kv(geom, k, v, kp, vp)
    for b, h in check:
        for tid, got in ((S.K_ID, kp), (S.V_ID, vp)):
            exact = O.pool(host_f64(w, tid, b, h), g)
            err = np.abs(to_f64(got[b, h]) - exact)
            assert (err <= _bf16_ulp(exact)).all(), err.max()


def test_pool_small_geometries(V):
    import torch
    for grid, tile, pool, d in [((4, 8, 8), (2, 4, 4), (1, 2, 2), 64), ((6, 12, 20), (2, 4, 4), (3, 2, 5), 128),
                                ((3, 8, 8), (3, 8, 8), (1, 8, 8), 128)]:
        w = S.small_workload("pool", 7, 2, 3, d, grid, tile, (1, 1, 1), pool)
        g = O.geom_of(w)
        geom = geom_for(V, w)
        check = [(b, h) for b in range(2) for h in range(3)]
        k = _permute(V, geom, gpu_tensor(w, S.K_ID, check))
        v = _permute(V, geom, gpu_tensor(w, S.V_ID, check))
        kp = torch.empty((2, 3, g.n_pooled, d), dtype=torch.bfloat16, device="cuda")
        vp = torch.empty_like(kp)
        V.vattn_pool_kv(geom, k, v, kp, vp)
        for b, h in check:
            exact = O.pool(host_f64(w, S.V_ID, b, h), g)
            assert (np.abs(to_f64(vp[b, h]) - exact) <= _bf16_ulp(exact)).all()


# ------------------------------------------------------------------ attention forward

def _sta_gpu(V, w, check):
    import torch
    geom = geom_for(V, w)
    q, k, v = (_permute(V, geom, gpu_tensor(w, i, check)) for i in (S.Q_ID, S.K_ID, S.V_ID))
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    V.vattn_sta_fwd(geom, q, k, v, 1 / math.sqrt(w.head_dim), o, lse)
    o_r = _unpermute(V, geom, o)
    lse_r = torch.empty_like(lse)
    V.vattn_tile_unpermute(geom, lse, lse_r, 4)
    torch.cuda.synchronize()
    assert V.vattn_get_status() == 0
    return o_r, lse_r


def _check_sta(w, o_r, lse_r, check, tiles):
    g = O.geom_of(w)
    scale = 1 / math.sqrt(w.head_dim)
    for b, h in check:
        q, k, v = (host_f64(w, i, b, h) for i in (S.Q_ID, S.K_ID, S.V_ID))
        ids, o_ref, lse_ref = O.sta_attention_tiles(q, k, v, g, scale, tiles)
        assert_close(to_f64(o_r[b, h])[ids], o_ref, O_MAX_ABS, O_MEAN_ABS, f"O b{b} h{h}")
        assert_close(lse_r[b, h].cpu().numpy().astype(np.float64)[ids], lse_ref, LSE_MAX_ABS, what=f"LSE b{b} h{h}")


def test_sta_fwd_tiny_full(V):
    w = S.WORKLOADS["tiny"]
    check = [(0, 0), (0, 1)]
    o_r, lse_r = _sta_gpu(V, w, check)
    _check_sta(w, o_r, lse_r, check, range(math.prod(O.geom_of(w).tiles_per_dim)))


def test_sta_fwd_720p_sampled(V):
    w = S.WORKLOADS["720p"]
    check = [(0, 0), (0, w.heads - 1)]
    o_r, lse_r = _sta_gpu(V, w, check)
    _check_sta(w, o_r, lse_r, check, sample_tiles(O.geom_of(w).tiles_per_dim, 10))


@pytest.mark.parametrize("grid,tile,window,d,batch,heads", [
    ((4, 8, 8), (2, 4, 4), (2, 2, 2), 64, 1, 2),         # window covers the grid: full attention
    ((6, 16, 24), (3, 8, 8), (1, 1, 3), 128, 1, 2),      # tile 192: ragged second query block
    ((6, 16, 32), (6, 8, 8), (1, 3, 3), 64, 2, 1),       # tile 384, d = 64, batch 2
    ((4, 8, 16), (2, 4, 4), (1, 1, 1), 128, 1, 3),       # window of one tile
    ((2, 8, 8), (2, 4, 4), (3, 5, 7), 128, 1, 1),        # window wider than the grid in every dim
    # tiles of 192 and 64 rows: adjacent tiles along w share query blocks, the
    # straddling block over windows that coincide (edges) or start a tile apart
    ((3, 16, 40), (3, 8, 8), (1, 3, 3), 128, 1, 2),      # 5 tiles along w: two pairs and a tile of its own
    ((2, 16, 48), (1, 8, 8), (1, 1, 3), 64, 1, 2),       # tile 64: every query block straddles two tiles
    ((3, 8, 64), (3, 8, 8), (1, 1, 5), 128, 1, 1),       # window of 5 along w: interior pairs a tile apart
    ((3, 8, 48), (3, 8, 8), (1, 2, 2), 128, 1, 1),       # even window
])
def test_sta_fwd_small_full(V, grid, tile, window, d, batch, heads):
    w = S.small_workload("sta", 11, batch, heads, d, grid, tile, window, (1, 1, 1))
    check = [(b, h) for b in range(batch) for h in range(heads)]
    o_r, lse_r = _sta_gpu(V, w, check)
    g = O.geom_of(w)
    _check_sta(w, o_r, lse_r, check, range(math.prod(g.tiles_per_dim)))
    if all(wi >= ni for wi, ni in zip(window, g.tiles_per_dim)):
        q, k, v = (host_f64(w, i, 0, 0)[None, None] for i in (S.Q_ID, S.K_ID, S.V_ID))
        o_full, _ = O.full_attention(q, k, v, 1 / math.sqrt(d))
        assert_close(to_f64(o_r[0, 0]), o_full[0, 0], O_MAX_ABS, O_MEAN_ABS, "full")


def _dual_gpu(V, w, check, saved=True):
    import torch
    g = O.geom_of(w)
    geom = geom_for(V, w)
    q, k, v = (_permute(V, geom, gpu_tensor(w, i, check)) for i in (S.Q_ID, S.K_ID, S.V_ID))
    gvec = torch.from_numpy(S.blend_g(w)).cuda()
    scale = 1 / math.sqrt(w.head_dim)
    o = torch.empty_like(q)
    out = {}
    if saved:
        o_l, o_g = torch.empty_like(q), torch.empty_like(q)
        lse_l = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
        lse_g = torch.empty_like(lse_l)
        kp = torch.empty((w.batch, w.heads, g.n_pooled, w.head_dim), dtype=torch.bfloat16, device="cuda")
        vp = torch.empty_like(kp)
        V.vattn_dual_fwd(geom, q, k, v, gvec, scale, o, o_l, lse_l, o_g, lse_g, kp, vp)
        out.update(O_l=_unpermute(V, geom, o_l), O_g=_unpermute(V, geom, o_g))
        for name, t in (("LSE_l", lse_l), ("LSE_g", lse_g)):
            r = torch.empty_like(t)
            V.vattn_tile_unpermute(geom, t, r, 4)
            out[name] = r
    else:
        ws = torch.empty(V.vattn_workspace_size(V.VATTN_OP_DUAL_FWD, geom), dtype=torch.uint8, device="cuda")
        V.vattn_dual_fwd(geom, q, k, v, gvec, scale, o, workspace=ws)
    out["O"] = _unpermute(V, geom, o)
    torch.cuda.synchronize()
    assert V.vattn_get_status() == 0
    return out


def _check_dual(w, out, check, tiles):
    g = O.geom_of(w)
    scale = 1 / math.sqrt(w.head_dim)
    gv = S.blend_g(w).astype(np.float64)
    for b, h in check:
        q, k, v = (host_f64(w, i, b, h) for i in (S.Q_ID, S.K_ID, S.V_ID))
        ids, ol, lsel = O.sta_attention_tiles(q, k, v, g, scale, tiles)
        og, lseg = O.global_attention_rows(q, O.pool(k, g), O.pool(v, g), scale, ids)
        o_ref = gv[h] * ol + (1 - gv[h]) * og
        assert_close(to_f64(out["O"][b, h])[ids], o_ref, O_MAX_ABS, O_MEAN_ABS, f"O b{b} h{h}")
        if "O_l" in out:
            assert_close(to_f64(out["O_l"][b, h])[ids], ol, O_MAX_ABS, O_MEAN_ABS, "O_l")
            assert_close(to_f64(out["O_g"][b, h])[ids], og, O_MAX_ABS, O_MEAN_ABS, "O_g")
            assert_close(out["LSE_l"][b, h].cpu().numpy().astype(np.float64)[ids], lsel, LSE_MAX_ABS, what="LSE_l")
            assert_close(out["LSE_g"][b, h].cpu().numpy().astype(np.float64)[ids], lseg, LSE_MAX_ABS, what="LSE_g")


@pytest.mark.parametrize("grid,tile,window,pool,d,batch,heads", [
    ((4, 8, 8), (2, 4, 4), (1, 2, 2), (1, 2, 2), 64, 1, 2),
    ((3, 20, 24), (3, 4, 4), (1, 3, 3), (1, 2, 2), 128, 2, 3),    # N, N_p not multiples of 128
    ((3, 8, 8), (1, 4, 4), (3, 1, 1), (1, 1, 1), 128, 1, 2),      # pool 1: global = full attention
    ((3, 24, 16), (3, 8, 8), (1, 3, 1), (1, 2, 2), 128, 1, 2),    # 192-token tiles: 5 local, 3 pooled key blocks
    ((3, 16, 40), (3, 8, 8), (1, 3, 3), (1, 2, 2), 128, 1, 2),    # 192-token tiles paired along w
])
def test_dual_fwd_small_full(V, grid, tile, window, pool, d, batch, heads):
    w = S.small_workload("dual", 13, batch, heads, d, grid, tile, window, pool)
    check = [(b, h) for b in range(batch) for h in range(heads)]
    g = O.geom_of(w)
    out = _dual_gpu(V, w, check, saved=True)
    _check_dual(w, out, check, range(math.prod(g.tiles_per_dim)))
    out2 = _dual_gpu(V, w, check, saved=False)
    import torch
    assert torch.equal(out2["O"], out["O"])


def test_dual_fwd_1080p_sampled(V):
    w = S.WORKLOADS["1080p"]
    check = [(0, 0), (0, w.heads - 1)]
    out = _dual_gpu(V, w, check, saved=True)
    _check_dual(w, out, check, sample_tiles(O.geom_of(w).tiles_per_dim, 6))


def test_dual_fwd_4k_sampled(V):
    """The 4K-shaped launch with its saved outputs.  Every head from 12 on
    starts past byte 2^31 of every [B, h, N, d] bf16 tensor, and the last
    query tiles of head 23 lie past element 2^31 (23 * 725760 * 128 + 725759 *
    128 > 2^31), so they are addressed only through 64-bit offsets: O, O_l,
    O_g, LSE_l and LSE_g of heads 0 and 23 are compared on query tiles
    covering every boundary class, the last tiles included."""
    w = S.WORKLOADS["4k"]
    check = [(0, 0), (0, w.heads - 1)]
    assert 12 * w.n_tokens * w.head_dim * 2 > 2 ** 31
    assert ((w.heads - 1) * w.n_tokens + w.n_tokens - 1) * w.head_dim > 2 ** 31
    out = _dual_gpu(V, w, check, saved=True)
    _check_dual(w, out, check, sample_tiles(O.geom_of(w).tiles_per_dim, 4))


def _global_gpu(V, w, check, kp_bits, vp_bits):
    """vattn_global_fwd on raster Q (the global branch has no tile order: every
    query sees every pooled key) and host-pooled K_p, V_p given as bf16 bits
    [B, h, N_p, d]."""
    import torch
    from helpers import bits_to_gpu
    geom = geom_for(V, w)
    q = gpu_tensor(w, S.Q_ID, check)
    kp, vp = bits_to_gpu(kp_bits), bits_to_gpu(vp_bits)
    o = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device="cuda")
    V.vattn_global_fwd(geom, q, kp, vp, 1 / math.sqrt(w.head_dim), o, lse)
    torch.cuda.synchronize()
    assert V.vattn_get_status() == 0, V.vattn_last_error()
    return o, lse


@pytest.mark.parametrize("grid,tile,pool,d,batch,heads", [
    ((3, 20, 24), (3, 4, 4), (1, 2, 2), 128, 2, 3),   # N = 1440, N_p = 360: both ragged against 128
    ((4, 8, 24), (2, 4, 4), (2, 4, 3), 64, 1, 2),     # temporal pooling, N_p = 32 (one partial key block)
    ((2, 8, 16), (1, 4, 4), (1, 1, 1), 128, 1, 2),    # pool 1: the global branch is full attention
])
def test_global_fwd_direct(V, grid, tile, pool, d, batch, heads):
    """vattn_global_fwd called on its own, with K_p and V_p pooled on the host
    (the exact block mean rounded to bf16), against the oracle's dense softmax
    attention over those pooled keys; with pool 1 also against full attention
    over the unpooled K, V."""
    w = S.small_workload("global", 17, batch, heads, d, grid, tile, (1, 1, 1), pool)
    g = O.geom_of(w)
    check = [(b, h) for b in range(batch) for h in range(heads)]
    kp_bits = np.empty((batch, heads, g.n_pooled, d), dtype=np.uint16)
    vp_bits = np.empty_like(kp_bits)
    for b, h in check:
        kp_bits[b, h] = S.bf16_round_bits(O.pool(host_f64(w, S.K_ID, b, h), g).astype(np.float32))
        vp_bits[b, h] = S.bf16_round_bits(O.pool(host_f64(w, S.V_ID, b, h), g).astype(np.float32))
    o, lse = _global_gpu(V, w, check, kp_bits, vp_bits)
    scale = 1 / math.sqrt(d)
    for b, h in check:
        q = host_f64(w, S.Q_ID, b, h)
        kp, vp = S.bf16_bits_to_f64(kp_bits[b, h]), S.bf16_bits_to_f64(vp_bits[b, h])
        o_ref, lse_ref = O.global_attention(q[None, None], kp[None, None], vp[None, None], scale)
        assert_close(to_f64(o[b, h]), o_ref[0, 0], O_MAX_ABS, O_MEAN_ABS, f"O b{b} h{h}")
        assert_close(lse[b, h].cpu().numpy().astype(np.float64), lse_ref[0, 0], LSE_MAX_ABS, what=f"LSE b{b} h{h}")
        if pool == (1, 1, 1):
            k, v = host_f64(w, S.K_ID, b, h), host_f64(w, S.V_ID, b, h)
            o_full, lse_full = O.full_attention(q[None, None], k[None, None], v[None, None], scale)
            assert_close(to_f64(o[b, h]), o_full[0, 0], O_MAX_ABS, O_MEAN_ABS, f"full O b{b} h{h}")
            assert_close(lse[b, h].cpu().numpy().astype(np.float64), lse_full[0, 0], LSE_MAX_ABS,
                         what=f"full LSE b{b} h{h}")


# ------------------------------------------------------------------ failure detection

def test_device_timeout_is_reported_and_context_survives(V):
    """The load warp skips its first arrival (test hook); the MMA warp's
    bounded wait runs out, the kernel records the timeout and returns; the
    context stays usable and the next call is correct."""
    import torch
    w = S.WORKLOADS["tiny"]
    geom = geom_for(V, w)
    q = torch.zeros((1, 2, w.n_tokens, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    V.vattn_debug_set(1, 200_000_000)
    try:
        V.vattn_sta_fwd(geom, q, q, q, 0.125, o)
        st = V.vattn_get_status()
    finally:
        V.vattn_debug_set(0, 0)
    assert st == V.binding.VATTN_ERR_DEVICE_TIMEOUT
    assert V.vattn_get_status() == 0
    check = [(0, 0), (0, 1)]
    o_r, lse_r = _sta_gpu(V, w, check)
    _check_sta(w, o_r, lse_r, check, range(8))


def test_polynomial_exp2_against_cuda_exp2f(V):
    """The FMA-pipe 2^x that the forward can run for one chunk of its
    exponentials (a compile-time option, off in the default build) against
    CUDA's exp2f (torch.exp2): relative error <= 1e-4 on the range the forward
    feeds it (x <= 8); at or below the clamp the result is tiny."""
    import torch
    x = torch.cat([torch.linspace(-124.0, 8.0, 1 << 20, device="cuda"),
                   torch.rand(1 << 20, device="cuda") * 16 - 8]).contiguous()
    y = torch.empty_like(x)
    V.vattn_debug_exp2(x, y)
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref).abs() / ref).max().item()
    assert rel <= 1e-4, rel
    z = torch.tensor([-float("inf"), -1e30, -300.0, -126.0], device="cuda")
    yz = torch.empty_like(z)
    V.vattn_debug_exp2(z, yz)
    assert (yz >= 0).all() and (yz <= 2.0 ** -124).all()
