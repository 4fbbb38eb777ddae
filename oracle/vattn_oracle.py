"""Plain fp64 definitions of every result on the attention hot path.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module.  All arrays are float64 NumPy; inputs arrive as exact
float64 copies of bfloat16 values, in RASTER token order
(token n = (t*H + y)*W + x), shaped [B, heads, N, d].

Readings taken where the pages leave a step open (each one is also listed in
the design notes):
  * window start: start = clamp(a - floor(w/2), 0, max(N_tiles - w, 0)),
    extent = min(w, N_tiles); a clamped window always keeps prod(min(w, N))
    tiles ("Fast Video Generation with Sliding Tile Attention", abstract,
    tile-by-tile sliding window; the clamp is the plainest reading that keeps
    every query tile's window fully inside the grid);
  * tile order and intra-tile order are both raster, t-major, w fastest;
  * only K and V are pooled (average over p_t x p_h x p_w token blocks); the
    queries keep full resolution ("AtlasVid ...", abstract, asymmetric
    global-local attention; "UltraGen ..." §4.2, compressed global modelling);
  * the fusion factor of "UltraGen ..." §4.1 is a given per-head g in [0, 1]:
    O = g * O_local + (1 - g) * O_global;
  * LSE is the natural log of the softmax denominator, scale included.

Parity: pinned by invariants, brute force and finite differences in
tests/test_oracle.py; the pages print no worked numeric example.
"""
from __future__ import annotations

import math
from typing import NamedTuple

import numpy as np


class Geom(NamedTuple):
    """Latent grid (T, H, W), tile, window (in tiles) and pool sizes, (t, h, w) order."""
    T: int
    H: int
    W: int
    tile: tuple
    window: tuple
    pool: tuple = (1, 1, 1)

    @property
    def n(self) -> int:
        return self.T * self.H * self.W

    @property
    def tiles_per_dim(self) -> tuple:
        return (self.T // self.tile[0], self.H // self.tile[1], self.W // self.tile[2])

    @property
    def tile_volume(self) -> int:
        return self.tile[0] * self.tile[1] * self.tile[2]

    @property
    def pooled_dims(self) -> tuple:
        return (self.T // self.pool[0], self.H // self.pool[1], self.W // self.pool[2])

    @property
    def n_pooled(self) -> int:
        a, b, c = self.pooled_dims
        return a * b * c


def geom_of(workload) -> Geom:
    T, H, W = workload.grid
    return Geom(T, H, W, tuple(workload.tile), tuple(workload.window), tuple(workload.pool))


# ---------------------------------------------------------------------------
# a1: raster <-> tile-major reorder ("AtlasVid ...", abstract: reordered
# spatiotemporal windows; "Fast Video Generation with Sliding Tile Attention",
# abstract: tile-by-tile operation)
# ---------------------------------------------------------------------------

def token_coords(g: Geom) -> np.ndarray:
    """[N, 3] (t, y, x) of every raster token."""
    n = np.arange(g.n)
    x = n % g.W
    y = (n // g.W) % g.H
    t = n // (g.W * g.H)
    return np.stack([t, y, x], axis=1)


def tile_major_index(g: Geom) -> np.ndarray:
    """m[n] = tile-major position of raster token n:
    m = tile_id * s + local_id, tile_id = ((t/t_t)*N_h + y/t_h)*N_w + x/t_w,
    local_id = ((t%t_t)*t_h + y%t_h)*t_w + x%t_w."""
    tt, th, tw = g.tile
    _, nh, nw = g.tiles_per_dim
    c = token_coords(g)
    t, y, x = c[:, 0], c[:, 1], c[:, 2]
    tile_id = ((t // tt) * nh + y // th) * nw + x // tw
    local = ((t % tt) * th + y % th) * tw + x % tw
    return tile_id * g.tile_volume + local


def permute(x_raster: np.ndarray, g: Geom) -> np.ndarray:
    """Raster -> tile-major along axis -2 (a pure row gather)."""
    m = tile_major_index(g)
    out = np.empty_like(x_raster)
    out[..., m, :] = x_raster
    return out


def unpermute(x_tiled: np.ndarray, g: Geom) -> np.ndarray:
    """Tile-major -> raster along axis -2."""
    m = tile_major_index(g)
    return x_tiled[..., m, :]


# ---------------------------------------------------------------------------
# a2: kept-tile list ("Fast Video Generation with Sliding Tile Attention",
# abstract: each query tile attends to a 3D window of tiles around it)
# ---------------------------------------------------------------------------

def window_range(a: int, w: int, n: int) -> range:
    """Tiles kept along one dim for query tile coordinate a: the window of
    min(w, n) tiles centred on a and shifted inward at the grid boundary."""
    ext = min(w, n)
    start = min(max(a - w // 2, 0), max(n - w, 0))
    return range(start, start + ext)


def kept_tiles(g: Geom) -> np.ndarray:
    """[n_tiles, kept] int32: for every query tile (tile-major id order) the ids
    of its kept key tiles, t outermost, w fastest."""
    nt, nh, nw = g.tiles_per_dim
    rows = []
    for at in range(nt):
        for ah in range(nh):
            for aw in range(nw):
                ids = [(kt * nh + kh) * nw + kw
                       for kt in window_range(at, g.window[0], nt)
                       for kh in window_range(ah, g.window[1], nh)
                       for kw in window_range(aw, g.window[2], nw)]
                rows.append(ids)
    return np.asarray(rows, dtype=np.int32)


def kept_count_closed_form(g: Geom) -> int:
    return math.prod(min(w, n) for w, n in zip(g.window, g.tiles_per_dim))


def _tile_token_box(g: Geom, lo: tuple, hi: tuple) -> np.ndarray:
    """Raster ids of all tokens with tile coordinates in [lo, hi) per dim."""
    tt, th, tw = g.tile
    ts = np.arange(lo[0] * tt, hi[0] * tt)
    ys = np.arange(lo[1] * th, hi[1] * th)
    xs = np.arange(lo[2] * tw, hi[2] * tw)
    return ((ts[:, None, None] * g.H + ys[None, :, None]) * g.W + xs[None, None, :]).reshape(-1)


# ---------------------------------------------------------------------------
# softmax attention over an explicit key set (the definition of "UltraGen ..."
# §3: S = q k^T * scale, softmax over keys, O = P V)
# ---------------------------------------------------------------------------

def _softmax_attend(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    s = (q @ k.T) * scale
    mx = s.max(axis=1, keepdims=True)
    e = np.exp(s - mx)
    den = e.sum(axis=1, keepdims=True)
    p = e / den
    return p @ v, (mx + np.log(den))[:, 0], p


def full_attention(q, k, v, scale):
    """Dense softmax attention over all keys; [B,h,N,d] -> (O, LSE)."""
    B, nh, n, d = q.shape
    o = np.empty_like(q)
    lse = np.empty((B, nh, n))
    for b in range(B):
        for h in range(nh):
            o[b, h], lse[b, h], _ = _softmax_attend(q[b, h], k[b, h], v[b, h], scale)
    return o, lse


# ---------------------------------------------------------------------------
# a3: sliding-tile (local) attention
# ---------------------------------------------------------------------------

def _query_tiles(g: Geom):
    """Yield (query token ids, key token ids) per query tile, both raster."""
    nt, nh, nw = g.tiles_per_dim
    for at in range(nt):
        for ah in range(nh):
            for aw in range(nw):
                qi = _tile_token_box(g, (at, ah, aw), (at + 1, ah + 1, aw + 1))
                rt = window_range(at, g.window[0], nt)
                rh = window_range(ah, g.window[1], nh)
                rw = window_range(aw, g.window[2], nw)
                kj = _tile_token_box(g, (rt.start, rh.start, rw.start), (rt.stop, rh.stop, rw.stop))
                yield qi, kj


def sta_attention(q, k, v, g: Geom, scale: float):
    """Local branch: every query attends only to the tokens of its query tile's
    kept tiles.  Raster in, raster out: (O [B,h,N,d], LSE [B,h,N])."""
    B, nh, n, d = q.shape
    o = np.empty_like(q)
    lse = np.empty((B, nh, n))
    for b in range(B):
        for h in range(nh):
            for qi, kj in _query_tiles(g):
                o[b, h, qi], lse[b, h, qi], _ = _softmax_attend(q[b, h, qi], k[b, h, kj], v[b, h, kj], scale)
    return o, lse


def sta_mask_bruteforce(g: Geom) -> np.ndarray:
    """[N, N] bool, built token by token: key j is visible to query i iff j's
    tile lies in the clamped window of i's tile along every dim."""
    c = token_coords(g)
    tc = c // np.asarray(g.tile)
    dims = g.tiles_per_dim
    mask = np.ones((g.n, g.n), dtype=bool)
    for ax in range(3):
        w, nd = g.window[ax], dims[ax]
        start = np.array([window_range(a, w, nd).start for a in range(nd)])
        ext = min(w, nd)
        s_i = start[tc[:, ax]][:, None]
        mask &= (tc[None, :, ax] >= s_i) & (tc[None, :, ax] < s_i + ext)
    return mask


def sta_attention_bruteforce(q, k, v, g: Geom, scale: float):
    """Local branch as a masked dense softmax (tiny grids only)."""
    mask = sta_mask_bruteforce(g)
    B, nh, n, d = q.shape
    o = np.empty_like(q)
    lse = np.empty((B, nh, n))
    for b in range(B):
        for h in range(nh):
            s = (q[b, h] @ k[b, h].T) * scale
            s = np.where(mask, s, -np.inf)
            mx = s.max(axis=1, keepdims=True)
            e = np.exp(s - mx)
            den = e.sum(axis=1, keepdims=True)
            o[b, h] = (e / den) @ v[b, h]
            lse[b, h] = (mx + np.log(den))[:, 0]
    return o, lse


# ---------------------------------------------------------------------------
# a4: K/V average pooling ("UltraGen ..." §4.2: downsample before global
# attention, fewer spatial tokens; the spec form is average pooling)
# ---------------------------------------------------------------------------

def pooled_index(g: Geom) -> np.ndarray:
    """u[n] = pooled-raster id of the block containing raster token n."""
    pt, ph, pw = g.pool
    _, PH, PW = g.pooled_dims
    c = token_coords(g)
    return ((c[:, 0] // pt) * PH + c[:, 1] // ph) * PW + c[:, 2] // pw


def pool(x_raster: np.ndarray, g: Geom) -> np.ndarray:
    """Exact fp64 mean over every p_t x p_h x p_w block; [..., N, d] -> [..., N_p, d]."""
    u = pooled_index(g)
    cnt = g.pool[0] * g.pool[1] * g.pool[2]
    # group the tokens of each block together (every block has cnt tokens),
    # then sum each group
    order = np.argsort(u, kind="stable")
    d = x_raster.shape[-1]
    grouped = x_raster[..., order, :].reshape(x_raster.shape[:-2] + (g.n_pooled, cnt, d))
    return grouped.sum(axis=-2) / cnt


def pool_transpose(y_pooled: np.ndarray, g: Geom) -> np.ndarray:
    """Adjoint of pool: x[n] = y[u(n)] / count."""
    cnt = g.pool[0] * g.pool[1] * g.pool[2]
    return y_pooled[..., pooled_index(g), :] / cnt


# ---------------------------------------------------------------------------
# a5/a6: global branch and blend ("UltraGen ..." §4.1, §4.2)
# ---------------------------------------------------------------------------

def global_attention(q, kp, vp, scale):
    """Every full-resolution query attends to all pooled keys."""
    return full_attention(q, kp, vp, scale)


def dual_forward(q, k, v, gvec, g: Geom, scale: float):
    """Returns dict with O, O_l, LSE_l, O_g, LSE_g, K_p, V_p (all raster)."""
    o_l, lse_l = sta_attention(q, k, v, g, scale)
    kp, vp = pool(k, g), pool(v, g)
    o_g, lse_g = global_attention(q, kp, vp, scale)
    gb = np.asarray(gvec, dtype=np.float64)[None, :, None, None]
    o = gb * o_l + (1.0 - gb) * o_g
    return dict(O=o, O_l=o_l, LSE_l=lse_l, O_g=o_g, LSE_g=lse_g, K_p=kp, V_p=vp)


# ---------------------------------------------------------------------------
# a7: backward, restated from the softmax Jacobian (no saved-statistics split)
# ---------------------------------------------------------------------------

def _softmax_attend_bwd(q, k, v, do, scale):
    """Gradients of O = softmax(q k^T scale) v w.r.t. q, k, v for upstream do."""
    _, _, p = _softmax_attend(q, k, v, scale)
    dv = p.T @ do
    dp = do @ v.T
    # dS_ij = sum_l dP_il * dP_il/dS_ij with dP/dS the softmax Jacobian
    # diag(p) - p p^T per row.
    ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
    dq = scale * (ds @ k)
    dk = scale * (ds.T @ q)
    return dq, dk, dv


def sta_backward(q, k, v, do, g: Geom, scale: float):
    """Local-branch gradients (raster)."""
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    B, nh = q.shape[:2]
    for b in range(B):
        for h in range(nh):
            for qi, kj in _query_tiles(g):
                a, bk, c = _softmax_attend_bwd(q[b, h, qi], k[b, h, kj], v[b, h, kj], do[b, h, qi], scale)
                dq[b, h, qi] += a
                dk[b, h, kj] += bk
                dv[b, h, kj] += c
    return dq, dk, dv


def global_backward(q, kp, vp, do, scale):
    """Global-branch gradients w.r.t. q and the pooled k_p, v_p."""
    dq = np.zeros_like(q)
    dkp = np.zeros_like(kp)
    dvp = np.zeros_like(vp)
    B, nh = q.shape[:2]
    for b in range(B):
        for h in range(nh):
            dq[b, h], dkp[b, h], dvp[b, h] = _softmax_attend_bwd(q[b, h], kp[b, h], vp[b, h], do[b, h], scale)
    return dq, dkp, dvp


def dual_backward(q, k, v, gvec, do, g: Geom, scale: float):
    """Gradients of the blended output w.r.t. q, k, v (through the pooling) and g.

    O = g O_l + (1-g) O_g  =>  branch upstream gradients g*dO and (1-g)*dO;
    dK = dK_l + pool^T(dK_p), dV likewise; dg_h = sum_{b,n} dO . (O_l - O_g).
    """
    gb = np.asarray(gvec, dtype=np.float64)[None, :, None, None]
    dq_l, dk_l, dv_l = sta_backward(q, k, v, gb * do, g, scale)
    kp, vp = pool(k, g), pool(v, g)
    dq_g, dkp, dvp = global_backward(q, kp, vp, (1.0 - gb) * do, scale)
    o_l, _ = sta_attention(q, k, v, g, scale)
    o_g, _ = global_attention(q, kp, vp, scale)
    dg = (do * (o_l - o_g)).sum(axis=(0, 2, 3))
    return dict(dQ=dq_l + dq_g, dK=dk_l + pool_transpose(dkp, g), dV=dv_l + pool_transpose(dvp, g),
                dK_p=dkp, dV_p=dvp, dg=dg, dQ_l=dq_l, dQ_g=dq_g)


# ---------------------------------------------------------------------------
# work accounting ("UltraGen ..." App. B complexity model; effective FLOPs)
# ---------------------------------------------------------------------------

def kept_pairs_local(g: Geom, batch: int, heads: int) -> int:
    """Query-key pairs the local branch computes: every query sees kept*s keys."""
    return batch * heads * g.n * kept_count_closed_form(g) * g.tile_volume


def pairs_global(g: Geom, batch: int, heads: int) -> int:
    return batch * heads * g.n * g.n_pooled


def ultragen_cost_ratio(K: int) -> float:
    """App. B of "UltraGen ...": (5/(4K^2) + 1/K^4) of full attention's cost."""
    return 5.0 / (4.0 * K * K) + 1.0 / K ** 4


# ---------------------------------------------------------------------------
# sampled evaluation (large grids): the same definitions restricted to a few
# query tiles / rows of one (batch, head) slice
# ---------------------------------------------------------------------------

def tile_coords_of(g: Geom, tile_id: int) -> tuple:
    nt, nh, nw = g.tiles_per_dim
    return (tile_id // (nh * nw), (tile_id // nw) % nh, tile_id % nw)


def sta_attention_tiles(q, k, v, g: Geom, scale: float, tile_ids):
    """Local branch for the listed query tiles of one head ([N, d] raster
    inputs).  Returns (raster query ids, O [n, d], LSE [n]) concatenated over
    the tiles in the given order."""
    nt, nh, nw = g.tiles_per_dim
    ids, outs, lses = [], [], []
    for tid in tile_ids:
        at, ah, aw = tile_coords_of(g, int(tid))
        qi = _tile_token_box(g, (at, ah, aw), (at + 1, ah + 1, aw + 1))
        rt = window_range(at, g.window[0], nt)
        rh = window_range(ah, g.window[1], nh)
        rw = window_range(aw, g.window[2], nw)
        kj = _tile_token_box(g, (rt.start, rh.start, rw.start), (rt.stop, rh.stop, rw.stop))
        o, lse, _ = _softmax_attend(q[qi], k[kj], v[kj], scale)
        ids.append(qi)
        outs.append(o)
        lses.append(lse)
    return np.concatenate(ids), np.concatenate(outs), np.concatenate(lses)


def global_attention_rows(q, kp, vp, scale: float, rows):
    """Global branch for the listed raster query rows of one head."""
    o, lse, _ = _softmax_attend(q[np.asarray(rows)], kp, vp, scale)
    return o, lse


def dual_backward_sampled(q, k, v, gval: float, do, g: Geom, scale: float, q_tiles, k_tiles, chunk: int = 8192,
                          symmetric: bool = False):
    """dual_backward (or, with symmetric=True, dual_sym_backward) for one head
    ([N, d] raster inputs) restricted to the tokens of `q_tiles` (dQ) and of
    `k_tiles` (dK, dV).  Every softmax row it uses is the full row of the
    definition; only the outputs are restricted.

    Returns dict(q_ids, dQ, k_ids, dK, dV) with rows in the order of the ids.
    """
    nt, nh, nw = g.tiles_per_dim
    gl, gg = float(gval), 1.0 - float(gval)

    def window_ids(tid):
        at, ah, aw = tile_coords_of(g, int(tid))
        rt = window_range(at, g.window[0], nt)
        rh = window_range(ah, g.window[1], nh)
        rw = window_range(aw, g.window[2], nw)
        qi = _tile_token_box(g, (at, ah, aw), (at + 1, ah + 1, aw + 1))
        kj = _tile_token_box(g, (rt.start, rh.start, rw.start), (rt.stop, rh.stop, rw.stop))
        return qi, kj

    kp, vp = pool(k, g), pool(v, g)
    u_all = pooled_index(g)
    cnt = g.pool[0] * g.pool[1] * g.pool[2]
    if symmetric:
        # the pooled branch is small: its gradients are computed in full
        qp = pool(q, g)
        do_p = upsample_transpose(gg * do, g)
        dqp, dkp_s, dvp_s = _softmax_attend_bwd(qp, kp, vp, do_p, scale)
    # dQ rows: local branch of the query tile, global branch of the same rows
    q_ids, dq_rows = [], []
    for tid in q_tiles:
        qi, kj = window_ids(tid)
        dq_l, _, _ = _softmax_attend_bwd(q[qi], k[kj], v[kj], gl * do[qi], scale)
        if symmetric:
            dq_g = dqp[u_all[qi]] / cnt
        else:
            dq_g, _, _ = _softmax_attend_bwd(q[qi], kp, vp, gg * do[qi], scale)
        q_ids.append(qi)
        dq_rows.append(dq_l + dq_g)
    # dK/dV rows, local branch: every query tile whose window holds the key tile
    k_ids = [_tile_token_box(g, tile_coords_of(g, int(t)), tuple(c + 1 for c in tile_coords_of(g, int(t))))
             for t in k_tiles]
    want = np.concatenate(k_ids)
    pos = {int(t): i for i, t in enumerate(want)}
    dk = np.zeros((len(want), q.shape[1]))
    dv = np.zeros_like(dk)
    kept = kept_tiles(g)
    wanted_tiles = set(int(t) for t in k_tiles)
    for a in range(kept.shape[0]):
        if not wanted_tiles.intersection(int(x) for x in kept[a]):
            continue
        qi, kj = window_ids(a)
        _, dk_a, dv_a = _softmax_attend_bwd(q[qi], k[kj], v[kj], gl * do[qi], scale)
        for col, tok in enumerate(kj):
            r = pos.get(int(tok))
            if r is not None:
                dk[r] += dk_a[col]
                dv[r] += dv_a[col]
    if symmetric:
        dk += dkp_s[u_all[want]] / cnt
        dv += dvp_s[u_all[want]] / cnt
        return dict(q_ids=np.concatenate(q_ids), dQ=np.concatenate(dq_rows), k_ids=want, dK=dk, dV=dv)
    # pooled branch: dK_p, dV_p at the pool blocks of the wanted tokens, summed
    # over every query (row chunks of the full softmax)
    cols = np.unique(u_all[want])
    dkp = np.zeros((len(cols), q.shape[1]))
    dvp = np.zeros_like(dkp)
    for r0 in range(0, g.n, chunk):
        qc, doc = q[r0:r0 + chunk], gg * do[r0:r0 + chunk]
        s = (qc @ kp.T) * scale
        mx = s.max(axis=1, keepdims=True)
        e = np.exp(s - mx)
        p = e / e.sum(axis=1, keepdims=True)
        dp = doc @ vp.T
        row = (p * dp).sum(axis=1, keepdims=True)
        pc = p[:, cols]
        ds = pc * (dp[:, cols] - row)
        dvp += pc.T @ doc
        dkp += scale * (ds.T @ qc)
    cidx = {int(c): i for i, c in enumerate(cols)}
    for r, tok in enumerate(want):
        c = cidx[int(u_all[tok])]
        dk[r] += dkp[c] / cnt
        dv[r] += dvp[c] / cnt
    return dict(q_ids=np.concatenate(q_ids), dQ=np.concatenate(dq_rows), k_ids=want, dK=dk, dV=dv)


# ---------------------------------------------------------------------------
# cross-window local attention ("UltraGen ..." §4.3: window partitions that
# alternate between adjacent layers, K x K windows and shifted (K+1) x (K+1)
# partitions).  Reading taken: along each dim the tile grid is cut into
# consecutive blocks; mode "partition" uses blocks of `window` tiles starting
# at tile 0, mode "shifted" uses blocks of `window + 1` tiles whose cuts are
# moved by floor((window + 1) / 2); blocks at the grid edge are truncated.  A
# query tile attends to every tile of its own block (in all three dims).
# ---------------------------------------------------------------------------

def partition_range(a: int, w: int, n: int, shifted: bool) -> range:
    """Tiles of the block holding tile a along one dim."""
    size = w + 1 if shifted else w
    off = (w + 1) // 2 if shifted else 0
    b = (a + off) // size
    lo = max(b * size - off, 0)
    hi = min((b + 1) * size - off, n)
    return range(lo, hi)


def xwin_query_tiles(g: Geom, shifted: bool):
    """Yield (query token ids, key token ids) per query tile, both raster."""
    nt, nh, nw = g.tiles_per_dim
    for at in range(nt):
        for ah in range(nh):
            for aw in range(nw):
                qi = _tile_token_box(g, (at, ah, aw), (at + 1, ah + 1, aw + 1))
                rt = partition_range(at, g.window[0], nt, shifted)
                rh = partition_range(ah, g.window[1], nh, shifted)
                rw = partition_range(aw, g.window[2], nw, shifted)
                kj = _tile_token_box(g, (rt.start, rh.start, rw.start), (rt.stop, rh.stop, rw.stop))
                yield qi, kj


def xwin_attention(q, k, v, g: Geom, scale: float, shifted: bool):
    """Cross-window local attention: raster in, raster out (O, LSE)."""
    B, nh, n, d = q.shape
    o = np.empty_like(q)
    lse = np.empty((B, nh, n))
    for b in range(B):
        for h in range(nh):
            for qi, kj in xwin_query_tiles(g, shifted):
                o[b, h, qi], lse[b, h, qi], _ = _softmax_attend(q[b, h, qi], k[b, h, kj], v[b, h, kj], scale)
    return o, lse


def xwin_backward(q, k, v, do, g: Geom, scale: float, shifted: bool):
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    B, nh = q.shape[:2]
    for b in range(B):
        for h in range(nh):
            for qi, kj in xwin_query_tiles(g, shifted):
                a, bk, c = _softmax_attend_bwd(q[b, h, qi], k[b, h, kj], v[b, h, kj], do[b, h, qi], scale)
                dq[b, h, qi] += a
                dk[b, h, kj] += bk
                dv[b, h, kj] += c
    return dq, dk, dv


# ---------------------------------------------------------------------------
# symmetric compressed global branch ("UltraGen ..." §4.2: latents are
# downsampled before global attention and restored afterwards by upsampling).
# Reading taken: queries, keys and values are all average-pooled; the pooled
# queries attend to all pooled keys; the result is brought back to the full
# grid by separable linear interpolation along t, y and x with half-pixel
# centres (source coordinate (i + 1/2) / p - 1/2, clamped to the pooled grid at
# the edges).  The learned convolutions of the pages need trained weights and
# are not part of this definition.
# ---------------------------------------------------------------------------

def _interp_weights(n_out: int, n_in: int, p: int) -> np.ndarray:
    """[n_out, n_in] linear interpolation matrix along one dim."""
    m = np.zeros((n_out, n_in))
    for i in range(n_out):
        src = (i + 0.5) / p - 0.5
        src = min(max(src, 0.0), n_in - 1.0)
        i0 = int(math.floor(src))
        i1 = min(i0 + 1, n_in - 1)
        f = src - i0
        m[i, i0] += 1.0 - f
        m[i, i1] += f
    return m


def upsample(x_pooled: np.ndarray, g: Geom) -> np.ndarray:
    """Pooled-raster [..., N_p, d] -> raster [..., N, d] by the separable
    interpolation above."""
    PT, PH, PW = g.pooled_dims
    lead = x_pooled.shape[:-2]
    d = x_pooled.shape[-1]
    x = x_pooled.reshape(lead + (PT, PH, PW, d))
    mt = _interp_weights(g.T, PT, g.pool[0])
    mh = _interp_weights(g.H, PH, g.pool[1])
    mw = _interp_weights(g.W, PW, g.pool[2])
    y = np.einsum("tT,...THWd->...tHWd", mt, x)
    y = np.einsum("hH,...tHWd->...thWd", mh, y)
    y = np.einsum("wW,...thWd->...thwd", mw, y)
    return y.reshape(lead + (g.n, d))


def upsample_transpose(y: np.ndarray, g: Geom) -> np.ndarray:
    """Adjoint of upsample: raster [..., N, d] -> pooled-raster [..., N_p, d]."""
    PT, PH, PW = g.pooled_dims
    lead = y.shape[:-2]
    d = y.shape[-1]
    z = y.reshape(lead + (g.T, g.H, g.W, d))
    mt = _interp_weights(g.T, PT, g.pool[0])
    mh = _interp_weights(g.H, PH, g.pool[1])
    mw = _interp_weights(g.W, PW, g.pool[2])
    z = np.einsum("tT,...thwd->...Thwd", mt, z)
    z = np.einsum("hH,...Thwd->...THwd", mh, z)
    z = np.einsum("wW,...THwd->...THWd", mw, z)
    return z.reshape(lead + (g.n_pooled, d))


def global_sym_forward(q, k, v, g: Geom, scale: float):
    """Symmetric global branch: (O_g [raster, full grid], O_p, LSE_p [pooled])."""
    qp, kp, vp = pool(q, g), pool(k, g), pool(v, g)
    o_p, lse_p = full_attention(qp, kp, vp, scale)
    return upsample(o_p, g), o_p, lse_p


def dual_sym_forward(q, k, v, gvec, g: Geom, scale: float):
    o_l, lse_l = sta_attention(q, k, v, g, scale)
    o_g, o_p, lse_p = global_sym_forward(q, k, v, g, scale)
    gb = np.asarray(gvec, dtype=np.float64)[None, :, None, None]
    return dict(O=gb * o_l + (1.0 - gb) * o_g, O_l=o_l, LSE_l=lse_l, O_p=o_p, LSE_p=lse_p)


def dual_sym_backward(q, k, v, gvec, do, g: Geom, scale: float):
    """Gradients of g*O_l + (1-g)*upsample(attn(pool q, pool k, pool v))."""
    gb = np.asarray(gvec, dtype=np.float64)[None, :, None, None]
    dq_l, dk_l, dv_l = sta_backward(q, k, v, gb * do, g, scale)
    qp, kp, vp = pool(q, g), pool(k, g), pool(v, g)
    do_p = upsample_transpose((1.0 - gb) * do, g)
    dqp, dkp, dvp = global_backward(qp, kp, vp, do_p, scale)
    return dict(dQ=dq_l + pool_transpose(dqp, g), dK=dk_l + pool_transpose(dkp, g),
                dV=dv_l + pool_transpose(dvp, g), dQ_p=dqp, dK_p=dkp, dV_p=dvp)


# ---------------------------------------------------------------------------
# symmetric global branch, learned variant ("UltraGen ..." §4.2: the latents
# are compressed by a depthwise convolution of stride k before global
# attention; after it, bilinear upsampling and a 3D convolution restore the
# full grid, processing space and time jointly).  Readings taken: the
# compression kernel equals its stride (p_t x p_h x p_w taps, non-overlapping,
# no bias), one kernel per head and channel, applied to Q, K and V with
# separate weights; the restoring convolution is depthwise as well, 3 x 3 x 3
# with zero padding (output on the full grid), no bias, applied to the
# upsampled global output before the blend; convolution means
# cross-correlation (out[t] = sum_a w[a] x[t + a]).  The weights are inputs:
# the method's trained values are not available, so tests draw them at random.
# ---------------------------------------------------------------------------

def conv_compress(x_raster: np.ndarray, g: Geom, w: np.ndarray) -> np.ndarray:
    """Depthwise strided convolution; x [B, h, N, d] raster, w [h, P, d] with
    the P = p_t*p_h*p_w taps in (dt, dy, dx) raster order:
    x_p[t', y', x', c] = sum_taps w[h, tap, c] * x[t' p_t + dt, y' p_h + dy, x' p_w + dx, c]."""
    PT, PH, PW = g.pooled_dims
    pt, ph, pw = g.pool
    B, nh, _, d = x_raster.shape
    x = x_raster.reshape(B, nh, PT, pt, PH, ph, PW, pw, d)
    wr = np.asarray(w, dtype=np.float64).reshape(nh, pt, ph, pw, d)
    y = np.einsum("bhTiHjWkd,hijkd->bhTHWd", x, wr)
    return y.reshape(B, nh, g.n_pooled, d)


def conv3d_depthwise(x_raster: np.ndarray, g: Geom, w3: np.ndarray) -> np.ndarray:
    """3 x 3 x 3 depthwise convolution with zero padding on the full grid;
    x [B, h, N, d] raster, w3 [h, 27, d] with taps (a, b, e) in {-1, 0, 1}^3,
    raster order: y[t, y, x, c] = sum w3[h, tap, c] * x[t + a, y + b, x + e, c]."""
    B, nh, _, d = x_raster.shape
    x = x_raster.reshape(B, nh, g.T, g.H, g.W, d)
    xp = np.zeros((B, nh, g.T + 2, g.H + 2, g.W + 2, d))
    xp[:, :, 1:-1, 1:-1, 1:-1, :] = x
    w = np.asarray(w3, dtype=np.float64)
    y = np.zeros_like(x)
    tap = 0
    for a in (-1, 0, 1):
        for b in (-1, 0, 1):
            for e in (-1, 0, 1):
                y += w[None, :, tap, None, None, None, :] * xp[:, :, 1 + a:1 + a + g.T, 1 + b:1 + b + g.H,
                                                                1 + e:1 + e + g.W, :]
                tap += 1
    return y.reshape(B, nh, g.n, d)


def dual_sym_learned_forward(q, k, v, gvec, wq, wk, wv, w3, g: Geom, scale: float):
    """Blend of the local branch and the learned compressed global branch
    (raster in, raster out): O_g = conv3d(upsample(attn(cq(Q), ck(K), cv(V))))."""
    o_l, lse_l = sta_attention(q, k, v, g, scale)
    qp, kp, vp = conv_compress(q, g, wq), conv_compress(k, g, wk), conv_compress(v, g, wv)
    o_p, lse_p = full_attention(qp, kp, vp, scale)
    o_g = conv3d_depthwise(upsample(o_p, g), g, w3)
    gb = np.asarray(gvec, dtype=np.float64)[None, :, None, None]
    return dict(O=gb * o_l + (1.0 - gb) * o_g, O_l=o_l, LSE_l=lse_l, Q_p=qp, K_p=kp, V_p=vp, O_p=o_p,
                LSE_p=lse_p, O_g=o_g)


# ---------------------------------------------------------------------------
# NEXT-2: hierarchical local attention ("UltraGen ..." §4.3, hierarchical local
# attention: intermediate-scale attention over coarse windows).  Reading: the
# local branch also sees K and V average-pooled by a medium factor h_pool,
# through a window of coarse tiles -- the pooled grid cut into tiles of the
# same shape, one coarse tile covering h_pool fine tiles per dim -- around the
# coarse tile that holds the query tile; fine and coarse keys share one
# softmax.
# ---------------------------------------------------------------------------

def hier_geom(g: Geom, hpool: tuple) -> Geom:
    """The medium-pooled grid with the fine tile shape and window (its tiles
    are the coarse tiles)."""
    pt, ph, pw = hpool
    return Geom(g.T // pt, g.H // ph, g.W // pw, g.tile, g.window)


def coarse_tile_of(a: tuple, hpool: tuple) -> tuple:
    """Coarse tile holding fine tile a: a coarse tile spans h_pool fine tiles
    per dim (the same tile shape over a grid pooled by h_pool)."""
    return tuple(x // p for x, p in zip(a, hpool))


def _hier_query_tiles(g: Geom, hpool: tuple):
    """Yield (query ids, fine key ids, coarse key ids) per query tile: raster
    ids in the fine grid, and in the medium-pooled grid for the coarse keys."""
    gc = hier_geom(g, hpool)
    ncd = gc.tiles_per_dim
    nt, nh, nw = g.tiles_per_dim
    fine = _query_tiles(g)
    for at in range(nt):
        for ah in range(nh):
            for aw in range(nw):
                qi, kj = next(fine)
                c = coarse_tile_of((at, ah, aw), hpool)
                r = [window_range(c[ax], g.window[ax], ncd[ax]) for ax in range(3)]
                kc = _tile_token_box(gc, (r[0].start, r[1].start, r[2].start), (r[0].stop, r[1].stop, r[2].stop))
                yield qi, kj, kc


def hier_attention(q, k, v, g: Geom, hpool: tuple, scale: float):
    """Joint softmax over each query tile's fine sliding-tile keys and its
    coarse-window medium-pooled keys.  Raster in and out: (O, LSE)."""
    gh = g._replace(pool=tuple(hpool))
    kh, vh = pool(k, gh), pool(v, gh)
    B, nh, n, d = q.shape
    o = np.empty_like(q)
    lse = np.empty((B, nh, n))
    for b in range(B):
        for h in range(nh):
            for qi, kj, kc in _hier_query_tiles(g, hpool):
                keys = np.concatenate([k[b, h, kj], kh[b, h, kc]])
                vals = np.concatenate([v[b, h, kj], vh[b, h, kc]])
                o[b, h, qi], lse[b, h, qi], _ = _softmax_attend(q[b, h, qi], keys, vals, scale)
    return o, lse


def hier_backward(q, k, v, do, g: Geom, hpool: tuple, scale: float):
    """Gradients of hier_attention w.r.t. q, k, v (the coarse keys' gradients
    flow back through the medium pooling)."""
    gh = g._replace(pool=tuple(hpool))
    kh, vh = pool(k, gh), pool(v, gh)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dkh = np.zeros_like(kh)
    dvh = np.zeros_like(vh)
    B, nh = q.shape[:2]
    for b in range(B):
        for h in range(nh):
            for qi, kj, kc in _hier_query_tiles(g, hpool):
                keys = np.concatenate([k[b, h, kj], kh[b, h, kc]])
                vals = np.concatenate([v[b, h, kj], vh[b, h, kc]])
                a, dkeys, dvals = _softmax_attend_bwd(q[b, h, qi], keys, vals, do[b, h, qi], scale)
                nf = len(kj)
                dq[b, h, qi] += a
                dk[b, h, kj] += dkeys[:nf]
                dv[b, h, kj] += dvals[:nf]
                dkh[b, h, kc] += dkeys[nf:]
                dvh[b, h, kc] += dvals[nf:]
    return dq, dk + pool_transpose(dkh, gh), dv + pool_transpose(dvh, gh)


def hier_attention_tiles(q, k, v, g: Geom, hpool: tuple, scale: float, tile_ids):
    """hier_attention for the listed query tiles of one head (2-D q, k, v):
    returns (raster query ids, O rows, LSE rows)."""
    gh = g._replace(pool=tuple(hpool))
    kh, vh = pool(k, gh), pool(v, gh)
    want = set(int(t) for t in tile_ids)
    ids, os_, ls_ = [], [], []
    for t, (qi, kj, kc) in enumerate(_hier_query_tiles(g, hpool)):
        if t not in want:
            continue
        o, l, _ = _softmax_attend(q[qi], np.concatenate([k[kj], kh[kc]]), np.concatenate([v[kj], vh[kc]]), scale)
        ids.append(qi)
        os_.append(o)
        ls_.append(l)
    return np.concatenate(ids), np.concatenate(os_), np.concatenate(ls_)


def hier_backward_dq_tiles(q, k, v, do, g: Geom, hpool: tuple, scale: float, tile_ids):
    """dQ of hier_backward for the listed query tiles of one head (2-D arrays):
    a query's dQ depends only on its own row of the joint softmax.  Returns
    (raster query ids, dQ rows)."""
    gh = g._replace(pool=tuple(hpool))
    kh, vh = pool(k, gh), pool(v, gh)
    want = set(int(t) for t in tile_ids)
    ids, rows = [], []
    for t, (qi, kj, kc) in enumerate(_hier_query_tiles(g, hpool)):
        if t not in want:
            continue
        dq, _, _ = _softmax_attend_bwd(q[qi], np.concatenate([k[kj], kh[kc]]), np.concatenate([v[kj], vh[kc]]),
                                       do[qi], scale)
        ids.append(qi)
        rows.append(dq)
    return np.concatenate(ids), np.concatenate(rows)


def hier_backward_dkdv_tiles(q, k, v, do, g: Geom, hpool: tuple, scale: float, k_tiles):
    """dK and dV of hier_backward for the tokens of the listed fine key tiles
    of one head (2-D arrays).  A fine key token receives gradient twice: as a
    fine key of every query tile whose sliding window holds its tile, and
    through the medium pooling, as 1/|block| of the gradient of the pooled key
    holding it, which every query tile whose coarse window holds that pooled
    key contributes to.  Only the query tiles that see a wanted fine or pooled
    key are evaluated; each is the full joint-softmax row of the definition.
    Returns (raster key ids, dK rows, dV rows)."""
    gh = g._replace(pool=tuple(hpool))
    kh, vh = pool(k, gh), pool(v, gh)
    u = pooled_index(gh)
    cnt = hpool[0] * hpool[1] * hpool[2]
    want = np.concatenate([_tile_token_box(g, tile_coords_of(g, int(t)), tuple(c + 1 for c in tile_coords_of(g, int(t))))
                           for t in k_tiles])
    want_set = set(int(x) for x in want)
    coarse_set = set(int(x) for x in u[want])
    dk_f = {t: np.zeros(q.shape[1]) for t in want_set}
    dv_f = {t: np.zeros(q.shape[1]) for t in want_set}
    dk_c = {c: np.zeros(q.shape[1]) for c in coarse_set}
    dv_c = {c: np.zeros(q.shape[1]) for c in coarse_set}
    for qi, kj, kc in _hier_query_tiles(g, hpool):
        hit_f = [i for i, t in enumerate(kj) if int(t) in want_set]
        hit_c = [i for i, c in enumerate(kc) if int(c) in coarse_set]
        if not hit_f and not hit_c:
            continue
        _, dkeys, dvals = _softmax_attend_bwd(q[qi], np.concatenate([k[kj], kh[kc]]),
                                              np.concatenate([v[kj], vh[kc]]), do[qi], scale)
        nf = len(kj)
        for i in hit_f:
            dk_f[int(kj[i])] += dkeys[i]
            dv_f[int(kj[i])] += dvals[i]
        for i in hit_c:
            dk_c[int(kc[i])] += dkeys[nf + i]
            dv_c[int(kc[i])] += dvals[nf + i]
    dk = np.stack([dk_f[int(t)] + dk_c[int(u[t])] / cnt for t in want])
    dv = np.stack([dv_f[int(t)] + dv_c[int(u[t])] / cnt for t in want])
    return want, dk, dv
