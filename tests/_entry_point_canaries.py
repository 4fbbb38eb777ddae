"""Runs every data entry point of the library once on a small grid, with each
output and workspace surrounded by canary bytes, and saves the outputs.

    python tests/_entry_point_canaries.py OUT.npz

Run in its own process: the environment decides which build is loaded
(VATTN_DEBUG_BUILD=1: the debug build with device-side bounds checks).  After
every call the status word must read VATTN_OK and every canary must be
intact; a failure exits non-zero with the entry point's name.  The saved
outputs let a caller compare two builds bit for bit.
"""
import math
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

import torch  # noqa: E402

import video_dit_local_b200 as V  # noqa: E402
from helpers import geom_for, gpu_tensor  # noqa: E402
from synth import inputs as S  # noqa: E402

PAD = 4096          # canary bytes on each side (keeps 16-byte alignment)
CANARY = 0xA5
_buffers = []       # (name, padded uint8 buffer) of every guarded allocation


def guarded(name, shape, dtype, device="cuda", fill=None):
    """A tensor of `shape` inside a uint8 buffer with PAD canary bytes on both sides."""
    nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    buf = torch.full((nbytes + 2 * PAD,), CANARY, dtype=torch.uint8, device=device)
    t = buf[PAD:PAD + nbytes].view(dtype).view(shape)
    if fill is not None:
        t.copy_(fill)
    _buffers.append((name, buf, nbytes))
    return t


def guarded_like(name, x):
    return guarded(name, tuple(x.shape), x.dtype, x.device.type, None)


def workspace(name, op, geom):
    return guarded(name, (V.vattn_workspace_size(op, geom),), torch.uint8)


def check(what):
    torch.cuda.synchronize()
    st = V.vattn_get_status()
    if st != 0:
        sys.exit(f"{what}: device status {st} ({V.vattn_last_error()})")
    for name, buf, nbytes in _buffers:
        head, tail = buf[:PAD], buf[PAD + nbytes:]
        if not (bool((head == CANARY).all()) and bool((tail == CANARY).all())):
            sys.exit(f"{what}: canary around {name} overwritten")


def main(out_path):
    saved = {}
    # small grids: tile 192 (a ragged second query block), pool 4x4; d = 128
    w = S.small_workload("canary", 91, 1, 2, 128, (6, 16, 24), (3, 8, 8), (1, 3, 3), (1, 4, 4))
    geom = geom_for(V, w)
    check_heads = [(0, 0), (0, 1)]
    scale = 1 / math.sqrt(w.head_dim)
    qr, kr, vr, dor = (gpu_tensor(w, t, check_heads) for t in (S.Q_ID, S.K_ID, S.V_ID, S.DO_ID))
    lse_shape = tuple(qr.shape[:3])
    gvec = torch.from_numpy(S.blend_g(w)).cuda()
    n_pooled = (w.grid[0] // w.pool[0]) * (w.grid[1] // w.pool[1]) * (w.grid[2] // w.pool[2])
    pooled_shape = (w.batch, w.heads, n_pooled, w.head_dim)

    # a1 permute / unpermute, a2 kept tiles
    q, k, v, do = (guarded_like(f"{n} tiled", x) for n, x in (("q", qr), ("k", kr), ("v", vr), ("dO", dor)))
    for src, dst in ((qr, q), (kr, k), (vr, v), (dor, do)):
        V.vattn_tile_permute(geom, src, dst)
    check("vattn_tile_permute")
    back = guarded_like("unpermuted", q)
    V.vattn_tile_unpermute(geom, q, back)
    check("vattn_tile_unpermute")
    saved["unpermute"] = back.cpu().view(torch.int16).numpy()
    n_tiles = math.prod(a // b for a, b in zip(w.grid, w.tile))
    kept = guarded("kept", (n_tiles, math.prod(w.window)), torch.int32)
    V.vattn_kept_tiles(geom, kept)
    check("vattn_kept_tiles")
    saved["kept"] = kept.cpu().numpy()

    def fwd_outputs(tag):
        return guarded(f"{tag} O", tuple(q.shape), torch.bfloat16), guarded(f"{tag} LSE", lse_shape, torch.float32)

    # a3 sliding tile, raster, cross-window, FP8, hierarchical
    o, lse = fwd_outputs("sta")
    V.vattn_sta_fwd(geom, q, k, v, scale, o, lse)
    check("vattn_sta_fwd")
    saved["sta_o"], saved["sta_lse"] = o.cpu().view(torch.int16).numpy(), lse.cpu().numpy()
    orr, lser = fwd_outputs("raster")
    V.vattn_sta_fwd_raster(geom, qr, kr, vr, scale, orr, lser)
    check("vattn_sta_fwd_raster")
    saved["raster_o"] = orr.cpu().view(torch.int16).numpy()
    for shifted in (0, 1):
        ox, lx = fwd_outputs(f"xwin{shifted}")
        V.vattn_xwin_fwd(geom, shifted, q, k, v, scale, ox, lx)
        check(f"vattn_xwin_fwd shifted={shifted}")
        saved[f"xwin{shifted}_o"] = ox.cpu().view(torch.int16).numpy()
    of8, lf8 = fwd_outputs("fp8")
    V.vattn_sta_fwd_fp8(geom, q, k, v, scale, of8, lf8, workspace("fp8 ws", V.VATTN_OP_STA_FWD_FP8, geom))
    check("vattn_sta_fwd_fp8")
    saved["fp8_o"] = of8.cpu().view(torch.int16).numpy()
    wh = S.small_workload("canary_hier", 92, 1, 2, 128, (6, 16, 32), (3, 8, 8), (1, 3, 3), (1, 2, 2))
    gh = geom_for(V, wh)
    hq, hk, hv, hdo = (gpu_tensor(wh, t, [(0, 0), (0, 1)]) for t in (S.Q_ID, S.K_ID, S.V_ID, S.DO_ID))
    oh = guarded("hier O", tuple(hq.shape), torch.bfloat16)
    lh = guarded("hier LSE", tuple(hq.shape[:3]), torch.float32)
    V.vattn_hier_fwd(gh, hq, hk, hv, scale, oh, lh, workspace("hier ws", V.VATTN_OP_HIER_FWD, gh))
    check("vattn_hier_fwd")
    saved["hier_o"] = oh.cpu().view(torch.int16).numpy()

    # a4 pooling, a5 global, a6 dual (saved outputs), no-alloc, FP8 dual, symmetric dual
    kp, vp = (guarded(n, pooled_shape, torch.bfloat16) for n in ("K_p", "V_p"))
    V.vattn_pool_kv(geom, k, v, kp, vp)
    check("vattn_pool_kv")
    saved["kp"] = kp.cpu().view(torch.int16).numpy()
    og, lg = fwd_outputs("global")
    V.vattn_global_fwd(geom, q, kp, vp, scale, og, lg)
    check("vattn_global_fwd")
    saved["global_o"] = og.cpu().view(torch.int16).numpy()
    od, (o_l, lse_l), (o_g, lse_g) = fwd_outputs("dual")[0], fwd_outputs("dual local"), fwd_outputs("dual global")
    kp2, vp2 = (guarded(n, pooled_shape, torch.bfloat16) for n in ("dual K_p", "dual V_p"))
    V.vattn_dual_fwd(geom, q, k, v, gvec, scale, od, o_l, lse_l, o_g, lse_g, kp2, vp2)
    check("vattn_dual_fwd")
    saved["dual_o"] = od.cpu().view(torch.int16).numpy()
    on = guarded("noalloc O", tuple(q.shape), torch.bfloat16)
    V.vattn_dual_fwd_noalloc(geom, q, k, v, gvec, scale, on)
    check("vattn_dual_fwd_noalloc")
    saved["noalloc_o"] = on.cpu().view(torch.int16).numpy()
    odf = guarded("dual fp8 O", tuple(q.shape), torch.bfloat16)
    V.vattn_dual_fwd_fp8(geom, q, k, v, gvec, scale, odf, workspace("dual fp8 ws", V.VATTN_OP_DUAL_FWD_FP8, geom))
    check("vattn_dual_fwd_fp8")
    saved["dual_fp8_o"] = odf.cpu().view(torch.int16).numpy()
    osy, (osl, lsl) = guarded("sym O", tuple(q.shape), torch.bfloat16), fwd_outputs("sym local")
    qps, kps, vps, ops = (guarded(f"sym {n}", pooled_shape, torch.bfloat16) for n in ("Q_p", "K_p", "V_p", "O_p"))
    lps = guarded("sym LSE_p", pooled_shape[:3], torch.float32)
    V.vattn_dual_sym_fwd(geom, q, k, v, gvec, scale, osy, osl, lsl, qps, kps, vps, ops, lps)
    check("vattn_dual_sym_fwd")
    saved["sym_o"] = osy.cpu().view(torch.int16).numpy()
    wts = {n: guarded(f"learned {n}", tuple(a.shape), torch.float32, fill=torch.from_numpy(a).cuda())
           for n, a in S.learned_weights(w).items()}
    olr = guarded("sym learned O", tuple(q.shape), torch.bfloat16)
    V.vattn_dual_sym_learned_fwd(geom, q, k, v, gvec, wts["wq"], wts["wk"], wts["wv"], wts["w3"], scale, olr,
                                 workspace("sym learned ws", V.VATTN_OP_DUAL_SYM_LEARNED_FWD, geom))
    check("vattn_dual_sym_learned_fwd")
    saved["sym_learned_o"] = olr.cpu().view(torch.int16).numpy()

    # host-buffer forward: host outputs with canaries in host memory
    ohh = guarded("host O", tuple(qr.shape), torch.bfloat16, device="cpu")
    lhh = guarded("host LSE", lse_shape, torch.float32, device="cpu")
    qh, kh, vh = (x.cpu().pin_memory() for x in (qr, kr, vr))
    g1 = V.make_geom(1, 1, w.head_dim, w.grid, w.tile, w.window, w.pool)  # one slice per chunk
    wsh = guarded("host ws", (2 * V.vattn_workspace_size(V.VATTN_OP_STA_FWD_HOST, g1),), torch.uint8)
    V.vattn_sta_fwd_host(geom, qh, kh, vh, scale, ohh, lhh, 1, wsh)
    check("vattn_sta_fwd_host")
    saved["host_o"] = ohh.view(torch.int16).numpy().copy()

    # a7 backward passes
    def grads(tag, like):
        return tuple(guarded(f"{tag} {n}", tuple(like.shape), torch.bfloat16) for n in ("dQ", "dK", "dV"))

    dq, dk, dv = grads("sta", q)
    V.vattn_sta_bwd(geom, q, k, v, o, lse, do, scale, dq, dk, dv, workspace("sta bwd ws", V.VATTN_OP_STA_BWD, geom))
    check("vattn_sta_bwd")
    saved["sta_dq"], saved["sta_dk"] = dq.cpu().view(torch.int16).numpy(), dk.cpu().view(torch.int16).numpy()
    ox, lx = fwd_outputs("xwin bwd in")
    V.vattn_xwin_fwd(geom, 1, q, k, v, scale, ox, lx)
    dq, dk, dv = grads("xwin", q)
    V.vattn_xwin_bwd(geom, 1, q, k, v, ox, lx, do, scale, dq, dk, dv,
                     workspace("xwin bwd ws", V.VATTN_OP_STA_BWD, geom))
    check("vattn_xwin_bwd")
    saved["xwin_dv"] = dv.cpu().view(torch.int16).numpy()
    dq, dk, dv = grads("dual", q)
    dg = guarded("dg", (w.heads,), torch.float32)
    V.vattn_dual_bwd(geom, q, k, v, gvec, o_l, lse_l, o_g, lse_g, kp2, vp2, do, scale, dq, dk, dv, dg,
                     workspace("dual bwd ws", V.VATTN_OP_DUAL_BWD, geom))
    check("vattn_dual_bwd")
    saved["dual_dk"], saved["dg"] = dk.cpu().view(torch.int16).numpy(), dg.cpu().numpy()
    dq, dk, dv = grads("hier", hq)
    V.vattn_hier_bwd(gh, hq, hk, hv, oh, lh, hdo, scale, dq, dk, dv, workspace("hier bwd ws", V.VATTN_OP_HIER_BWD, gh))
    check("vattn_hier_bwd")
    saved["hier_dk"] = dk.cpu().view(torch.int16).numpy()
    dq, dk, dv = grads("sym", q)
    V.vattn_dual_sym_bwd(geom, q, k, v, gvec, osl, lsl, qps, kps, vps, ops, lps, do, scale, dq, dk, dv,
                         workspace("sym bwd ws", V.VATTN_OP_DUAL_SYM_BWD, geom))
    check("vattn_dual_sym_bwd")
    saved["sym_dq"] = dq.cpu().view(torch.int16).numpy()
    np.savez(out_path, **saved)
    print(f"{len(saved)} outputs, {len(_buffers)} guarded buffers: status OK, canaries intact")


if __name__ == "__main__":
    main(sys.argv[1])
