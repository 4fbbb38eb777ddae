"""GPU parity of the pipelined host-buffer sliding-tile forward.

vattn_sta_fwd_host runs the same permute, sliding-tile and unpermute kernels
as the device path, one chunk of batch*head slices at a time, with the
host<->device copies of neighbouring chunks overlapping the compute.  Each
slice's arithmetic does not depend on how the slices are grouped, so the
outputs must equal the device path bit for bit; the seeded heads are also
compared with the fp64 oracle (O within 2e-2 max-abs, 2e-3 mean-abs; LSE
within 1e-3), for chunk sizes that divide the slices and ones that leave a
ragged last chunk.
"""
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


def _device_path(V, geom, qr, kr, vr, scale):
    import torch
    q, k, v = (torch.empty_like(qr) for _ in range(3))
    for src, dst in ((qr, q), (kr, k), (vr, v)):
        V.vattn_tile_permute(geom, src, dst)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    V.vattn_sta_fwd(geom, q, k, v, scale, o, lse)
    o_r, lse_r = torch.empty_like(o), torch.empty_like(lse)
    V.vattn_tile_unpermute(geom, o, o_r)
    V.vattn_tile_unpermute(geom, lse, lse_r, 4)
    torch.cuda.synchronize()
    return o_r.cpu(), lse_r.cpu()


def _host_path(V, geom, w, qh, kh, vh, scale, chunk, with_lse=True, rounds=1):
    import torch
    one = V.make_geom(1, chunk, w.head_dim, w.grid, w.tile, w.window, w.pool)
    need = V.vattn_workspace_size(V.VATTN_OP_STA_FWD_HOST, one)
    ws = torch.empty(2 * need, dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(rounds):
        o = torch.full(qh.shape, float("nan"), dtype=torch.bfloat16).pin_memory()
        lse = torch.full(qh.shape[:3], float("nan"), dtype=torch.float32).pin_memory() if with_lse else None
        V.vattn_sta_fwd_host(geom, qh, kh, vh, scale, o, lse, chunk, ws)
        torch.cuda.current_stream().synchronize()
        assert V.vattn_get_status() == 0, V.vattn_last_error()
        outs.append((o, lse))
    return outs


@pytest.mark.parametrize("name,seed,batch,heads,d,grid,tile,window,chunks", [
    ("host_small", 31, 2, 3, 128, (6, 16, 24), (3, 8, 8), (1, 3, 3), (1, 2, 4, 6)),
    ("host_d64", 32, 1, 5, 64, (4, 8, 16), (2, 4, 4), (2, 1, 3), (2, 3, 5)),
])
def test_sta_fwd_host_equals_device_path_and_oracle(V, name, seed, batch, heads, d, grid, tile, window, chunks):
    w = S.small_workload(name, seed, batch, heads, d, grid, tile, window, (1, 1, 1))
    check = [(b, h) for b in range(batch) for h in range(heads)]
    geom = geom_for(V, w)
    scale = 1 / math.sqrt(d)
    qr, kr, vr = (gpu_tensor(w, i, check) for i in (S.Q_ID, S.K_ID, S.V_ID))
    o_ref, lse_ref = _device_path(V, geom, qr, kr, vr, scale)
    qh, kh, vh = (x.cpu().pin_memory() for x in (qr, kr, vr))
    g = O.geom_of(w)
    for chunk in chunks:
        for o, lse in _host_path(V, geom, w, qh, kh, vh, scale, chunk, rounds=2):
            assert torch_equal_bits(o, o_ref), f"O differs from the device path (chunk {chunk})"
            assert torch_equal_bits(lse, lse_ref), f"LSE differs from the device path (chunk {chunk})"
    # the seeded heads against the oracle, on every query tile
    tiles = range(math.prod(g.tiles_per_dim))
    for b, h in check:
        q, k, v = (host_f64(w, i, b, h) for i in (S.Q_ID, S.K_ID, S.V_ID))
        ids, o_or, lse_or = O.sta_attention_tiles(q, k, v, g, scale, tiles)
        assert_close(to_f64(o_ref[b, h])[ids], o_or, O_MAX_ABS, O_MEAN_ABS, f"O b{b} h{h}")
        assert_close(lse_ref[b, h].numpy().astype(np.float64)[ids], lse_or, LSE_MAX_ABS, what=f"LSE b{b} h{h}")


def torch_equal_bits(a, b):
    import torch
    if a.dtype == torch.bfloat16:
        return torch.equal(a.view(torch.int16), b.view(torch.int16))
    return torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_sta_fwd_host_without_lse_and_pageable_output(V):
    """LSE may be omitted, and pageable (unpinned) host buffers still give the
    same result (CUDA then stages the copies through its own pinned buffers)."""
    import torch
    w = S.small_workload("host_nolse", 33, 1, 4, 128, (6, 16, 16), (3, 8, 8), (1, 1, 3), (1, 1, 1))
    check = [(0, h) for h in range(4)]
    geom = geom_for(V, w)
    scale = 1 / math.sqrt(128)
    qr, kr, vr = (gpu_tensor(w, i, check) for i in (S.Q_ID, S.K_ID, S.V_ID))
    o_ref, _ = _device_path(V, geom, qr, kr, vr, scale)
    qh, kh, vh = (x.cpu() for x in (qr, kr, vr))
    (o, lse), = _host_path(V, geom, w, qh, kh, vh, scale, 3, with_lse=False)
    assert lse is None
    assert torch_equal_bits(o, o_ref)


def test_sta_fwd_host_720p_sampled(V):
    """The benchmarked 720p workload (24 heads) in chunks of 3 slices, equal to
    the device path on the two seeded heads' full outputs."""
    import torch
    w = S.WORKLOADS["720p"]
    check = [(0, 0), (0, w.heads - 1)]
    geom = geom_for(V, w)
    scale = 1 / math.sqrt(w.head_dim)
    qr, kr, vr = (gpu_tensor(w, i, check) for i in (S.Q_ID, S.K_ID, S.V_ID))
    o_ref, lse_ref = _device_path(V, geom, qr, kr, vr, scale)
    qh, kh, vh = (x.cpu().pin_memory() for x in (qr, kr, vr))
    del qr, kr, vr
    (o, lse), = _host_path(V, geom, w, qh, kh, vh, scale, 3)
    assert torch_equal_bits(o, o_ref) and torch_equal_bits(lse, lse_ref)
    torch.cuda.empty_cache()


def test_sta_fwd_host_back_to_back_calls_from_two_streams(V):
    """Two calls with different inputs, issued from two streams and sharing
    one workspace: the library orders them on its own streams, so both
    results equal the device path."""
    import torch
    w = S.small_workload("host_2s", 34, 1, 4, 128, (6, 16, 16), (3, 8, 8), (1, 1, 3), (1, 1, 1))
    check = [(0, h) for h in range(4)]
    geom = geom_for(V, w)
    scale = 1 / math.sqrt(128)
    qr, kr, vr = (gpu_tensor(w, i, check) for i in (S.Q_ID, S.K_ID, S.V_ID))
    q2, k2, v2 = (x.flip(2).contiguous() for x in (qr, kr, vr))   # a second, different input set
    ref1, _ = _device_path(V, geom, qr, kr, vr, scale)
    ref2, _ = _device_path(V, geom, q2, k2, v2, scale)
    one = V.make_geom(1, 2, 128, w.grid, w.tile, w.window, w.pool)
    ws = torch.empty(2 * V.vattn_workspace_size(V.VATTN_OP_STA_FWD_HOST, one), dtype=torch.uint8, device="cuda")
    ins1 = [x.cpu().pin_memory() for x in (qr, kr, vr)]
    ins2 = [x.cpu().pin_memory() for x in (q2, k2, v2)]
    o1 = torch.empty(qr.shape, dtype=torch.bfloat16).pin_memory()
    o2 = torch.empty(qr.shape, dtype=torch.bfloat16).pin_memory()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    V.vattn_sta_fwd_host(geom, *ins1, scale, o1, None, 2, ws, stream=s1)
    V.vattn_sta_fwd_host(geom, *ins2, scale, o2, None, 2, ws, stream=s2)
    torch.cuda.synchronize()
    assert V.vattn_get_status() == 0, V.vattn_last_error()
    assert torch_equal_bits(o1, ref1) and torch_equal_bits(o2, ref2)


def test_shutdown_waits_for_the_pipeline_and_calls_recreate_it(V):
    """vattn_shutdown issued right after an asynchronous host-buffer call
    waits for that call's copies and kernels, releases the library streams,
    and the next call builds them again with the same result."""
    import torch
    w = S.small_workload("host_shutdown", 35, 1, 4, 128, (6, 16, 16), (3, 8, 8), (1, 1, 3), (1, 1, 1))
    check = [(0, h) for h in range(4)]
    geom = geom_for(V, w)
    scale = 1 / math.sqrt(128)
    qr, kr, vr = (gpu_tensor(w, i, check) for i in (S.Q_ID, S.K_ID, S.V_ID))
    ref, _ = _device_path(V, geom, qr, kr, vr, scale)
    ins = [x.cpu().pin_memory() for x in (qr, kr, vr)]
    one = V.make_geom(1, 1, 128, w.grid, w.tile, w.window, w.pool)
    ws = torch.empty(2 * V.vattn_workspace_size(V.VATTN_OP_STA_FWD_HOST, one), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        o = torch.full(qr.shape, float("nan"), dtype=torch.bfloat16).pin_memory()
        V.vattn_sta_fwd_host(geom, *ins, scale, o, None, 1, ws)
        V.vattn_shutdown()          # no synchronisation before it: shutdown waits
        torch.cuda.current_stream().synchronize()
        assert V.vattn_get_status() == 0, V.vattn_last_error()
        assert torch_equal_bits(o, ref)
