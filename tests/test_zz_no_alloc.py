"""The allocation-free dual forward against the allocating one.

vattn_dual_fwd_noalloc serves callers that cannot call cudaMalloc (a plug-in
inside a host framework whose pool has already reserved the device; a
latency-critical path that forbids allocation after start-up): it takes its
workspace from the library's static device scratch instead of a caller
buffer.  Its output must equal, bit for bit, vattn_dual_fwd's with a
caller-owned workspace, on two calls per geometry with another geometry's
call in between (the scratch keeps the previous call's contents), and
geometries that do not fit the scratch must be refused before any launch.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import math

import pytest

from helpers import geom_for, gpu_tensor
from synth import inputs as S

pytestmark = pytest.mark.gpu

CASES = [
    # one head of the 1080p-shaped dual workload: about 52 MB of scratch
    S.small_workload("noalloc_1080p_1h", 21, 1, 1, 128, (21, 72, 120), (3, 8, 8), (3, 3, 3), (1, 4, 4)),
    # a small grid with ragged N and N_p, d = 64
    S.small_workload("noalloc_small", 22, 2, 3, 64, (3, 20, 24), (3, 4, 4), (1, 3, 3), (1, 2, 2)),
]


def _inputs(V, w):
    import torch
    geom = geom_for(V, w)
    check = [(b, h) for b in range(w.batch) for h in range(w.heads)]
    tiled = []
    for tid in (S.Q_ID, S.K_ID, S.V_ID):
        x = gpu_tensor(w, tid, check)
        t = torch.empty_like(x)
        V.vattn_tile_permute(geom, x, t)
        tiled.append(t)
    g = torch.from_numpy(S.blend_g(w)).cuda()
    return geom, tiled, g


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    """Both geometries are called twice, interleaved (A, B, A, B), so every
    second call finds the scratch holding the other geometry's intermediates:
    a region of it that a call reads before writing would show.  The same
    kernels run on the same inputs as with a caller workspace, and the forward
    is deterministic (no atomics), so the outputs must be bit-identical."""
    import torch
    import video_dit_local_b200 as V
    runs = []
    for w in CASES:
        geom, (q, k, v), g = _inputs(V, w)
        need = V.vattn_workspace_size(V.VATTN_OP_DUAL_FWD, geom)
        assert need <= V.binding.VATTN_NOALLOC_SCRATCH_BYTES
        scale = 1 / math.sqrt(w.head_dim)
        ref = torch.empty_like(q)
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        V.vattn_dual_fwd(geom, q, k, v, g, scale, ref, workspace=ws)
        torch.cuda.synchronize()
        assert V.vattn_get_status() == 0, V.vattn_last_error()
        assert torch.isfinite(ref.float()).all(), f"{w.name}: non-finite reference"
        runs.append((w, geom, q, k, v, g, scale, ref))
    for call in range(2):
        for w, geom, q, k, v, g, scale, ref in runs:
            out = torch.full_like(q, float("nan"))
            V.vattn_dual_fwd_noalloc(geom, q, k, v, g, scale, out)
            torch.cuda.synchronize()
            assert V.vattn_get_status() == 0, V.vattn_last_error()
            assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"{w.name} call {call}: not bit-identical"


def test_noalloc_refuses_geometry_larger_than_scratch():
    import torch
    import video_dit_local_b200 as V
    w = S.WORKLOADS["1080p"]          # 24 heads: about 1.25 GB of workspace
    geom = geom_for(V, w)
    assert V.vattn_workspace_size(V.VATTN_OP_DUAL_FWD, geom) > V.binding.VATTN_NOALLOC_SCRATCH_BYTES
    t = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(V.VattnError) as e:
        V.vattn_dual_fwd_noalloc(geom, t, t, t, torch.zeros(24, device="cuda"), 0.1, t)
    assert e.value.code == V.binding.VATTN_ERR_WORKSPACE
    assert "static scratch" in str(e.value)
