"""Benchmark of the dual-branch 3D attention hot path (one JSON line on rank 0).

Default workload: the 720p-shaped sliding-tile forward (B1 h24 d128, grid
30x48x80, tile 6x8x8, window 3x3x3, per-head U(0.5, 2) scale).  One step =
one vattn_sta_fwd_raster call: raster Q, K, V in, raster O and LSE out, the
raster <-> tile-major reorder done by the kernel's tensor-map boxes and
epilogue stores (one launch).  `e2e` times vattn_sta_fwd_host on the same
workload from pinned host buffers, copies included.
Effective FLOPs count 4*d per kept query-key pair (masked work is not
counted).  Inputs (2.1 GB of Q/K/V) are larger than the 126 MB L2, so no flush
is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--no-extras]

Multi-GPU: one process per GPU (torchrun); each rank runs its own full
workload (batch/head slices are independent: no collective on the data path),
so scaling is weak and `value` sums all ranks' work over the max-over-ranks
time.  `--impl reference` times the fp64 CPU oracle on a bounded sample of the
same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "effective TFLOP/s & ms/call of 3D tile+global attention fwd/bwd; % BF16 TC peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# ncu DRAM traffic per launch of the sliding-tile forward kernel at the 720p
# workload (read+write bytes), and the hash of the kernel source it was taken
# from.  When the source changes the figure is stale and reported as null.
STA_FWD_TRAFFIC = 2721076224  # DRAM read + write bytes per launch: an ncu capture of the 2-head case x 12
STA_FWD_TRAFFIC_SRC_SHA = "657b6e246093eed6"


def reduce_max(values, world: int, device=None):
    """Max over ranks of a list of floats (the timing rule: every multi-GPU
    number is the slowest rank's); a no-op on one process."""
    if world <= 1:
        return list(values)
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def whole_job_tflops(flops_per_rank: float, ms: float, world: int) -> float:
    """Whole-job throughput: every rank runs its own full workload (weak
    scaling), so the job's work is world x per-rank work over the max time."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def _src_sha() -> str:
    h = hashlib.sha256()
    for f in ("attn_fwd.cu", "fwd_common.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "video_dit_local_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_index: int):
        self.dev = dev_index
        self.proc = None
        self.lines = []
        self.t = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "50", "-i", str(self.dev)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.25)
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.lines:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm, smax, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
                power.append(float(parts[3]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        loaded = [s for s, p in zip(sm, power) if p > 300] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm), "power_w_max": max(power) if power else None}


# ----------------------------------------------------------------------------- workloads

def _geom(V, w):
    return V.make_geom(w.batch, w.heads, w.head_dim, w.grid, w.tile, w.window, w.pool)


def _flops_fwd(w):
    from synth import inputs as S  # noqa: F401
    T, H, W = w.grid
    nt = [a // b for a, b in zip(w.grid, w.tile)]
    kept = math.prod(min(x, n) for x, n in zip(w.window, nt))
    s = math.prod(w.tile)
    n = T * H * W
    pairs_local = w.batch * w.heads * n * kept * s
    pairs_global = 0
    if w.dual:
        npool = (T // w.pool[0]) * (H // w.pool[1]) * (W // w.pool[2])
        pairs_global = w.batch * w.heads * n * npool
    return 4 * w.head_dim * pairs_local, 4 * w.head_dim * pairs_global


def _host_inputs_720p(w):
    """Seeded Q/K/V (bf16 bits, raster) from the shared generator."""
    import numpy as np
    from synth import inputs as S
    out = []
    for tid in (S.Q_ID, S.K_ID, S.V_ID):
        out.append(S.draw(w, tid).view(np.int16))
    return out


def _device_randn(shape, seed, std=1.0, scales=None):
    import torch
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    x = torch.randn(shape, generator=gen, device="cuda", dtype=torch.float32) * std
    if scales is not None:
        x *= torch.as_tensor(scales, device="cuda").view(1, -1, 1, 1)
    return x.to(torch.bfloat16)


def run_train_only(args, rank, world, local_rank):
    """Profiling mode: the training workload's fwd+bwd step alone (optionally
    with fewer heads), timed with CUDA events."""
    import dataclasses

    import torch

    import video_dit_local_b200 as V
    from synth import inputs as S
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = S.WORKLOADS["train"]
    if args.heads:
        w = dataclasses.replace(w, heads=args.heads)
    peaks, _ = _peaks()
    res = _bench_train(V, dev, peaks, w=w, n=args.steps, warm=args.warmup)
    return {"metric": METRIC, "value": res["step_eff_tflops"], "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": res["fwd_ms"] + res["bwd_ms"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded torch N(0,1))",
            "config": {"workload": f"train dual fwd+bwd: B{w.batch} h{w.heads} d128, grid 21x72x120, tile 3x8x8, "
                                   "window 3x3x3, pool 1x4x4"}, "train": res}


def run_fp8_only(args, rank, world, local_rank):
    """Profiling mode: the FP8 sliding-tile forward (e4m3 Q*K^T and P*V, the
    quantisation included) of the 720p workload alone (optionally with fewer
    heads), timed with CUDA events."""
    import dataclasses

    import torch

    import video_dit_local_b200 as V
    from synth import inputs as S
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = S.WORKLOADS["720p"]
    if args.heads:
        w = dataclasses.replace(w, heads=args.heads)
    geom = _geom(V, w)
    shape = (w.batch, w.heads, w.n_tokens, w.head_dim)
    q, k, v = (_device_randn(shape, 800 + i) for i in range(3))
    o = torch.empty_like(q)
    lse = torch.empty(shape[:3], dtype=torch.float32, device=dev)
    ws = torch.empty(V.vattn_workspace_size(V.VATTN_OP_STA_FWD_FP8, geom), dtype=torch.uint8, device=dev)
    fl, _ = _flops_fwd(w)
    ms = _time_ms(lambda: V.vattn_sta_fwd_fp8(geom, q, k, v, 1 / math.sqrt(w.head_dim), o, lse, ws), args.steps,
                  warm=args.warmup)
    return {"metric": METRIC, "value": round(fl / ms / 1e9, 1), "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3", "data": "synthetic (seeded torch N(0,1))",
            "config": {"workload": f"720p sliding-tile fwd, FP8: B1 h{w.heads} d128, grid 30x48x80, tile 6x8x8, "
                                   "window 3x3x3"}, "status": V.vattn_get_status()}


def run_dual_only(args, rank, world, local_rank):
    """Profiling mode: the inference dual forward (pool, sliding-tile branch,
    global branch with the blend) of the 1080p or 4K workload alone (optionally
    with fewer heads), timed with CUDA events."""
    import dataclasses

    import torch

    import video_dit_local_b200 as V
    from synth import inputs as S
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = S.WORKLOADS[args.workload]
    if args.heads:
        w = dataclasses.replace(w, heads=args.heads)
    geom = _geom(V, w)
    shape = (w.batch, w.heads, w.n_tokens, w.head_dim)
    q, k, v = (_device_randn(shape, 100 * w.seed + i) for i in range(3))
    gvec = torch.rand(w.heads, device=dev)
    o = torch.empty_like(q)
    ws = torch.empty(V.vattn_workspace_size(V.VATTN_OP_DUAL_FWD, geom), dtype=torch.uint8, device=dev)
    fl, fg = _flops_fwd(w)
    ms = _time_ms(lambda: V.vattn_dual_fwd(geom, q, k, v, gvec, 1 / math.sqrt(w.head_dim), o, workspace=ws),
                  args.steps, warm=args.warmup)
    T, H, W = w.grid
    return {"metric": METRIC, "value": round((fl + fg) / ms / 1e9, 1), "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded torch N(0,1))",
            "config": {"workload": f"{w.name} dual fwd: B{w.batch} h{w.heads} d{w.head_dim}, grid {T}x{H}x{W}, "
                                   f"tile {'x'.join(map(str, w.tile))}, window {'x'.join(map(str, w.window))}, "
                                   f"pool {'x'.join(map(str, w.pool))}"}, "status": V.vattn_get_status()}


def run_sym_learned_only(args, rank, world, local_rank):
    """Profiling mode: the 1080p dual forward with the learned symmetric
    global branch alone (seeded random weights), timed with CUDA events."""
    import torch

    import video_dit_local_b200 as V
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    peaks, _ = _peaks()
    res = _bench_sym_learned(V, dev, peaks, n=args.steps, warm=args.warmup, heads=args.heads)
    return {"metric": METRIC, "value": res["eff_tflops"], "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": res["ms"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded torch N(0,1), seeded random weights)",
            "config": {"workload": f"1080p dual fwd, learned symmetric global branch: B1 h{args.heads or 24} d128, "
                                   "grid 21x72x120, tile 3x8x8, window 3x3x3, pool 1x4x4"}, "status": res["status"]}


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch

    import video_dit_local_b200 as V
    from synth import inputs as S

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = S.WORKLOADS["720p"]
    if args.heads and args.heads != w.heads:   # reduced case for profiling only
        import dataclasses
        w = dataclasses.replace(w, heads=args.heads)
    geom = _geom(V, w)
    scale = 1.0 / math.sqrt(w.head_dim)
    flops_local, _ = _flops_fwd(w)

    host = _host_inputs_720p(w)
    pinned = [torch.from_numpy(h).pin_memory() for h in host]
    shape = (w.batch, w.heads, w.n_tokens, w.head_dim)
    qr, kr, vr = (p.to(dev).view(torch.bfloat16) for p in pinned)
    o_r = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    lse_r = torch.empty(shape[:3], dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    kernel_events = []

    def step(record=False):
        # raster Q, K, V in, raster O and LSE out: the tile reorder is done by
        # the kernel's tensor-map boxes and epilogue stores (one launch)
        if record:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        V.vattn_sta_fwd_raster(geom, qr, kr, vr, scale, o_r, lse_r)
        if record:
            e1.record(stream)
            kernel_events.append((e0, e1))

    launches_per_step = 1
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if V.vattn_get_status() != 0:
        raise RuntimeError("device status after warm-up: " + V.vattn_last_error())

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            step(record=True)
        t1.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms_total = t0.elapsed_time(t1)
    ms_kernel = sum(a.elapsed_time(b) for a, b in kernel_events) / len(kernel_events)
    if V.vattn_get_status() != 0:
        raise RuntimeError("device status after timing: " + V.vattn_last_error())
    ms_step = ms_total / args.steps
    ms_step, ms_kernel = reduce_max([ms_step, ms_kernel], world, dev)

    # end to end through the C ABI from pinned host buffers
    o_host = torch.empty(shape, dtype=torch.bfloat16, pin_memory=True)
    lse_host = torch.empty(shape[:3], dtype=torch.float32, pin_memory=True)

    def serial_step():   # copies, then the device step, then copies, on one stream
        for p, dst in zip(pinned, (qr, kr, vr)):
            dst.view(torch.int16).copy_(p, non_blocking=True)
        step()
        o_host.copy_(o_r, non_blocking=True)
        lse_host.copy_(lse_r, non_blocking=True)

    # the library's pipelined host-buffer entry point: chunks of batch*head
    # slices, copies in both directions overlapping the compute
    chunk = min(args.e2e_chunk, w.batch * w.heads)
    one = V.make_geom(1, chunk, w.head_dim, w.grid, w.tile, w.window, w.pool)
    host_ws = torch.empty(2 * V.vattn_workspace_size(V.VATTN_OP_STA_FWD_HOST, one), dtype=torch.uint8, device=dev)

    def e2e_step():
        V.vattn_sta_fwd_host(geom, pinned[0], pinned[1], pinned[2], scale, o_host, lse_host, chunk, host_ws)

    def time_steps(fn, n):
        fn()
        torch.cuda.synchronize()
        barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(n):
            fn()
        a1.record(stream)
        torch.cuda.synchronize()
        return reduce_max([a0.elapsed_time(a1) / n], world, dev)[0]

    e2e_steps = max(3, min(args.steps, 10))
    ms_e2e = time_steps(e2e_step, e2e_steps)
    if V.vattn_get_status() != 0:
        raise RuntimeError("device status after the host-buffer steps: " + V.vattn_last_error())
    ms_serial = time_steps(serial_step, e2e_steps)
    del host_ws
    h2d = sum(p.numel() * p.element_size() for p in pinned)
    d2h = o_host.numel() * 2 + lse_host.numel() * 4

    peaks, peak_src = _peaks()
    achieved = flops_local / (ms_kernel * 1e-3) / 1e12
    traffic = STA_FWD_TRAFFIC if STA_FWD_TRAFFIC_SRC_SHA == _src_sha() else None
    result = {
        "metric": METRIC,
        "value": round(whole_job_tflops(flops_local, ms_step, world), 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16, per-head U(0.5,2) scale)",
        "config": {"workload": f"720p sliding-tile fwd: B1 h{w.heads} d128, grid 30x48x80, tile 6x8x8, window 3x3x3",
                   "global_batch": w.batch * world, "seq_len": w.n_tokens, "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (2.1 GB Q/K/V), no flush",
                   "step": "sta_fwd on raster Q,K,V -> raster O,LSE (tile reorder fused into the kernel)"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1),
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(achieved / peaks["bf16_tflops"], 4),
                     "frac_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
                     "peak_source": f"{peak_src} bf16 (burst)", "traffic": traffic,
                     "kernel": "fwd::attn_fwd_kernel<128> (sliding tile, raster tensor-map boxes)",
                     "kernel_ms": round(ms_kernel, 4),
                     "algorithmic_flop_per_launch": flops_local},
        "e2e": {"value": round(whole_job_tflops(flops_local, ms_e2e, world), 2), "unit": "TFLOP/s",
                "ms_per_step": round(ms_e2e, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "call": f"vattn_sta_fwd_host, pinned host buffers, chunks of {chunk} slices",
                "serial_ms_per_step": round(ms_serial, 3)},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_extras and args.workload == "720p":
        result["extras"] = run_extras(V, dev)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    return result


def run_extras(V, dev):
    """Other shipped workloads, kernel-timed (not part of `value`)."""
    import torch
    from synth import inputs as S
    out = {}
    peaks, _ = _peaks()
    for name in ("1080p", "4k"):
        w = S.WORKLOADS[name]
        geom = _geom(V, w)
        shape = (w.batch, w.heads, w.n_tokens, w.head_dim)
        q, k, v = (_device_randn(shape, 100 * w.seed + i) for i in range(3))
        gvec = torch.rand(w.heads, device=dev)
        o = torch.empty_like(q)
        ws = torch.empty(V.vattn_workspace_size(V.VATTN_OP_DUAL_FWD, geom), dtype=torch.uint8, device=dev)
        scale = 1 / math.sqrt(w.head_dim)
        fl, fg = _flops_fwd(w)

        def call():
            V.vattn_dual_fwd(geom, q, k, v, gvec, scale, o, workspace=ws)
        with ClockSampler(dev.index) as clk:
            ms = _time_ms(call, 4)
        out[f"{name}_dual_fwd"] = {"ms": round(ms, 3), "eff_tflops": round((fl + fg) / ms / 1e9, 1),
                                   "frac": round((fl + fg) / ms / 1e9 / peaks["bf16_tflops"], 4),
                                   "status": V.vattn_get_status(), "clocks": clk.summary()}
        del q, k, v, o, ws
        torch.cuda.empty_cache()
    def clocked(fn):
        with ClockSampler(dev.index) as clk:
            res = fn()
        res["clocks"] = clk.summary()
        return res

    out["train_fwd_bwd"] = clocked(lambda: _bench_train(V, dev, peaks))
    with ClockSampler(dev.index) as clk:
        xw = _bench_xwin(V, dev, peaks)
    for name, res in xw.items():
        res["clocks"] = clk.summary()
        out[name] = res
    out["1080p_dual_sym_fwd"] = clocked(lambda: _bench_sym(V, dev, peaks))
    out["1080p_dual_sym_learned_fwd"] = clocked(lambda: _bench_sym_learned(V, dev, peaks))
    out["720p_hier_fwd_bwd"] = clocked(lambda: _bench_hier(V, dev, peaks))
    out["720p_sta_fwd_fp8"] = clocked(lambda: _bench_fp8(V, dev, peaks))
    out["1080p_dual_fwd_fp8"] = clocked(lambda: _bench_dual_fp8(V, dev, peaks))
    out["memory_bound"] = clocked(lambda: _bench_memory_bound(V, dev, peaks))
    return out


def _time_ms(fn, n, warm=2):
    import torch
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / n


def _bench_memory_bound(V, dev, peaks):
    """The HBM-bound kernels on their own, algorithmic bytes over time: the
    tile permute of one 720p tensor (read + write of every row) and the K/V
    pooling at 1080p and 4K (K and V read, K_p and V_p written)."""
    import torch
    from synth import inputs as S
    out = {}
    w = S.WORKLOADS["720p"]
    shape = (w.batch, w.heads, w.n_tokens, w.head_dim)
    x = _device_randn(shape, 600)
    y = torch.empty_like(x)
    geom = _geom(V, w)
    ms = _time_ms(lambda: V.vattn_tile_permute(geom, x, y), 10)
    nbytes = 2 * x.numel() * 2
    out["permute_720p"] = {"ms": round(ms, 4), "gbs": round(nbytes / ms / 1e6, 1),
                           "frac_hbm": round(nbytes / ms / 1e6 / peaks["hbm_gbs"], 4)}
    del x, y
    for name in ("1080p", "4k"):
        w = S.WORKLOADS[name]
        geom = _geom(V, w)
        shape = (w.batch, w.heads, w.n_tokens, w.head_dim)
        k, v = (_device_randn(shape, 610 + i) for i in range(2))
        npool = w.n_tokens // (w.pool[0] * w.pool[1] * w.pool[2])
        kp = torch.empty((w.batch, w.heads, npool, w.head_dim), dtype=torch.bfloat16, device=dev)
        vp = torch.empty_like(kp)
        ms = _time_ms(lambda: V.vattn_pool_kv(geom, k, v, kp, vp), 10)
        nbytes = 2 * k.numel() * 2 + 2 * kp.numel() * 2
        out[f"pool_kv_{name}"] = {"ms": round(ms, 4), "gbs": round(nbytes / ms / 1e6, 1),
                                  "frac_hbm": round(nbytes / ms / 1e6 / peaks["hbm_gbs"], 4)}
        del k, v, kp, vp
        torch.cuda.empty_cache()
    out["status"] = V.vattn_get_status()
    return out


def _bench_dual_fp8(V, dev, peaks):
    """The 1080p dual forward with e4m3 Q*K^T in both branches (pooling and
    quantisation included in the timed call); effective FLOPs as the bf16
    dual forward, fraction of the bf16 peak."""
    import torch
    from synth import inputs as S
    w = S.WORKLOADS["1080p"]
    geom = _geom(V, w)
    shape = (w.batch, w.heads, w.n_tokens, w.head_dim)
    q, k, v = (_device_randn(shape, 900 + i) for i in range(3))
    gvec = torch.rand(w.heads, device=dev)
    o = torch.empty_like(q)
    ws = torch.empty(V.vattn_workspace_size(V.VATTN_OP_DUAL_FWD_FP8, geom), dtype=torch.uint8, device=dev)
    fl, fg = _flops_fwd(w)
    scale = 1 / math.sqrt(w.head_dim)
    for _ in range(2):
        V.vattn_dual_fwd_fp8(geom, q, k, v, gvec, scale, o, ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(4):
        V.vattn_dual_fwd_fp8(geom, q, k, v, gvec, scale, o, ws)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / 4
    res = {"ms": round(ms, 3), "eff_tflops": round((fl + fg) / ms / 1e9, 1),
           "frac_of_bf16_peak": round((fl + fg) / ms / 1e9 / peaks["bf16_tflops"], 4), "status": V.vattn_get_status()}
    del q, k, v, o, ws
    torch.cuda.empty_cache()
    return res


def _bench_fp8(V, dev, peaks):
    """The 720p sliding-tile forward with e4m3 Q*K^T (quantisation included in
    the timed call); effective FLOPs as the bf16 forward; the fraction is of
    the bf16 peak (half the Q*K^T work ran at the e4m3 rate)."""
    import torch
    from synth import inputs as S
    w = S.WORKLOADS["720p"]
    geom = _geom(V, w)
    shape = (w.batch, w.heads, w.n_tokens, w.head_dim)
    q, k, v = (_device_randn(shape, 800 + i) for i in range(3))
    o = torch.empty_like(q)
    lse = torch.empty(shape[:3], dtype=torch.float32, device=dev)
    ws = torch.empty(V.vattn_workspace_size(V.VATTN_OP_STA_FWD_FP8, geom), dtype=torch.uint8, device=dev)
    fl, _ = _flops_fwd(w)
    scale = 1 / math.sqrt(w.head_dim)
    for _ in range(2):
        V.vattn_sta_fwd_fp8(geom, q, k, v, scale, o, lse, ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(5):
        V.vattn_sta_fwd_fp8(geom, q, k, v, scale, o, lse, ws)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / 5
    res = {"ms": round(ms, 3), "eff_tflops": round(fl / ms / 1e9, 1),
           "frac_of_bf16_peak": round(fl / ms / 1e9 / peaks["bf16_tflops"], 4), "status": V.vattn_get_status()}
    del q, k, v, o, lse, ws
    torch.cuda.empty_cache()
    return res


def _bench_hier(V, dev, peaks):
    """Hierarchical local attention at the 720p workload with h_pool 1x2x2
    (coarse tiles 5x3x5): effective FLOPs count the fine and the coarse pairs
    (27 kept tiles of 384 tokens each, per query)."""
    import torch
    from synth import inputs as S
    w = S.WORKLOADS["720p"]
    hp = (1, 2, 2)
    geom = V.make_geom(w.batch, w.heads, w.head_dim, w.grid, w.tile, w.window, hp)
    shape = (w.batch, w.heads, w.n_tokens, w.head_dim)
    q, k, v = (_device_randn(shape, 700 + i) for i in range(3))
    o = torch.empty_like(q)
    lse = torch.empty(shape[:3], dtype=torch.float32, device=dev)
    ws = torch.empty(V.vattn_workspace_size(V.VATTN_OP_HIER_FWD, geom), dtype=torch.uint8, device=dev)
    nc = [g // t // p for g, t, p in zip(w.grid, w.tile, hp)]
    s = math.prod(w.tile)
    coarse_keys = math.prod(min(win, n) for win, n in zip(w.window, nc)) * s
    fl, _ = _flops_fwd(w)
    fl += 4 * w.head_dim * w.batch * w.heads * w.n_tokens * coarse_keys
    scale = 1 / math.sqrt(w.head_dim)
    for _ in range(2):
        V.vattn_hier_fwd(geom, q, k, v, scale, o, lse, ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(4):
        V.vattn_hier_fwd(geom, q, k, v, scale, o, lse, ws)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / 4
    # backward: 10*d effective FLOPs per pair (the forward counts 4*d)
    do = _device_randn(shape, 703)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    wsb = torch.empty(V.vattn_workspace_size(V.VATTN_OP_HIER_BWD, geom), dtype=torch.uint8, device=dev)
    for _ in range(2):
        V.vattn_hier_bwd(geom, q, k, v, o, lse, do, scale, dq, dk, dv, wsb)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(3):
        V.vattn_hier_bwd(geom, q, k, v, o, lse, do, scale, dq, dk, dv, wsb)
    e1.record()
    torch.cuda.synchronize()
    ms_b = e0.elapsed_time(e1) / 3
    fl_b = fl * 10 // 4
    res = {"fwd_ms": round(ms, 3), "fwd_eff_tflops": round(fl / ms / 1e9, 1),
           "fwd_frac": round(fl / ms / 1e9 / peaks["bf16_tflops"], 4),
           "bwd_ms": round(ms_b, 3), "bwd_eff_tflops": round(fl_b / ms_b / 1e9, 1),
           "bwd_frac": round(fl_b / ms_b / 1e9 / peaks["bf16_tflops"], 4), "status": V.vattn_get_status(),
           "h_pool": list(hp)}
    del q, k, v, o, lse, ws, do, dq, dk, dv, wsb
    torch.cuda.empty_cache()
    return res


def _bench_sym_learned(V, dev, peaks, n=4, warm=2, heads=None):
    """Dual forward with the learned symmetric global branch (depthwise
    strided compression, 3x3x3 depthwise restoration, seeded random weights)
    at the 1080p workload; effective FLOPs as the average-pooling form (the
    convolutions are HBM / L2 work, reported with it, not counted)."""
    import torch
    from synth import inputs as S
    w = S.WORKLOADS["1080p"]
    if heads:   # reduced case for profiling only
        import dataclasses
        w = dataclasses.replace(w, heads=heads)
    geom = _geom(V, w)
    T, H, W = w.grid
    npool = (T // w.pool[0]) * (H // w.pool[1]) * (W // w.pool[2])
    shape = (w.batch, w.heads, w.n_tokens, w.head_dim)
    q, k, v = (_device_randn(shape, 700 + i) for i in range(3))
    gvec = torch.rand(w.heads, device=dev)
    wts = {n: torch.from_numpy(a).to(dev) for n, a in S.learned_weights(w).items()}
    o = torch.empty_like(q)
    ws = torch.empty(V.vattn_workspace_size(V.VATTN_OP_DUAL_SYM_LEARNED_FWD, geom), dtype=torch.uint8, device=dev)
    fl, _ = _flops_fwd(w)
    fl += 4 * w.head_dim * w.batch * w.heads * npool * npool
    scale = 1 / math.sqrt(w.head_dim)

    def call():
        V.vattn_dual_sym_learned_fwd(geom, q, k, v, gvec, wts["wq"], wts["wk"], wts["wv"], wts["w3"], scale, o, ws)
    ms = _time_ms(call, n, warm=warm)
    res = {"ms": round(ms, 3), "eff_tflops": round(fl / ms / 1e9, 1),
           "frac": round(fl / ms / 1e9 / peaks["bf16_tflops"], 4), "status": V.vattn_get_status()}
    del q, k, v, o, ws
    torch.cuda.empty_cache()
    return res


def _bench_sym(V, dev, peaks):
    """Dual forward with the symmetric (query-pooled) global branch at the
    1080p workload; effective FLOPs: local pairs + pooled N_p x N_p pairs."""
    import torch
    from synth import inputs as S
    w = S.WORKLOADS["1080p"]
    geom = _geom(V, w)
    T, H, W = w.grid
    npool = (T // w.pool[0]) * (H // w.pool[1]) * (W // w.pool[2])
    shape = (w.batch, w.heads, w.n_tokens, w.head_dim)
    q, k, v = (_device_randn(shape, 600 + i) for i in range(3))
    gvec = torch.rand(w.heads, device=dev)
    o = torch.empty_like(q)
    ws = torch.empty(V.vattn_workspace_size(V.VATTN_OP_DUAL_SYM_FWD, geom), dtype=torch.uint8, device=dev)
    fl, _ = _flops_fwd(w)
    fl += 4 * w.head_dim * w.batch * w.heads * npool * npool
    scale = 1 / math.sqrt(w.head_dim)
    for _ in range(2):
        V.vattn_dual_sym_fwd(geom, q, k, v, gvec, scale, o, workspace=ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(4):
        V.vattn_dual_sym_fwd(geom, q, k, v, gvec, scale, o, workspace=ws)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / 4
    res = {"ms": round(ms, 3), "eff_tflops": round(fl / ms / 1e9, 1),
           "frac": round(fl / ms / 1e9 / peaks["bf16_tflops"], 4), "status": V.vattn_get_status()}
    del q, k, v, o, ws
    torch.cuda.empty_cache()
    return res


def _xwin_pairs(w, shifted: bool) -> int:
    """Query-key pairs of cross-window attention: the block extents are
    separable per dim, so the sum over query tiles factorises."""
    sizes = 1
    for n_t, win in zip([a // b for a, b in zip(w.grid, w.tile)], w.window):
        size = win + 1 if shifted else win
        off = (win + 1) // 2 if shifted else 0
        tot = 0
        for a in range(n_t):
            b = (a + off) // size
            tot += min((b + 1) * size - off, n_t) - max(b * size - off, 0)
        sizes *= tot
    s = math.prod(w.tile)
    return w.batch * w.heads * s * s * sizes


def _bench_xwin(V, dev, peaks):
    """Cross-window local attention at the 1080p grid (window 3x3x3), both
    partitions, forward kernel timed alone."""
    import torch
    from synth import inputs as S
    w = S.WORKLOADS["1080p"]
    geom = _geom(V, w)
    shape = (w.batch, w.heads, w.n_tokens, w.head_dim)
    q, k, v = (_device_randn(shape, 500 + i) for i in range(3))
    o = torch.empty_like(q)
    lse = torch.empty(shape[:3], dtype=torch.float32, device=dev)
    res = {}
    for shifted in (0, 1):
        fl = 4 * w.head_dim * _xwin_pairs(w, bool(shifted))
        for _ in range(2):
            V.vattn_xwin_fwd(geom, shifted, q, k, v, 1 / math.sqrt(w.head_dim), o, lse)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(5):
            V.vattn_xwin_fwd(geom, shifted, q, k, v, 1 / math.sqrt(w.head_dim), o, lse)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / 5
        res[f"1080p_xwin_fwd_{'shifted' if shifted else 'partition'}"] = {
            "ms": round(ms, 3), "eff_tflops": round(fl / ms / 1e9, 1),
            "frac": round(fl / ms / 1e9 / peaks["bf16_tflops"], 4), "status": V.vattn_get_status()}
    del q, k, v, o, lse
    torch.cuda.empty_cache()
    return res


def _bench_train(V, dev, peaks, w=None, n=3, warm=2):
    """Training workload (B2 h24 d128, 1080p grid): dual forward with saved
    outputs, then the dual backward; effective FLOPs 4d (fwd) + 10d (bwd) per
    computed pair."""
    import torch
    from synth import inputs as S
    w = w or S.WORKLOADS["train"]
    geom = _geom(V, w)
    T, H, W = w.grid
    npool = (T // w.pool[0]) * (H // w.pool[1]) * (W // w.pool[2])
    shape = (w.batch, w.heads, w.n_tokens, w.head_dim)
    q, k, v = (_device_randn(shape, 400 + i) for i in range(3))
    do = _device_randn(shape, 404, std=0.1)
    gvec = torch.rand(w.heads, device=dev)
    scale = 1 / math.sqrt(w.head_dim)
    o, o_l, o_g, dq, dk, dv = (torch.empty_like(q) for _ in range(6))
    lse_l = torch.empty(shape[:3], dtype=torch.float32, device=dev)
    lse_g = torch.empty_like(lse_l)
    kp = torch.empty((w.batch, w.heads, npool, w.head_dim), dtype=torch.bfloat16, device=dev)
    vp = torch.empty_like(kp)
    ws = torch.empty(V.vattn_workspace_size(V.VATTN_OP_DUAL_BWD, geom), dtype=torch.uint8, device=dev)
    fl, fg = _flops_fwd(w)
    bwd_flops = 2.5 * (fl + fg)

    def fwd():
        V.vattn_dual_fwd(geom, q, k, v, gvec, scale, o, o_l, lse_l, o_g, lse_g, kp, vp)

    def bwd():
        V.vattn_dual_bwd(geom, q, k, v, gvec, o_l, lse_l, o_g, lse_g, kp, vp, do, scale, dq, dk, dv, None, ws)
    for _ in range(warm):
        fwd()
        bwd()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    tf = tb = 0.0
    for _ in range(n):
        ev[0].record()
        fwd()
        ev[1].record()
        bwd()
        ev[2].record()
        torch.cuda.synchronize()
        tf += ev[0].elapsed_time(ev[1])
        tb += ev[1].elapsed_time(ev[2])
    tf, tb = tf / n, tb / n
    res = {"fwd_ms": round(tf, 3), "bwd_ms": round(tb, 3),
           "fwd_eff_tflops": round((fl + fg) / tf / 1e9, 1), "bwd_eff_tflops": round(bwd_flops / tb / 1e9, 1),
           "step_eff_tflops": round((fl + fg + bwd_flops) / (tf + tb) / 1e9, 1),
           "step_frac": round((fl + fg + bwd_flops) / (tf + tb) / 1e9 / peaks["bf16_tflops"], 4),
           "status": V.vattn_get_status()}
    del q, k, v, do, o, o_l, o_g, dq, dk, dv, ws
    torch.cuda.empty_cache()
    return res


def cpu_baseline(budget_s: float):
    """The fp64 oracle, as it stands, on a bounded sample of the 720p workload:
    one head (b=0, h=0), query tiles taken in a fixed order until the time
    budget is spent."""
    import numpy as np

    from oracle import vattn_oracle as O
    from synth import inputs as S
    w = S.WORKLOADS["720p"]
    g = O.geom_of(w)
    q, k, v = (S.bf16_bits_to_f64(S.draw_head(w, i, 0, 0)) for i in (S.Q_ID, S.K_ID, S.V_ID))
    scale = 1 / math.sqrt(w.head_dim)
    kept = O.kept_count_closed_form(g)
    s = g.tile_volume
    n_tiles = math.prod(g.tiles_per_dim)
    order = np.random.default_rng(0).permutation(n_tiles)
    done = 0
    t0 = time.perf_counter()
    while done < n_tiles and time.perf_counter() - t0 < budget_s:
        O.sta_attention_tiles(q, k, v, g, scale, [int(order[done])])
        done += 1
    dt = time.perf_counter() - t0
    flops = 4 * w.head_dim * done * s * kept * s
    cores = len(os.sched_getaffinity(0))
    return {"value": round(flops / dt / 1e12, 5), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"720p STA fwd, head (0,0), {done} of {n_tiles} query tiles ({done * s} queries), "
                      f"{dt:.1f} s, numpy fp64 BLAS threads={_blas_threads()}"}


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 0) for i in threadpool_info()), default=None)
    except Exception:
        return None


def run_reference(args):
    """Reference arm: the fp64 oracle on the host cores, a bounded sample per step."""
    import numpy as np

    from oracle import vattn_oracle as O
    from synth import inputs as S
    w = S.WORKLOADS["720p"]
    g = O.geom_of(w)
    q, k, v = (S.bf16_bits_to_f64(S.draw_head(w, i, 0, 0)) for i in (S.Q_ID, S.K_ID, S.V_ID))
    scale = 1 / math.sqrt(w.head_dim)
    kept = O.kept_count_closed_form(g)
    s = g.tile_volume
    n_tiles = math.prod(g.tiles_per_dim)
    tiles_per_step = 2
    order = np.random.default_rng(0).permutation(n_tiles)
    for i in range(args.warmup):
        O.sta_attention_tiles(q, k, v, g, scale, [int(t) for t in order[:tiles_per_step]])
    t0 = time.perf_counter()
    for i in range(args.steps):
        sel = [int(order[(i * tiles_per_step + j) % n_tiles]) for j in range(tiles_per_step)]
        O.sta_attention_tiles(q, k, v, g, scale, sel)
    dt = time.perf_counter() - t0
    flops = 4 * w.head_dim * args.steps * tiles_per_step * s * kept * s
    value = flops / dt / 1e12
    cores = len(os.sched_getaffinity(0))
    sample = (f"720p STA fwd, head (0,0), {tiles_per_step} query tiles ({tiles_per_step * s} queries) per step, "
              f"numpy fp64")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "TFLOP/s", "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1) bf16, per-head U(0.5,2) scale)",
            "config": {"workload": f"720p sliding-tile fwd: B1 h{w.heads} d128, grid 30x48x80, tile 6x8x8, window 3x3x3",
                       "sample": sample},
            "cpu_baseline": {"value": round(value, 5), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 5), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--e2e-chunk", type=int, default=1, help="batch*head slices per host-copy chunk (e2e)")
    ap.add_argument("--heads", type=int, default=0, help="profiling only: fewer heads than the workload")
    ap.add_argument("--workload", choices=["720p", "train", "fp8", "1080p", "4k", "sym_learned"], default="720p",
                    help="720p: the benchmark line; train, fp8, 1080p, 4k, sym_learned: profiling of the training "
                         "step, the FP8 forward, the 1080p / 4K dual forward or the learned symmetric branch alone")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        if args.workload == "train":
            result = run_train_only(args, rank, world, local_rank)
        elif args.workload == "fp8":
            result = run_fp8_only(args, rank, world, local_rank)
        elif args.workload in ("1080p", "4k"):
            result = run_dual_only(args, rank, world, local_rank)
        elif args.workload == "sym_learned":
            result = run_sym_learned_only(args, rank, world, local_rank)
        else:
            result = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(result), flush=True)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
