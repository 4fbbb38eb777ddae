"""The multi-process plumbing of the benchmark on CPU (gloo, world size 2):
the max-over-ranks timing reduction, the whole-job throughput, and the
reference arm printing one line under torchrun.  The attention path itself
has no exchange step (batch/head slices are independent), so N GPUs run N
replicas; these tests cover everything the replicas share."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out_dir):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        got = bench.reduce_max([1.0 + rank, 10.0 - rank, 0.5 * rank], world)
        dist.barrier()
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump(got, f)
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks(tmp_path):
    import random

    import torch.multiprocessing as mp
    port = random.randint(20000, 40000)
    mp.spawn(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        with open(tmp_path / f"r{r}.json") as f:
            assert json.load(f) == [2.0, 10.0, 0.5]


def test_whole_job_value_is_weak_scaling_sum():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.whole_job_tflops(1.4676e13, 15.0, 1)
    assert abs(bench.whole_job_tflops(1.4676e13, 15.0, 4) - 4 * one) < 1e-9
    assert abs(one - 1.4676e13 / 0.015 / 1e12) < 1e-9
    assert bench.reduce_max([3.0, 1.0], 1) == [3.0, 1.0]


@pytest.mark.slow
def test_reference_arm_prints_once_under_torchrun():
    import random
    port = random.randint(40001, 60000)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["value"] > 0


def test_bench_xwin_pair_count_matches_oracle_tiles():
    sys.path.insert(0, ROOT)
    import bench
    from oracle import vattn_oracle as O
    from synth import inputs as S
    w = S.small_workload("x", 1, 1, 2, 64, (6, 24, 40), (3, 8, 8), (2, 2, 2), (1, 1, 1))
    g = O.geom_of(w)
    for shifted in (False, True):
        brute = sum(len(qi) * len(kj) for qi, kj in O.xwin_query_tiles(g, shifted)) * w.batch * w.heads
        assert bench._xwin_pairs(w, shifted) == brute
