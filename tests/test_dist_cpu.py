"""The multi-process plumbing of bench.py on the CPU (gloo, world size 2):
replicas report their own device time, the job's time is the slowest rank's,
and the whole-job rate counts every rank's units. The GPU path runs the same
functions over NCCL."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    got = bench.max_over_ranks([10.0 + rank, 5.0 - rank])
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, got))


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1] == [11.0, 5.0]


def test_whole_job_rate_and_single_process_identity():
    import bench
    assert bench.max_over_ranks([3.0, 4.5]) == [3.0, 4.5]       # not distributed
    # 2 ranks x 100 units each, slowest rank 50 ms -> 4000 units / s
    assert bench.whole_job_rate(100, 50.0, 2) == pytest.approx(4000.0)


def test_reference_arm_runs_the_oracle_on_cpu():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "2", "--warmup", "1", "--ref-step-seconds", "0.3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_bench_spawns_its_own_ranks():
    # `bench.py --gpus 2` outside torchrun relaunches itself as two ranks; the
    # reference arm then runs on rank 0 only (gloo on a host without GPUs) and
    # prints one line that reports the world size it ran under.
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--steps", "1", "--warmup", "1",
                          "--ref-step-seconds", "0.2"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert out.returncode == 0, out.stderr[-3000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0


def test_peak_follows_observed_conditions():
    import bench
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    capped = {"reasons": ["sw_power_cap"]}
    assert bench.pick_peak(peaks, 5.0, capped) == (1400.0, "sustained")
    assert bench.pick_peak(peaks, 0.5, capped) == (1600.0, "burst")      # too short
    assert bench.pick_peak(peaks, 5.0, {"reasons": []}) == (1600.0, "burst")
    assert bench.pick_peak(peaks, 5.0, None) == (1600.0, "burst")
