"""Multi-rank host logic of the benchmark on CPU: two gloo ranks (one process
each, like one process per GPU) take the slowest rank's time, draw distinct
batches of the same workload, aggregate whole-job throughput, and only rank 0
reports.  No GPU and no data-path collective is involved (the path shards by
rows, so ranks are independent replicas)."""
import datetime
import json
import multiprocessing as mp
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    import hyena_workloads as hw
    t = bench.max_over_ranks(10.0 + 5.0 * rank, world)
    w = hw.make("c1", seed=bench.rank_seed("c1", rank), B=1, D=2, L=64)
    dist.barrier()
    q.put((rank, t, float(w.v.f32.sum()), w.v.f32.shape))
    dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_distinct_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    assert out[0][1] == out[1][1] == 15.0          # both see the slowest rank's time
    assert out[0][2] != out[1][2]                   # distinct batches
    assert out[0][3] == out[1][3]                   # same per-rank shape (weak scaling)


def test_job_value_aggregates_all_ranks():
    sys.path.insert(0, ROOT)
    import bench
    v1 = bench.job_value(1, 10, 1e9, 100.0)
    v4 = bench.job_value(4, 10, 1e9, 100.0)
    assert v1 == pytest.approx(100.0) and v4 == pytest.approx(4 * v1)
    # a slower slowest-rank lowers the whole-job number
    assert bench.job_value(4, 10, 1e9, 200.0) == pytest.approx(2 * v1)


def test_reference_arm_only_rank0_prints(tmp_path):
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True, env=env,
                       timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "c1", "--steps", "2", "--warmup", "0"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["fft_reference"]["value"] > 0
    # the steps it reports are the steps it timed
    assert line["steps"] == 2 and line["ms_per_step"] * line["steps"] <= 1e3 * line["wall_s"] * 1.05
    sys.path.insert(0, ROOT)
    import bench
    import hyena_workloads as hw
    assert line["config"] == bench.workload_config("c1", hw.make("c1", with_signals=False).spec, 1)


@pytest.mark.parametrize("name,over", [("c3", dict(D=2, L=1 << 15)), ("c4", dict(D=2, grid=(8, 8, 8))),
                                       ("c5", dict(H=2, Dh=4, L=64))])
def test_cpu_samples_of_every_workload(name, over):
    """The CPU baselines (direct oracle and naive FFT reference) run on a
    bounded sample of every workload kind and report a positive rate."""
    sys.path.insert(0, ROOT)
    import bench
    import hyena_workloads as hw
    w = hw.make(name, **over)
    cb = bench.cpu_baseline(w)
    assert cb["value"] > 0 and cb["fft_reference"]["value"] > 0 and cb["cores"] >= 1
