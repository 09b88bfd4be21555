"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2): the
whole-job value is all ranks' bytes over the slowest rank's device time, and
the reference arm runs on rank 0 only."""
import datetime
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    sys.path.insert(0, ROOT)
    import bench

    value, ms = bench.weak_scaling_value(2.0e9, 1.0 + rank, world)  # rank 1 is the slow one
    mx = bench.max_over_ranks(float(10 - rank), world)
    q.put((rank, value, ms, mx))
    dist.barrier()
    dist.destroy_process_group()


def test_weak_scaling_value_uses_slowest_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, value, ms, mx in got:
        assert ms == 2.0                      # max over ranks of the step time
        assert value == pytest.approx(2 * 2.0e9 / 2.0e-3 / 1e9)
        assert mx == 10.0


def _run_reference(rank: int, world: int):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                           "--warmup", "3"], env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_runs_on_rank_zero_only():
    r1 = _run_reference(1, 2)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _run_reference(0, 2)
    assert r0.returncode == 0
    import json

    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["higher_is_better"] is True
    required = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"}
    assert required <= set(line)
    sys.path.insert(0, ROOT)
    import bench

    assert line["metric"] == bench.METRIC and line["unit"] == "GB/s" and line["steps"] == 1
    assert line["config"]["workload"] == "ht_prefill" and line["e2e"]["value"] == line["value"] > 0
