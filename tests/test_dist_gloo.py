"""Multi-rank host logic on CPU (gloo, world size 2): the benchmark's
whole-job value is all ranks' bytes over the slowest rank's device time, the
reference arm runs on rank 0 only, and the host side of expert parallelism
across GPUs (gathered counts, identical plans, exchanged IPC handles) agrees
with the oracle's routing of the concatenated batch."""
import datetime
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
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


# ---------------------------------------------------------------------------
# Expert parallelism across ranks, host side: per-rank counts gathered with
# the package's own collective (combine_ep_dispatch_03_b200.world), then
# every rank's plan from the gathered counts, against the oracle's routing of
# the concatenated batch.

def _first_rows(dest_row, idx, lo, hi, K, E):
    """Row of the first pair (in (t, k) order) of expert e among tokens
    [lo, hi) of a routing, or -1."""
    first = np.full(E, -1, np.int64)
    flat = idx[lo:hi].reshape(-1)
    rows = dest_row[lo * K:hi * K]
    for p in range(flat.size - 1, -1, -1):
        e = flat[p]
        if 0 <= e < E and rows[p] >= 0:
            first[e] = rows[p]
    return first


def _world_worker(rank, world, port, q, balanced):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    sys.path.insert(0, ROOT)
    import oracle
    from combine_ep_dispatch_03_b200 import synth, world as wmod

    oracle.build()
    Tl, E, K = 300, 64, 4
    idx_all, _ = synth.routing(Tl * world, E, K, zipf_s=1.0, seed=17)
    idx_all = idx_all.numpy()
    mine = idx_all[rank * Tl:(rank + 1) * Tl]
    local = oracle.route(mine, E=E, R=1)  # this rank's per-expert counts
    counts = wmod.gather_counts(torch.from_numpy(local.cnt.astype(np.int32)))
    wc = counts.numpy()
    # the world's plan from the gathered counts alone: a batch with those
    # counts, rank by rank (one choice per token), has the same plan, and the
    # stable index of rank r's first pair of expert e is the pairs of e on
    # ranks below r
    fake = np.concatenate([np.repeat(np.arange(E), wc[r]) for r in range(world)]).astype(np.int32)[:, None]
    plan = oracle.route(fake, E=E, R=world, balanced=balanced)
    off = np.concatenate([[0], np.cumsum(wc.sum(axis=1))])
    bases = _first_rows(plan.dest_row, fake, int(off[rank]), int(off[rank + 1]), 1, E)
    res = {"counts": wc.tolist(), "rank_off": (plan.plan["rank_off"] if balanced else
                                               np.concatenate([[0], np.cumsum(plan.cnt)])[::E // world]).tolist(),
           "replica": plan.plan["replica_expert"].tolist() if balanced else None,
           "bases": bases.tolist()}
    handles = wmod.exchange_handles({"recv_x": (bytes([rank]) * 64, 1000 + rank)})
    res["handles"] = [(h["recv_x"][0][0], h["recv_x"][1]) for h in handles]
    q.put((rank, res))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("balanced", [False, True])
def test_world_plan_from_gathered_counts(balanced):
    """Both ranks gather the same [R, E] counts, derive the same plan, rank
    offsets and rows, and these equal the oracle's routing of the concatenated
    batch: rank r's first row of expert e is the row the concatenated routing
    gives rank r's first pair of e. The IPC handles come back in rank order."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_world_worker, args=(r, world, port, q, balanced)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    sys.path.insert(0, ROOT)
    import oracle
    from combine_ep_dispatch_03_b200 import synth

    Tl, E, K = 300, 64, 4
    idx_all, _ = synth.routing(Tl * world, E, K, zipf_s=1.0, seed=17)
    idx_all = idx_all.numpy()
    ref = oracle.route(idx_all, E=E, R=world, balanced=balanced)
    assert got[0]["counts"] == got[1]["counts"]
    for r in range(world):
        np.testing.assert_array_equal(got[r]["counts"][r], oracle.route(idx_all[r * Tl:(r + 1) * Tl], E=E, R=1).cnt)
    assert got[0]["rank_off"] == got[1]["rank_off"]
    if balanced:
        np.testing.assert_array_equal(got[0]["rank_off"], ref.plan["rank_off"])
        assert got[0]["replica"] == got[1]["replica"] == ref.plan["replica_expert"].tolist()
    else:
        np.testing.assert_array_equal(got[0]["rank_off"], np.concatenate([[0], np.cumsum(ref.cnt)])[::E // world])
    for r in range(world):
        want = _first_rows(ref.dest_row, idx_all, r * Tl, (r + 1) * Tl, K, E)
        np.testing.assert_array_equal(got[r]["bases"], want)
        assert got[r]["handles"] == [(0, 1000), (1, 1001)]
