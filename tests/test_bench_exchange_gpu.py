"""bench.py --exchange on one GPU: the workload's R ranks as separate buffers,
through the peer-table calls, prints a line whose bytes are the single-GPU
step's and whose status word is clean."""
import json
import os
import subprocess
import sys

import pytest
import torch

from conftest import ROOT

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.mark.parametrize("workload", ["tiny", "ll_decode"])
def test_bench_exchange_line(workload):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--exchange", "--workload", workload,
                        "--steps", "3", "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "native-exchange" and line["value"] > 0 and line["device_flags"] == 0
    sys.path.insert(0, ROOT)
    import bench

    wl = bench.WORKLOADS[workload]
    placed = wl["T"] * wl["K"] if wl["mode"] == "ht" else None
    if placed is not None:
        want = sum(bench.algorithmic_bytes(wl["T"], wl["H"], wl["K"], placed, wl["fp8"]).values())
        assert line["bytes_per_step"] == want
    assert set(line["per_call_us"]) == {"plan", "dispatch", "combine"}
