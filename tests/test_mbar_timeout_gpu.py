"""The bf16 dispatch waits on an mbarrier for its own bulk copy of a row, and
that wait is bounded: past its limit the kernel sets EP_FLAG_WAIT_TIMEOUT
and returns, so a copy that never completes cannot hang the GPU. This runs
the same wait code (csrc/bulk.cuh) on a barrier phase armed for bytes that
no copy ever delivers, a condition that needs no fault: the wait must give
up at its limit, while a real copy on the same barrier completes."""
import os
import re
import subprocess

import pytest

from combine_ep_dispatch_03_b200 import build

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    exe = str(tmp_path_factory.mktemp("mbar") / "mbar_timeout")
    subprocess.check_call([build.NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                           "-I", os.path.join(build.PKG, "csrc"), "-o", exe,
                           os.path.join(HERE, "mbar_timeout.cu")])
    return exe


def _run(exe, arg):
    out = subprocess.run([exe, arg], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    m = re.search(r"copy_ok (\d+) data_ok (\d+) gave_up (\d+) waited_ns (\d+) limit_ns (\d+)", out.stdout)
    return tuple(map(int, m.groups()))


@pytest.mark.gpu
@pytest.mark.parametrize("arg", ["50", "default"])
def test_wait_gives_up_at_its_limit(probe, arg):
    copy_ok, data_ok, gave_up, waited, limit = _run(probe, arg)
    assert copy_ok == 1 and data_ok == 1  # a copy that lands completes its phase
    assert gave_up == 1                   # a phase whose bytes never arrive does not
    assert limit <= waited < limit + 500_000_000
    if arg == "default":
        assert limit == 2_000_000_000     # the limit the dispatch kernel uses
