"""The FP8 cast divides by each block's scale with Markstein's reciprocal-
and-correction method (csrc/fast_div.cuh). It must give the bits of a
correctly rounded division, which the oracle's e4m3 codes are pinned to:
this checks it against CUDA's __fdiv_rn on every bf16 input the cast can see."""
import os
import re
import subprocess

import pytest

from combine_ep_dispatch_03_b200 import build

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.gpu
def test_fast_division_matches_fdiv_rn_on_every_bf16_pair(tmp_path):
    exe = str(tmp_path / "fast_div_exhaustive")
    subprocess.check_call([build.NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                           "-I", os.path.join(build.PKG, "csrc"), "-I", os.path.join(build.ROOT, "include"),
                           "-o", exe, os.path.join(HERE, "fast_div_exhaustive.cu")])
    out = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stdout + out.stderr
    m = re.search(r"pairs (\d+) fast (\d+) mismatches (\d+)", out.stdout)
    pairs, fast, bad = map(int, m.groups())
    assert bad == 0
    assert pairs > 10**9 and fast > pairs // 2  # the guarded path covers most of the domain
