"""Seeded random routing without a plan against the oracle: HT and LL
layouts (random capacities, some overflowing), any top-K including those
that do not divide a warp (the routing cluster's per-token repeat check then
reads across warp ranges), and ids that are masked (-1), out of range or
repeated within a token, at batch sizes across every routing path (one CTA,
the cluster of 8 or 16 CTAs, three kernels). Each case compares the status
bits, destination rows, counts, source rows and dispatched rows with the
oracle, and the combine's output."""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_dispatch_03_b200 import synth

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

PAIRS = (1, 31, 500, 1024, 1025, 5000, 8192, 8193, 16384, 16385, 30000, 32768, 32769, 50000)


def _case(i):
    rng = np.random.default_rng(9000 + i)
    E = int(rng.choice([4, 8, 16, 33, 64, 129, 256, 384]))
    R = int(rng.choice([r for r in (1, 2, 4, 8) if E % r == 0]))
    K = int(rng.integers(1, min(E, 12) + 1))
    L = int(PAIRS[i % len(PAIRS)])
    T = max(1, (L + K - 1) // K)
    mode = "ll" if rng.random() < 0.4 else "ht"
    cap = int(rng.integers(1, max(2, 2 * T * K // E) + 1)) if mode == "ll" else 0
    s = float(rng.choice([0.0, 1.0, 2.5]))
    dirt = float(rng.choice([0.0, 0.0, 0.02, 0.1]))  # share of ids made masked, bad or repeated
    return T, E, K, R, mode, cap, s, dirt, 9000 + i


CASES = [_case(i) for i in range(120)]


def _dirty(idx, E, dirt, seed):
    """Masked, out-of-range and repeated ids, each on about dirt/3 of the pairs."""
    if dirt == 0.0:
        return idx
    rng = np.random.default_rng(seed)
    a = idx.numpy().copy()
    T, K = a.shape
    u = rng.random((T, K))
    a[u < dirt / 3] = -1
    bad = (u >= dirt / 3) & (u < 2 * dirt / 3)
    a[bad] = rng.choice([E, E + 7, -2, -1000], size=int(bad.sum()))
    if K > 1:
        rep = (u >= 2 * dirt / 3) & (u < dirt)
        rep[:, 0] = False
        ts, ks = np.nonzero(rep)
        a[ts, ks] = a[ts, rng.integers(0, ks)]  # an earlier choice of the same token
    return torch.from_numpy(a)


@pytest.mark.parametrize("T,E,K,R,mode,cap,s,dirt,seed", CASES)
def test_random_routing(T, E, K, R, mode, cap, s, dirt, seed):
    import gpu_cases as g

    H = 32
    idx, w = synth.routing(T, E, K, zipf_s=s, seed=seed)
    idx = _dirty(idx, E, dirt, seed)
    r = g.run_forward(T, H, E, K, R, mode=mode, cap=cap, idx=idx, w=w, seed=seed)
    ref = r["ref"]
    if dirt == 0.0:
        assert not (r["flags"] & (oracle.FLAG_BAD_EXPERT_ID | oracle.FLAG_DUP_EXPERT_ID))
    placed = ref.dest_row[ref.dest_row >= 0]
    assert len(np.unique(placed)) == len(placed)  # a row is never given twice
    r["h"].close()
