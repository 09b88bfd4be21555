"""Seeded random balanced plans against the oracle: expert counts, ranks,
replica slots, direct overflow, skew and batch sizes drawn so that every
routing path builds plans (one CTA up to 1024 pairs, the routing cluster of
8 or 16 CTAs up to 32768, three kernels beyond), including plans whose slots
run out (the planner's one-thread walk). Each case compares the destination
rows, counts, per-rank tables, replica and direct tables and the dispatched
rows with the oracle; without direct overflow it also runs the backward with
the replica-gradient reduce, and it copies the filled slots' weights with the
prefetch."""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_dispatch_03_b200 import ep, synth

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

PAIRS = (64, 700, 1024, 1025, 3000, 8192, 8193, 16384, 20000, 32768, 40000)


def _case(i):
    rng = np.random.default_rng(7000 + i)
    E = int(rng.choice([8, 16, 24, 32, 64, 96, 128, 256, 384]))
    R = int(rng.choice([r for r in (2, 4, 8, 16) if E % r == 0 and E // r >= 1]))
    K = int(rng.choice([k for k in (1, 2, 4, 6, 8) if k <= E]))
    L = int(PAIRS[i % len(PAIRS)])
    T = max(1, (L + K - 1) // K)
    g = E // R
    S = int(rng.integers(1, g + 1)) if rng.random() < 0.7 else 0  # 0: the default, E/R slots
    direct = bool(S > 0 and rng.random() < 0.4)
    s = float(rng.choice([0.0, 0.7, 1.2, 2.0, 3.0]))
    return T, E, K, R, S, direct, s


CASES = [_case(i) for i in range(120)]


def _gc():
    import gpu_cases

    return gpu_cases


@pytest.mark.parametrize("T,E,K,R,S,direct,s", CASES)
def test_random_balanced_plans(T, E, K, R, S, direct, s):
    g = _gc()
    H = 64
    r = g.run_forward(T, H, E, K, R, balanced=True, slots=S, direct=direct, zipf_s=s, seed=T + E + K,
                      check_combine=False, G=0 if direct else 32)
    h, ref = r["h"], r["ref"]
    assert ep.plan_launches(h) == (1 if T * K <= 32768 else 3)
    _, load = h.get_plan()
    if not (r["flags"] & oracle.FLAG_PLAN_SLOTS):
        assert max(load) - min(load) <= 1  # every rank floor or ceil of L/R
    # the filled slots' weights, copied by the prefetch (through its slot list)
    Sh = h.S
    gen = torch.Generator().manual_seed(T + E)
    B = 48
    weights = torch.randint(0, 256, (E, B), dtype=torch.uint8, generator=gen)
    slots0 = torch.randint(0, 256, (R, Sh, B), dtype=torch.uint8, generator=gen)
    wd, sd = weights.cuda(), slots0.cuda()
    h.prefetch_replica_weights(wd, sd)
    want = oracle.prefetch(ref.plan["replica_expert"], weights.numpy(), slots0.numpy().reshape(R * Sh, B))
    np.testing.assert_array_equal(sd.cpu().numpy().reshape(R * Sh, B), want)
    if not direct:
        g.run_backward(r, seed=T)
    h.close()
