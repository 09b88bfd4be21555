"""GPU parity for the two steps around the path: the router top-K that feeds
ep_plan, and the replica weight prefetch driven by the balanced plan.

Router tolerance: expert ids bit-exact (both sides compare the same fp32
logits, ties to the lower id). Weights: the kernel computes
exp(l_k - l_0) / sum_j exp(l_j - l_0) in fp32. That is one rounded
subtraction (a relative error of |l_k - l_0| * 2^-24 after the exponential),
CUDA's expf (at most 2 ulp), K - 1 rounded additions and one rounded division.
The oracle computes it in double and rounds once. So
|w_gpu - w_oracle| <= (8 + K + |l_k - l_0|) * 2^-24 * w_oracle.
Prefetch: bit-exact copies, empty slots untouched.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_dispatch_03_b200 import ep, synth

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from combine_ep_dispatch_03_b200 import build

    build.build()
    oracle.build()
    ep.lib()


def _router_gpu(logits, K):
    T, E = logits.shape
    lg = logits.cuda()
    idx = torch.full((T, K), -5, dtype=torch.int32, device="cuda")
    w = torch.full((T, K), -1.0, dtype=torch.float32, device="cuda")
    ep.router_topk(lg, K, idx, w)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy()


def _check_router(logits, K):
    gi, gw = _router_gpu(logits, K)
    oi, ow = oracle.router_topk(logits, K)
    np.testing.assert_array_equal(gi, oi)
    lg = logits.numpy().astype(np.float64)
    sel = np.take_along_axis(lg, oi, axis=1)
    spread = np.abs(sel - sel[:, :1])
    bound = (8 + K + spread) * 2.0 ** -24 * ow.astype(np.float64)
    assert (np.abs(gw.astype(np.float64) - ow) <= bound + 1e-38).all()


@pytest.mark.parametrize("T,E,K,s", [
    (32768, 256, 8, 0.0),   # HT prefill router
    (1024, 256, 8, 0.0),    # LL decode router
    (32768, 128, 8, 1.5),   # imbalance sweep, strongest skew
    (4096, 384, 8, 1.0),    # large training step shape (fewer tokens)
    (128, 16, 2, 0.0),      # tiny
    (100, 100, 3, 0.5),     # E not a multiple of 32
    (50, 1024, 32, 0.5),    # the largest E and K
    (64, 8, 8, 0.0),        # K = E
    (37, 33, 1, 0.0),       # K = 1, one lane holds two experts
    # four lanes a token (K <= 8, E a multiple of 16): a last warp with fewer
    # than 8 tokens, an odd count of 16-byte vectors a lane, K < 8, E = 1024
    (1001, 48, 3, 0.0),
    (777, 1024, 8, 0.0),
    (513, 64, 1, 0.5),
    (9, 16, 8, 0.0),
])
def test_router_topk_parity(T, E, K, s):
    _check_router(synth.router_logits(T, E, zipf_s=s, seed=T + E + K), K)


def test_router_topk_ties():
    """Logits rounded to one decimal: many exact ties, all broken to the lower id."""
    logits = torch.round(synth.router_logits(2000, 64, seed=3) * 10) / 10
    _check_router(logits.contiguous(), 8)


@pytest.mark.parametrize("T,E,K", [(3000, 256, 8), (200, 1024, 32), (500, 40, 5), (300, 1024, 8), (257, 48, 6)])
def test_router_topk_near_ties(T, E, K):
    """Each token's logits agree in all but their lowest 11 mantissa bits: the
    choices and their order must follow the full fp32 values."""
    g = torch.Generator().manual_seed(T + E)
    base = torch.randn(T, 1, generator=g).expand(T, E).contiguous()
    low = torch.randint(0, 1 << 11, (T, E), generator=g, dtype=torch.int32)
    _check_router((base.view(torch.int32) ^ low).view(torch.float32).contiguous(), K)


def _fuzz_case(i):
    rng = np.random.default_rng(11000 + i)
    if i % 2 == 0:  # four lanes a token: K <= 8, E a multiple of 16
        E = int(rng.choice([16, 32, 48, 64, 128, 256, 384, 512, 1024]))
        K = int(rng.integers(1, min(E, 8) + 1))
    else:  # a warp a token
        E = int(rng.integers(1, 1025))
        K = int(rng.integers(1, min(E, 32) + 1))
    T = int(rng.choice([1, 7, 8, 9, 63, 64, 65, 500, 2049]))
    kind = ["normal", "ties", "near", "signed_zero", "wide"][i % 5]
    return T, E, K, kind, 11000 + i


@pytest.mark.parametrize("T,E,K,kind,seed", [_fuzz_case(i) for i in range(60)])
def test_router_topk_random(T, E, K, kind, seed):
    """Random sizes on both router kernels and logits that stress the
    selection: exact ties (values on a coarse grid), near-ties (all but the
    low mantissa bits equal), signed zeros among them, and a wide range of
    magnitudes and signs. Ids bit-exact; weights within the derived bound."""
    g = torch.Generator().manual_seed(seed)
    if kind == "normal":
        lg = torch.randn(T, E, generator=g)
    elif kind == "ties":
        lg = torch.randint(-3, 4, (T, E), generator=g).to(torch.float32) * 0.5
    elif kind == "near":
        base = torch.randn(T, 1, generator=g).expand(T, E).contiguous()
        low = torch.randint(0, 1 << 9, (T, E), generator=g, dtype=torch.int32)
        lg = (base.view(torch.int32) ^ low).view(torch.float32)
    elif kind == "signed_zero":
        lg = torch.randint(-1, 2, (T, E), generator=g).to(torch.float32) * 1e-3
        zero = torch.rand(T, E, generator=g) < 0.5
        lg[zero] = torch.where(torch.rand(int(zero.sum()), generator=g) < 0.5, torch.tensor(0.0),
                               torch.tensor(-0.0))
    else:
        lg = torch.randn(T, E, generator=g) * torch.exp(torch.randn(T, E, generator=g) * 8)
    _check_router(lg.contiguous(), K)


def test_router_feeds_plan_dispatch_combine():
    """Router -> plan -> dispatch -> combine on the GPU equals the oracle chain."""
    import gpu_cases

    T, H, E, K, R = 2048, 1024, 64, 8, 8
    logits = synth.router_logits(T, E, zipf_s=0.5, seed=11)
    idx, w = _router_gpu(logits, K)
    oi, ow = oracle.router_topk(logits, K)
    np.testing.assert_array_equal(idx, oi)
    r = gpu_cases.run_forward(T, H, E, K, R, idx=torch.from_numpy(idx), w=torch.from_numpy(w), seed=11)
    assert r["combine_diff"] == 0


def test_router_rejects_bad_sizes():
    lg = torch.zeros((4, 2048), device="cuda")
    with pytest.raises(ep.EpError):
        _ = ep.router_topk(lg, 8, torch.empty((4, 8), dtype=torch.int32, device="cuda"),
                           torch.empty((4, 8), device="cuda"))


@pytest.mark.parametrize("E,R,slots,s,B", [(384, 16, 0, 1.0, 4096 + 16), (64, 8, 2, 2.0, 1040), (16, 4, 0, 1.5, 16)])
def test_prefetch_replica_weights(E, R, slots, s, B):
    T, K, H = 4096, 8, 128
    idx, w = synth.routing(T, E, K, zipf_s=s, seed=E)
    h = ep.Ep(T, H, E, K, R, balanced=True, replica_slots=slots)
    h.plan(idx.cuda())
    S = h.S
    g = torch.Generator().manual_seed(E)
    weights = torch.randint(0, 256, (E, B), dtype=torch.uint8, generator=g)
    slots_init = torch.randint(0, 256, (R, S, B), dtype=torch.uint8, generator=g)
    wd, sd = weights.cuda(), slots_init.cuda()
    h.prefetch_replica_weights(wd, sd)
    ref = oracle.route(idx, E=E, R=R, balanced=True, slots=S)
    rep, _ = h.get_plan()
    np.testing.assert_array_equal(np.array(rep).reshape(R, S), ref.plan["replica_expert"])
    want = oracle.prefetch(ref.plan["replica_expert"], weights.numpy(), slots_init.numpy().reshape(R * S, B))
    np.testing.assert_array_equal(sd.cpu().numpy().reshape(R * S, B), want)
    assert (np.array(rep) >= 0).any()


def test_prefetch_needs_a_plan():
    h = ep.Ep(16, 128, 8, 2, 2)
    h.plan(torch.zeros((16, 2), dtype=torch.int32, device="cuda"))
    with pytest.raises(ep.EpError):
        h.prefetch_replica_weights(torch.zeros((8, 16), dtype=torch.uint8, device="cuda"),
                                   torch.zeros((2, 1, 16), dtype=torch.uint8, device="cuda"))
