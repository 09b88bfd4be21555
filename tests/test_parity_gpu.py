"""GPU parity: the CUDA path (through the C-ABI) against the CPU oracle, element
by element, on seeded synthetic inputs. Tolerances are in tests/gpu_cases.py."""
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


def _gc():
    import gpu_cases

    return gpu_cases


# --------------------------------------------------------------- the workloads

def test_tiny_identity_expert_returns_x():
    """Tiny workload: HT, identity expert, weights summing to 1 -> x."""
    g = _gc()
    r = g.run_forward(128, 1024, 16, 2, 4, y_kind="identity")
    np.testing.assert_array_equal(g.bits16(r["combine_out"]), g.bits16(r["x"]))
    g.run_backward(r)


def test_ll_decode_full_size():
    """LL decode workload at its full size: 1024 tokens, H=7168, E=256, top-8,
    R=8, capacity 1024, combine of the affine expert 1.5 x + 0.25."""
    g = _gc()
    r = g.run_forward(1024, 7168, 256, 8, 8, mode="ll", cap=1024, check_combine=False)
    h, ref, dev = r["h"], r["ref"], torch.device("cuda")
    y = synth.affine_expert(r["bufs"]["recv_x"])
    o = torch.empty((1024, 7168), dtype=torch.bfloat16, device=dev)
    h.combine(y, r["w"].to(dev), o)
    want = oracle.combine(y.cpu(), r["w"], ref.dest_row, 1024, 8)
    g.assert_bf16_close(g.bits16(o), want, "LL combine")
    # padding rows of the 3D buffer are never targeted
    counts = r["bufs"]["recv_counts"].cpu().numpy()
    assert counts.sum() == 1024 * 8 and counts.max() <= 1024


def test_ht_prefill_fp8_reduced():
    """HT prefill shape (H=7168, E=256, top-8, R=8, FP8) on 2048 tokens."""
    g = _gc()
    r = g.run_forward(2048, 7168, 256, 8, 8, fp8=True)
    assert r["fp8_diff"] == 0  # IEEE division + RNE on both sides
    assert r["combine_diff"] == 0


@pytest.mark.parametrize("s", [0.0, 0.5, 1.0, 1.5])
@pytest.mark.parametrize("balanced", [False, True])
def test_imbalance_sweep_reduced(s, balanced):
    """Imbalance-sweep shape (H=4096, E=128, top-8, R=8) on 4096 tokens."""
    g = _gc()
    r = g.run_forward(4096, 4096, 128, 8, 8, balanced=balanced, zipf_s=s, seed=int(s * 10))
    if balanced:
        _, load = r["h"].get_plan()
        assert max(load) - min(load) <= 1  # flat whatever the skew


def test_large_train_reduced_forward_backward():
    """Large training-step shape (E=384, top-8, R=16, Zipf 1.0, balanced plan)
    with fewer tokens and a narrower hidden size; forward, backward and the
    replica-gradient reduce."""
    g = _gc()
    r = g.run_forward(4096, 1024, 384, 8, 16, balanced=True, zipf_s=1.0, seed=3, G=4096 + 12)
    g.run_backward(r, seed=3)
    rep, load = r["h"].get_plan()
    assert max(load) - min(load) <= 1
    assert sum(e >= 0 for e in rep) > 0


# --------------------------------------------------------------- random shapes

def _random_cases(n=24):
    rng = np.random.default_rng(2024)
    cases = []
    for i in range(n):
        E = int(rng.choice([4, 8, 16, 32]))
        R = int(rng.choice([r for r in (1, 2, 4, 8) if E % r == 0]))
        K = int(rng.integers(1, min(8, E) + 1))
        T = int(rng.integers(1, 301))
        fp8 = bool(i % 3 == 1)
        H = int(rng.choice([128, 256, 1024])) if not fp8 else int(rng.choice([128, 640, 1024]))
        mode = "ll" if i % 4 == 3 else "ht"
        balanced = mode == "ht" and i % 4 == 2
        cap = int(rng.integers(1, T + 1)) if mode == "ll" else 0
        cases.append((T, H, E, K, R, mode, cap, fp8, balanced, float(rng.choice([0.0, 1.0, 2.0])), i))
    return cases


@pytest.mark.parametrize("T,H,E,K,R,mode,cap,fp8,balanced,s,seed", _random_cases())
def test_random_small_shapes(T, H, E, K, R, mode, cap, fp8, balanced, s, seed):
    g = _gc()
    r = g.run_forward(T, H, E, K, R, mode=mode, cap=cap, fp8=fp8, balanced=balanced, zipf_s=s, seed=seed,
                      G=64 if balanced else 0)
    if not fp8:
        g.run_backward(r, seed=seed)


@pytest.mark.parametrize("T,K", [(3000, 2), (2049, 1), (777, 3), (300, 32)])
def test_several_tiles_ragged_tail(T, K):
    """Routing tiles hold about 2048 pairs: these span several tiles with a
    ragged last one (and K = 32, the largest top-k)."""
    g = _gc()
    E = 64
    r = g.run_forward(T, 256, E, K, 4, seed=T)
    g.run_backward(r, seed=T)


@pytest.mark.parametrize("T,E,K,mode,cap", [(1100, 129, 6, "ht", 0), (4096, 256, 8, "ll", 100),
                                             (2000, 1024, 5, "ht", 0), (1024, 384, 32, "ht", 0),
                                             (3001, 200, 3, "ll", 64)])
def test_cluster_routing_with_bad_and_repeated_ids(T, E, K, mode, cap):
    """Batches of 1025..32768 pairs are routed by one launch of a cluster of
    8 CTAs: expert counts that are not powers of two, top-k that does not
    divide a warp (a token's earlier choices in the previous warp's range),
    capacity drops, and masked, bad and repeated ids."""
    g = _gc()
    H, R = 256, 4 if E % 4 == 0 else 1
    x, idx, w = g.make_inputs(T, H, E, K, zipf_s=1.0, seed=T)
    idx = idx.clone()
    flat = idx.view(-1)
    rng = np.random.default_rng(T)
    # a repeat on a pair that starts a 32-pair word (its earlier choices sit
    # in the previous word), elsewhere too
    for p in list(range(32, T * K, 32 * 7)) + rng.integers(0, T * K, 40).tolist():
        if p % K:
            flat[p] = flat[p - 1]
    flat[rng.integers(0, T * K, 25)] = -1
    flat[rng.integers(0, T * K, 5)] = E + 3
    h = ep.Ep(T, H, E, K, R, mode=mode, ll_capacity=cap)
    assert ep.plan_launches(h) == 1
    r = g.run_forward(T, H, E, K, R, mode=mode, cap=cap, idx=idx, w=w, x=x)
    assert r["flags"] & oracle.FLAG_BAD_EXPERT_ID and r["flags"] & oracle.FLAG_DUP_EXPERT_ID
    g.run_backward(r, seed=T)


@pytest.mark.parametrize("T,K", [(1025, 1), (8192, 1), (8193, 1), (2048, 8), (16385, 1), (32767, 1),
                                 (4096, 8), (32769, 1)])
def test_routing_shape_boundaries(T, K):
    """Batches on either side of each switch of the routing's shape: one CTA
    up to 1024 pairs; a cluster of 8 CTAs x 16 warps up to 8192; 16 x 16 up
    to 16384; 16 x 32 up to 32768; three kernels beyond."""
    g = _gc()
    r = g.run_forward(T, 128, 64, K, 4, seed=T + K, check_combine=False)
    assert r["flags"] == 0


@pytest.mark.parametrize("T,K,E,R,direct", [(128, 8, 256, 8, False), (129, 8, 256, 8, False),
                                             (128, 8, 256, 8, True), (1024, 1, 64, 4, False),
                                             (1025, 1, 64, 4, True), (300, 3, 384, 16, False),
                                             (1024, 8, 256, 8, True), (2048, 8, 384, 16, False),
                                             (4096, 8, 256, 8, False), (4097, 8, 256, 8, False),
                                             (4097, 8, 128, 8, True)])
def test_balanced_plan_shape_boundaries(T, K, E, R, direct):
    """The balanced plan is built inside the one-CTA routing kernel up to
    1024 pairs, by every CTA of the one-launch routing cluster up to 32768
    pairs (CTA 0 writes the tables out), and by the three-kernel path beyond: both
    sides of each switch, with skewed routing, training and inference plans
    (two slots a rank for the inference plan), forward and backward with the
    replica reduce."""
    g = _gc()
    h = ep.Ep(T, 128, E, K, R, balanced=True, replica_slots=2 if direct else 0, direct_overflow=direct)
    assert ep.plan_launches(h) == (1 if T * K <= 32768 else 3)
    h.close()
    r = g.run_forward(T, 128, E, K, R, balanced=True, slots=2 if direct else 0, direct=direct, zipf_s=1.0,
                      seed=T + K, G=0 if direct else 256)
    assert r["flags"] == 0
    if not direct:
        g.run_backward(r, seed=T)


@pytest.mark.parametrize("T,H,fp8", [(1000, 7176, False), (1000, 7296, True), (300, 2056, False),
                                      (64, 20480, False), (64, 40960, True)])
def test_rows_split_across_ctas(T, H, fp8):
    """Batches too small for several waves of one-row CTAs cut each row into
    parts of whole warps of vectors, the last part ragged (897 vectors as
    7 x 128 and 1 left over, 456 FP8 chunks as 3 x 128 + 72, 257 vectors as
    96 + 96 + 65)."""
    g = _gc()
    r = g.run_forward(T, H, 32, 4, 4, fp8=fp8, seed=H)
    if not fp8:
        g.run_backward(r, seed=H)


def test_long_rows_use_slab_loop():
    """Rows longer than one CTA's registers hold (2050 bf16 vectors, 2056 FP8
    chunks) in a batch large enough to keep one CTA per row, and FP8 rows of
    768 chunks, four a thread (the instance rows of 8193..16384 elements use)."""
    g = _gc()
    T = 40 * torch.cuda.get_device_properties(0).multi_processor_count
    r = g.run_forward(T, 16400, 4, 1, 4, seed=9)
    g.run_backward(r, seed=9)
    g.run_forward(T, 32896, 4, 1, 4, fp8=True, seed=9)
    g.run_forward(T, 12288, 4, 1, 4, fp8=True, seed=10)


# --------------------------------------------------------------- edge cases

def test_empty_batch():
    g = _gc()
    h = ep.Ep(0, 1024, 16, 2, 4)
    idx = torch.empty((0, 2), dtype=torch.int32, device="cuda")
    h.plan(idx)
    b = h.empty_recv()
    x = torch.empty((0, 1024), dtype=torch.bfloat16, device="cuda")
    w = torch.empty((0, 2), dtype=torch.float32, device="cuda")
    h.dispatch(x, idx, w, b["recv_x"], None, b["recv_w"], b["recv_expert"], b["recv_counts"])
    assert (b["recv_counts"] == 0).all()
    h.combine(b["recv_x"], w, x)
    assert h.status() == 0


def test_masked_bad_and_duplicate_ids_are_skipped_and_flagged():
    g = _gc()
    T, H, E, K, R = 200, 256, 16, 4, 4
    x, idx, w = g.make_inputs(T, H, E, K, seed=5)
    idx = idx.clone()
    idx[3, 1] = -1          # masked: skipped, no flag
    idx[7, :] = -1          # fully masked token: combine gives 0
    idx[10, 2] = E + 5      # bad id
    idx[11, 0] = -7         # bad id
    idx[12, 3] = idx[12, 1]  # repeat within a token
    r = g.run_forward(T, H, E, K, R, idx=idx, w=w, x=x)
    assert r["flags"] == oracle.FLAG_BAD_EXPERT_ID | oracle.FLAG_DUP_EXPERT_ID
    assert (r["combine_out"][7].float() == 0).all()
    g.run_backward(r)


def test_all_masked():
    g = _gc()
    T, H, E, K, R = 64, 128, 8, 2, 2
    x, idx, w = g.make_inputs(T, H, E, K)
    idx = torch.full_like(idx, -1)
    r = g.run_forward(T, H, E, K, R, idx=idx, w=w, x=x)
    assert r["flags"] == 0 and r["ref"].cnt.sum() == 0
    assert (r["combine_out"].float() == 0).all()


def test_ll_capacity_overflow_drops_and_flags():
    g = _gc()
    r = g.run_forward(512, 256, 8, 2, 2, mode="ll", cap=40, zipf_s=2.0, seed=4)
    assert r["flags"] & oracle.FLAG_CAPACITY
    g.run_backward(r, seed=4)


def test_hand_worked_plans():
    """The hand-worked balanced plans of tests/golden/plan_worked.txt (a normal
    case, slot overflow with and without a tail between kept rows, the
    inference plan, and a case decided by the spill and receiver orders) run
    on the GPU: loads and replica table equal to the worked values, routing,
    rows and combine equal to the oracle."""
    from test_oracle_pins import _golden_plans, _idx_from_counts

    g = _gc()
    for n, c in enumerate(_golden_plans()):
        E, R, S = c["E"][0], c["R"][0], c["S"][0]
        idx = torch.from_numpy(_idx_from_counts(c["cnt"]))
        T = idx.shape[0]
        r = g.run_forward(T, 128, E, 1, R, balanced=True, slots=S, direct=bool(c.get("direct", [0])[0]),
                          idx=idx, w=torch.ones((T, 1), dtype=torch.float32), seed=40 + n)
        rep, load = r["h"].get_plan()
        assert rep == c["replica_expert"] and load == c["rank_load"]
        assert r["flags"] == c["flags"][0]


@pytest.mark.parametrize("T", [2048, 8192, 16384])
def test_balanced_plan_slot_overflow_keeps_rows_on_owner(T):
    """Replica slots limited to 1 per rank under heavy skew: the plan runs out
    of slots (the planner's one-thread walk), raises PLAN_SLOTS and keeps the
    leftover rows on the owner; the layout stays a permutation and matches the
    oracle. 8192 pairs route in a cluster of 8 CTAs, 32768 in one of 16, and
    65536 in three kernels."""
    g = _gc()
    r = g.run_forward(T, 256, 32, 4, 8, balanced=True, slots=1, zipf_s=2.0, seed=6, G=128)
    assert ep.plan_launches(r["h"]) == (1 if T * 4 <= 32768 else 3)
    assert r["flags"] & oracle.FLAG_PLAN_SLOTS
    assert sorted(r["ref"].dest_row.tolist()) == list(range(T * 4))
    g.run_backward(r, seed=6)


@pytest.mark.parametrize("E,R,S,s", [(64, 8, 1, 2.0), (32, 8, 1, 2.0), (384, 16, 2, 1.0), (16, 4, 1, 1.5)])
def test_inference_plan_direct_overflow(E, R, S, s):
    """Inference plan (a few prefetch slots, overflow read from the owner):
    loads always exact, direct pieces and rows identical to the oracle, and
    dispatch / combine / backward / replica reduce on top of it."""
    g = _gc()
    T, K = 4096, 8
    r = g.run_forward(T, 512, E, K, R, balanced=True, slots=S, direct=True, zipf_s=s, seed=E + S, G=256)
    assert r["flags"] == 0
    _, load = r["h"].get_plan()
    assert max(load) - min(load) <= 1
    assert r["h"].tensor(ep.T_DIRECT_COUNT).sum().item() > 0  # the slots did run out
    g.run_backward(r, seed=E)


def test_zero_blocks_and_large_values_fp8():
    g = _gc()
    T, H, E, K, R = 64, 1024, 16, 2, 4
    x, idx, w = g.make_inputs(T, H, E, K, seed=8)
    x[0, :] = 0
    x[1, 128:256] = 0
    x[2, :128] = 3.0e38
    x[3, 256:384] *= 1e-30
    x[4, 384:512] = -448.0
    r = g.run_forward(T, H, E, K, R, fp8=True, idx=idx, w=w, x=x)
    assert r["fp8_diff"] == 0


def test_fp8_cast_across_the_bf16_range():
    """Blocks scaled from 2^-133 to 2^120, with elements spread 2^40 below
    the block's largest and some exact zeros of either sign. The cast's
    division takes its reciprocal-and-correction path inside a range of
    block scales and elements and the full division outside it; both must
    give the oracle's e4m3 codes and scales bit for bit."""
    g = _gc()
    T, H, E, K, R = 256, 1024, 16, 2, 4
    _, idx, w = g.make_inputs(T, H, E, K, seed=21)
    rng = np.random.default_rng(21)
    nb = T * H // 128
    block_exp = rng.integers(-133, 121, nb).astype(np.float64)
    spread = rng.uniform(-40.0, 0.0, (nb, 128))  # each element up to 2^40 below its block's top
    mant = rng.uniform(1.0, 2.0, (nb, 128)) * rng.choice([-1.0, 1.0], (nb, 128))
    vals = mant * np.exp2(block_exp[:, None] + np.floor(spread))
    vals[rng.random((nb, 128)) < 0.02] = 0.0
    neg0 = rng.random((nb, 128)) < 0.01
    x = torch.from_numpy(vals.reshape(T, H)).to(torch.bfloat16)
    x[torch.from_numpy(neg0.reshape(T, H))] = -0.0
    assert torch.isfinite(x.float()).all()
    r = g.run_forward(T, H, E, K, R, fp8=True, idx=idx, w=w, x=x, check_combine=False)
    assert r["fp8_diff"] == 0
    # byte for byte, so that a zero of the wrong sign shows too
    ref = r["ref"]
    codes = oracle.dispatch(x, idx, w, ref.dest_row, ref.recv_rows, fp8=True)[0]
    np.testing.assert_array_equal(g.bits8(r["bufs"]["recv_x"])[r["rows"]], codes[r["rows"]])


def test_plan_is_reused_by_backward_after_other_work():
    """Routing state lives in the handle from one ep_plan to the next (forward
    and backward share it); a second plan with new routing replaces it."""
    g = _gc()
    r1 = g.run_forward(300, 256, 16, 2, 4, seed=1)
    g.run_backward(r1, seed=1)
    x, idx, w = g.make_inputs(300, 256, 16, 2, seed=2)
    h = r1["h"]
    h.plan(idx.cuda())
    dest = h.tensor(ep.T_DEST_ROW).cpu().numpy()
    np.testing.assert_array_equal(dest, oracle.route(idx, E=16, R=4).dest_row)


def test_direct_overflow_needs_a_plan():
    with pytest.raises(ep.EpError):
        ep.Ep(16, 128, 8, 2, 2, direct_overflow=True)


def test_host_argument_errors():
    h = ep.Ep(16, 128, 8, 2, 2)
    x = torch.zeros((16, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ep.EpError):  # before any plan
        h.combine(torch.zeros((32, 128), dtype=torch.bfloat16, device="cuda"),
                  torch.zeros((16, 2), device="cuda"), x)
    from combine_ep_dispatch_03_b200.ep import lib
    import ctypes

    idx = torch.zeros((16, 2), dtype=torch.int32, device="cuda")
    h.plan(idx)
    # misaligned token pointer
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    bad = ctypes.c_void_p(x.data_ptr() + 2)
    assert lib().ep_combine(h._h, bad, ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(x.data_ptr()), st) == 1
    assert lib().ep_reduce_replica_grads(h._h, None, None, st) == 3  # no plan -> unsupported
