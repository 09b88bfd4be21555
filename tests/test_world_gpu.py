"""Expert parallelism across ranks through a peer table, on one GPU.

R ranks are R handles, each with its own T_local tokens, and R separate
receive buffers stand in for the R GPUs' symmetric buffers. Every rank counts
its pairs (ep_plan_local_counts), the count rows are stacked (the all-gather
of a real world), every rank completes its plan (ep_plan_world), sends its
rows through the table (ep_dispatch_peers), signals and waits on the
completion flags, and combines from the table (ep_combine_peers). The calls
of all ranks run in stream order, so every wait finds flags that kernels
before it have set: no kernel waits on another that runs at the same time.

The oracle routes the concatenation of all ranks' tokens (rank order) as one
batch: rank q's receive buffer must equal rows [rank_off[q], rank_off[q+1])
of the oracle's receive buffer, bit for bit (FP8 codes within the tolerance
of gpu_cases), and every rank's combined tokens the oracle's combine of the
concatenated expert outputs. A bounded wait on flags nobody sets must give up
and report EP_FLAG_WAIT_TIMEOUT.
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


def _gc():
    import gpu_cases

    return gpu_cases


def _world(Tl, H, E, K, R, mode="ht", cap=0, fp8=False, balanced=False, slots=0, direct=False, zipf_s=0.0,
           seed=0, idx=None, capacity=None, epoch=1):
    g = _gc()
    dev = torch.device("cuda")
    T = Tl * R
    x = synth.tokens_bf16(T, H, seed=seed)
    if idx is None:
        idx, w = synth.routing(T, E, K, zipf_s=zipf_s, seed=seed)
    else:
        _, w = synth.routing(T, E, K, zipf_s=zipf_s, seed=seed)
    ref = oracle.route(idx, E=E, R=R, mode=mode, cap=cap, balanced=balanced, slots=slots or None, direct=direct)
    rx, rs, rw, re = oracle.dispatch(x, idx, w, ref.dest_row, ref.recv_rows, fp8=fp8)

    hs = [ep.Ep(Tl, H, E, K, R, mode=mode, ll_capacity=cap, fp8=fp8, balanced=balanced, replica_slots=slots,
                direct_overflow=direct) for _ in range(R)]
    cap_rows = ep.world_recv_rows(hs[0].cfg) if capacity is None else capacity
    xs = [x[q * Tl:(q + 1) * Tl].to(dev) for q in range(R)]
    ids = [idx[q * Tl:(q + 1) * Tl].contiguous().to(dev) for q in range(R)]
    ws = [w[q * Tl:(q + 1) * Tl].contiguous().to(dev) for q in range(R)]
    dt = torch.float8_e4m3fn if fp8 else torch.bfloat16
    recv_x = [torch.zeros((max(cap_rows, 1), H), dtype=dt, device=dev) for _ in range(R)]
    recv_s = [torch.zeros((max(cap_rows, 1), H // 128), dtype=torch.float32, device=dev) for _ in range(R)] \
        if fp8 else None
    recv_w = [torch.zeros(max(cap_rows, 1), dtype=torch.float32, device=dev) for _ in range(R)]
    recv_e = [torch.full((max(cap_rows, 1),), -7, dtype=torch.int32, device=dev) for _ in range(R)]
    flags = [torch.zeros(R, dtype=torch.int32, device=dev) for _ in range(R)]
    table = ep.peer_table(cap_rows, recv_x, flags, recv_s, recv_w, recv_e)

    counts = torch.zeros((R, E), dtype=torch.int32, device=dev)
    for q in range(R):
        hs[q].plan_local_counts(ids[q], counts[q])
    for q in range(R):
        hs[q].plan_world(counts, q)
    for q in range(R):
        hs[q].dispatch_peers(xs[q], ids[q], ws[q], table)
    for q in range(R):
        hs[q].signal_peers(table, epoch)
    for q in range(R):
        hs[q].wait_peers(flags[q], epoch, timeout_us=2_000_000)
    torch.cuda.synchronize()

    # every flag of every rank carries the epoch
    for q in range(R):
        assert (flags[q].cpu().numpy() == epoch).all()
    # the world plan, the same on every rank; each rank's own rows
    roff = hs[0].tensor(ep.T_RANK_OFFSET).cpu().numpy()
    for q in range(R):
        np.testing.assert_array_equal(hs[q].tensor(ep.T_RANK_OFFSET).cpu().numpy(), roff)
        np.testing.assert_array_equal(hs[q].tensor(ep.T_EXPERT_COUNTS).cpu().numpy(), ref.cnt)
        np.testing.assert_array_equal(hs[q].tensor(ep.T_DEST_ROW).cpu().numpy(),
                                      ref.dest_row[q * Tl * K:(q + 1) * Tl * K])
    g_ = E // R
    if mode == "ll":
        np.testing.assert_array_equal(roff, np.arange(R + 1) * g_ * cap)
    elif not balanced:
        np.testing.assert_array_equal(roff, [int(ref.cnt[:q * g_].sum()) for q in range(R + 1)])
    if balanced:
        np.testing.assert_array_equal(roff, ref.plan["rank_off"])
        for q in range(R):
            rep, load = hs[q].get_plan()
            np.testing.assert_array_equal(np.array(rep), ref.plan["replica_expert"].reshape(-1))
            np.testing.assert_array_equal(np.array(load), ref.plan["rank_load"])
    # each rank's receive buffer is its region of the oracle's buffer
    placed = np.unique(ref.dest_row[ref.dest_row >= 0])
    nflag = 0
    for q in range(R):
        rows = placed[(placed >= roff[q]) & (placed < roff[q + 1])]
        kept = rows[rows - roff[q] < cap_rows]
        nflag += len(rows) - len(kept)
        lr = torch.from_numpy((kept - roff[q]).astype(np.int64)).to(dev)
        if fp8:
            g.assert_fp8_close(g.bits8(recv_x[q][lr]), rx[kept], f"fp8 rows of rank {q}")
            np.testing.assert_array_equal(recv_s[q][lr].cpu().numpy(), rs[kept])
        else:
            np.testing.assert_array_equal(g.bits16(recv_x[q][lr]), rx[kept])
        np.testing.assert_array_equal(recv_w[q][lr].cpu().numpy(), rw[kept])
        np.testing.assert_array_equal(recv_e[q][lr].cpu().numpy(), re[kept])
    want_flags = ref.flags | (oracle.FLAG_CAPACITY if nflag else 0)
    got_flags = 0
    for q in range(R):
        got_flags |= hs[q].status()
    assert got_flags == want_flags, (got_flags, want_flags)

    # combine: the expert outputs stand in a fresh buffer per rank
    ys = [synth.tokens_bf16(max(cap_rows, 1), H, seed=seed + 50 + q).to(dev) for q in range(R)]
    ytab = ep.peer_table(cap_rows, ys, None)
    outs = [torch.empty((Tl, H), dtype=torch.bfloat16, device=dev) for _ in range(R)]
    for q in range(R):
        hs[q].combine_peers(ytab, ws[q], outs[q])
    torch.cuda.synchronize()
    # the oracle's combine reads the same rows from one global buffer; rows
    # beyond a rank's capacity were never written and are not read
    yglob = np.zeros((ref.recv_rows, H), np.uint16)
    for q in range(R):
        n = min(roff[q + 1] - roff[q], cap_rows)
        yglob[roff[q]:roff[q] + n] = g.bits16(ys[q][:n])
    dest = ref.dest_row.copy()
    for q in range(R):
        dest[(dest >= roff[q] + cap_rows) & (dest < roff[q + 1])] = -1
    want = oracle.combine(yglob, w, dest, T, K)
    got = np.concatenate([g.bits16(o) for o in outs])
    g.assert_bf16_close(got, want, "combine across ranks")
    for h in hs:
        h.close()
    return ref


@pytest.mark.parametrize("Tl,H,E,K,R", [(300, 256, 64, 4, 4), (129, 1024, 32, 8, 8), (1, 128, 8, 2, 2)])
def test_world_ht_bf16(Tl, H, E, K, R):
    _world(Tl, H, E, K, R, seed=Tl)


def test_world_ht_fp8():
    _world(512, 1024, 256, 8, 8, fp8=True, seed=3)


@pytest.mark.parametrize("direct", [False, True])
def test_world_balanced_plan(direct):
    ref = _world(500, 256, 64, 6, 4, balanced=True, slots=2 if direct else 0, direct=direct, zipf_s=1.0, seed=4)
    load = ref.plan["rank_load"]
    assert max(load) - min(load) <= 1  # the world's loads are flat


def test_world_ll():
    _world(200, 512, 32, 4, 4, mode="ll", cap=150, zipf_s=1.0, seed=5)


def test_world_bad_and_repeated_ids():
    R, Tl, E, K = 4, 100, 16, 3
    idx, _ = synth.routing(R * Tl, E, K, seed=6)
    idx = idx.clone()
    idx[Tl + 3, 1] = idx[Tl + 3, 0]  # a repeat on rank 1
    idx[2 * Tl + 5, 2] = E + 1       # a bad id on rank 2
    idx[7, 0] = -1                   # a masked choice on rank 0
    ref = _world(Tl, 128, E, K, R, idx=idx, seed=6)
    assert ref.flags & oracle.FLAG_BAD_EXPERT_ID and ref.flags & oracle.FLAG_DUP_EXPERT_ID


def test_world_capacity_overflow_is_skipped_and_flagged():
    # skewed routing without a plan sends rank 0 far more rows than 300
    _world(256, 128, 16, 4, 4, zipf_s=2.0, seed=7, capacity=300)


def test_world_refuses_mixed_calls():
    h = ep.Ep(16, 128, 8, 2, 2)
    idx, w = synth.routing(16, 8, 2, seed=1)
    dev = torch.device("cuda")
    counts = torch.zeros((2, 8), dtype=torch.int32, device=dev)
    h.plan_local_counts(idx.to(dev), counts[0])
    h.plan_local_counts(idx.to(dev), counts[1])
    h.plan_world(counts, 0)
    x = torch.zeros((16, 128), dtype=torch.bfloat16, device=dev)
    bufs = h.empty_recv()
    with pytest.raises(ep.EpError) as e:
        h.dispatch(x, idx.to(dev), w.to(dev), **bufs)
    assert e.value.status == 3  # EP_ERR_UNSUPPORTED: the rows are global
    h.plan(idx.to(dev))
    tab = ep.peer_table(64, [bufs["recv_x"], bufs["recv_x"]], None)
    with pytest.raises(ep.EpError) as e:
        h.dispatch_peers(x, idx.to(dev), w.to(dev), tab)
    assert e.value.status == 3
    h.close()


def test_wait_gives_up_on_flags_nobody_sets():
    """A bounded wait whose flags never reach the epoch gives up after its
    limit, sets EP_FLAG_WAIT_TIMEOUT and returns; the context stays usable
    and a wait on flags that are set passes at once."""
    dev = torch.device("cuda")
    h = ep.Ep(16, 128, 8, 2, 2)
    idx, _ = synth.routing(16, 8, 2, seed=2)
    h.plan(idx.to(dev))  # clears the status word
    flags = torch.zeros(2, dtype=torch.int32, device=dev)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    h.wait_peers(flags, 5, timeout_us=50_000)
    e.record()
    torch.cuda.synchronize()
    waited = s.elapsed_time(e)
    assert h.status() & ep.FLAG_WAIT_TIMEOUT
    assert 45.0 <= waited < 1000.0, waited
    h.plan(idx.to(dev))
    flags.fill_(5)
    s.record()
    h.wait_peers(flags, 5, timeout_us=50_000)
    e.record()
    torch.cuda.synchronize()
    assert h.status() == 0
    assert s.elapsed_time(e) < 40.0
    h.close()


def test_world_empty_batches():
    """Ranks with no tokens: counts of zero, an empty plan, and dispatch and
    combine calls that launch nothing and succeed."""
    dev = torch.device("cuda")
    R, E, K, H = 2, 8, 2, 128
    hs = [ep.Ep(0, H, E, K, R) for _ in range(R)]
    cap = ep.world_recv_rows(hs[0].cfg)
    assert cap == 0
    counts = torch.full((R, E), 7, dtype=torch.int32, device=dev)
    ids = torch.empty((0, K), dtype=torch.int32, device=dev)
    x = torch.empty((0, H), dtype=torch.bfloat16, device=dev)
    w = torch.empty((0, K), dtype=torch.float32, device=dev)
    bufs = [torch.zeros((1, H), dtype=torch.bfloat16, device=dev) for _ in range(R)]
    flags = [torch.zeros(R, dtype=torch.int32, device=dev) for _ in range(R)]
    table = ep.peer_table(cap, bufs, flags)
    for q in range(R):
        hs[q].plan_local_counts(ids, counts[q])
    for q in range(R):
        hs[q].plan_world(counts, q)
        hs[q].dispatch_peers(x, ids, w, table)
        hs[q].signal_peers(table, 3)
    for q in range(R):
        hs[q].wait_peers(flags[q], 3, timeout_us=1_000_000)
        hs[q].combine_peers(table, w, torch.empty((0, H), dtype=torch.bfloat16, device=dev))
    torch.cuda.synchronize()
    assert (counts == 0).all()
    for q in range(R):
        assert hs[q].status() == 0
        assert (flags[q] == 3).all()
        np.testing.assert_array_equal(hs[q].tensor(ep.T_RANK_OFFSET).cpu().numpy(), np.zeros(R + 1))
        hs[q].close()


def _plan_world_ranks(idx, Tl, H, E, K, R, balanced=False, G=0):
    dev = torch.device("cuda")
    hs = [ep.Ep(Tl, H, E, K, R, balanced=balanced, grad_elems_per_expert=G) for _ in range(R)]
    ids = [idx[q * Tl:(q + 1) * Tl].contiguous().to(dev) for q in range(R)]
    counts = torch.zeros((R, E), dtype=torch.int32, device=dev)
    for q in range(R):
        hs[q].plan_local_counts(ids[q], counts[q])
    for q in range(R):
        hs[q].plan_world(counts, q)
    return hs, ids


@pytest.mark.parametrize("balanced", [False, True])
def test_world_backward(balanced):
    """The backward pass across ranks against the oracle on the concatenated
    batch: combine backward (weighted rows stored to the owning ranks),
    dispatch backward (rows gathered and summed in k order), and, with a plan,
    the replica gradients reduced into each owner's rows. Two steps alternate
    two sets of gradient buffers (double buffering), each checked."""
    g = _gc()
    dev = torch.device("cuda")
    R, Tl, H, E, K = 4, 300, 256, 32, 4
    T = R * Tl
    G = 1024 if balanced else 0
    idx, w = synth.routing(T, E, K, zipf_s=1.0, seed=31)
    ref = oracle.route(idx, E=E, R=R, balanced=balanced)
    hs, ids = _plan_world_ranks(idx, Tl, H, E, K, R, balanced, G)
    cap = ep.world_recv_rows(hs[0].cfg)
    roff = hs[0].tensor(ep.T_RANK_OFFSET).cpu().numpy()
    ws = [w[q * Tl:(q + 1) * Tl].contiguous().to(dev) for q in range(R)]
    flags = [torch.zeros(R, dtype=torch.int32, device=dev) for _ in range(R)]
    sets = [[torch.zeros((cap, H), dtype=torch.bfloat16, device=dev) for _ in range(R)] for _ in range(2)]
    placed = np.unique(ref.dest_row[ref.dest_row >= 0])
    epoch = 0
    for step in range(2):
        bufs = sets[step % 2]
        tab = ep.peer_table(cap, bufs, flags)
        gout = synth.tokens_bf16(T, H, seed=40 + step)
        gout_d = [gout[q * Tl:(q + 1) * Tl].to(dev) for q in range(R)]
        for q in range(R):
            hs[q].combine_backward_peers(gout_d[q], ws[q], tab)
        epoch += 1
        for q in range(R):
            hs[q].signal_peers(tab, epoch)
        for q in range(R):
            hs[q].wait_peers(flags[q], epoch, timeout_us=2_000_000)
        torch.cuda.synchronize()
        want = oracle.combine_backward(gout, w, ref.dest_row, ref.recv_rows)
        for q in range(R):
            rows = placed[(placed >= roff[q]) & (placed < roff[q + 1])]
            lr = torch.from_numpy((rows - roff[q]).astype(np.int64)).to(dev)
            g.assert_bf16_close(g.bits16(bufs[q][lr]), want[rows], f"combine backward, rank {q}, step {step}")
        # dispatch backward: each rank's gradient rows (fresh values) summed per token
        grecv = synth.tokens_bf16(ref.recv_rows, H, seed=50 + step)
        for q in range(R):
            n = roff[q + 1] - roff[q]
            bufs[q][:n] = grecv[roff[q]:roff[q + 1]].to(dev)
        torch.cuda.synchronize()
        gx = [torch.empty((Tl, H), dtype=torch.bfloat16, device=dev) for _ in range(R)]
        for q in range(R):
            hs[q].dispatch_backward_peers(tab, gx[q])
        torch.cuda.synchronize()
        want2 = oracle.combine(grecv, None, ref.dest_row, T, K)
        got2 = np.concatenate([g.bits16(o) for o in gx])
        g.assert_bf16_close(got2, want2, f"dispatch backward, step {step}")
    if balanced:
        S = hs[0].S
        gen = torch.Generator().manual_seed(61)
        rep = torch.randn((R, S, G), generator=gen)
        own = torch.randn((E, G), generator=gen)
        rep_d = [rep[q].contiguous().to(dev) for q in range(R)]
        own_d = [own[q * (E // R):(q + 1) * (E // R)].contiguous().to(dev) for q in range(R)]
        gtab = ep.peer_table(0, rep_d, None)
        for q in range(R):
            hs[q].reduce_replica_grads_peers(gtab, own_d[q])
        torch.cuda.synchronize()
        want3 = oracle.replica_reduce(ref.plan["replica_expert"], rep.numpy(), own.numpy())
        np.testing.assert_array_equal(torch.cat([o.cpu() for o in own_d]).numpy(), want3)
        assert (ref.plan["replica_expert"] >= 0).any()  # the plan has replicas to reduce
    for q in range(R):
        assert hs[q].status() == 0
        hs[q].close()


def test_world_prefetch_from_owners():
    """Each rank's filled replica slots receive their experts' weights from the
    owning ranks' tables; empty slots keep their contents (the oracle's
    prefetch on the world's plan)."""
    dev = torch.device("cuda")
    R, Tl, E, K, B = 4, 400, 32, 4, 4096
    g_ = E // R
    idx, _ = synth.routing(R * Tl, E, K, zipf_s=1.5, seed=71)
    ref = oracle.route(idx, E=E, R=R, balanced=True)
    hs, _ = _plan_world_ranks(idx, Tl, 128, E, K, R, balanced=True)
    S = hs[0].S
    rng = np.random.default_rng(72)
    weights = rng.integers(0, 256, size=(E, B), dtype=np.uint8)
    slots0 = rng.integers(0, 256, size=(R * S, B), dtype=np.uint8)
    wd = [torch.from_numpy(weights[q * g_:(q + 1) * g_].copy()).to(dev) for q in range(R)]
    sd = [torch.from_numpy(slots0[q * S:(q + 1) * S].copy()).to(dev) for q in range(R)]
    tab = ep.peer_table(0, wd, None)
    for q in range(R):
        hs[q].prefetch_replica_weights_peers(tab, B, sd[q])
    torch.cuda.synchronize()
    want = oracle.prefetch(ref.plan["replica_expert"], weights, slots0)
    got = np.concatenate([s_.cpu().numpy() for s_ in sd])
    np.testing.assert_array_equal(got, want)
    assert (ref.plan["replica_expert"] >= 0).any() and (ref.plan["replica_expert"] < 0).any()
    for h in hs:
        h.close()


def _world_case(i):
    rng = np.random.default_rng(13000 + i)
    R = int(rng.choice([2, 4, 8]))
    E = R * int(rng.choice([1, 2, 4, 8, 16, 32]))
    K = int(rng.integers(1, min(E, 8) + 1))
    Tl = int(rng.choice([1, 3, 64, 129, 300, 700, 2000]))
    H = int(rng.choice([128, 256]))
    mode = "ll" if rng.random() < 0.3 else "ht"
    cap = int(rng.integers(1, max(2, 2 * Tl * R * K // E) + 1)) if mode == "ll" else 0
    fp8 = bool(mode == "ht" and rng.random() < 0.3)
    balanced = bool(mode == "ht" and rng.random() < 0.4)
    slots = int(rng.integers(0, E // R + 1)) if balanced else 0
    direct = bool(balanced and slots > 0 and rng.random() < 0.4)
    s = float(rng.choice([0.0, 1.0, 2.0]))
    return Tl, H, E, K, R, mode, cap, fp8, balanced, slots, direct, s, 13000 + i


@pytest.mark.parametrize("Tl,H,E,K,R,mode,cap,fp8,balanced,slots,direct,s,seed",
                         [_world_case(i) for i in range(40)])
def test_world_random(Tl, H, E, K, R, mode, cap, fp8, balanced, slots, direct, s, seed):
    """Seeded random worlds: ranks, experts, top-K, tokens a rank, HT or LL
    (random capacities), FP8, and balanced plans with slots and direct
    overflow, each against the oracle's routing of the concatenated batch."""
    _world(Tl, H, E, K, R, mode=mode, cap=cap, fp8=fp8, balanced=balanced, slots=slots, direct=direct, zipf_s=s,
           seed=seed)
