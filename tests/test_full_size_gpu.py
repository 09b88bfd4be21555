"""Parity at full workload sizes, in the launch configuration the benchmark
times. The oracle recomputes the complete routing and a sample of tokens one
by one; properties that hold at any size (permutation, counts, identity
expert) are checked on every element."""
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


def _sample_tokens(T, n, seed):
    rng = np.random.default_rng(seed)
    s = rng.choice(T, size=n, replace=False)
    return np.sort(np.concatenate([s, [0, T - 1]]))


def test_ht_prefill_full_size_sampled():
    """HT prefill: T=32768, H=7168, E=256, top-8, R=8, FP8 dispatch, bf16
    combine; the benchmark's workload and launch configuration."""
    g = _gc()
    T, H, E, K, R = 32768, 7168, 256, 8, 8
    dev = torch.device("cuda")
    x = synth.tokens_bf16(T, H, seed=0)
    idx, w = synth.routing(T, E, K, seed=0)
    h = ep.Ep(T, H, E, K, R, fp8=True)
    bufs = h.empty_recv()
    xd, idxd, wd = x.to(dev), idx.to(dev), w.to(dev)
    h.plan(idxd)
    h.dispatch(xd, idxd, wd, **bufs)
    gen = torch.Generator(device=dev).manual_seed(77)
    y = torch.randn((h.recv_rows, H), generator=gen, device=dev).to(torch.bfloat16)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    h.combine(y, wd, out)
    assert h.status() == 0

    ref = oracle.route(idx, E=E, R=R)
    dest = h.tensor(ep.T_DEST_ROW).cpu().numpy()
    np.testing.assert_array_equal(dest, ref.dest_row)  # all 262144 pairs
    np.testing.assert_array_equal(bufs["recv_counts"].cpu().numpy(), ref.cnt)
    assert np.array_equal(np.sort(dest), np.arange(T * K))  # every pair exactly once

    toks = _sample_tokens(T, 64, 1)
    pairs = (toks[:, None] * K + np.arange(K)[None, :]).reshape(-1)
    rows = dest[pairs]
    compact = np.arange(pairs.size, dtype=np.int32)
    rx, rs, rw, re = oracle.dispatch(x[toks], idx[toks], w[toks], compact, pairs.size, fp8=True)
    got = g.bits8(bufs["recv_x"][torch.from_numpy(rows).to(dev)])
    g.assert_fp8_close(got, rx, "fp8 payload (sampled)")
    np.testing.assert_array_equal(bufs["recv_scales"][torch.from_numpy(rows).to(dev)].cpu().numpy(), rs)
    np.testing.assert_array_equal(bufs["recv_w"].cpu().numpy()[rows], rw)
    np.testing.assert_array_equal(bufs["recv_expert"].cpu().numpy()[rows], re)

    ysub = y[torch.from_numpy(rows).to(dev)].cpu()
    want = oracle.combine(ysub, w[toks], compact, toks.size, K)
    g.assert_bf16_close(g.bits16(out[torch.from_numpy(toks).to(dev)]), want, "combine (sampled)")


def test_large_train_full_size_sampled():
    """Large training step: T=131072, H=7168, E=384, top-8, R=16, Zipf 1.0,
    balanced plan; forward with the identity expert (combine returns x on
    every element), backward and the replica-gradient reduce sampled."""
    g = _gc()
    T, H, E, K, R = 131072, 7168, 384, 8, 16
    G = 7168 * 256
    dev = torch.device("cuda")
    x = synth.tokens_bf16(T, H, seed=0)
    idx, w = synth.routing(T, E, K, zipf_s=1.0, seed=0)
    h = ep.Ep(T, H, E, K, R, balanced=True, grad_elems_per_expert=G)
    bufs = h.empty_recv()
    xd, idxd, wd = x.to(dev), idx.to(dev), w.to(dev)
    h.plan(idxd)
    h.dispatch(xd, idxd, wd, **bufs)
    out = torch.empty_like(xd)
    h.combine(bufs["recv_x"], wd, out)
    assert h.status() == 0
    assert torch.equal(out.view(torch.int16), xd.view(torch.int16))  # identity expert returns x

    ref = oracle.route(idx, E=E, R=R, balanced=True)
    dest = h.tensor(ep.T_DEST_ROW).cpu().numpy()
    np.testing.assert_array_equal(dest, ref.dest_row)
    rep_e, load = h.get_plan()
    np.testing.assert_array_equal(np.array(rep_e), ref.plan["replica_expert"].reshape(-1))
    q = T * K // R
    assert set(load) <= {q, q + 1}
    np.testing.assert_array_equal(bufs["recv_counts"].cpu().numpy(), ref.recv_counts.reshape(-1))

    toks = _sample_tokens(T, 48, 2)
    pairs = (toks[:, None] * K + np.arange(K)[None, :]).reshape(-1)
    rows = torch.from_numpy(dest[pairs]).to(dev)
    compact = np.arange(pairs.size, dtype=np.int32)
    gout = torch.randn((T, H), generator=torch.Generator(device=dev).manual_seed(5), device=dev).to(torch.bfloat16)
    gy = bufs["recv_x"]  # reuse the dispatch buffer for the expert-output gradient
    h.combine_backward(gout, wd, gy)
    want_gy = oracle.combine_backward(gout[torch.from_numpy(toks).to(dev)].cpu(), w[toks], compact, pairs.size)
    g.assert_bf16_close(g.bits16(gy[rows]), want_gy, "combine backward (sampled)")
    gx = out
    h.dispatch_backward(gy, gx)
    want_gx = oracle.combine(want_gy, None, compact, toks.size, K)
    g.assert_bf16_close(g.bits16(gx[torch.from_numpy(toks).to(dev)]), want_gx, "dispatch backward (sampled)")

    del bufs, gy, gx, gout, xd
    torch.cuda.empty_cache()
    S = E // R
    gen = torch.Generator(device=dev).manual_seed(9)
    rep = torch.randn((R, S, G), generator=gen, device=dev)
    own = torch.randn((E, G), generator=gen, device=dev)
    cols = torch.from_numpy(np.sort(np.random.default_rng(3).choice(G, 4096, replace=False))).to(dev)
    rep_s, own_s = rep[:, :, cols].cpu().numpy(), own[:, cols].cpu().numpy()
    h.reduce_replica_grads(rep, own)
    want = oracle.replica_reduce(ref.plan["replica_expert"], rep_s, own_s)
    np.testing.assert_array_equal(own[:, cols].cpu().numpy(), want)
