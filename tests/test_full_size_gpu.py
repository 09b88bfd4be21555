"""Parity at full workload sizes, in the launch configuration the benchmark
times. The oracle recomputes the complete routing; at HT prefill it also
recomputes every dispatched row and every combined token, in chunks of
tokens. At the large training step it recomputes the backward over a whole
source-rank region and the replica reduce on sampled columns, and properties
that hold at any size (permutation, counts, identity expert) are checked on
every element."""
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


def test_ht_prefill_full_size_complete():
    """HT prefill: T=32768, H=7168, E=256, top-8, R=8, FP8 dispatch, bf16
    combine; the benchmark's workload and launch configuration. Every one of
    the 262144 rows is compared: all FP8 codes against the tolerance (at most
    1 e4m3 ulp, on at most 0.1% of all codes), every scale, weight and expert
    id bit-exact, and every combined element within 1 bf16 ulp. The oracle
    works through the tokens in chunks."""
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
    recv_w, recv_e = bufs["recv_w"].cpu().numpy(), bufs["recv_expert"].cpu().numpy()

    chunk = 2048
    differ = codes = 0
    for t0 in range(0, T, chunk):
        toks = np.arange(t0, min(T, t0 + chunk))
        pairs = (toks[:, None] * K + np.arange(K)[None, :]).reshape(-1)
        rows = dest[pairs]
        rows_d = torch.from_numpy(rows).to(dev)
        compact = np.arange(pairs.size, dtype=np.int32)
        rx, rs, rw, re = oracle.dispatch(x[toks], idx[toks], w[toks], compact, pairs.size, fp8=True)
        got = g.bits8(bufs["recv_x"][rows_d])
        d = g.e4m3_ulp_diff(got, rx)
        assert d.max(initial=0) <= g.FP8_MAX_ULP, f"fp8 payload: {int(d.max())} e4m3 ulps at tokens {t0}+"
        differ += int((d > 0).sum())
        codes += d.size
        np.testing.assert_array_equal(bufs["recv_scales"][rows_d].cpu().numpy(), rs)
        np.testing.assert_array_equal(recv_w[rows], rw)
        np.testing.assert_array_equal(recv_e[rows], re)
        want = oracle.combine(y[rows_d].cpu(), w[toks], compact, toks.size, K)
        g.assert_bf16_close(g.bits16(out[t0:t0 + toks.size]), want, f"combine at tokens {t0}+")
    assert codes == T * K * H
    assert differ <= g.FP8_MAX_FRAC * codes, f"fp8 payload: {differ} of {codes} codes differ"


def test_large_train_full_size():
    """Large training step: T=131072, H=7168, E=384, top-8, R=16, Zipf 1.0,
    balanced plan; forward with the identity expert (combine returns x on
    every element), the backward pair on every element of one whole
    source-rank region (8192 tokens), and the replica-gradient reduce on 4096
    sampled columns of every slot."""
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

    # backward over one whole source-rank region (tokens 0 .. T/R-1, 65536
    # rows), the oracle in chunks of 1024 tokens
    gout = torch.randn((T, H), generator=torch.Generator(device=dev).manual_seed(5), device=dev).to(torch.bfloat16)
    gy = bufs["recv_x"]  # reuse the dispatch buffer for the expert-output gradient
    h.combine_backward(gout, wd, gy)
    gx = out
    h.dispatch_backward(gy, gx)
    region = T // R
    for t0 in range(0, region, 1024):
        toks = np.arange(t0, t0 + 1024)
        pairs = (toks[:, None] * K + np.arange(K)[None, :]).reshape(-1)
        rows = torch.from_numpy(dest[pairs]).to(dev)
        compact = np.arange(pairs.size, dtype=np.int32)
        want_gy = oracle.combine_backward(gout[t0:t0 + 1024].cpu(), w[toks], compact, pairs.size)
        g.assert_bf16_close(g.bits16(gy[rows]), want_gy, f"combine backward at tokens {t0}+")
        # the dispatch backward's input is the oracle's own expert-output gradient
        want_gx = oracle.combine(want_gy, None, compact, toks.size, K)
        g.assert_bf16_close(g.bits16(gx[t0:t0 + 1024]), want_gx, f"dispatch backward at tokens {t0}+")

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
