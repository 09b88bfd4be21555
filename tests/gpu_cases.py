"""Shared driver for the GPU parity tests: run the CUDA path through the C-ABI
binding and the oracle on the same seeded inputs, and compare.

Tolerances (written here, used by every GPU test):
* routing (counts, destination rows, plan tables), bf16 dispatch rows,
  recv_w / recv_expert, FP8 scales: bit-exact;
* FP8 payload: at most 1 e4m3 ulp, on at most 0.1% of elements;
* combine / backward bf16 outputs: at most 1 bf16 ulp (fp32 accumulation in
  the same fixed k order on both sides, so 0 is expected);
* replica-gradient reduce: bit-exact (fp32 adds in the same slot order).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from combine_ep_dispatch_03_b200 import ep, synth

FP8_MAX_ULP, FP8_MAX_FRAC = 1, 1e-3
BF16_MAX_ULP = 1


def bits16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bits8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.uint8).numpy()


def _ordered(b: np.ndarray, sign: int, mag: int) -> np.ndarray:
    b = b.astype(np.int64)
    m = b & mag
    return np.where(b & sign, -m, m)


def bf16_ulp_diff(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    return np.abs(_ordered(a, 0x8000, 0x7FFF) - _ordered(b, 0x8000, 0x7FFF))


def e4m3_ulp_diff(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    return np.abs(_ordered(a, 0x80, 0x7F) - _ordered(b, 0x80, 0x7F))


def assert_bf16_close(got: np.ndarray, want: np.ndarray, what: str) -> int:
    d = bf16_ulp_diff(got, want)
    assert d.max(initial=0) <= BF16_MAX_ULP, f"{what}: {int(d.max())} bf16 ulps"
    return int((d > 0).sum())


def assert_fp8_close(got: np.ndarray, want: np.ndarray, what: str) -> int:
    d = e4m3_ulp_diff(got, want)
    n = int((d > 0).sum())
    assert d.max(initial=0) <= FP8_MAX_ULP, f"{what}: {int(d.max())} e4m3 ulps"
    assert n <= FP8_MAX_FRAC * max(1, d.size), f"{what}: {n} of {d.size} codes differ"
    return n


def make_inputs(T, H, E, K, zipf_s=0.0, seed=0):
    x = synth.tokens_bf16(T, H, seed=seed)
    idx, w = synth.routing(T, E, K, zipf_s=zipf_s, seed=seed)
    return x, idx, w


def run_forward(T, H, E, K, R, mode="ht", cap=0, fp8=False, balanced=False, slots=0, zipf_s=0.0, seed=0,
                idx=None, w=None, x=None, check_combine=True, y_kind="random", G=0, direct=False):
    """Plan + dispatch + combine on the GPU and in the oracle; assert parity.
    Returns a dict of what was compared (for the tests to add checks)."""
    if x is None:
        x = synth.tokens_bf16(T, H, seed=seed)
    if idx is None:
        idx, w = synth.routing(T, E, K, zipf_s=zipf_s, seed=seed)
    dev = torch.device("cuda")
    h = ep.Ep(T, H, E, K, R, mode=mode, ll_capacity=cap, fp8=fp8, balanced=balanced, replica_slots=slots,
              grad_elems_per_expert=G, direct_overflow=direct)
    xd, idxd, wd = x.to(dev), idx.to(dev), w.to(dev)
    bufs = h.empty_recv()
    h.plan(idxd)
    h.dispatch(xd, idxd, wd, bufs["recv_x"], bufs["recv_scales"], bufs["recv_w"], bufs["recv_expert"],
               bufs["recv_counts"])
    flags = h.status()

    ref = oracle.route(idx, E=E, R=R, mode=mode, cap=cap, balanced=balanced, slots=slots or None, direct=direct)
    assert flags == ref.flags, (flags, ref.flags)
    dest = h.tensor(ep.T_DEST_ROW).cpu().numpy()
    np.testing.assert_array_equal(dest, ref.dest_row)
    np.testing.assert_array_equal(h.tensor(ep.T_EXPERT_COUNTS).cpu().numpy(), ref.cnt)
    np.testing.assert_array_equal(bufs["recv_counts"].cpu().numpy(), ref.recv_counts.reshape(-1))
    placed_rows = np.unique(ref.dest_row[ref.dest_row >= 0])
    np.testing.assert_array_equal(h.tensor(ep.T_SRC_ROW).cpu().numpy()[placed_rows], ref.src_row[placed_rows])
    if balanced:
        rep, load = h.get_plan()
        np.testing.assert_array_equal(np.array(rep), ref.plan["replica_expert"].reshape(-1))
        np.testing.assert_array_equal(np.array(load), ref.plan["rank_load"])
        np.testing.assert_array_equal(h.tensor(ep.T_RANK_OFFSET).cpu().numpy(), ref.plan["rank_off"])
        if direct:
            dn = h.tensor(ep.T_DIRECT_COUNT).cpu().numpy()
            np.testing.assert_array_equal(dn, ref.plan["direct_n"])
            de = h.tensor(ep.T_DIRECT_EXPERT).cpu().numpy().reshape(R, E)
            dl = h.tensor(ep.T_DIRECT_LEN).cpu().numpy().reshape(R, E)
            for rr in range(R):
                np.testing.assert_array_equal(de[rr, :dn[rr]], ref.plan["direct_expert"][rr, :dn[rr]])
                np.testing.assert_array_equal(dl[rr, :dn[rr]], ref.plan["direct_len"][rr, :dn[rr]])
                assert (de[rr, dn[rr]:] == -1).all()

    rx, rs, rw, re = oracle.dispatch(x, idx, w, ref.dest_row, ref.recv_rows, fp8=fp8)
    rows = np.unique(ref.dest_row[ref.dest_row >= 0])
    out = {"h": h, "ref": ref, "rows": rows, "x": x, "idx": idx, "w": w, "bufs": bufs, "flags": flags}
    if fp8:
        out["fp8_diff"] = assert_fp8_close(bits8(bufs["recv_x"])[rows], rx[rows], "fp8 payload")
        np.testing.assert_array_equal(bufs["recv_scales"].cpu().numpy()[rows], rs[rows])
    else:
        np.testing.assert_array_equal(bits16(bufs["recv_x"])[rows], rx[rows])
    np.testing.assert_array_equal(bufs["recv_w"].cpu().numpy()[rows], rw[rows])
    np.testing.assert_array_equal(bufs["recv_expert"].cpu().numpy()[rows], re[rows])

    if check_combine:
        if y_kind == "identity" and not fp8:
            y = bufs["recv_x"]
        else:
            y = synth.tokens_bf16(ref.recv_rows, H, seed=seed + 101).to(dev)
        o = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        h.combine(y, wd, o)
        want = oracle.combine(y.cpu(), w, ref.dest_row, T, K)
        out["combine_diff"] = assert_bf16_close(bits16(o), want, "combine")
        out["combine_out"] = o
        out["y"] = y
    torch.cuda.synchronize()
    return out


def run_backward(res, seed=0):
    """Combine-grad dispatch, dispatch-grad combine and (with a plan and a
    gradient width G set on the handle) the replica-gradient reduce, against
    the oracle."""
    h, ref, w, idx = res["h"], res["ref"], res["w"], res["idx"]
    G = h.G
    T, H, K = h.T, h.H, h.K
    dev = torch.device("cuda")
    g = synth.tokens_bf16(T, H, seed=seed + 202)
    gy = torch.zeros((h.recv_rows, H), dtype=torch.bfloat16, device=dev)
    h.combine_backward(g.to(dev), w.to(dev), gy)
    want = oracle.combine_backward(g, w, ref.dest_row, ref.recv_rows)
    rows = res["rows"]
    assert_bf16_close(bits16(gy)[rows], want[rows], "combine backward")
    grecv = synth.tokens_bf16(h.recv_rows, H, seed=seed + 303).to(dev)
    gx = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    h.dispatch_backward(grecv, gx)
    want2 = oracle.combine(grecv.cpu(), None, ref.dest_row, T, K)
    assert_bf16_close(bits16(gx), want2, "dispatch backward")
    if h.balanced and G:
        rng = torch.Generator().manual_seed(seed + 404)
        rep = torch.randn((h.R, h.S, G), generator=rng)
        own = torch.randn((h.E, G), generator=rng)
        own_d = own.to(dev)
        h.reduce_replica_grads(rep.to(dev), own_d)
        want3 = oracle.replica_reduce(ref.plan["replica_expert"], rep.numpy(), own.numpy())
        np.testing.assert_array_equal(own_d.cpu().numpy(), want3)
    torch.cuda.synchronize()
