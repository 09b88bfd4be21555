"""ep_route_noalloc: routing for callers that cannot allocate device memory.

Serving engines that hand nearly all of HBM to their own memory pool, and
plugin hosts that forbid allocation after start-up, cannot let a library call
cudaMalloc on the hot path. ep_route_noalloc computes the same routing as
ep_plan (HT layout, no balanced plan) with its scratch in a fixed static
device array instead of a handle's workspace. These tests check, through the
C ABI, that it returns exactly what the handle-based entry point and the CPU
oracle return, on two calls in a row with different sizes (so the second call
runs over the first call's leftover scratch), and that oversized inputs are
refused.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from combine_ep_dispatch_03_b200 import ep, synth

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _routing(T, E, K, s, seed, corrupt=False):
    idx, _ = synth.routing(T, E, K, zipf_s=s, seed=seed)
    if corrupt:
        idx = idx.clone()
        idx[1, 0] = -1            # masked choice
        idx[2, 0] = E + 3         # bad id
        if K > 1:
            idx[3, 1] = idx[3, 0]  # repeated id
    return idx.cuda()


def _reference(idx, E):
    """The existing entry point: a handle, ep_plan, and its routing state."""
    T, K = idx.shape
    h = ep.Ep(T, 128, E, K, 1)
    h.plan(idx)
    out = (h.tensor(ep.T_DEST_ROW).cpu().numpy(), h.tensor(ep.T_EXPERT_COUNTS).cpu().numpy(), h.status())
    h.close()
    return out


def _noalloc(idx, E):
    T, K = idx.shape
    dest = torch.full((T * K,), 12345, dtype=torch.int32, device="cuda")
    cnt = torch.full((E,), 777, dtype=torch.int32, device="cuda")
    flags = torch.full((1,), 99, dtype=torch.int32, device="cuda")
    ep.route_noalloc(idx, E, dest, cnt, flags)
    torch.cuda.synchronize()
    return dest.cpu().numpy(), cnt.cpu().numpy(), int(flags.item())


def _check_against_oracle(idx, E, got):
    """The CPU oracle's routing for one logical rank (plain HT layout)."""
    want = oracle.route(idx.cpu(), E=E, R=1)
    np.testing.assert_array_equal(got[0], want.dest_row)
    np.testing.assert_array_equal(got[1], want.cnt)
    assert got[2] == want.flags


def test_noalloc_matches_plan_on_two_calls_in_a_row():
    cases = [
        (65536, 64, 8, 0.0, 0, False),   # 524288 pairs: the tile, scan and assignment kernels with their scratch
        (3000, 64, 2, 1.5, 1, True),     # smaller, skewed, with masked / bad / repeated ids
        (32768, 256, 8, 0.0, 2, False),  # the HT prefill routing
    ]
    for T, E, K, s, seed, corrupt in cases:  # later calls reuse the earlier calls' scratch
        idx = _routing(T, E, K, s, seed, corrupt)
        want = _reference(idx, E)
        got = _noalloc(idx, E)
        np.testing.assert_array_equal(got[0], want[0])  # routing is bit-exact
        np.testing.assert_array_equal(got[1], want[1])
        assert got[2] == want[2]
        assert want[2] == ((ep.FLAG_BAD_EXPERT_ID | ep.FLAG_DUP_EXPERT_ID) if corrupt else 0)
        _check_against_oracle(idx, E, got)


def test_noalloc_small_and_empty_batches():
    for T, E, K in [(7, 16, 2), (0, 16, 2)]:
        idx = _routing(T, E, K, 0.0, 3) if T else torch.empty((0, K), dtype=torch.int32, device="cuda")
        want = _reference(idx, E)
        got = _noalloc(idx, E)
        np.testing.assert_array_equal(got[0], want[0])
        np.testing.assert_array_equal(got[1], want[1])
        assert got[2] == want[2] == 0
        _check_against_oracle(idx, E, got)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """1M pairs need more scratch than the fixed array holds: the call returns
    EP_ERR_TOO_LARGE and launches nothing. The buffers are real and of the
    right sizes, so even a call that wrongly went ahead would stay in bounds;
    the outputs must keep their fill values."""
    T, K, E = 131072, 8, 384
    L = ep.lib()
    idx = _routing(T, E, K, 0.0, 4)
    dest = torch.full((T * K,), 12345, dtype=torch.int32, device="cuda")
    cnt = torch.full((E,), 777, dtype=torch.int32, device="cuda")
    flags = torch.full((1,), 99, dtype=torch.int32, device="cuda")
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    assert L.ep_route_noalloc(ptr(idx), T, K, E, ptr(dest), ptr(cnt), ptr(flags), st) == 6  # EP_ERR_TOO_LARGE
    assert L.ep_status_string(6) == b"EP_ERR_TOO_LARGE"
    torch.cuda.synchronize()
    assert (dest == 12345).all() and (cnt == 777).all() and int(flags.item()) == 99
