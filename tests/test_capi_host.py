"""The C-ABI library loads and exports every entry point include/ep.h
declares; the host-only queries validate configurations without a GPU."""
import ctypes
import os
import re

import pytest

from conftest import ROOT


@pytest.fixture(scope="module")
def L():
    from combine_ep_dispatch_03_b200 import build, ep

    build.build()
    return ep.lib()


def _declared() -> list[str]:
    src = open(os.path.join(ROOT, "include", "ep.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ep_[a-z_]+)\s*\(", src)))


def test_header_declares_the_api():
    names = _declared()
    for n in ["ep_create", "ep_destroy", "ep_plan", "ep_dispatch", "ep_combine", "ep_combine_backward",
              "ep_dispatch_backward", "ep_reduce_replica_grads", "ep_get_plan", "ep_get_status"]:
        assert n in names


def test_library_exports_every_declared_symbol(L):
    from combine_ep_dispatch_03_b200 import ep

    for name in _declared():
        assert hasattr(L, name), name
        assert name in ep.SIGNATURES, f"binding lacks {name}"


def test_version_and_status_strings(L):
    assert L.ep_version().decode().count(".") == 2
    assert L.ep_status_string(0) == b"EP_OK"
    assert L.ep_status_string(1) == b"EP_ERR_INVALID_ARG"


def _cfg(**kw):
    from combine_ep_dispatch_03_b200 import ep

    base = dict(T=128, H=1024, E=16, K=2, R=4)
    base.update(kw)
    return ep.make_config(**base)


@pytest.mark.parametrize("kw,status", [
    ({}, 0),
    (dict(T=0), 0),
    (dict(H=1004), 1),                # not a multiple of 8
    (dict(H=1032, fp8=True), 1),      # fp8 needs 128-element blocks
    (dict(E=18), 1),                  # E % R != 0
    (dict(K=17), 1),                  # K > E
    (dict(K=33, E=64), 1),            # K > 32
    (dict(E=8192, R=8), 1),           # too many experts
    (dict(mode="ll", ll_capacity=0), 1),
    (dict(mode="ll", ll_capacity=64, balanced=True), 3),
    (dict(balanced=True, replica_slots=5), 1),  # more than E/R slots
    (dict(balanced=True, replica_slots=4), 0),
    (dict(replica_slots=2), 1),       # slots without a plan
    (dict(grad_elems_per_expert=6), 1),
    (dict(T=-1), 1),
    # a balanced plan's tables fit one CTA's shared memory (the limit ep.h states)
    (dict(E=1696, R=8, K=8, balanced=True), 0),
    (dict(E=2048, R=8, K=8, balanced=True), 3),  # unsupported, not malformed
    (dict(E=2048, R=8, K=8, balanced=True, replica_slots=2), 0),
    (dict(E=2048, R=8, K=8), 0),      # no plan: no such limit
])
def test_validate(L, kw, status):
    cfg = _cfg(**kw)
    assert L.ep_validate_config(ctypes.byref(cfg)) == status


def test_recv_rows_and_counts(L):
    rows, n = ctypes.c_int64(), ctypes.c_int64()
    cfg = _cfg()
    assert L.ep_recv_rows(ctypes.byref(cfg), ctypes.byref(rows)) == 0 and rows.value == 256
    assert L.ep_recv_counts_len(ctypes.byref(cfg), ctypes.byref(n)) == 0 and n.value == 16
    cfg = _cfg(mode="ll", ll_capacity=100)
    assert L.ep_recv_rows(ctypes.byref(cfg), ctypes.byref(rows)) == 0 and rows.value == 1600
    cfg = _cfg(balanced=True)
    assert L.ep_recv_counts_len(ctypes.byref(cfg), ctypes.byref(n)) == 0 and n.value == 4 * (4 + 4)
    b = ctypes.c_size_t()
    assert L.ep_workspace_bytes(ctypes.byref(cfg), ctypes.byref(b)) == 0 and b.value > 0


def test_output_shape(L):
    """HT: one row per (token, k) pair, [T*K, H]; LL: [R, E/R, cap, H]."""
    from combine_ep_dispatch_03_b200 import ep

    assert ep.output_shape(_cfg()) == (256, 1024)
    assert ep.output_shape(_cfg(fp8=True)) == (256, 1024)
    assert ep.output_shape(_cfg(mode="ll", ll_capacity=100)) == (4, 4, 100, 1024)
    dims, nd = (ctypes.c_int64 * 4)(), ctypes.c_int32()
    assert L.ep_output_shape(ctypes.byref(_cfg(E=18)), dims, ctypes.byref(nd)) == 1  # E % R != 0
    assert L.ep_output_shape(ctypes.byref(_cfg()), None, ctypes.byref(nd)) == 1


@pytest.mark.parametrize("kw,count", [
    (dict(T=100, E=256, K=8, R=8), 1),            # 800 pairs: one CTA
    (dict(T=32768, E=256, K=8, R=8), 3),          # 262144 pairs: three kernels
    (dict(T=100, E=256, K=8, R=8, balanced=True), 1),    # 800 pairs with a plan: one CTA
    (dict(T=128, E=256, K=8, R=8, balanced=True), 1),    # 1024 pairs: the largest one-CTA plan
    (dict(T=129, E=256, K=8, R=8, balanced=True), 3),
    (dict(T=1024, E=256, K=8, R=8, balanced=True), 3),
])
def test_plan_kernel_count(L, kw, count):
    """Counts that do not depend on the device (the cluster path, 1025 to
    32768 pairs, asks the GPU whether its cluster fits)."""
    n = ctypes.c_int32()
    assert L.ep_plan_kernel_count(ctypes.byref(_cfg(**kw)), ctypes.byref(n)) == 0
    assert n.value == count


def test_null_arguments_rejected_without_gpu(L):
    assert L.ep_create(None, None) == 1
    assert L.ep_destroy(None) == 0
    assert L.ep_plan(None, None, None) == 1
    assert L.ep_get_status(None, None, None) == 1


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="host-only check: needs no GPU")
def test_noalloc_refuses_misaligned_pointers_before_any_launch(L):
    """ep_route_noalloc checks every int32 pointer for 4-byte alignment and
    returns EP_ERR_INVALID_ARG (1) before it touches the device: here there is
    no GPU, so a call that got past the checks would report EP_ERR_CUDA (2)
    instead. The addresses are never dereferenced."""
    ok, odd = ctypes.c_void_p(4096), ctypes.c_void_p(4098)
    T, K, E = 64, 2, 16
    for i in range(4):
        args = [ok, ok, ok, ok]
        args[i] = odd
        idx, dest, cnt, fl = args
        assert L.ep_route_noalloc(idx, T, K, E, dest, cnt, fl, None) == 1, i
    # the same call with aligned pointers gets as far as the device lookup
    assert L.ep_route_noalloc(ok, T, K, E, ok, ok, ok, None) == 2


class _FakeCudaTensor:
    """Stands in for a CUDA tensor (no GPU here): only what the binding's
    pointer marshalling reads."""

    def __init__(self, index):
        import torch

        self.is_cuda = True
        self.device = type("D", (), {"index": index})()
        self.dtype = torch.float32

    def is_contiguous(self):
        return True

    def numel(self):
        return 4

    def data_ptr(self):
        return 4096


def test_binding_rejects_a_tensor_on_another_device():
    import torch

    from combine_ep_dispatch_03_b200 import ep

    with pytest.raises(ValueError, match="cuda:1, the handle on cuda:0"):
        ep._ptr(_FakeCudaTensor(1), torch.float32, 4, "x", device=0)
    assert ep._ptr(_FakeCudaTensor(1), torch.float32, 4, "x", device=1).value == 4096
    assert ep._ptr(_FakeCudaTensor(1), torch.float32, 4, "x").value == 4096  # no handle: no device to match
    with pytest.raises(ValueError, match="must have 8 elements"):
        ep._ptr(_FakeCudaTensor(0), torch.float32, 8, "x", device=0)


def test_shape_queries_agree_with_the_oracle_layout(L):
    """ep_recv_rows / ep_recv_counts_len (host-only) against the receive
    buffer the oracle lays out, over random HT, LL and planned configs."""
    import numpy as np

    import oracle
    from combine_ep_dispatch_03_b200 import ep, synth

    oracle.build()
    rng = np.random.default_rng(5)
    for i in range(40):
        R = int(rng.choice([1, 2, 4, 8]))
        E = R * int(rng.choice([1, 2, 4, 8]))
        K = int(rng.integers(1, min(E, 8) + 1))
        T = int(rng.integers(1, 200))
        mode = "ll" if i % 3 == 0 else "ht"
        cap = int(rng.integers(1, T + 1)) if mode == "ll" else 0
        balanced = mode == "ht" and i % 3 == 1
        direct = balanced and i % 2 == 0
        idx, _ = synth.routing(T, E, K, zipf_s=1.0, seed=i)
        ref = oracle.route(idx, E=E, R=R, mode=mode, cap=cap, balanced=balanced, direct=direct)
        cfg = ep.make_config(T, 128, E, K, R, mode=mode, ll_capacity=cap, balanced=balanced,
                             direct_overflow=direct)
        rows, n = ctypes.c_int64(), ctypes.c_int64()
        assert L.ep_recv_rows(ctypes.byref(cfg), ctypes.byref(rows)) == 0
        assert L.ep_recv_counts_len(ctypes.byref(cfg), ctypes.byref(n)) == 0
        assert rows.value == ref.recv_rows
        assert n.value == ref.recv_counts.size
        shape = ep.output_shape(cfg)
        assert int(np.prod(shape)) == ref.recv_rows * 128
