"""Thin ctypes binding of the C ABI in include/ep.h (argument marshalling only).

Every step of dispatch / combine runs in libep_b200.so's CUDA kernels; this
module checks tensor shapes and dtypes, passes raw device pointers and the
current CUDA stream, and turns status codes into exceptions. PyTorch is used
for device memory and streams only. There is no fallback: if the library is
missing, ``lib()`` raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libep_b200.so")

MODE_LL, MODE_HT = 0, 1
FLAG_BAD_EXPERT_ID, FLAG_DUP_EXPERT_ID, FLAG_CAPACITY, FLAG_PLAN_SLOTS = 0x1, 0x2, 0x4, 0x8
FLAG_WAIT_TIMEOUT = 0x10  # a bounded wait inside a kernel gave up; that call's outputs are incomplete
(T_DEST_ROW, T_EXPERT_COUNTS, T_RECV_COUNTS, T_RANK_LOAD, T_RANK_OFFSET, T_REPLICA_EXPERT, T_DIRECT_COUNT,
 T_DIRECT_EXPERT, T_DIRECT_LEN, T_SRC_ROW) = range(10)


class EpConfig(ctypes.Structure):
    _fields_ = [
        ("num_tokens", ctypes.c_int32),
        ("hidden", ctypes.c_int32),
        ("num_experts", ctypes.c_int32),
        ("topk", ctypes.c_int32),
        ("num_ranks", ctypes.c_int32),
        ("mode", ctypes.c_int32),
        ("ll_capacity", ctypes.c_int32),
        ("fp8", ctypes.c_int32),
        ("balanced", ctypes.c_int32),
        ("replica_slots", ctypes.c_int32),
        ("grad_elems_per_expert", ctypes.c_int64),
        ("direct_overflow", ctypes.c_int32),
    ]


MAX_PEERS = 64  # EP_MAX_PEERS


class EpPeerTable(ctypes.Structure):
    """ep_peer_table_t: every rank's receive arrays as device addresses."""
    _fields_ = [
        ("num_ranks", ctypes.c_int32),
        ("capacity_rows", ctypes.c_int64),
        ("recv_x", ctypes.c_void_p * MAX_PEERS),
        ("recv_scales", ctypes.c_void_p * MAX_PEERS),
        ("recv_w", ctypes.c_void_p * MAX_PEERS),
        ("recv_expert", ctypes.c_void_p * MAX_PEERS),
        ("flags", ctypes.c_void_p * MAX_PEERS),
    ]


class EpError(RuntimeError):
    def __init__(self, call: str, status: int):
        self.status = status
        super().__init__(f"{call} failed: {_lib_status_string(status)} ({status})")


# name -> (restype, argtypes); every entry point of include/ep.h
_P, _I32, _I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
_CFG = ctypes.POINTER(EpConfig)
SIGNATURES = {
    "ep_validate_config": (ctypes.c_int, [_CFG]),
    "ep_recv_rows": (ctypes.c_int, [_CFG, ctypes.POINTER(_I64)]),
    "ep_output_shape": (ctypes.c_int, [_CFG, ctypes.POINTER(_I64), ctypes.POINTER(ctypes.c_int32)]),
    "ep_recv_counts_len": (ctypes.c_int, [_CFG, ctypes.POINTER(_I64)]),
    "ep_workspace_bytes": (ctypes.c_int, [_CFG, ctypes.POINTER(ctypes.c_size_t)]),
    "ep_plan_kernel_count": (ctypes.c_int, [_CFG, ctypes.POINTER(_I32)]),
    "ep_version": (ctypes.c_char_p, []),
    "ep_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "ep_create": (ctypes.c_int, [_CFG, ctypes.POINTER(_P)]),
    "ep_destroy": (ctypes.c_int, [_P]),
    "ep_plan": (ctypes.c_int, [_P, _P, _P]),
    "ep_dispatch": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "ep_combine": (ctypes.c_int, [_P, _P, _P, _P, _P]),
    "ep_combine_backward": (ctypes.c_int, [_P, _P, _P, _P, _P]),
    "ep_dispatch_backward": (ctypes.c_int, [_P, _P, _P, _P]),
    "ep_reduce_replica_grads": (ctypes.c_int, [_P, _P, _P, _P]),
    "ep_prefetch_replica_weights": (ctypes.c_int, [_P, _P, _I64, _P, _P]),
    "ep_get_plan": (ctypes.c_int, [_P, _P, _P, _P]),
    "ep_get_status": (ctypes.c_int, [_P, ctypes.POINTER(_I32), _P]),
    "ep_get_tensor": (ctypes.c_int, [_P, ctypes.c_int, ctypes.POINTER(_P), ctypes.POINTER(_I64)]),
    "ep_route_noalloc": (ctypes.c_int, [_P, _I32, _I32, _I32, _P, _P, _P, _P]),
    "ep_world_recv_rows": (ctypes.c_int, [_CFG, ctypes.POINTER(_I64)]),
    "ep_plan_local_counts": (ctypes.c_int, [_P, _P, _P, _P]),
    "ep_plan_world": (ctypes.c_int, [_P, _P, _I32, _P]),
    "ep_dispatch_peers": (ctypes.c_int, [_P, _P, _P, _P, ctypes.POINTER(EpPeerTable), _P]),
    "ep_signal_peers": (ctypes.c_int, [_P, ctypes.POINTER(EpPeerTable), ctypes.c_uint32, _P]),
    "ep_wait_peers": (ctypes.c_int, [_P, _P, ctypes.c_uint32, _I64, _P]),
    "ep_combine_peers": (ctypes.c_int, [_P, ctypes.POINTER(EpPeerTable), _P, _P, _P]),
    "ep_combine_backward_peers": (ctypes.c_int, [_P, _P, _P, ctypes.POINTER(EpPeerTable), _P]),
    "ep_dispatch_backward_peers": (ctypes.c_int, [_P, ctypes.POINTER(EpPeerTable), _P, _P]),
    "ep_reduce_replica_grads_peers": (ctypes.c_int, [_P, ctypes.POINTER(EpPeerTable), _P, _P]),
    "ep_prefetch_replica_weights_peers": (ctypes.c_int, [_P, ctypes.POINTER(EpPeerTable), _I64, _P, _P]),
    "ep_ipc_export": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_uint8 * 64), ctypes.POINTER(_I64)]),
    "ep_ipc_import": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint8 * 64), _I64, ctypes.POINTER(_P),
                                     ctypes.POINTER(_P)]),
    "ep_ipc_close": (ctypes.c_int, [_P]),
    "ep_router_topk": (ctypes.c_int, [_P, _I32, _I32, _I32, _P, _P, _P]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libep_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m combine_ep_dispatch_03_b200.build` "
                "(there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _lib_status_string(status: int) -> str:
    try:
        return lib().ep_status_string(status).decode()
    except Exception:  # pragma: no cover
        return "status"


def _check(call: str, status: int) -> None:
    if status != 0:
        raise EpError(call, status)


def make_config(T: int, H: int, E: int, K: int, R: int, mode: str = "ht", ll_capacity: int = 0,
                fp8: bool = False, balanced: bool = False, replica_slots: int = 0,
                grad_elems_per_expert: int = 0, direct_overflow: bool = False) -> EpConfig:
    return EpConfig(T, H, E, K, R, MODE_LL if mode == "ll" else MODE_HT, ll_capacity, int(fp8), int(balanced),
                    replica_slots, grad_elems_per_expert, int(direct_overflow))


def validate(cfg: EpConfig) -> int:
    return lib().ep_validate_config(ctypes.byref(cfg))


def output_shape(cfg: "EpConfig") -> tuple:
    """Receive-buffer shape in elements: (rows, H) in HT, (R, E/R, cap, H) in LL."""
    dims = (_I64 * 4)()
    nd = ctypes.c_int32()
    _check("ep_output_shape", lib().ep_output_shape(ctypes.byref(cfg), dims, ctypes.byref(nd)))
    return tuple(dims[i] for i in range(nd.value))


def plan_launches(h: "Ep") -> int:
    """Kernels one ep_plan of this handle's configuration launches."""
    n = ctypes.c_int32()
    _check("ep_plan_kernel_count", lib().ep_plan_kernel_count(ctypes.byref(h.cfg), ctypes.byref(n)))
    return n.value


def _ptr(t: torch.Tensor | None, dtype: torch.dtype | None = None, numel: int | None = None,
         name: str = "tensor", device: int | None = None) -> ctypes.c_void_p | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device.index != device:
        raise ValueError(f"{name} is on cuda:{t.device.index}, the handle on cuda:{device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} must have {numel} elements, got {t.numel()}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream: torch.cuda.Stream | None) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def router_topk(logits: torch.Tensor, K: int, topk_idx: torch.Tensor, topk_w: torch.Tensor, stream=None) -> None:
    """Top-K experts and renormalised softmax weights per token (ep_router_topk):
    logits fp32 [T, E] -> topk_idx int32 [T, K], topk_w fp32 [T, K]."""
    T, E = logits.shape
    _check("ep_router_topk", lib().ep_router_topk(
        _ptr(logits, torch.float32, T * E, "logits"), T, E, K, _ptr(topk_idx, torch.int32, T * K, "topk_idx"),
        _ptr(topk_w, torch.float32, T * K, "topk_w"), _stream(stream)))


def route_noalloc(topk_idx: torch.Tensor, num_experts: int, dest_row: torch.Tensor, expert_counts: torch.Tensor,
                  flags: torch.Tensor, stream=None) -> None:
    """Routing without any device allocation (ep_route_noalloc): for callers
    that own all device memory up front. All tensors are caller-provided
    int32 CUDA tensors: topk_idx [T, K], dest_row [T*K], expert_counts [E],
    flags [1]."""
    T, K = topk_idx.shape
    _check("ep_route_noalloc", lib().ep_route_noalloc(
        _ptr(topk_idx, torch.int32, T * K, "topk_idx"), T, K, num_experts,
        _ptr(dest_row, torch.int32, T * K, "dest_row"), _ptr(expert_counts, torch.int32, num_experts,
                                                             "expert_counts"),
        _ptr(flags, torch.int32, 1, "flags"), _stream(stream)))


def world_recv_rows(cfg: EpConfig) -> int:
    """Rows one rank's receive buffer needs in a world of cfg.num_ranks GPUs."""
    rows = ctypes.c_int64()
    _check("ep_world_recv_rows", lib().ep_world_recv_rows(ctypes.byref(cfg), ctypes.byref(rows)))
    return rows.value


def _addr(t) -> int | None:
    """Device address of a CUDA tensor, or an int address as it is (peer
    buffers mapped through IPC have no tensor), or None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("peer buffers must be contiguous CUDA tensors or device addresses")
    return t.data_ptr()


def peer_table(capacity_rows: int, recv_x, flags, recv_scales=None, recv_w=None, recv_expert=None) -> EpPeerTable:
    """An ep_peer_table_t from per-rank lists (entry r: rank r's buffer, a CUDA
    tensor or a device address; the optional lists may be None)."""
    R = len(recv_x)
    if R > MAX_PEERS:
        raise ValueError(f"at most {MAX_PEERS} ranks")
    tab = EpPeerTable()
    tab.num_ranks = R
    tab.capacity_rows = capacity_rows
    for r in range(R):
        tab.recv_x[r] = _addr(recv_x[r])
        tab.flags[r] = _addr(flags[r]) if flags is not None else None
        tab.recv_scales[r] = _addr(recv_scales[r]) if recv_scales is not None else None
        tab.recv_w[r] = _addr(recv_w[r]) if recv_w is not None else None
        tab.recv_expert[r] = _addr(recv_expert[r]) if recv_expert is not None else None
    return tab


def ipc_export(t: torch.Tensor) -> tuple[bytes, int]:
    """(64-byte CUDA IPC handle of the allocation holding t, t's offset in it)."""
    h = (ctypes.c_uint8 * 64)()
    off = ctypes.c_int64()
    _check("ep_ipc_export", lib().ep_ipc_export(ctypes.c_void_p(t.data_ptr()), ctypes.byref(h), ctypes.byref(off)))
    return bytes(h), off.value


def ipc_import(handle: bytes, offset: int) -> tuple[int, int]:
    """Map a peer's exported buffer: (device address of the buffer, mapping
    base to pass to ipc_close)."""
    h = (ctypes.c_uint8 * 64).from_buffer_copy(handle)
    p, base = ctypes.c_void_p(), ctypes.c_void_p()
    _check("ep_ipc_import", lib().ep_ipc_import(ctypes.byref(h), offset, ctypes.byref(p), ctypes.byref(base)))
    return p.value, base.value


def ipc_close(base: int) -> None:
    _check("ep_ipc_close", lib().ep_ipc_close(ctypes.c_void_p(base)))


class _DeviceArray:
    """__cuda_array_interface__ view of a device pointer owned by the handle."""

    def __init__(self, ptr: int, n: int, typestr: str = "<i4"):
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": typestr, "data": (ptr, False), "version": 3}


class Ep:
    """One EP configuration and its routing state (group + handle in one)."""

    def __init__(self, T: int, H: int, E: int, K: int, R: int, mode: str = "ht", ll_capacity: int = 0,
                 fp8: bool = False, balanced: bool = False, replica_slots: int = 0,
                 grad_elems_per_expert: int = 0, direct_overflow: bool = False):
        L = lib()
        self.cfg = make_config(T, H, E, K, R, mode, ll_capacity, fp8, balanced, replica_slots,
                               grad_elems_per_expert, direct_overflow)
        self.direct = direct_overflow
        self.T, self.H, self.E, self.K, self.R = T, H, E, K, R
        self.mode, self.fp8, self.balanced = mode, fp8, balanced
        self.S = (replica_slots or E // R) if balanced else 0
        self.G = grad_elems_per_expert
        self.device = torch.cuda.current_device()  # ep_create allocates on the current device
        rows, clen = ctypes.c_int64(), ctypes.c_int64()
        _check("ep_recv_rows", L.ep_recv_rows(ctypes.byref(self.cfg), ctypes.byref(rows)))
        _check("ep_recv_counts_len", L.ep_recv_counts_len(ctypes.byref(self.cfg), ctypes.byref(clen)))
        self.recv_rows, self.counts_len = rows.value, clen.value
        h = ctypes.c_void_p()
        _check("ep_create", L.ep_create(ctypes.byref(self.cfg), ctypes.byref(h)))
        self._h = h

    # -- lifetime
    def close(self) -> None:
        if getattr(self, "_h", None):
            _check("ep_destroy", lib().ep_destroy(self._h))
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def _p(self, t, dtype=None, numel=None, name="tensor"):
        """A tensor's device pointer, checked to be on this handle's device."""
        return _ptr(t, dtype, numel, name, device=self.device)

    # -- output allocation helpers (plumbing)
    def empty_recv(self, device="cuda") -> dict:
        rows, H = self.recv_rows, self.H
        out = {
            "recv_x": torch.empty((rows, H), dtype=torch.float8_e4m3fn if self.fp8 else torch.bfloat16,
                                  device=device),
            "recv_scales": torch.empty((rows, H // 128), dtype=torch.float32, device=device) if self.fp8 else None,
            "recv_w": torch.empty(rows, dtype=torch.float32, device=device),
            "recv_expert": torch.empty(rows, dtype=torch.int32, device=device),
            "recv_counts": torch.empty(self.counts_len, dtype=torch.int32, device=device),
        }
        return out

    # -- forward
    def plan(self, topk_idx: torch.Tensor, stream=None) -> None:
        _check("ep_plan", lib().ep_plan(self._h, self._p(topk_idx, torch.int32, self.T * self.K, "topk_idx"),
                                        _stream(stream)))

    def dispatch(self, x, topk_idx, topk_w, recv_x, recv_scales=None, recv_w=None, recv_expert=None,
                 recv_counts=None, stream=None) -> None:
        """Rows, scales (FP8), weights, expert ids and per-slot counts into the
        caller's receive buffers (see empty_recv)."""
        rows, H = self.recv_rows, self.H
        _check("ep_dispatch", lib().ep_dispatch(
            self._h, self._p(x, torch.bfloat16, self.T * H, "x"),
            self._p(topk_idx, torch.int32, self.T * self.K, "topk_idx"),
            self._p(topk_w, torch.float32, self.T * self.K, "topk_w"),
            self._p(recv_x, torch.float8_e4m3fn if self.fp8 else torch.bfloat16, rows * H, "recv_x"),
            self._p(recv_scales, torch.float32, rows * (H // 128), "recv_scales"),
            self._p(recv_w, torch.float32, rows, "recv_w"),
            self._p(recv_expert, torch.int32, rows, "recv_expert"),
            self._p(recv_counts, torch.int32, self.counts_len, "recv_counts"),
            _stream(stream)))

    def combine(self, expert_out, topk_w, out, stream=None) -> None:
        _check("ep_combine", lib().ep_combine(
            self._h, self._p(expert_out, torch.bfloat16, self.recv_rows * self.H, "expert_out"),
            self._p(topk_w, torch.float32, self.T * self.K, "topk_w"),
            self._p(out, torch.bfloat16, self.T * self.H, "out"), _stream(stream)))

    # -- backward
    def combine_backward(self, grad_out, topk_w, grad_expert_out, stream=None) -> None:
        _check("ep_combine_backward", lib().ep_combine_backward(
            self._h, self._p(grad_out, torch.bfloat16, self.T * self.H, "grad_out"),
            self._p(topk_w, torch.float32, self.T * self.K, "topk_w"),
            self._p(grad_expert_out, torch.bfloat16, self.recv_rows * self.H, "grad_expert_out"), _stream(stream)))

    def dispatch_backward(self, grad_recv, grad_x, stream=None) -> None:
        _check("ep_dispatch_backward", lib().ep_dispatch_backward(
            self._h, self._p(grad_recv, torch.bfloat16, self.recv_rows * self.H, "grad_recv"),
            self._p(grad_x, torch.bfloat16, self.T * self.H, "grad_x"), _stream(stream)))

    def reduce_replica_grads(self, replica_grad, owner_grad, stream=None) -> None:
        _check("ep_reduce_replica_grads", lib().ep_reduce_replica_grads(
            self._h, self._p(replica_grad, torch.float32, self.R * max(self.S, 1) * self.G, "replica_grad"),
            self._p(owner_grad, torch.float32, self.E * self.G, "owner_grad"), _stream(stream)))

    def prefetch_replica_weights(self, expert_weights, prefetch_slots, stream=None) -> None:
        """Copy each filled replica slot's expert weights into it: expert_weights
        [E, ...] and prefetch_slots [R, S, ...] of the same row size in bytes."""
        total = expert_weights.numel() * expert_weights.element_size()
        if total % self.E:
            raise ValueError("expert_weights must hold E rows of equal size")
        nbytes = total // self.E
        if prefetch_slots.numel() * prefetch_slots.element_size() != self.R * max(self.S, 1) * nbytes:
            raise ValueError("prefetch_slots must hold R*S rows of one expert's weights")
        _check("ep_prefetch_replica_weights", lib().ep_prefetch_replica_weights(
            self._h, self._p(expert_weights), nbytes, self._p(prefetch_slots), _stream(stream)))

    # -- expert parallelism across GPUs (one rank per GPU; see include/ep.h)
    def plan_local_counts(self, topk_idx, counts, stream=None) -> None:
        """This rank's routed pairs per expert into counts (int32 [E])."""
        _check("ep_plan_local_counts", lib().ep_plan_local_counts(
            self._h, self._p(topk_idx, torch.int32, self.T * self.K, "topk_idx"),
            self._p(counts, torch.int32, self.E, "counts"), _stream(stream)))

    def plan_world(self, world_counts, rank: int, stream=None) -> None:
        """The world's plan from every rank's counts (int32 [R, E], rank order)."""
        _check("ep_plan_world", lib().ep_plan_world(
            self._h, self._p(world_counts, torch.int32, self.R * self.E, "world_counts"), rank, _stream(stream)))

    def dispatch_peers(self, x, topk_idx, topk_w, table: EpPeerTable, stream=None) -> None:
        _check("ep_dispatch_peers", lib().ep_dispatch_peers(
            self._h, self._p(x, torch.bfloat16, self.T * self.H, "x"),
            self._p(topk_idx, torch.int32, self.T * self.K, "topk_idx"),
            self._p(topk_w, torch.float32, self.T * self.K, "topk_w"), ctypes.byref(table), _stream(stream)))

    def signal_peers(self, table: EpPeerTable, epoch: int, stream=None) -> None:
        _check("ep_signal_peers", lib().ep_signal_peers(self._h, ctypes.byref(table), epoch, _stream(stream)))

    def wait_peers(self, flags, epoch: int, timeout_us: int = 0, stream=None) -> None:
        """Wait (bounded) until every source has signalled `epoch` into flags
        (this rank's uint32 [R], given as an int32 CUDA tensor)."""
        _check("ep_wait_peers", lib().ep_wait_peers(
            self._h, self._p(flags, torch.int32, self.R, "flags"), epoch, timeout_us, _stream(stream)))

    def combine_peers(self, table: EpPeerTable, topk_w, out, stream=None) -> None:
        _check("ep_combine_peers", lib().ep_combine_peers(
            self._h, ctypes.byref(table), self._p(topk_w, torch.float32, self.T * self.K, "topk_w"),
            self._p(out, torch.bfloat16, self.T * self.H, "out"), _stream(stream)))

    def combine_backward_peers(self, grad_out, topk_w, grad_rows: EpPeerTable, stream=None) -> None:
        _check("ep_combine_backward_peers", lib().ep_combine_backward_peers(
            self._h, self._p(grad_out, torch.bfloat16, self.T * self.H, "grad_out"),
            self._p(topk_w, torch.float32, self.T * self.K, "topk_w"), ctypes.byref(grad_rows), _stream(stream)))

    def dispatch_backward_peers(self, grad_rows: EpPeerTable, grad_x, stream=None) -> None:
        _check("ep_dispatch_backward_peers", lib().ep_dispatch_backward_peers(
            self._h, ctypes.byref(grad_rows), self._p(grad_x, torch.bfloat16, self.T * self.H, "grad_x"),
            _stream(stream)))

    def reduce_replica_grads_peers(self, replica_grads: EpPeerTable, owner_grad, stream=None) -> None:
        """This rank's experts' gradients [E/R, G] += their replicas' gradients,
        read through the table (entry r: rank r's [S, G] fp32)."""
        _check("ep_reduce_replica_grads_peers", lib().ep_reduce_replica_grads_peers(
            self._h, ctypes.byref(replica_grads), self._p(owner_grad, torch.float32, (self.E // self.R) * self.G,
                                                          "owner_grad"), _stream(stream)))

    def prefetch_replica_weights_peers(self, weights: EpPeerTable, bytes_per_expert: int, prefetch_slots,
                                       stream=None) -> None:
        """This rank's filled replica slots [S, bytes] receive their experts'
        weights, read from the owners' entries of the table ([E/R, bytes] each)."""
        if prefetch_slots.numel() * prefetch_slots.element_size() != max(self.S, 1) * bytes_per_expert:
            raise ValueError("prefetch_slots must hold S rows of one expert's weights")
        _check("ep_prefetch_replica_weights_peers", lib().ep_prefetch_replica_weights_peers(
            self._h, ctypes.byref(weights), bytes_per_expert, self._p(prefetch_slots), _stream(stream)))

    # -- inspection
    def get_plan(self, stream=None) -> tuple[list[int], list[int]]:
        rep = (ctypes.c_int32 * (self.R * self.S))()
        load = (ctypes.c_int32 * self.R)()
        rep_p = ctypes.cast(rep, _P) if self.S > 0 else None
        _check("ep_get_plan", lib().ep_get_plan(self._h, rep_p, ctypes.cast(load, _P), _stream(stream)))
        return list(rep), list(load)

    def status(self, stream=None) -> int:
        f = ctypes.c_int32()
        _check("ep_get_status", lib().ep_get_status(self._h, ctypes.byref(f), _stream(stream)))
        return f.value

    def tensor(self, which: int) -> torch.Tensor:
        """A copy of one piece of the routing state (int32, on the device)."""
        p, n = ctypes.c_void_p(), ctypes.c_int64()
        _check("ep_get_tensor", lib().ep_get_tensor(self._h, which, ctypes.byref(p), ctypes.byref(n)))
        if n.value == 0:
            return torch.empty(0, dtype=torch.int32, device="cuda")
        return torch.as_tensor(_DeviceArray(p.value, n.value), device="cuda").clone()
