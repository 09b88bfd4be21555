"""CPU oracle for MoE expert-parallel dispatch and combine.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package. The product
path (``combine_ep_dispatch_03_b200``) never imports it and the two share no
code. The arithmetic lives in ``ep_oracle.c`` (plain single-threaded C); this
module only marshals numpy / torch CPU arrays into it.

Every function cites the passage it follows in ``ep_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ep_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "libep_oracle.so")

FLAG_BAD_EXPERT_ID = 1
FLAG_DUP_EXPERT_ID = 2
FLAG_CAPACITY = 4
FLAG_PLAN_SLOTS = 8


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no contraction of multiply-adds)."""
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC):
        return _LIB_PATH
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(
        ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
         "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
    )
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def configure(cdll: ctypes.CDLL) -> ctypes.CDLL:
    """Declare the argument and result types of the oracle's C functions."""
    P = ctypes.c_void_p
    i32, i64 = ctypes.c_int, ctypes.c_int64
    sig = {
        "orc_bf16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
        "orc_bf16_from_f32": (ctypes.c_uint16, [ctypes.c_float]),
        "orc_e4m3_from_f32": (ctypes.c_uint8, [ctypes.c_float]),
        "orc_e4m3_to_f32": (ctypes.c_float, [ctypes.c_uint8]),
        "orc_bf16_from_f32_n": (None, [P, i64, P]),
        "orc_e4m3_from_f32_n": (None, [P, i64, P]),
        "orc_router_topk": (None, [i32, i32, i32, P, P, P]),
        "orc_route": (i32, [i32, i32, i32, P, P, P]),
        "orc_layout_ht": (None, [i32, i32, i32, P, P, P, P]),
        "orc_layout_ll": (i32, [i32, i32, i32, P, P, P]),
        "orc_plan_balanced": (i32, [i32, i32, i32, P, P, P, P, P, P, P, P, P]),
        "orc_layout_balanced": (None, [i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P, P, P]),
        "orc_plan_direct": (i32, [i32, i32, i32, P, P, P, P, P, P, P, P, P, P, P, P, P]),
        "orc_layout_direct": (None, [i32, i32, i32, i32, i32] + [P] * 14),
        "orc_dispatch": (None, [i32, i32, i32, i32, P, P, P, P, P, P, P, P]),
        "orc_combine": (None, [i32, i32, i32, P, P, P, P]),
        "orc_combine_backward": (None, [i32, i32, i32, P, P, P, P]),
        "orc_replica_reduce": (None, [i32, i32, i32, i64, P, P, P]),
        "orc_prefetch": (None, [i32, i32, i64, P, P, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(cdll, name)
        f.restype = res
        f.argtypes = args
    return cdll


def compile_to(src: str, out: str) -> str:
    """Compile an oracle source file with the oracle's flags."""
    subprocess.check_call(["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
                           "-Wall", "-o", out, src, "-lm"])
    return out


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = configure(ctypes.CDLL(build()))
    return _lib


def _np(a, dtype) -> np.ndarray:
    """Contiguous numpy view/copy of a numpy array or CPU torch tensor."""
    try:
        import torch

        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().contiguous()
            if a.dtype == torch.bfloat16:
                a = a.view(torch.int16).numpy().view(np.uint16)
            elif a.dtype == torch.float8_e4m3fn:
                a = a.view(torch.uint8).numpy()
            else:
                a = a.numpy()
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        if dtype == np.uint16 and a.dtype == np.int16:
            a = a.view(np.uint16)
        else:
            a = a.astype(dtype)
    return a


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- formats

def bf16_from_f32(v: np.ndarray) -> np.ndarray:
    """Element-wise RNE float32 -> bf16 bits (uint16)."""
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float32).ravel())
    out = np.zeros(v.size, np.uint16)
    lib().orc_bf16_from_f32_n(_p(v), v.size, _p(out))
    return out


def e4m3_from_f32(v: np.ndarray) -> np.ndarray:
    """Element-wise float32 -> e4m3 code (uint8), RNE, saturating to +-448."""
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float32).ravel())
    out = np.zeros(v.size, np.uint8)
    lib().orc_e4m3_from_f32_n(_p(v), v.size, _p(out))
    return out


def e4m3_to_f32(q: np.ndarray) -> np.ndarray:
    L = lib()
    q = np.asarray(q, dtype=np.uint8).ravel()
    return np.array([L.orc_e4m3_to_f32(int(c)) for c in q], dtype=np.float32)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bits -> float32 values (exact; the bits are the float's top half)."""
    b = np.asarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------- router

def router_topk(logits, K: int):
    """(topk_idx [T, K] int32, topk_w [T, K] float32) from logits [T, E]."""
    lg = _np(logits, np.float32)
    T, E = lg.shape
    idx = np.zeros((T, K), np.int32)
    w = np.zeros((T, K), np.float32)
    lib().orc_router_topk(T, E, K, _p(lg), _p(idx), _p(w))
    return idx, w


# ---------------------------------------------------------------- routing

@dataclass
class Routing:
    cnt: np.ndarray          # [E] routed pairs per expert
    j: np.ndarray            # [T*K] stable index within the expert, -1 if not routed
    dest_row: np.ndarray     # [T*K] row in the receive buffer, -1 if not placed
    flags: int
    recv_rows: int           # rows of the receive buffer
    recv_counts: np.ndarray  # HT: [E] or [R, g+S] under a plan; LL: [E] rows kept
    plan: dict | None = None

    @property
    def src_row(self) -> np.ndarray:
        """[recv_rows]: the pair index t*K+k placed in each receive row, -1 for
        rows no pair targets. By definition the inverse of dest_row, which is
        one-to-one on the placed pairs."""
        src = np.full(self.recv_rows, -1, np.int64)
        placed = np.nonzero(self.dest_row >= 0)[0]
        src[self.dest_row[placed]] = placed
        return src.astype(np.int32)


def route(idx, E: int, R: int, mode: str = "ht", cap: int = 0, balanced: bool = False,
          slots: int | None = None, direct: bool = False) -> Routing:
    """Counts, stable slots and destination rows (HT, LL or balanced HT; with
    `direct`, the inference plan whose overflow pieces read the owner's
    weights directly)."""
    L = lib()
    idx = _np(idx, np.int32)
    T, K = idx.shape
    cnt = np.zeros(E, np.int32)
    j = np.zeros(T * K, np.int32)
    flags = L.orc_route(T, K, E, _p(idx), _p(cnt), _p(j))
    dest = np.zeros(T * K, np.int32)
    g = E // R
    if mode == "ll":
        flags |= L.orc_layout_ll(T, K, cap, _p(idx), _p(j), _p(dest))
        return Routing(cnt, j, dest, flags, E * cap, np.minimum(cnt, cap).astype(np.int32))
    if not balanced:
        L.orc_layout_ht(T, K, E, _p(idx), _p(cnt), _p(j), _p(dest))
        return Routing(cnt, j, dest, flags, T * K, cnt.copy())
    S = g if slots is None else int(slots)
    keep = np.zeros(E, np.int32)
    tail_start = np.zeros(E, np.int32)
    tail_len = np.zeros(E, np.int32)
    rep = np.zeros(R * S, np.int32)
    sstart = np.zeros(R * S, np.int32)
    slen = np.zeros(R * S, np.int32)
    load = np.zeros(R, np.int32)
    roff = np.zeros(R + 1, np.int32)
    plan = {}
    if direct:
        dn = np.zeros(R, np.int32)
        de = np.zeros(R * E, np.int32)
        ds = np.zeros(R * E, np.int32)
        dl = np.zeros(R * E, np.int32)
        flags |= L.orc_plan_direct(E, R, S, _p(cnt), _p(keep), _p(tail_start), _p(tail_len), _p(rep), _p(sstart),
                                   _p(slen), _p(dn), _p(de), _p(ds), _p(dl), _p(load), _p(roff))
        L.orc_layout_direct(T, K, E, R, S, _p(idx), _p(j), _p(keep), _p(tail_start), _p(tail_len), _p(rep),
                            _p(sstart), _p(slen), _p(dn), _p(de), _p(ds), _p(dl), _p(roff), _p(dest))
        plan.update(direct_n=dn, direct_expert=de.reshape(R, E), direct_start=ds.reshape(R, E),
                    direct_len=dl.reshape(R, E))
    else:
        flags |= L.orc_plan_balanced(E, R, S, _p(cnt), _p(keep), _p(tail_start), _p(tail_len), _p(rep),
                                     _p(sstart), _p(slen), _p(load), _p(roff))
        L.orc_layout_balanced(T, K, E, R, S, _p(idx), _p(j), _p(keep), _p(tail_start), _p(tail_len), _p(rep),
                              _p(sstart), _p(slen), _p(roff), _p(dest))
    own = (keep + tail_len).reshape(R, g)
    counts = np.concatenate([own, slen.reshape(R, S)], axis=1).astype(np.int32)
    plan.update(keep=keep, tail_start=tail_start, tail_len=tail_len, replica_expert=rep.reshape(R, S),
                slot_start=sstart.reshape(R, S), slot_len=slen.reshape(R, S), rank_load=load, rank_off=roff)
    return Routing(cnt, j, dest, flags, T * K, counts, plan)


# ---------------------------------------------------------------- data path

def dispatch(x, idx, w, dest_row, recv_rows: int, fp8: bool = False):
    """Rows of the receive buffer; returns (recv, scales, recv_w, recv_expert).

    Rows that no pair targets are zero here (the kernels leave them untouched;
    tests only compare targeted rows)."""
    L = lib()
    xb = _np(x, np.uint16)
    T, H = xb.shape
    idx = _np(idx, np.int32)
    K = idx.shape[1]
    w = _np(w, np.float32)
    dest = _np(dest_row, np.int32).ravel()
    if fp8:
        recv = np.zeros((recv_rows, H), np.uint8)
        scales = np.zeros((recv_rows, H // 128), np.float32)
    else:
        recv = np.zeros((recv_rows, H), np.uint16)
        scales = None
    rw = np.zeros(recv_rows, np.float32)
    re = np.full(recv_rows, -1, np.int32)
    L.orc_dispatch(T, K, H, int(fp8), _p(xb), _p(idx), _p(w), _p(dest), _p(recv), _p(scales), _p(rw), _p(re))
    return recv, scales, rw, re


def combine(y, w, dest_row, T: int, K: int) -> np.ndarray:
    """out[T, H] bf16 bits; w=None gives the unweighted (dispatch-gradient) sum."""
    L = lib()
    yb = _np(y, np.uint16)
    H = yb.shape[1]
    dest = _np(dest_row, np.int32).ravel()
    wa = None if w is None else _np(w, np.float32)
    out = np.zeros((T, H), np.uint16)
    L.orc_combine(T, K, H, _p(yb), _p(wa), _p(dest), _p(out))
    return out


def combine_backward(g, w, dest_row, recv_rows: int) -> np.ndarray:
    """grad of the expert outputs [recv_rows, H] bf16 bits (untargeted rows 0)."""
    L = lib()
    gb = _np(g, np.uint16)
    T, H = gb.shape
    wa = _np(w, np.float32)
    K = wa.shape[1]
    dest = _np(dest_row, np.int32).ravel()
    gy = np.zeros((recv_rows, H), np.uint16)
    L.orc_combine_backward(T, K, H, _p(gb), _p(wa), _p(dest), _p(gy))
    return gy


def replica_reduce(replica_expert, rep, owner) -> np.ndarray:
    """owner [E, G] fp32 after adding every replica slot's gradient."""
    L = lib()
    re = _np(replica_expert, np.int32)
    R, S = re.shape
    rep = _np(rep, np.float32).reshape(R * S, -1)
    out = _np(owner, np.float32).copy()
    E, G = out.shape
    L.orc_replica_reduce(E, R, S, G, _p(re), _p(rep), _p(out))
    return out


def prefetch(replica_expert, weights, slots) -> np.ndarray:
    """slots [R, S, B] bytes after copying each filled slot's expert weights
    (weights [E, B] bytes); empty slots keep their contents."""
    re = _np(replica_expert, np.int32)
    R, S = re.shape
    wt = np.ascontiguousarray(np.asarray(weights, dtype=np.uint8))
    out = np.ascontiguousarray(np.asarray(slots, dtype=np.uint8)).copy()
    B = wt.shape[1]
    lib().orc_prefetch(R, S, B, _p(re), _p(wt), _p(out))
    return out
