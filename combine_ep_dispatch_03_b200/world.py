"""Host plumbing of expert parallelism across GPUs (one rank per GPU).

The device work (counts, the world plan, peer dispatch and combine, flags)
is in libep_b200.so (include/ep.h, the "across GPUs" section). This module
only moves host-side data between the ranks with torch.distributed:

* gather_counts: the all-gather of every rank's per-expert counts into the
  [R, E] table ep_plan_world reads (one collective of R*E int32);
* exchange_handles: every rank's CUDA IPC handles of its receive buffers, so
  that each rank can map its peers' buffers into its own peer table;
* peer_table_from_handles: the mapped table (ep_ipc_import for the peers,
  the rank's own buffers as they are).

There is no data-path fallback here: all row movement is in the library.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import ep


def gather_counts(local_counts: torch.Tensor, group=None) -> torch.Tensor:
    """[R, E] int32: row r = rank r's counts (rank order), on local_counts'
    device. local_counts: this rank's int32 [E] (ep_plan_local_counts)."""
    R, E = dist.get_world_size(group), local_counts.numel()
    out = torch.empty(R * E, dtype=local_counts.dtype, device=local_counts.device)
    dist.all_gather_into_tensor(out, local_counts.contiguous().view(-1), group=group)
    return out.view(R, E)


def exchange_handles(local: dict, group=None) -> list[dict]:
    """Every rank's entry of `local` (name -> picklable value, e.g. an
    ep.ipc_export result), in rank order."""
    R = dist.get_world_size(group)
    out = [None] * R
    dist.all_gather_object(out, local, group=group)
    return out


def export_buffers(bufs: dict) -> dict:
    """name -> (IPC handle bytes, offset) of each CUDA tensor in bufs (None
    entries stay None)."""
    return {k: (ep.ipc_export(t) if t is not None else None) for k, t in bufs.items()}


def peer_table_from_handles(rank: int, own: dict, handles: list[dict], capacity_rows: int):
    """(ep_peer_table_t, mapping bases to release with ep.ipc_close): entry r
    of every array is rank r's buffer; this rank's own entries are its own
    tensors, the others are mapped from their IPC handles. Keys of `own`:
    recv_x, flags and optionally recv_scales, recv_w, recv_expert."""
    R = len(handles)
    bases = []
    cols = {k: [None] * R for k in ("recv_x", "recv_scales", "recv_w", "recv_expert", "flags")}
    for r in range(R):
        for k in cols:
            if own.get(k) is None:
                continue
            if r == rank:
                cols[k][r] = own[k]
            else:
                h, off = handles[r][k]
                p, base = ep.ipc_import(h, off)
                cols[k][r] = p
                bases.append(base)
    table = ep.peer_table(capacity_rows, cols["recv_x"], cols["flags"],
                          cols["recv_scales"] if own.get("recv_scales") is not None else None,
                          cols["recv_w"] if own.get("recv_w") is not None else None,
                          cols["recv_expert"] if own.get("recv_expert") is not None else None)
    return table, bases
