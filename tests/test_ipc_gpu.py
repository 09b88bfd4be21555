"""CUDA IPC helpers of the peer table (ep_ipc_export / ep_ipc_import /
ep_ipc_close), between two processes on one GPU: the owner exports a buffer
at an offset inside its allocation, the peer maps it, reads the owner's
pattern and writes its own, and the owner sees it. The processes order their
steps through host queues; no kernel waits on another process's work."""
import multiprocessing as mp

import pytest
import torch

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

N = 4096


def _owner(q_out, q_in, q_res):
    import torch

    from combine_ep_dispatch_03_b200 import ep

    torch.cuda.set_device(0)
    big = torch.zeros(3 * N, dtype=torch.int32, device="cuda")
    buf = big[N:2 * N]  # inside the allocation, not at its start
    buf.copy_(torch.arange(N, dtype=torch.int32, device="cuda") * 3 + 1)
    torch.cuda.synchronize()
    h, off = ep.ipc_export(buf)
    q_out.put((h, off))
    assert q_in.get(timeout=120) == "written"
    torch.cuda.synchronize()
    ok = bool(torch.equal(buf.cpu(), torch.arange(N, dtype=torch.int32) * 7 - 2))
    ok &= bool((big[:N] == 0).all().item() and (big[2 * N:] == 0).all().item())
    q_res.put(("owner", ok, off))


def _peer(q_in, q_out, q_res):
    import torch

    from combine_ep_dispatch_03_b200 import ep

    torch.cuda.set_device(0)
    h, off = q_in.get(timeout=120)
    ptr, base = ep.ipc_import(h, off)
    view = torch.as_tensor(ep._DeviceArray(ptr, N), device="cuda")
    ok = bool(torch.equal(view.cpu(), torch.arange(N, dtype=torch.int32) * 3 + 1))
    view.copy_(torch.arange(N, dtype=torch.int32, device="cuda") * 7 - 2)
    torch.cuda.synchronize()
    del view
    q_out.put("written")
    ep.ipc_close(base)
    q_res.put(("peer", ok, ptr - base))


def test_ipc_export_import_round_trip():
    from combine_ep_dispatch_03_b200 import build

    build.build()
    ctx = mp.get_context("spawn")
    a2b, b2a, res = ctx.Queue(), ctx.Queue(), ctx.Queue()
    pa = ctx.Process(target=_owner, args=(a2b, b2a, res))
    pb = ctx.Process(target=_peer, args=(a2b, b2a, res))
    pa.start()
    pb.start()
    got = {r[0]: r[1:] for r in (res.get(timeout=180), res.get(timeout=180))}
    pa.join(timeout=60)
    pb.join(timeout=60)
    assert pa.exitcode == 0 and pb.exitcode == 0
    assert got["peer"][0], "the peer did not read the owner's pattern"
    assert got["owner"][0], "the owner did not see the peer's pattern"
    # the buffer's offset inside its allocation (the caching allocator may place
    # the tensor anywhere in a larger block; the slice adds N elements)
    assert got["owner"][1] == got["peer"][1] and got["owner"][1] >= N * 4
