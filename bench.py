#!/usr/bin/env python3
"""Benchmark: MoE expert-parallel dispatch + combine on B200.

One step = one pass of the hot path over one batch: ep_plan (routing
histogram, scan, layout/plan, stable slots) + ep_dispatch + ep_combine.
Default workload: HT prefill (T=32768, H=7168, E=256, top-8, R=8 logical ranks,
FP8 e4m3 dispatch with per-128 scales, bf16 combine with fp32 accumulation),
seeded synthetic routing. Its step moves 6.6 GB, far more than L2 (126 MB), so
no L2 flush is needed between its steps; workloads whose step moves at most four
times the L2 (LL decode, tiny, router) are timed one step at a time, each after
a write of a buffer twice the L2's size.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

Prints ONE JSON line on rank 0. With N > 1 (torchrun), every rank runs its
own independent EP world (weak scaling, no data-path collective); the time is
the max over ranks of the device-timed region.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "dispatch+combine GB/s and tokens/s on 1 B200; % of HBM roofline vs skew"
FALLBACK_HBM_GBS = 6650.0
NVLINK_PEER_GBS = 770.0  # measured peer copy per direction per GPU on this B200 type (context only)


# ------------------------------------------------------------------ bytes

def algorithmic_bytes(T, H, K, rows_placed, fp8):
    """Minimum bytes each call must move (per step), by call."""
    L = T * K
    plan = 4 * L + 4 * L + 4 * rows_placed                  # topk_idx read; dest_row, src_row written
    payload = rows_placed * H * (1 if fp8 else 2)
    scales = rows_placed * (H // 128) * 4 if fp8 else 0
    dispatch = 2 * T * H + payload + scales + 12 * L + 8 * rows_placed  # x, rows, scales, idx+w+dest, recv_w+recv_expert
    combine = 2 * rows_placed * H + 2 * T * H + 8 * L       # expert rows, out, w + dest
    return {"plan": plan, "dispatch": dispatch, "combine": combine}


def compute_dtype(wl: dict) -> str:
    """What the path computes in: bf16 rows (e4m3 codes with fp32 scales when
    the dispatch casts), fp32 accumulation in combine and the backward."""
    return "bf16+e4m3 (fp32 accumulate)" if wl["fp8"] else "bf16 (fp32 accumulate)"


def workload_config(name: str, wl: dict, world: int, l2_note: str) -> dict:
    """The `config` object of the JSON line; both arms print the same one."""
    return {"workload": name, "T": wl["T"], "H": wl["H"], "E": wl["E"], "topk": wl["K"],
            "logical_ranks": wl["R"], "layout": wl["mode"], "ll_capacity": wl["cap"],
            "balanced_plan": wl["balanced"], "zipf_s": wl["s"], "backward": wl["backward"],
            "payload": ("bf16 x -> fp8 e4m3 dispatch (per-128 fp32 scales)" if wl["fp8"]
                        else "bf16 dispatch") + " -> bf16 combine (fp32 accumulation)",
            "l2": l2_note,
            "parallelism": f"{world} independent EP worlds (one per GPU), R logical ranks each"}


def l2_note_for(step_bytes: int, l2: int, flushed) -> str:
    if flushed == "clean":
        return (f"flushed, clean: before every timed step a {2 * l2 / 2**20:.0f} MiB buffer is written and then a "
                "second one read, so the step finds none of its data in L2 and no dirty lines of the flush to write "
                "back (the write alone leaves up to an L2 of them)")
    if flushed:
        return (f"flushed: each step moves {step_bytes / 1e6:.1f} MB, at most 4x L2 ({l2 / 2**20:.0f} MiB), so "
                f"a {2 * l2 / 2**20:.0f} MiB buffer is written before every timed step and the steps are "
                "timed one by one")
    if needs_l2_flush(step_bytes, l2):
        return "not flushed (--no-flush): the working set is partly L2-resident"
    return f"no flush: each step moves {step_bytes / 1e9:.2f} GB, more than 4x L2 ({l2 / 2**20:.0f} MiB)"


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def code_sha(paths) -> str:
    """sha256[:16] of the C/CUDA code in `paths` (repo-relative), with comments
    removed and whitespace collapsed: an edit to a comment keeps a committed
    counter record valid, while any change to the code voids it."""
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel)) as f:
            s = f.read()
        s = re.sub(r"/\*.*?\*/", " ", s, flags=re.S)
        s = re.sub(r"//[^\n]*", "", s)
        h.update((rel + "\0" + " ".join(s.split()) + "\0").encode())
    return h.hexdigest()[:16]


def committed_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary of this kernel on
    this workload ("kernel@workload"), if it was taken on the current code of
    the kernel's sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)[f"{kernel}@{workload}"]
        if code_sha(rec["sources"]) != rec["code_sha"] or rec["workload"] != workload:
            return None
        return int(rec["dram_bytes_per_launch"])
    except Exception:
        return None


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling SM clocks and throttle reasons every 20 ms, with a
    timestamp on each sample. stop() summarises every sample; window() those
    taken within a host-time interval (a timed region shorter than the sampling
    period is given the samples of the surrounding interval it names)."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.samples = []  # (host epoch seconds, sm MHz, max MHz, set of reasons)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "20",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def _parse(self, out: str):
        import datetime

        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                sm, smax = float(parts[2]), float(parts[3])
            except ValueError:
                continue
            reasons = {n for n, v in zip(self.REASONS, parts[6:10]) if v.lower() == "active"}
            self.samples.append((ts, sm, smax, reasons))

    @staticmethod
    def _summary(samples):
        if not samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = set().union(*(r for _, _, _, r in samples))
        return {"sm_mhz": statistics.median(s for _, s, _, _ in samples), "sm_max_mhz": samples[-1][2],
                "reasons": sorted(reasons), "samples": len(samples)}

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self._parse(out)
        self.proc = None
        return self._summary(self.samples)

    def window(self, t0: float, t1: float, margin: float = 0.1):
        """Samples taken from t0 - margin to t1 + margin (host epoch seconds),
        widened step by step to at least 5 samples where the region is short."""
        sel = []
        while margin <= 1.6:
            sel = [x for x in self.samples if t0 - margin <= x[0] <= t1 + margin]
            if len(sel) >= 5:
                break
            margin *= 2
        rec = self._summary(sel)
        rec["window_s"] = round(t1 - t0 + 2 * min(margin, 1.6), 3)
        return rec


def clocks_rejected(c: dict):
    """Why a timed region's clock record rejects its number, or None: a
    hardware or thermal slowdown seen, or a median SM clock well below the
    maximum with no reason given (a leftover clock lock). sw_power_cap alone
    is kept (and noted in the record)."""
    bad = [r for r in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown") if r in c.get("reasons", [])]
    if bad:
        return ",".join(bad)
    sm, smax = c.get("sm_mhz"), c.get("sm_max_mhz")
    if sm and smax and sm < 0.8 * smax and not c.get("reasons"):
        return f"sm clock {sm:.0f} of {smax:.0f} MHz with no reason"
    return None


# ------------------------------------------------------------------ distributed

def dist_setup(gpus: int):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """The largest value over all ranks (every rank must call it)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(step_bytes: float, ms_local: float, world: int):
    """Whole-job GB/s when every rank moves step_bytes per step: all ranks'
    bytes over the slowest rank's step time. Returns (GB/s, max ms)."""
    ms = max_over_ranks(ms_local, world)
    return world * step_bytes / (ms * 1e-3) / 1e9, ms


# ------------------------------------------------------------------ workloads

# The five workloads of the hot path (synthetic routing from combine_ep_dispatch_03_b200.synth).
WORKLOADS = {
    "ht_prefill": dict(T=32768, H=7168, E=256, K=8, R=8, mode="ht", cap=0, fp8=True, balanced=False, s=0.0,
                       backward=False, G=0),
    "ll_decode": dict(T=1024, H=7168, E=256, K=8, R=8, mode="ll", cap=1024, fp8=False, balanced=False, s=0.0,
                      backward=False, G=0),
    "imbalance": dict(T=32768, H=4096, E=128, K=8, R=8, mode="ht", cap=0, fp8=False, balanced=False, s=0.0,
                      backward=False, G=0),
    "large_train": dict(T=131072, H=7168, E=384, K=8, R=16, mode="ht", cap=0, fp8=False, balanced=True, s=1.0,
                        backward=True, G=7168 * 256),
    "tiny": dict(T=128, H=1024, E=16, K=2, R=4, mode="ht", cap=0, fp8=False, balanced=False, s=0.0,
                 backward=False, G=0),
    # the two steps around the path (next rows): router top-K on the HT
    # prefill logits, and replica weight prefetch under the large step's plan
    # (stand-in weights: one 7168 x 2048 bf16 projection per expert)
    "router": dict(T=32768, H=7168, E=256, K=8, R=8, mode="ht", cap=0, fp8=False, balanced=False, s=0.0,
                   backward=False, G=0, kind="router"),
    "prefetch": dict(T=131072, H=7168, E=384, K=8, R=16, mode="ht", cap=0, fp8=False, balanced=True, s=1.0,
                     backward=False, G=0, kind="prefetch", wbytes=7168 * 2048 * 2),
    # the inference plan at decode size (a few prefetch slots, overflow rows
    # read the owner's weights in place) on skewed routing, and the same batch
    # without a plan
    "inference_decode": dict(T=1024, H=7168, E=256, K=8, R=8, mode="ht", cap=0, fp8=False, balanced=True, s=1.0,
                             backward=False, G=0, slots=2, direct=True),
    "ht_decode": dict(T=1024, H=7168, E=256, K=8, R=8, mode="ht", cap=0, fp8=False, balanced=False, s=1.0,
                      backward=False, G=0),
}
# the workloads timed beside the headline in the default run (sub-records)
SIDE_WORKLOADS = ("ll_decode", "large_train", "tiny", "router", "prefetch", "inference_decode", "ht_decode")
HT = WORKLOADS["ht_prefill"]
SWEEP = WORKLOADS["imbalance"]

KERNEL_OF = {"plan": "k_route_*", "combine": "k_combine", "combine_backward": "k_combine_bwd",
             "dispatch_backward": "k_combine", "replica_reduce": "k_replica_reduce", "router": "k_router_topk",
             "prefetch": "k_prefetch"}


class Step:
    """One pass of the hot path for a workload: buffers, the calls in order,
    and the algorithmic bytes of each call."""

    def __init__(self, wl: dict, dev, seed: int, host_inputs: bool = True):
        import torch

        from combine_ep_dispatch_03_b200 import ep, synth

        self.wl = wl
        T, H, E, K, R = wl["T"], wl["H"], wl["E"], wl["K"], wl["R"]
        self.T, self.H, self.E, self.K, self.R = T, H, E, K, R
        self.kind = wl.get("kind", "path")
        if self.kind == "router":
            self._init_router(wl, dev, seed, host_inputs)
            return
        if self.kind == "prefetch":
            self._init_prefetch(wl, dev, seed)
            return
        x = synth.tokens_bf16(T, H, seed=seed)
        idx, w = synth.routing(T, E, K, zipf_s=wl["s"], seed=seed)
        self.x_host = x.pin_memory() if host_inputs else x
        self.idx_host = idx.pin_memory() if host_inputs else idx
        self.w_host = w.pin_memory() if host_inputs else w
        self.xd, self.idxd, self.wd = self.x_host.to(dev), self.idx_host.to(dev), self.w_host.to(dev)
        h = ep.Ep(T, H, E, K, R, mode=wl["mode"], ll_capacity=wl["cap"], fp8=wl["fp8"], balanced=wl["balanced"],
                  replica_slots=wl.get("slots", 0), grad_elems_per_expert=wl["G"],
                  direct_overflow=wl.get("direct", False))
        self.h = h
        self.bufs = h.empty_recv(dev)
        g = torch.Generator(device=dev).manual_seed(1000 + seed)
        if wl["backward"]:
            # identity expert: combine reads the dispatched rows (no second row buffer)
            self.y = self.bufs["recv_x"]
        else:
            # the expert-FFN output stand-in, resident on the device (not timed)
            self.y = torch.randn((h.recv_rows, H), generator=g, device=dev).to(torch.bfloat16)
        self.out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        self.calls = [("plan", lambda st: h.plan(self.idxd, st)),
                      ("dispatch", lambda st: h.dispatch(self.xd, self.idxd, self.wd, stream=st, **self.bufs)),
                      ("combine", lambda st: h.combine(self.y, self.wd, self.out, st))]
        self.outputs = [self.out]
        if wl["backward"]:
            self.gout_host = synth.tokens_bf16(T, H, seed=seed + 5)
            if host_inputs:
                self.gout_host = self.gout_host.pin_memory()
            self.gout = self.gout_host.to(dev)
            self.gy = torch.empty((h.recv_rows, H), dtype=torch.bfloat16, device=dev)
            self.gx = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
            self.rep = torch.randn((R, h.S, wl["G"]), generator=g, device=dev)
            self.owner = torch.randn((E, wl["G"]), generator=g, device=dev)
            self.calls += [
                ("combine_backward", lambda st: h.combine_backward(self.gout, self.wd, self.gy, st)),
                ("dispatch_backward", lambda st: h.dispatch_backward(self.gy, self.gx, st)),
                ("replica_reduce", lambda st: h.reduce_replica_grads(self.rep, self.owner, st)),
            ]
            self.outputs.append(self.gx)
        self.bytes = None

    def _init_router(self, wl, dev, seed, host_inputs):
        import torch

        from combine_ep_dispatch_03_b200 import ep, synth

        T, E, K = self.T, self.E, self.K
        lg = synth.router_logits(T, E, zipf_s=wl["s"], seed=seed)
        self.logits_host = lg.pin_memory() if host_inputs else lg
        self.logits = self.logits_host.to(dev)
        self.idx = torch.empty((T, K), dtype=torch.int32, device=dev)
        self.w = torch.empty((T, K), dtype=torch.float32, device=dev)
        self.h = None
        self.calls = [("router", lambda st: ep.router_topk(self.logits, K, self.idx, self.w, st))]
        self.ins = [(self.logits_host, self.logits)]
        self.outputs = [self.idx, self.w]

    def _init_prefetch(self, wl, dev, seed):
        import torch

        from combine_ep_dispatch_03_b200 import ep, synth

        T, E, K, R = self.T, self.E, self.K, self.R
        idx, _ = synth.routing(T, E, K, zipf_s=wl["s"], seed=seed)
        self.h = ep.Ep(T, 128, E, K, R, balanced=True)
        self.h.plan(idx.to(dev))
        nb = wl["wbytes"]
        g = torch.Generator(device=dev).manual_seed(3000 + seed)
        self.weights = torch.randint(0, 256, (E, nb), dtype=torch.uint8, device=dev, generator=g)
        self.slots = torch.empty((R, self.h.S, nb), dtype=torch.uint8, device=dev)
        self.calls = [("prefetch", lambda st: self.h.prefetch_replica_weights(self.weights, self.slots, st))]
        self.ins, self.outputs = [], []

    def run(self, st):
        for _, f in self.calls:
            f(st)

    def e2e_sets(self):
        """Two sets of device inputs and outputs for the end-to-end leg, each
        with the step's calls bound to it: (host->device copies, device
        outputs, run(stream)). Set 0 is the step's own buffers; set 1 twins
        them, so that one set's copies can run while the other's kernels do.
        The handle, the receive buffers and the resident stand-ins are shared
        (the kernels of consecutive steps run in order on one stream)."""
        import torch

        from combine_ep_dispatch_03_b200 import ep

        def twin(t, b):
            return t if b == 0 else torch.empty_like(t)

        sets = []
        for b in range(2):
            if self.kind == "router":
                lg, idx, w = twin(self.logits, b), twin(self.idx, b), twin(self.w, b)
                K = self.K

                def run(st, lg=lg, idx=idx, w=w):
                    ep.router_topk(lg, K, idx, w, st)

                sets.append(([(self.logits_host, lg)], [idx, w], run))
                continue
            h, bufs, back = self.h, self.bufs, self.wl["backward"]
            xd, idxd, wd, out = twin(self.xd, b), twin(self.idxd, b), twin(self.wd, b), twin(self.out, b)
            ins = [(self.x_host, xd), (self.idx_host, idxd), (self.w_host, wd)]
            outs = [out]
            gout = gx = None
            if back:
                gout, gx = twin(self.gout, b), twin(self.gx, b)
                ins.append((self.gout_host, gout))
                outs.append(gx)

            def run(st, xd=xd, idxd=idxd, wd=wd, out=out, gout=gout, gx=gx):
                h.plan(idxd, st)
                h.dispatch(xd, idxd, wd, stream=st, **bufs)
                h.combine(self.y, wd, out, st)
                if back:
                    h.combine_backward(gout, wd, self.gy, st)
                    h.dispatch_backward(self.gy, gx, st)
                    h.reduce_replica_grads(self.rep, self.owner, st)

            sets.append((ins, outs, run))
        return sets

    def measure_bytes(self, st):
        """Algorithmic bytes per call, from the routing of one untimed step."""
        self.run(st)
        st.synchronize()  # recv_counts is written on `st`
        T, H, K, wl = self.T, self.H, self.K, self.wl
        if self.kind == "router":
            self.placed = T * K
            self.bytes = {"router": 4 * T * self.E + 8 * T * K}
            return self.bytes
        if self.kind == "prefetch":
            rep, _ = self.h.get_plan(st)
            used = sum(1 for e in rep if e >= 0)
            self.placed = used
            self.bytes = {"prefetch": 2 * wl["wbytes"] * used}
            return self.bytes
        L = T * K
        placed = int(self.bufs["recv_counts"].sum().item())
        b = algorithmic_bytes(T, H, K, placed, wl["fp8"])
        if wl["backward"]:
            b["combine_backward"] = 2 * T * H + 2 * placed * H + 8 * L
            b["dispatch_backward"] = 2 * placed * H + 2 * T * H + 4 * L
            rep, _ = self.h.get_plan(st)
            used = [e for e in rep if e >= 0]
            b["replica_reduce"] = 4 * wl["G"] * (len(used) + 2 * len(set(used)))
        self.bytes = b
        self.placed = placed
        return b

    def launches(self):
        from combine_ep_dispatch_03_b200.ep import plan_launches

        if self.kind != "path":
            return len(self.calls)
        return plan_launches(self.h) + len(self.calls) - 1


class WorldStep:
    """One pass of the path across ranks through the peer table (ep_plan_local_counts,
    the gathered counts, ep_plan_world, ep_dispatch_peers, signal and wait,
    ep_combine_peers). With one process the workload's R ranks are R handles
    with R separate buffers on this GPU, run in stream order (every wait finds
    flags that earlier kernels set); with N processes (N = R GPUs) each process
    is one rank, the counts are all-gathered with NCCL and the peers' buffers
    are mapped through CUDA IPC."""

    def __init__(self, wl: dict, dev, seed: int, world: int, rank: int):
        import torch

        from combine_ep_dispatch_03_b200 import ep, synth
        from combine_ep_dispatch_03_b200 import world as wmod

        self.wl, self.kind, self.h = wl, "world", None
        T, H, E, K, R = wl["T"], wl["H"], wl["E"], wl["K"], wl["R"]
        self.T, self.H, self.E, self.K, self.R = T, H, E, K, R
        self.multi = world > 1
        if self.multi and world != R:
            raise ValueError(f"--exchange across GPUs needs --gpus equal to the workload's R ({R})")
        Tl = T // R
        x = synth.tokens_bf16(T, H, seed=seed)
        idx, w = synth.routing(T, E, K, zipf_s=wl["s"], seed=seed)
        mine = [rank] if self.multi else list(range(R))
        self.hs = {q: ep.Ep(Tl, H, E, K, R, mode=wl["mode"], ll_capacity=wl["cap"], fp8=wl["fp8"],
                            balanced=wl["balanced"], replica_slots=wl.get("slots", 0),
                            direct_overflow=wl.get("direct", False)) for q in mine}
        cap = ep.world_recv_rows(next(iter(self.hs.values())).cfg)
        self.cap = cap
        self.xs = {q: x[q * Tl:(q + 1) * Tl].to(dev) for q in mine}
        self.ids = {q: idx[q * Tl:(q + 1) * Tl].contiguous().to(dev) for q in mine}
        self.ws = {q: w[q * Tl:(q + 1) * Tl].contiguous().to(dev) for q in mine}
        dt = torch.float8_e4m3fn if wl["fp8"] else torch.bfloat16
        g = torch.Generator(device=dev).manual_seed(2000 + seed)
        own = {}
        for q in mine:
            own[q] = {"recv_x": torch.empty((cap, H), dtype=dt, device=dev),
                      "recv_scales": torch.empty((cap, H // 128), dtype=torch.float32, device=dev) if wl["fp8"] else None,
                      "recv_w": torch.empty(cap, dtype=torch.float32, device=dev),
                      "recv_expert": torch.empty(cap, dtype=torch.int32, device=dev),
                      "flags": torch.zeros(R, dtype=torch.int32, device=dev)}
            # the expert-FFN output stand-in of rank q, resident (not timed)
            own[q]["y"] = torch.randn((cap, H), generator=g, device=dev).to(torch.bfloat16)
        self.own = own
        self.bases = []
        if self.multi:
            handles = wmod.exchange_handles(wmod.export_buffers({k: v for k, v in own[rank].items()}))
            self.table, b1 = wmod.peer_table_from_handles(rank, own[rank], handles, cap)
            ytab_own = {"recv_x": own[rank]["y"], "flags": own[rank]["flags"]}
            yh = [{"recv_x": h["y"], "flags": h["flags"]} for h in handles]
            self.ytable, b2 = wmod.peer_table_from_handles(rank, ytab_own, yh, cap)
            self.bases = b1 + b2
        else:
            col = lambda k: [own[q][k] for q in range(R)]
            self.table = ep.peer_table(cap, col("recv_x"), col("flags"), col("recv_scales") if wl["fp8"] else None,
                                       col("recv_w"), col("recv_expert"))
            self.ytable = ep.peer_table(cap, col("y"), col("flags"))
        self.counts = torch.zeros((R, E), dtype=torch.int32, device=dev)
        self.local = torch.zeros(E, dtype=torch.int32, device=dev)
        self.outs = {q: torch.empty((Tl, H), dtype=torch.bfloat16, device=dev) for q in mine}
        self.epoch = 0
        self.mine = mine
        self.rank = rank
        self.calls = [("plan", self._plan), ("dispatch", self._dispatch), ("combine", self._combine)]
        self.outputs = list(self.outs.values())

    def _plan(self, st):
        from combine_ep_dispatch_03_b200 import world as wmod

        if self.multi:
            h = self.hs[self.rank]
            h.plan_local_counts(self.ids[self.rank], self.local, st)
            import torch

            with torch.cuda.stream(st):
                self.counts.copy_(wmod.gather_counts(self.local))
            h.plan_world(self.counts, self.rank, st)
        else:
            for q in self.mine:
                self.hs[q].plan_local_counts(self.ids[q], self.counts[q], st)
            for q in self.mine:
                self.hs[q].plan_world(self.counts, q, st)

    def _exchange(self, table, st):
        self.epoch += 1
        for q in self.mine:
            self.hs[q].signal_peers(table, self.epoch, st)
        for q in self.mine:
            self.hs[q].wait_peers(self.own[q]["flags"], self.epoch, 0, st)

    def _dispatch(self, st):
        for q in self.mine:
            self.hs[q].dispatch_peers(self.xs[q], self.ids[q], self.ws[q], self.table, st)
        self._exchange(self.table, st)

    def _combine(self, st):
        self._exchange(self.table, st)  # every rank's expert outputs are ready
        for q in self.mine:
            self.hs[q].combine_peers(self.ytable, self.ws[q], self.outs[q], st)

    def run(self, st):
        for _, f in self.calls:
            f(st)

    def measure_bytes(self, st):
        """The same algorithmic bytes as the single-GPU step of this workload
        (this process's share with one rank per GPU)."""
        self.run(st)
        st.synchronize()
        from combine_ep_dispatch_03_b200 import ep

        T, H, K = self.T, self.H, self.K
        placed = 0
        for q in self.mine:
            dest = self.hs[q].tensor(ep.T_DEST_ROW)
            placed += int((dest >= 0).sum().item())
        share = len(self.mine) / self.R
        b = algorithmic_bytes(int(T * share), H, K, placed, self.wl["fp8"])
        self.bytes, self.placed = b, placed
        return b

    def launches(self):
        per_rank = 2 + 2 + 1 + 2 + 2 + 1  # counts (2), world plan (2), dispatch, signal+wait, signal+wait, combine
        return per_rank * len(self.mine)

    def status(self, st):
        f = 0
        for h in self.hs.values():
            f |= h.status(st)
        return f

    def close(self):
        from combine_ep_dispatch_03_b200 import ep

        for b in self.bases:
            ep.ipc_close(b)
        for h in self.hs.values():
            h.close()


L2_FALLBACK_BYTES = 126 * 2**20


def l2_bytes(dev) -> int:
    import torch

    return int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 0) or L2_FALLBACK_BYTES)


def needs_l2_flush(step_bytes: int, l2: int) -> bool:
    """A step that moves less than four times the L2 could find a good part of
    its inputs still in L2 from the step before, so such steps are timed one by
    one, each after a write of a buffer twice the L2's size."""
    return step_bytes <= 4 * l2


def timed(step: Step, steps, warmup, stream, breakdown_steps=None, graph=True, flush=None):
    """Warm-up, then `steps` steps back to back between two CUDA events on the
    launching stream (the step time), then `breakdown_steps` more with an
    event between every two calls (the per-call split; events between calls
    stop consecutive kernels from overlapping their launches, so this loop
    runs slightly slower). Returns (total_ms, {call: [ms per step]}).

    With `graph`, the timed steps are replays of CUDA graphs captured from the
    same calls (a graph of up to 10 steps, and one of a single step for the
    remainder): the same kernels with the same programmatic launch edges,
    without the host's per-launch cost, which otherwise bounds steps of a few
    microseconds.

    With a `flush` buffer (larger than L2), every timed step, and every step
    of the per-call loop, follows a write of that buffer outside its events:
    the step is timed alone (a replay of a one-step graph, with `graph`), on
    cold L2, and the step time is the sum of the steps' own times. A pair of
    buffers (written, then read) leaves L2 cold and clean."""
    import torch

    if flush is not None:
        return _timed_flushed(step, steps, warmup, stream, breakdown_steps, graph, flush)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step.run(stream)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if graph:
        chunk = min(steps, 10)
        graphs = {}
        for n in sorted({chunk, steps % chunk} - {0}):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for _ in range(n):
                    step.run(stream)
            graphs[n] = g
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            for _ in range(max(1, warmup // chunk)):
                graphs[chunk].replay()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(steps // chunk):
                graphs[chunk].replay()
            if steps % chunk:
                graphs[steps % chunk].replay()
            end.record(stream)
        torch.cuda.synchronize()
        del graphs
    else:
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(steps):
                step.run(stream)
            end.record(stream)
        torch.cuda.synchronize()
    total = start.elapsed_time(end)
    nb = steps if breakdown_steps is None else breakdown_steps
    n = len(step.calls)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(nb)]
    with torch.cuda.stream(stream):
        for s in range(nb):
            ev[s][0].record(stream)
            for i, (_, f) in enumerate(step.calls):
                f(stream)
                ev[s][i + 1].record(stream)
    torch.cuda.synchronize()
    per = {name: [e[i].elapsed_time(e[i + 1]) for e in ev] for i, (name, _) in enumerate(step.calls)}
    return total, per


def _flush_l2(flush, i):
    """Write the flush buffer (and read the second one of a pair)."""
    if isinstance(flush, tuple):
        flush[0].fill_(i & 0x7F)
        flush[1].sum()
    else:
        flush.fill_(i & 0x7F)


def _timed_flushed(step: Step, steps, warmup, stream, breakdown_steps, graph, flush):
    import torch

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step.run(stream)
    torch.cuda.synchronize()
    g = None
    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step.run(stream)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            g.replay()  # untimed: a graph's first replay may carry one-time set-up
        torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    with torch.cuda.stream(stream):
        for i in range(steps):
            _flush_l2(flush, i)
            ev[i][0].record(stream)
            if g is not None:
                g.replay()
            else:
                step.run(stream)
            ev[i][1].record(stream)
    torch.cuda.synchronize()
    total = sum(a.elapsed_time(b) for a, b in ev)
    del g
    nb = steps if breakdown_steps is None else breakdown_steps
    n = len(step.calls)
    pev = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(nb)]
    with torch.cuda.stream(stream):
        for s in range(nb):
            _flush_l2(flush, s)
            pev[s][0].record(stream)
            for i, (_, f) in enumerate(step.calls):
                f(stream)
                pev[s][i + 1].record(stream)
    torch.cuda.synchronize()
    per = {name: [e[i].elapsed_time(e[i + 1]) for e in pev] for i, (name, _) in enumerate(step.calls)}
    return total, per


def run_native(args):
    import torch

    from combine_ep_dispatch_03_b200 import build, ep

    rank, world, local = dist_setup(args.gpus)
    if rank == 0 or local == 0:
        build.build()
    barrier(world)
    ep.lib()
    dev = torch.device("cuda", local if world > 1 else 0)
    stream = torch.cuda.Stream(device=dev)
    wl = dict(WORKLOADS[args.workload])
    if args.tokens:
        wl["T"] = args.tokens
    if args.hidden:
        wl["H"] = args.hidden
    if args.zipf is not None:
        wl["s"] = args.zipf
    if args.balanced is not None:
        wl["balanced"] = bool(args.balanced)
    if args.capacity:
        wl["cap"] = args.capacity
    if args.grad_elems:
        wl["G"] = args.grad_elems
    if args.weight_bytes:
        wl["wbytes"] = args.weight_bytes
    name = args.workload if wl == WORKLOADS[args.workload] else args.workload + "_custom"
    if args.exchange:
        return run_exchange(args, wl, name, rank, world, dev, stream)
    seed = rank  # each rank: its own EP world (weak scaling)
    step = Step(wl, dev, seed)
    nbytes = step.measure_bytes(stream)
    step_bytes = sum(nbytes.values())
    torch.cuda.synchronize()

    l2 = l2_bytes(dev)
    flush = None
    if not args.no_flush and needs_l2_flush(step_bytes, l2):
        flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
    remeasured = None
    for attempt in range(2):  # a run whose clocks reject it is timed once more
        sampler = ClockSampler(torch.cuda.current_device() if world == 1 else local)
        sampler.start()
        time.sleep(0.3)  # nvidia-smi's first samples arrive after its start-up
        barrier(world)
        torch.cuda.synchronize()
        t0 = time.time()
        total_ms, per = timed(step, args.steps, args.warmup, stream, min(args.steps, 50), graph=not args.no_graph,
                              flush=flush)
        t1 = time.time()
        sampler.stop()
        clocks = sampler.window(t0, t1)
        barrier(world)
        why = clocks_rejected(clocks)
        if attempt == 1 or max_over_ranks(1.0 if why else 0.0, world) == 0.0:
            break
        remeasured = {"first_clocks": clocks, "why": why or "another rank's clocks"}
    value, ms_step = weak_scaling_value(step_bytes, total_ms / args.steps, world)
    flags = step.h.status(stream) if step.h is not None else 0

    avg = {k: sum(v) / len(v) for k, v in per.items()}
    peak, peak_kind = hbm_peak()
    dom = max((k for k in avg if k != "plan" or len(avg) == 1), key=lambda k: avg[k])
    kname = KERNEL_OF.get(dom) or ("k_dispatch_fp8" if wl["fp8"] else "k_dispatch_bulk")
    achieved = nbytes[dom] / (avg[dom] * 1e-3) / 1e9
    roofline = {"bound": "hbm", "call": dom, "kernel": kname, "achieved": round(achieved, 1), "peak": peak,
                "unit": "GB/s", "frac": round(achieved / peak, 4), "peak_source": f"{peak_kind} hbm_gbs (copy)",
                "traffic": committed_traffic(kname, name), "algorithmic_bytes_per_launch": nbytes[dom]}

    e2e = None if (args.no_e2e or step.kind == "prefetch") else run_e2e(step, dev, stream, max(3, min(args.steps, 20)),
                                                                        world, step_bytes)
    l2_note = l2_note_for(step_bytes, l2, flush is not None)
    del flush
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": compute_dtype(wl),
        "data": "synthetic",
        "config": workload_config(name, wl, world, l2_note),
        "launch": ("stream" if args.no_graph else "CUDA graph replay of the captured step calls")
                  + (", one step per timed interval" if l2_note.startswith("flushed") else ""),
        "tokens_per_s": round(world * wl["T"] / (ms_step * 1e-3), 1),
        "rows_per_s": round(world * step.placed / (ms_step * 1e-3), 1),
        "frac_of_hbm": round(step_bytes / (ms_step * 1e-3) / 1e9 / peak, 4),
        "frac_of_8tbs_nominal": round(step_bytes / (ms_step * 1e-3) / 1e9 / 8000.0, 4),
        "per_call_us": {k: round(v * 1e3, 2) for k, v in avg.items()},
        "per_call_note": "separate loop with an event between calls (blocks launch overlap)",
        "per_call_gbs": {k: round(nbytes[k] / (avg[k] * 1e-3) / 1e9, 1) for k in avg},
        "bytes_per_step": step_bytes,
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": step.launches() * args.steps,
        "clocks": clocks,
        "device_flags": flags,
    }
    if remeasured is not None:
        result["remeasured"] = remeasured
    if step.kind == "path" and (wl["balanced"] or wl["mode"] == "ht"):
        load = step.h.tensor(ep.T_RANK_LOAD).cpu().tolist()
        result["rank_load_max_over_mean"] = round(max(load) / (sum(load) / len(load)), 4) if sum(load) else None
    if step.h is not None:
        step.h.close()
    del step
    torch.cuda.empty_cache()
    if not args.no_sweep and args.workload == "ht_prefill":
        result["skew_sweep"] = run_sweep(dev, stream, seed, peak)
    if not args.no_side and args.workload == "ht_prefill" and name == "ht_prefill":
        result["workloads"] = run_side_workloads(dev, stream, seed, peak, world, args.no_graph)
    if world == 1 and rank == 0 and not args.no_cpu_baseline and args.workload == "ht_prefill":
        result["cpu_baseline"] = cpu_baseline(args.cpu_sample_tokens)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def run_exchange(args, wl, name, rank, world, dev, stream):
    """--exchange: the path across ranks through the peer table (WorldStep).
    Stream launches (the flags' epochs change every step), no L2 flush (the
    workloads it serves move far more than L2). With N GPUs the whole job is
    one EP world of N ranks, so the total work is fixed ("strong")."""
    import torch

    step = WorldStep(wl, dev, 0, world, rank)
    nbytes = step.measure_bytes(stream)
    step_bytes = sum(nbytes.values())
    torch.cuda.synchronize()
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    sampler.start()
    time.sleep(0.3)
    barrier(world)
    t0 = time.time()
    total_ms, per = timed(step, args.steps, args.warmup, stream, min(args.steps, 20), graph=False)
    t1 = time.time()
    sampler.stop()
    barrier(world)
    ms_local = total_ms / args.steps
    ms = max_over_ranks(ms_local, world)
    total_bytes = step_bytes * (world if step.multi else 1)
    value = total_bytes / (ms * 1e-3) / 1e9
    peak, _ = hbm_peak()
    avg = {k: sum(v) / len(v) for k, v in per.items()}
    flags = step.status(stream)
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "strong" if step.multi else "weak", "vs_baseline": None, "dtype": compute_dtype(wl),
        "data": "synthetic", "impl": "native-exchange",
        "config": dict(workload_config(name, wl, world, l2_note_for(step_bytes, l2_bytes(dev), False)),
                       parallelism=(f"one EP world of {world} GPUs (one rank each), peer stores and loads"
                                    if step.multi else
                                    f"{wl['R']} ranks as separate buffers on one GPU, peer-table path")),
        "launch": "stream",
        "tokens_per_s": round(wl["T"] / (ms * 1e-3), 1),
        "frac_of_hbm": round(value / max(world, 1) / peak, 4),
        "per_call_us": {k: round(v * 1e3, 2) for k, v in avg.items()},
        "per_call_note": "per call over all of this process's ranks, including the signal and wait kernels",
        "bytes_per_step": total_bytes, "capacity_rows_per_rank": step.cap,
        "gpu_launches": step.launches() * args.steps, "clocks": sampler.window(t0, t1), "device_flags": flags,
    }
    step.close()
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def run_e2e(step: Step, dev, stream, steps, world, step_bytes):
    """The same step through the public API, its inputs copied from pinned
    host memory and its results (combined tokens, and the input gradient with
    a backward pass) read back to pinned host memory, inside the timed region.

    Steps are pipelined over three streams (uploads, kernels, read-backs) and
    two sets of device inputs and outputs, used by alternate steps: step
    i+1's inputs go up while step i's kernels run and step i-1's results come
    down, so both directions of the link stay busy. Events order each step: a
    set's inputs are overwritten only after the kernels of the step that last
    used them have finished, and its outputs only after that step's results
    have been read back."""
    import torch

    sets = step.e2e_sets()
    host_outs = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in sets[0][1]]
    h2d_st, d2h_st = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    computed, drained = [None, None], [None, None]
    counter = [0]

    def one():
        b = counter[0] % 2
        counter[0] += 1
        ins, outs, run = sets[b]
        if computed[b] is not None:  # the kernels that last read this set's inputs
            h2d_st.wait_event(computed[b])
        with torch.cuda.stream(h2d_st):
            for src, dst in ins:
                dst.copy_(src, non_blocking=True)
        loaded = torch.cuda.Event()
        loaded.record(h2d_st)
        stream.wait_event(loaded)
        if drained[b] is not None:  # the read-back of this set's last outputs
            stream.wait_event(drained[b])
        run(stream)
        computed[b] = torch.cuda.Event()
        computed[b].record(stream)
        d2h_st.wait_event(computed[b])
        with torch.cuda.stream(d2h_st):
            for src, dst in zip(outs, host_outs):
                dst.copy_(src, non_blocking=True)
        drained[b] = torch.cuda.Event()
        drained[b].record(d2h_st)

    for _ in range(2):
        one()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    h2d_st.wait_event(s)
    d2h_st.wait_event(s)
    for _ in range(steps):
        one()
    stream.wait_event(drained[0])
    stream.wait_event(drained[1])
    e.record(stream)
    torch.cuda.synchronize()
    value, ms = weak_scaling_value(step_bytes, s.elapsed_time(e) / steps, world)
    h2d = sum(src.numel() * src.element_size() for src, _ in sets[0][0])
    d2h = sum(o.numel() * o.element_size() for o in sets[0][1])
    del sets
    return {"value": round(value, 2), "unit": "GB/s", "pipelined": True, "device_buffer_sets": 2,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 3), "steps": steps}


def modelled_exchange_ms(rank_loads, row_bytes: int, link_gbs: float = NVLINK_PEER_GBS) -> float:
    """What the skew would cost on R real GPUs: the busiest rank receives
    max(load) rows in dispatch and sends as many back in combine, each over a
    peer link of `link_gbs` per direction, one phase after the other."""
    return 2 * max(rank_loads) * row_bytes / link_gbs / 1e6


def run_sweep(dev, stream, seed, peak, steps=10, warmup=3):
    """Imbalance sweep: T=32768, H=4096, E=128, top-8, R=8, Zipf s, plan off/on."""
    import torch

    from combine_ep_dispatch_03_b200 import ep

    rows = []
    for balanced in (False, True):
        for s in (0.0, 0.5, 1.0, 1.5):
            wl = dict(SWEEP, s=s, balanced=balanced)
            step = Step(wl, dev, seed + 11, host_inputs=False)
            nb = step.measure_bytes(stream)
            total, per = timed(step, steps, warmup, stream)
            ms = total / steps
            load = step.h.tensor(ep.T_RANK_LOAD).cpu().tolist()
            mean = sum(load) / len(load)
            gbs = sum(nb.values()) / (ms * 1e-3) / 1e9
            modelled_ms = modelled_exchange_ms(load, wl["H"] * (1 if wl["fp8"] else 2))
            rows.append({"zipf_s": s, "balanced": balanced, "ms": round(ms, 4), "gbs": round(gbs, 1),
                         "frac": round(gbs / peak, 4), "load_max_over_mean": round(max(load) / mean, 4),
                         "modelled_ep_exchange_ms": round(modelled_ms, 3),
                         "plan_us": round(1e3 * sum(per["plan"]) / steps, 2), "flags": step.h.status(stream)})
            step.h.close()
            del step
            torch.cuda.empty_cache()
    return rows


def side_record(name: str, dev, stream, seed, peak, world, no_graph, steps, warmup, flushed):
    """One workload timed as the headline is (CUDA-graph replays, CUDA events
    on the launching stream, max over ranks), with or without an L2 flush
    before every step (flushed: True, False or "clean"): step time, GB/s of
    algorithmic bytes, fraction of the measured copy bandwidth, per-call split
    and the clocks seen."""
    import torch

    from combine_ep_dispatch_03_b200 import ep

    wl = WORKLOADS[name]
    step = Step(wl, dev, seed, host_inputs=False)
    nb = step.measure_bytes(stream)
    step_bytes = sum(nb.values())
    l2 = l2_bytes(dev)
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev) if flushed else None
    if flushed == "clean":
        flush = (flush, torch.zeros(2 * l2, dtype=torch.uint8, device=dev))
    torch.cuda.synchronize()
    t0 = time.time()
    total, per = timed(step, steps, warmup, stream, min(steps, 20), graph=not no_graph, flush=flush)
    t1 = time.time()
    gbs, ms = weak_scaling_value(step_bytes, total / steps, world)
    avg = {k: sum(v) / len(v) for k, v in per.items()}
    rec = {"ms": round(ms, 4), "gbs": round(gbs, 1), "frac": round(gbs / world / peak, 4),
           "frac_of_8tbs_nominal": round(gbs / world / 8000.0, 4), "bytes_per_step": step_bytes,
           "l2": l2_note_for(step_bytes, l2, flushed), "steps": steps,
           "per_call_us": {k: round(v * 1e3, 2) for k, v in avg.items()},
           "per_call_gbs": {k: round(nb[k] / (avg[k] * 1e-3) / 1e9, 1) for k in avg},
           "per_call_frac": {k: round(nb[k] / (avg[k] * 1e-3) / 1e9 / peak, 4) for k in avg},
           "timed_host_interval": (t0, t1)}  # replaced by the clocks seen in it
    if step.kind == "path":
        rec["tokens_per_s"] = round(world * wl["T"] / (ms * 1e-3), 1)
        rec["flags"] = step.h.status(stream)
        load = step.h.tensor(ep.T_RANK_LOAD).cpu().tolist()
        if sum(load):
            rec["load_max_over_mean"] = round(max(load) / (sum(load) / len(load)), 4)
    if step.h is not None:
        step.h.close()
    del step, flush
    torch.cuda.empty_cache()
    return rec


def run_side_workloads(dev, stream, seed, peak, world, no_graph):
    """The other workloads of the path, each its own sub-record of the line.
    Workloads whose step moves at most 4x L2 are timed after an L2 flush
    before every step (and, for LL decode and the two decode-size plan cases,
    also back to back without one)."""
    out = {}
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    sampler.start()
    for name in SIDE_WORKLOADS:
        big = name in ("large_train", "prefetch")
        steps, warmup = (10, 3) if big else (50, 5)
        small = name in ("ll_decode", "tiny", "router", "inference_decode", "ht_decode")
        cfg = WORKLOADS[name]
        rec = {"config": {k: v for k, v in cfg.items() if k not in ("kind",)}}
        if small:
            rec["flushed"] = side_record(name, dev, stream, seed, peak, world, no_graph, steps, warmup, True)
            if name in ("ll_decode", "inference_decode", "ht_decode"):
                rec["flushed_clean"] = side_record(name, dev, stream, seed, peak, world, no_graph, steps, warmup,
                                                   "clean")
                rec["back_to_back"] = side_record(name, dev, stream, seed, peak, world, no_graph, steps, warmup,
                                                  False)
        else:
            rec["back_to_back"] = side_record(name, dev, stream, seed, peak, world, no_graph, steps, warmup, False)
        out[name] = rec
    out["clocks"] = sampler.stop()  # every sample of the side workloads together
    for rec in out.values():
        for mode in ("flushed", "flushed_clean", "back_to_back"):
            if isinstance(rec, dict) and mode in rec:
                rec[mode]["clocks"] = sampler.window(*rec[mode].pop("timed_host_interval"))
    if "inference_decode" in out and "ht_decode" in out:
        a, b = out["inference_decode"]["flushed"]["ms"], out["ht_decode"]["flushed"]["ms"]
        out["inference_decode"]["over_unplanned_flushed"] = round(a / b, 4)
    return out


def cpu_baseline(sample_tokens: int):
    """The oracle as it stands, single-threaded on a host core, on a bounded
    sample of the HT prefill workload: full routing of all 32768 tokens, then
    FP8 dispatch and combine of `sample_tokens` tokens in chunks of 2048. The
    default is the whole step once: about 10 s on one core of a B200 server."""
    import numpy as np

    import oracle
    from combine_ep_dispatch_03_b200 import synth

    oracle.build()
    T, H, E, K, R = HT["T"], HT["H"], HT["E"], HT["K"], HT["R"]
    idx, w = synth.routing(T, E, K, seed=0)
    n = min(sample_tokens, T)
    x = synth.tokens_bf16(n, H, seed=0)
    chunk = 2048
    y = synth.tokens_bf16(chunk * K, H, seed=1)
    dest = np.arange(chunk * K, dtype=np.int32)
    t0 = time.perf_counter()
    oracle.route(idx, E=E, R=R)
    moved = 8 * T * K
    for c0 in range(0, n, chunk):
        c1 = min(n, c0 + chunk)
        m = c1 - c0
        oracle.dispatch(x[c0:c1], idx[c0:c1], w[c0:c1], dest[: m * K], m * K, fp8=True)
        oracle.combine(y, w[c0:c1], dest[: m * K], m, K)
        b = algorithmic_bytes(m, H, K, m * K, True)
        moved += b["dispatch"] + b["combine"]
    dt = time.perf_counter() - t0
    return {"value": round(moved / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "seconds": round(dt, 2),
            "sample": f"ht_prefill: routing of all {T} tokens + FP8 dispatch and combine of {n} "
                      f"tokens, once, in chunks of {chunk} tokens"}


def run_reference(args):
    """The oracle as the reference arm: rank 0 only, each step a bounded
    sample (1024 tokens) of the HT prefill workload on one host core."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import numpy as np

    import oracle
    from combine_ep_dispatch_03_b200 import synth

    oracle.build()
    T, H, E, K, R = HT["T"], HT["H"], HT["E"], HT["K"], HT["R"]
    n = 1024
    idx, w = synth.routing(T, E, K, seed=0)
    x = synth.tokens_bf16(n, H, seed=0)
    y = synth.tokens_bf16(n * K, H, seed=1)
    dest = np.arange(n * K, dtype=np.int32)
    sub_idx, sub_w = idx[:n], w[:n]

    def one():
        oracle.route(sub_idx, E=E, R=R)
        oracle.dispatch(x, sub_idx, sub_w, dest, n * K, fp8=True)
        oracle.combine(y, sub_w, dest, n, K)

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    dt = (time.perf_counter() - t0) / args.steps
    b = algorithmic_bytes(n, H, K, n * K, True)
    gbs = sum(b.values()) / dt / 1e9
    sample = f"ht_prefill: route + FP8 dispatch + combine of {n} of {T} tokens per step"
    # the GPU arm's config for the same workload (every pair of HT prefill is
    # placed, so its step bytes follow from the shape)
    full = algorithmic_bytes(T, H, K, T * K, True)
    l2 = L2_FALLBACK_BYTES
    try:
        import torch

        if torch.cuda.is_available():
            l2 = l2_bytes(torch.device("cuda", 0))
    except Exception:
        pass
    config = workload_config("ht_prefill", HT, world, l2_note_for(sum(full.values()), l2, False))
    print(json.dumps({
        "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": compute_dtype(HT), "data": "synthetic", "impl": "reference",
        "config": config,
        "tokens_per_s": round(n / dt, 1),
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="ht_prefill")
    ap.add_argument("--tokens", type=int, default=0, help="override T (smaller cases for profiling)")
    ap.add_argument("--hidden", type=int, default=0, help="override H (a multiple of 8; of 128 with FP8)")
    ap.add_argument("--zipf", type=float, default=None, help="override the router's Zipf bias s")
    ap.add_argument("--balanced", type=int, choices=[0, 1], default=None, help="override the balanced plan")
    ap.add_argument("--capacity", type=int, default=0, help="override the LL per-expert capacity (smaller buffers)")
    ap.add_argument("--grad-elems", type=int, default=0,
                    help="override the replica-gradient elements per expert (a multiple of 4)")
    ap.add_argument("--weight-bytes", type=int, default=0,
                    help="override the prefetch stand-in's bytes per expert (a multiple of 16)")
    ap.add_argument("--no-graph", action="store_true", help="time stream launches instead of CUDA-graph replays")
    ap.add_argument("--no-flush", action="store_true",
                    help="never flush L2 between timed steps (by default steps moving at most 4x L2 are flushed)")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-side", action="store_true", help="skip the other workloads' sub-records")
    ap.add_argument("--exchange", action="store_true",
                    help="the path across ranks through the peer table: the workload's R ranks as separate buffers "
                         "on one GPU, or one rank per GPU with --gpus R")
    ap.add_argument("--cpu-sample-tokens", type=int, default=32768)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
