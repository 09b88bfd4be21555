"""Seeded synthetic inputs for MoE expert-parallel dispatch and combine.

This module only draws inputs. It holds none of the dispatch / combine /
planning arithmetic: the CUDA path and the CPU oracle both receive the
tensors made here and nothing else is shared between them.

Input recipe (all CPU tensors, deterministic for a given torch version):

* tokens ``x[T, H]``: N(0, 1) samples from ``torch.randn`` (float32, drawn
  in fixed row chunks from one seeded ``torch.Generator``), rounded to bf16.
* router: logits ``l[t, e] = N(0, 1) + s * ln(1 / (e + 1))`` in float32,
  i.e. a Zipf-style bias of strength ``s`` on expert rank ``e + 1`` (``s = 0``
  is the balanced N(0, 1) router). Top-K by descending logit with ties broken
  towards the lower expert id (a stable sort), weights = softmax over the
  selected K logits computed in float64 and rounded to float32, which equals
  a full softmax followed by renormalisation over the top-K. The gating step
  itself is described in "Ultra-Large MoE Models: Open-Source Evolution and
  Heterogeneous Inference Adaptation", section 2.1 (top-K routing, K = 2 or 8).
* expert stand-ins used by tests and the benchmark harness (not part of the
  path): identity, and ``y = bf16(1.5 * float(r) + 0.25)``.
"""
from __future__ import annotations

import math

import torch

_CHUNK_ROWS = 4096


def _gen(seed: int, stream: int) -> torch.Generator:
    # one independent generator per (seed, tensor) pair
    g = torch.Generator(device="cpu")
    g.manual_seed((int(seed) * 1_000_003 + int(stream) * 7919 + 12345) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def tokens_bf16(T: int, H: int, seed: int = 0, stream: int = 1, out: torch.Tensor | None = None) -> torch.Tensor:
    """x[T, H] bf16 with N(0, 1) values (float32 samples rounded to bf16)."""
    g = _gen(seed, stream)
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16)
    for r0 in range(0, T, _CHUNK_ROWS):
        r1 = min(T, r0 + _CHUNK_ROWS)
        out[r0:r1].copy_(torch.randn((r1 - r0, H), generator=g, dtype=torch.float32))
    return out


def router_logits(T: int, E: int, zipf_s: float = 0.0, seed: int = 0, stream: int = 2) -> torch.Tensor:
    """logits[T, E] float32 = N(0, 1) + s * ln(1 / (e + 1))."""
    g = _gen(seed, stream)
    logits = torch.randn((T, E), generator=g, dtype=torch.float32)
    if zipf_s != 0.0:
        bias = torch.tensor([zipf_s * math.log(1.0 / (e + 1)) for e in range(E)], dtype=torch.float32)
        logits += bias
    return logits


def topk_route(logits: torch.Tensor, K: int) -> tuple[torch.Tensor, torch.Tensor]:
    """(topk_idx[T, K] int32, topk_w[T, K] float32) from router logits."""
    _, order = torch.sort(logits, dim=1, descending=True, stable=True)
    idx = order[:, :K].contiguous()
    top = torch.gather(logits, 1, idx).to(torch.float64)
    w = torch.softmax(top, dim=1).to(torch.float32)
    return idx.to(torch.int32).contiguous(), w.contiguous()


def routing(T: int, E: int, K: int, zipf_s: float = 0.0, seed: int = 0) -> tuple[torch.Tensor, torch.Tensor]:
    """Seeded synthetic router output for T tokens over E experts, top-K."""
    return topk_route(router_logits(T, E, zipf_s, seed), K)


def affine_expert(r: torch.Tensor) -> torch.Tensor:
    """Harness stand-in for an expert FFN: bf16(1.5 * r + 0.25), computed in float32."""
    return (r.to(torch.float32) * 1.5 + 0.25).to(torch.bfloat16)


# The workloads the benchmark and the parity tests use.
WORKLOADS = {
    # T, H, E, K, R, mode, ll_capacity, fp8, balanced, zipf_s
    "tiny": dict(T=128, H=1024, E=16, K=2, R=4, mode="ht", cap=0, fp8=False, balanced=False, s=0.0),
    "ll_decode": dict(T=1024, H=7168, E=256, K=8, R=8, mode="ll", cap=1024, fp8=False, balanced=False, s=0.0),
    "ht_prefill": dict(T=32768, H=7168, E=256, K=8, R=8, mode="ht", cap=0, fp8=True, balanced=False, s=0.0),
    "imbalance": dict(T=32768, H=4096, E=128, K=8, R=8, mode="ht", cap=0, fp8=False, balanced=False, s=0.0),
    "large_train": dict(T=131072, H=7168, E=384, K=8, R=16, mode="ht", cap=0, fp8=False, balanced=True, s=1.0),
}
