"""The router kernel's selection argument, checked on the host.

ep_router_topk selects each token's top K with one 32-bit word per
candidate: the logit's order-preserving key with its low B bits (B = 5..10,
enough for an id below 32 * EPL) replaced by (2^B - 1 - id). Lane l of the
warp holds experts l, l+32, ...; each lane sorts its words, and each of K
rounds takes the warp's largest head word, whose lane pops it. The words
order candidates as (logit descending, id ascending) does, except for two
candidates whose keys agree above the low B bits. The kernel therefore redoes
the selection with full keys whenever two chosen words agree there, or an
unchosen lane head agrees there with the last chosen word.

This is a numpy model of that selection and of its two votes. On inputs
built to trip the packing (exact ties, logits that differ only in their low
mantissa bits, signed zeros), every token where the packed choice differs
from the oracle's top-K must be one the votes flag. The same holds for the
four-lanes-per-token form (K <= 8), whose second check compares the last
choice with the largest unchosen word. These check the argument, not the CUDA
code; the GPU parity tests check the kernel."""
import numpy as np
import pytest

import oracle

_ID_BITS = {1: 5, 2: 6, 4: 7, 8: 8, 16: 9, 32: 10}


def _order_keys(v):
    v = np.where(v == 0, np.float32(0), v).astype(np.float32)
    u = v.view(np.uint32).astype(np.uint64)
    return np.where(u & 0x80000000, (~u) & 0xFFFFFFFF, u | 0x80000000).astype(np.uint64)


def _packed_selection(v, K):
    """(chosen ids, flagged) for one token, as the kernel's fast path sees it."""
    E = len(v)
    epl = 1
    while 32 * epl < E:
        epl *= 2
    M = (1 << _ID_BITS[epl]) - 1
    keys = _order_keys(v)
    lanes = []
    for lane in range(32):
        words = [int((int(keys[e]) & ~M) | (M - e)) if e < E else 0
                 for e in (lane + 32 * i for i in range(epl))]
        lanes.append(sorted(words, reverse=True))
    chosen = []
    for _ in range(K):
        m = max(w[0] for w in lanes)
        for w in lanes:
            if w[0] == m:
                w.pop(0)
                w.append(0)
                break
        chosen.append(m)
    high = ~M
    flagged = any((chosen[j] ^ chosen[j + 1]) & high == 0 for j in range(K - 1))
    flagged |= any((w[0] ^ chosen[-1]) & high == 0 for w in lanes)
    return [M - (m & M) for m in chosen], flagged


def _cases(rng, n):
    for i in range(n):
        epl = int(rng.choice([1, 2, 4, 8, 16, 32]))
        E = int(rng.integers(16 * epl + 1 if epl > 1 else 2, 32 * epl + 1))
        K = int(rng.integers(1, min(E, 32) + 1))
        kind = i % 4
        if kind == 0:    # exact ties
            v = rng.integers(-3, 4, E).astype(np.float32)
        elif kind == 1:  # agree in all but the low 11 mantissa bits
            base = np.full(E, np.float32(rng.standard_normal()), np.float32)
            v = (base.view(np.uint32) ^ rng.integers(0, 1 << 11, E).astype(np.uint32)).view(np.float32)
        elif kind == 2:  # dense near one value
            v = (1.0 + 1e-4 * rng.standard_normal(E)).astype(np.float32)
        else:            # signed zeros among a few nonzero logits
            v = np.where(rng.random(E) < 0.5, np.float32(0.0), np.float32(-0.0))
            v = np.where(rng.random(E) < 0.1, rng.standard_normal(E).astype(np.float32), v)
        yield v.astype(np.float32), K


def test_every_wrong_packed_choice_is_flagged():
    oracle.build()
    rng = np.random.default_rng(11)
    flagged_needed = 0
    for v, K in _cases(rng, 600):
        want = oracle.router_topk(v[None, :], K)[0][0].tolist()
        got, flagged = _packed_selection(v, K)
        if got != want:
            assert flagged, (v.tolist(), K, got, want)
            flagged_needed += 1
    assert flagged_needed > 0  # the inputs do reach the cases the votes exist for


# share of tokens that take the exact path: 8 replaced bits and 9 boundaries at
# E = 256, K = 8 (about 0.2 %); 10 bits and 33 boundaries at E = 1024, K = 32
# (about 10 %)
@pytest.mark.parametrize("E,K,most", [(256, 8, 0.02), (1024, 32, 0.2)])
def test_unflagged_choices_on_plain_logits_match_and_flags_are_rare(E, K, most):
    oracle.build()
    rng = np.random.default_rng(E + K)
    T = 200
    logits = rng.standard_normal((T, E)).astype(np.float32)
    want = oracle.router_topk(logits, K)[0]
    flags = 0
    for t in range(T):
        got, flagged = _packed_selection(logits[t], K)
        flags += flagged
        if not flagged:
            assert got == want[t].tolist()
    assert flags <= most * T


def _lanes_selection(v, K):
    """(chosen ids, flagged) as the four-lanes-per-token kernel sees a token
    (K <= 8, E a multiple of 16): the K largest packed words are chosen (its
    sorts and merges select them exactly), and a token is flagged when two
    chosen words, or the last chosen word and the largest unchosen one (the
    (K+1)-th largest word, which the merges carry along), agree above the low
    bits."""
    E = len(v)
    epl = 1
    while 32 * epl < E:
        epl *= 2
    M = (1 << _ID_BITS[epl]) - 1
    keys = _order_keys(v)
    words = sorted(((int(keys[e]) & ~M) | (M - e) for e in range(E)), reverse=True)
    chosen = words[:K]
    unchosen = words[K] if K < E else 0
    high = ~M
    flagged = any((chosen[j] ^ chosen[j + 1]) & high == 0 for j in range(K - 1))
    flagged |= (chosen[-1] ^ unchosen) & high == 0
    return [M - (m & M) for m in chosen], flagged


def test_every_wrong_lanes_choice_is_flagged():
    oracle.build()
    rng = np.random.default_rng(13)
    flagged_needed = 0
    for v, K in _cases(rng, 900):
        E = len(v) - len(v) % 16
        if E < 16:
            continue
        v, K = v[:E], min(K, 8)
        want = oracle.router_topk(v[None, :], K)[0][0].tolist()
        got, flagged = _lanes_selection(v, K)
        if got != want:
            assert flagged, (v.tolist(), K, got, want)
            flagged_needed += 1
    assert flagged_needed > 0


@pytest.mark.parametrize("E,K,most", [(256, 8, 0.02), (128, 8, 0.02), (384, 8, 0.02), (1024, 8, 0.05)])
def test_lanes_flags_are_rare_on_plain_logits(E, K, most):
    oracle.build()
    rng = np.random.default_rng(E + 7 * K)
    T = 200
    logits = rng.standard_normal((T, E)).astype(np.float32)
    want = oracle.router_topk(logits, K)[0]
    flags = 0
    for t in range(T):
        got, flagged = _lanes_selection(logits[t], K)
        flags += flagged
        if not flagged:
            assert got == want[t].tolist()
    assert flags <= most * T
