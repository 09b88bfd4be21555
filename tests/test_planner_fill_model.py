"""The balanced planner's parallel fill (csrc/route.cu, layout_balanced),
restated on the host and checked against the oracle's greedy walk (MoonEP
article paras. 3 and 5: the plan fills the ranks below their share from the
experts with rows left). The kernel finds the pieces with closed forms
instead of walking:

- the spilled rows of the experts in fill order are the intervals
  [A_i, A_i+1), the receivers' deficit rows [B_k, B_k+1); a piece is the
  overlap of one of each;
- expert i's pieces go to receivers q_first..q_last, the ones holding its
  first and last spilled rows;
- expert i's first piece is i plus the receivers' first rows that fall
  strictly inside the rows of the experts before it;
- a piece's slot is its expert's place minus that of the expert holding
  its receiver's first deficit row.

Here those formulas (and only they) build the plan from a count vector, and
the result must equal the oracle's plan table by table, on random counts
with every skew. Cases where a receiver needs more than S slots without
direct overflow take the kernel's one-thread walk, which is the oracle's
walk itself; they are only counted here."""
import numpy as np
import pytest

import oracle


def _last_le(a, v):
    """Last index i with a[i] <= v (a ascending, a[0] <= v)."""
    return int(np.searchsorted(a, v, side="right")) - 1


def closed_form_plan(cnt, R, S, direct):
    E = len(cnt)
    g = E // R
    L = int(cnt.sum())
    q, rem = divmod(L, R)
    cap = [q + (1 if r < rem else 0) for r in range(R)]
    keep = np.zeros(E, np.int64)
    for e in range(E):
        r, c = e // g, int(cnt[e])
        before = sum(int(cnt[e2]) for e2 in range(r * g, r * g + g)
                     if int(cnt[e2]) < c or (int(cnt[e2]) == c and e2 < e))
        keep[e] = max(0, min(c, cap[r] - before))
    used = [int(keep[r * g:(r + 1) * g].sum()) for r in range(R)]
    D = [cap[r] - used[r] for r in range(R)]
    assert min(D) >= 0
    spilled = sorted((e for e in range(E) if cnt[e] > keep[e]), key=lambda e: (-int(cnt[e]), e))
    recv = sorted((r for r in range(R) if D[r] > 0), key=lambda r: (-D[r], r))
    A = np.concatenate([[0], np.cumsum([int(cnt[e] - keep[e]) for e in spilled])]).astype(np.int64)
    B = np.concatenate([[0], np.cumsum([D[r] for r in recv])]).astype(np.int64)
    assert A[-1] == B[-1]  # the deficits add up to the spilled rows
    nsp, nrecv = len(spilled), len(recv)
    fe = [_last_le(A[:nsp], B[k]) for k in range(nrecv)]
    le = [_last_le(A[:nsp], B[k + 1] - 1) for k in range(nrecv)]
    if not direct and any(le[k] - fe[k] + 1 > S for k in range(nrecv)):
        return None  # the one-thread walk
    inner = [1 if (k > 0 and A[fe[k]] < B[k]) else 0 for k in range(nrecv)]
    rep = np.full((R, S), -1, np.int64)
    sstart = np.zeros((R, S), np.int64)
    slen = np.zeros((R, S), np.int64)
    dn = np.zeros(R, np.int64)
    de = np.full((R, E), -1, np.int64)
    ds = np.zeros((R, E), np.int64)
    dl = np.zeros((R, E), np.int64)
    pieces = 0
    for i, e in enumerate(spilled):
        qf, ql = _last_le(B[:nrecv], A[i]), _last_le(B[:nrecv], A[i + 1] - 1)
        assert i + sum(inner[1:qf + 1]) == pieces  # the first piece's closed form
        for k in range(qf, ql + 1):
            r = recv[k]
            lo, hi = max(A[i], B[k]), min(A[i + 1], B[k + 1])
            slot = i - fe[k]
            start = int(keep[e] + lo - A[i])
            if slot < S:
                assert rep[r, slot] == -1
                rep[r, slot], sstart[r, slot], slen[r, slot] = e, start, hi - lo
            else:
                de[r, slot - S], ds[r, slot - S], dl[r, slot - S] = e, start, hi - lo
                dn[r] = max(dn[r], slot - S + 1)
            pieces += 1
    load = np.array([used[r] + int(slen[r].sum()) + int(dl[r].sum()) for r in range(R)])
    return dict(keep=keep, rep=rep, sstart=sstart, slen=slen, dn=dn, de=de, ds=ds, dl=dl, load=load)


def _counts(rng, E):
    kind = rng.integers(0, 4)
    if kind == 0:
        c = rng.integers(0, 50, E)
    elif kind == 1:
        c = (rng.pareto(rng.uniform(0.3, 2.0), E) * 20).astype(np.int64)
    elif kind == 2:
        c = np.zeros(E, np.int64)
        c[rng.integers(0, E, rng.integers(1, 4))] = rng.integers(50, 5000)
        c += rng.integers(0, 3, E)
    else:
        c = rng.integers(0, 4, E) * rng.integers(1, 30)  # many equal counts
    return np.minimum(c, 100000).astype(np.int32)


CASES = list(range(400))


@pytest.mark.parametrize("seed", CASES[::40])
def test_closed_form_fill_equals_the_walk(seed):
    oracle.build()
    walked = 0
    for s in range(seed, seed + 40):
        rng = np.random.default_rng(5000 + s)
        E = int(rng.choice([4, 8, 16, 32, 48, 64, 128, 256, 384]))
        R = int(rng.choice([r for r in (1, 2, 4, 8, 16) if E % r == 0]))
        g = E // R
        S = int(rng.integers(1, g + 1))
        direct = bool(rng.random() < 0.5)
        cnt = _counts(rng, E)
        if cnt.sum() == 0:
            cnt[0] = 1
        idx = np.repeat(np.arange(E, dtype=np.int32), cnt)[:, None]  # a batch with these counts
        ref = oracle.route(idx, E=E, R=R, balanced=True, slots=S, direct=direct)
        np.testing.assert_array_equal(ref.cnt, cnt)
        m = closed_form_plan(cnt.astype(np.int64), R, S, direct)
        if m is None:
            walked += 1
            assert not direct
            continue
        p = ref.plan
        np.testing.assert_array_equal(m["keep"], p["keep"])
        assert (p["tail_len"] == 0).all()  # without the walk every spilled row finds a receiver
        np.testing.assert_array_equal(m["rep"], p["replica_expert"])
        filled = m["rep"] >= 0
        np.testing.assert_array_equal(m["sstart"][filled], p["slot_start"][filled])
        np.testing.assert_array_equal(m["slen"], p["slot_len"])
        np.testing.assert_array_equal(m["load"], p["rank_load"])
        if direct:
            np.testing.assert_array_equal(m["dn"], p["direct_n"])
            for r in range(R):
                n = int(m["dn"][r])
                np.testing.assert_array_equal(m["de"][r, :n], p["direct_expert"][r, :n])
                np.testing.assert_array_equal(m["ds"][r, :n], p["direct_start"][r, :n])
                np.testing.assert_array_equal(m["dl"][r, :n], p["direct_len"][r, :n])
    assert walked < 40
