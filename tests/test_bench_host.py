"""Host-side arithmetic of the benchmark (no GPU): the algorithmic bytes each
call must move, counted here term by term for a small case, and the guard
that ties a committed DRAM traffic figure to the source it was measured on."""
import sys

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_algorithmic_bytes_bf16_by_hand():
    T, H, K, P = 4, 128, 2, 7  # 8 pairs, 7 of them placed
    b = bench.algorithmic_bytes(T, H, K, P, fp8=False)
    L = T * K
    # plan: ids read (4 B each), dest_row written for every pair, src_row for placed ones
    assert b["plan"] == 4 * L + 4 * L + 4 * P
    # dispatch: x read once (bf16), every placed row written once, idx + w + dest read,
    # recv_w and recv_expert written per placed row
    assert b["dispatch"] == 2 * T * H + 2 * P * H + 12 * L + 8 * P
    # combine: every placed expert row read once, out written once, w + dest read
    assert b["combine"] == 2 * P * H + 2 * T * H + 8 * L


def test_algorithmic_bytes_fp8_by_hand():
    T, H, K, P = 4, 256, 2, 8
    b = bench.algorithmic_bytes(T, H, K, P, fp8=True)
    L = T * K
    # one byte per element and one fp32 scale per 128-element block of each placed row
    assert b["dispatch"] == 2 * T * H + P * H + P * (H // 128) * 4 + 12 * L + 8 * P
    assert b["combine"] == 2 * P * H + 2 * T * H + 8 * L


def test_ht_prefill_step_bytes_match_the_documented_total():
    # the HT prefill step with every pair placed: 6.64 GB
    wl = bench.WORKLOADS["ht_prefill"]
    T, H, K = wl["T"], wl["H"], wl["K"]
    b = bench.algorithmic_bytes(T, H, K, T * K, fp8=True)
    assert abs(sum(b.values()) / 1e9 - 6.645) < 0.002


def test_committed_traffic_is_tied_to_its_workload_and_source():
    assert bench.committed_traffic("k_combine", "not_a_workload") is None
    assert bench.committed_traffic("no_such_kernel", "ht_prefill") is None


def test_weak_scaling_value_single_rank():
    value, ms = bench.weak_scaling_value(2.0e9, 1.0, 1)
    assert ms == 1.0 and abs(value - 2000.0) < 1e-9


def test_code_sha_ignores_comments_but_not_code(tmp_path):
    a = tmp_path / "a.cu"
    a.write_text("// row mover\n__global__ void k(int* p) { p[0] = 1; /* store */ }\n")
    base = bench.code_sha([str(a)])
    a.write_text("/* another\n comment */ __global__ void k(int* p) {\n  p[0] = 1;  // same store\n}\n")
    assert bench.code_sha([str(a)]) == base
    a.write_text("__global__ void k(int* p) { p[0] = 2; }\n")
    assert bench.code_sha([str(a)]) != base


def test_committed_traffic_records_name_existing_sources():
    import json
    import os
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        recs = json.load(f)
    for rec in recs.values():
        assert rec["sources"] and all(os.path.exists(os.path.join(ROOT, s)) for s in rec["sources"])
        assert len(rec["code_sha"]) == 16 and rec["dram_bytes_per_launch"] > 0


def test_l2_flush_decision():
    l2 = bench.L2_FALLBACK_BYTES
    # HT prefill moves 6.6 GB a step: far beyond L2, no flush
    wl = bench.WORKLOADS["ht_prefill"]
    b = bench.algorithmic_bytes(wl["T"], wl["H"], wl["K"], wl["T"] * wl["K"], fp8=True)
    assert not bench.needs_l2_flush(sum(b.values()), l2)
    # LL decode moves about 265 MB (about 2x L2), the router 36 MB: flushed
    wl = bench.WORKLOADS["ll_decode"]
    b = bench.algorithmic_bytes(wl["T"], wl["H"], wl["K"], wl["T"] * wl["K"], fp8=False)
    assert bench.needs_l2_flush(sum(b.values()), l2)
    assert bench.needs_l2_flush(4 * 32768 * 256 + 8 * 32768 * 8, l2)
    # the three notes name what was done before each timed step
    assert bench.l2_note_for(264568832, l2, True).startswith("flushed: ")
    assert bench.l2_note_for(264568832, l2, "clean").startswith("flushed, clean: ")
    assert "read" in bench.l2_note_for(264568832, l2, "clean")
    assert bench.l2_note_for(264568832, l2, False).startswith("not flushed")


class _Buf:
    def __init__(self):
        self.calls = []

    def fill_(self, v):
        self.calls.append(("fill", v))

    def sum(self):
        self.calls.append(("sum",))


def test_flush_writes_then_reads_for_a_clean_l2():
    w, r = _Buf(), _Buf()
    bench._flush_l2((w, r), 130)
    assert w.calls == [("fill", 130 & 0x7F)] and r.calls == [("sum",)]
    one = _Buf()
    bench._flush_l2(one, 3)
    assert one.calls == [("fill", 3)]


def test_modelled_exchange_stays_flat_under_the_balanced_plan():
    """The sweep's derived column on the oracle's routing at the sweep's full
    size: with the balanced plan the busiest rank holds ceil(L/R) rows at
    every skew, so the modelled exchange time does not move; without it, it
    grows with the skew."""
    import numpy as np

    import oracle
    from combine_ep_dispatch_03_b200 import synth

    oracle.build()
    wl = bench.SWEEP
    T, H, E, K, R = wl["T"], wl["H"], wl["E"], wl["K"], wl["R"]
    L = T * K
    flat, plain = [], []
    for s in (0.0, 0.5, 1.0, 1.5):
        idx, _ = synth.routing(T, E, K, zipf_s=s, seed=11)
        bal = oracle.route(idx, E=E, R=R, balanced=True)
        assert bal.flags == 0 and max(bal.plan["rank_load"]) == -(-L // R)
        flat.append(bench.modelled_exchange_ms(bal.plan["rank_load"], 2 * H))
        loads = oracle.route(idx, E=E, R=R).cnt.reshape(R, E // R).sum(axis=1)
        plain.append(bench.modelled_exchange_ms(loads, 2 * H))
    assert flat == [flat[0]] * 4
    assert abs(flat[0] - 2 * (L // R) * 2 * H / 770e9 * 1e3) < 1e-9
    assert np.all(np.diff(plain) > 0) and plain[-1] > 5 * flat[0]


def test_clock_records_that_reject_a_number():
    ok = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert bench.clocks_rejected(ok) is None
    assert bench.clocks_rejected(dict(ok, reasons=["sw_power_cap"], sm_mhz=1500.0)) is None  # kept, noted
    assert "hw_thermal_slowdown" in bench.clocks_rejected(dict(ok, reasons=["hw_thermal_slowdown"]))
    assert "sw_thermal_slowdown" in bench.clocks_rejected(dict(ok, reasons=["sw_power_cap", "sw_thermal_slowdown"]))
    assert "no reason" in bench.clocks_rejected(dict(ok, sm_mhz=1000.0))  # a leftover clock lock
    assert bench.clocks_rejected({"sm_mhz": None, "sm_max_mhz": None, "reasons": []}) is None
