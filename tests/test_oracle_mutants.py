"""The pins are strong enough to catch plausible mistakes in the oracle.

Each case plants one mistake (one that keeps every access in bounds) in a
copy of oracle/ep_oracle.c: a dropped
term, a wrong operator, a flipped tie-break, an off-by-one, a wrong rounding,
a wrong order. It compiles the copy on the CPU, points the oracle wrapper at
it, and checks that at least one of the listed pins then fails. The real
oracle is restored afterwards.
"""
import ctypes
import os

import numpy as np
import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "ep_oracle.c")

# name, text to replace (must occur once), replacement, pins that must catch it;
# a mistake that needs several edits gives a list of (text, replacement) pairs
# and None for the replacement
MUTANTS = [
    ("combine drops the first choice",
     "            for (int k = 0; k < K; k++) {\n                int32_t row = dest_row[(int64_t)t * K + k];\n"
     "                if (row < 0) continue;\n                float v",
     "            for (int k = 1; k < K; k++) {\n                int32_t row = dest_row[(int64_t)t * K + k];\n"
     "                if (row < 0) continue;\n                float v",
     [lambda: pins.test_identity_expert_returns_x(oracle, "ht"), lambda: pins.test_combine_golden(oracle)]),
    ("FP8 scale multiplies instead of dividing",
     "float s = amax / 448.0f;", "float s = amax * 448.0f;",
     [lambda: pins.test_fp8_block_golden(oracle)]),
    ("plan keeps the higher id first on a count tie",
     "(cnt[order[b]] > cnt[v] || (cnt[order[b]] == cnt[v] && order[b] > v))",
     "(cnt[order[b]] > cnt[v] || (cnt[order[b]] == cnt[v] && order[b] < v))",
     [lambda: pins.test_plan_golden(oracle)]),
    ("stable index off by one",
     "j[(int64_t)t * K + k] = cnt[e];", "j[(int64_t)t * K + k] = cnt[e] + 1;",
     [lambda: pins.test_route_golden(oracle), lambda: pins.test_route_brute_force(oracle, 0)]),
    ("e4m3 rounds half away from zero",
     "double m = nearbyint((a / ldexp(1.0, ex) - 1.0) * 8.0);",
     "double m = round((a / ldexp(1.0, ex) - 1.0) * 8.0);",
     [lambda: pins.test_e4m3_golden_table(oracle),
      lambda: pins.test_e4m3_matches_torch_in_range_all_bf16_times_scales(oracle)]),
    ("bf16 conversion truncates",
     "if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))", "if (0)",
     [lambda: pins.test_bf16_rounding_matches_torch(oracle)]),
    ("replica gradients added in descending slot order",
     "for (int a = 0; a < n; a++) acc = acc + rep[(int64_t)list[a] * G + i];",
     "for (int a = n - 1; a >= 0; a--) acc = acc + rep[(int64_t)list[a] * G + i];",
     [lambda: pins.test_replica_reduce_order_is_slot_ascending(oracle)]),
    ("router breaks ties towards the higher id",
     "if (best < 0 || l[e] > l[best]) best = e;", "if (best < 0 || l[e] >= l[best]) best = e;",
     [lambda: pins.test_router_topk_ties_take_lower_id(oracle),
      lambda: pins.test_router_topk_matches_library_routines(oracle)]),
    ("combine backward forgets the router weight",
     "float prod = wk * orc_bf16_to_f32(g[(int64_t)t * H + i]);",
     "float prod = orc_bf16_to_f32(g[(int64_t)t * H + i]);",
     [lambda: pins.test_adjoint_identities_exact(oracle, False)]),
    ("LL keeps the pair at the capacity",
     "} else if (j[p] >= cap) {", "} else if (j[p] > cap) {",
     [lambda: pins.test_route_golden(oracle), lambda: pins.test_route_ll_capacity(oracle)]),
    ("inference plan never takes direct pieces",
     "if (D[r] > 0 && (nrep[r] < S || direct)) {", "if (D[r] > 0 && (nrep[r] < S || 0)) {",
     [lambda: pins.test_plan_golden(oracle), lambda: pins.test_direct_plan_invariants(oracle, 16, 4, 1)]),
    ("FP8 cast of an all-zero block divides by zero",
     "            if (amax == 0.0f)\n                q[b * 128 + i] = 0;\n            else\n"
     "                q[b * 128 + i] = orc_e4m3_from_f32(orc_bf16_to_f32(x[b * 128 + i]) / s);",
     "            q[b * 128 + i] = orc_e4m3_from_f32(orc_bf16_to_f32(x[b * 128 + i]) / s);",
     [lambda: pins.test_fp8_dequant_error_bound(oracle), lambda: pins.test_fp8_block_golden(oracle)]),
    ("FP8 cast multiplies by the reciprocal of the scale",
     "q[b * 128 + i] = orc_e4m3_from_f32(orc_bf16_to_f32(x[b * 128 + i]) / s);",
     "q[b * 128 + i] = orc_e4m3_from_f32(orc_bf16_to_f32(x[b * 128 + i]) * (1.0f / s));",
     [lambda: pins.test_fp8_cast_is_the_exactly_rounded_quotient(oracle)]),
    ("FP8 scale multiplies by a rounded 1/448",
     "float s = amax / 448.0f;", "float s = amax * (1.0f / 448.0f);",
     [lambda: pins.test_fp8_cast_is_the_exactly_rounded_quotient(oracle), lambda: pins.test_fp8_block_golden(oracle)]),
    ("combine rounds each product before adding it",
     "acc = fmaf(w[(int64_t)t * K + k], v, acc);", "acc = w[(int64_t)t * K + k] * v + acc;",
     [lambda: pins.test_combine_is_the_exact_fma_chain(oracle), lambda: pins.test_combine_golden(oracle),
      lambda: pins.test_affine_expert_and_fp64_error_bound(oracle)]),
    ("plan spills the coldest expert first",
     "(cnt[order[b]] < cnt[v] || (cnt[order[b]] == cnt[v] && order[b] > v))",
     "(cnt[order[b]] > cnt[v] || (cnt[order[b]] == cnt[v] && order[b] > v))",
     [lambda: pins.test_plan_golden(oracle)]),
    ("plan visits receivers by ascending deficit",
     "(D[recv[b]] < D[v] || (D[recv[b]] == D[v] && recv[b] > v))",
     "(D[recv[b]] > D[v] || (D[recv[b]] == D[v] && recv[b] > v))",
     [lambda: pins.test_plan_golden(oracle)]),
    ("router rounds each exponential to float before summing",
     "ex[k] = exp((double)l[idx[(int64_t)t * K + k]] - lmax);",
     "ex[k] = (float)exp((double)l[idx[(int64_t)t * K + k]] - lmax);",
     [lambda: pins.test_router_topk_matches_library_routines(oracle)]),
    ("combine backward uses the next choice's weight",
     "float wk = w[(int64_t)t * K + k];", "float wk = w[(int64_t)t * K + (k + 1) % K];",
     [lambda: pins.test_adjoint_identities_exact(oracle, False)]),
    ("replica reduce adds only the first replica",
     "for (int a = 0; a < n; a++) acc = acc + rep[(int64_t)list[a] * G + i];",
     "for (int a = 0; a < (n > 0 ? 1 : 0); a++) acc = acc + rep[(int64_t)list[a] * G + i];",
     [lambda: pins.test_replica_reduce_sums_exactly(oracle)]),
    ("replica reduce drops the owner's value",
     "float acc = owner[(int64_t)e * G + i];", "float acc = 0.0f;",
     [lambda: pins.test_replica_reduce_sums_exactly(oracle)]),
    ("dispatch records the token id as the expert",
     "if (recv_expert) recv_expert[row] = idx[p];", "if (recv_expert) recv_expert[row] = t;",
     [lambda: pins.test_dispatch_bf16_rows_follow_sorted_pairs(oracle)]),
    ("dispatch records the first choice's weight for every row",
     "if (recv_w) recv_w[row] = w[p];", "if (recv_w) recv_w[row] = w[(int64_t)t * K];",
     [lambda: pins.test_dispatch_bf16_rows_follow_sorted_pairs(oracle)]),
    ("e4m3 saturates to NaN instead of 448",
     "if (a > 448.0) return (uint8_t)(sign | 0x7e);", "if (a > 448.0) return (uint8_t)(sign | 0x7f);",
     [lambda: pins.test_e4m3_golden_table(oracle),
      lambda: pins.test_e4m3_matches_torch_in_range_all_bf16_times_scales(oracle)]),
    ("e4m3 loses the sign of a negative zero",
     "uint8_t sign = signbit(v) ? 0x80 : 0x00;", "uint8_t sign = (v < 0.0f) ? 0x80 : 0x00;",
     [lambda: pins.test_e4m3_golden_table(oracle),
      lambda: pins.test_e4m3_matches_torch_in_range_all_bf16_times_scales(oracle)]),
    ("owner's tail placed before its kept rows",
     "dest_row[p] = (int32_t)(rank_off[owner] + own_off + keep[e] + (j[p] - tail_start[e]));",
     "dest_row[p] = (int32_t)(rank_off[owner] + own_off + (j[p] - tail_start[e]));",
     [lambda: pins.test_plan_golden(oracle)]),
    ("later own experts ignore an earlier expert's tail",
     "for (int e2 = owner * g; e2 < e; e2++) own_off += keep[e2] + tail_len[e2];",
     "for (int e2 = owner * g; e2 < e; e2++) own_off += keep[e2];",
     [lambda: pins.test_plan_golden(oracle)]),
    ("direct pieces ignore earlier direct pieces",
     "for (int i2 = 0; i2 < i; i2++) off += direct_len[r * E + i2];",
     "for (int i2 = 0; i2 < 0; i2++) off += direct_len[r * E + i2];",
     [lambda: pins.test_direct_plan_invariants(oracle, 16, 4, 1)]),
    ("replica slot offset counts its own slot",
     "for (int s2 = 0; s2 < s; s2++) off += slot_len[r * S + s2];",
     "for (int s2 = 0; s2 <= s; s2++) off += slot_len[r * S + s2];",
     [lambda: pins.test_plan_golden(oracle)]),
    ("direct piece placed before the rank's slots",
     "                for (int s2 = 0; s2 < S; s2++) off += slot_len[r * S + s2];\n                for (int i2 = 0;",
     "                for (int s2 = 0; s2 < 0; s2++) off += slot_len[r * S + s2];\n                for (int i2 = 0;",
     [lambda: pins.test_plan_golden(oracle), lambda: pins.test_direct_plan_invariants(oracle, 16, 4, 1)]),
    ("dispatch-backward sum taken in reverse order",
     "            for (int k = 0; k < K; k++) {\n                int32_t row = dest_row[(int64_t)t * K + k];\n"
     "                if (row < 0) continue;\n                float v",
     "            for (int k0 = 0; k0 < K; k0++) {\n                int k = w ? k0 : K - 1 - k0;\n"
     "                int32_t row = dest_row[(int64_t)t * K + k];\n                if (row < 0) continue;\n"
     "                float v",
     [lambda: pins.test_dispatch_backward_is_the_exact_sum_chain(oracle)]),
    ("dispatch-backward sum taken as a pairwise tree",
     [("            float acc = 0.0f;", "            float acc = 0.0f, buf[32] = {0};"),
      ("                else\n                    acc = acc + v;", "                else\n                    buf[k] = v;"),
      ("            out[(int64_t)t * H + i] = orc_bf16_from_f32(acc);",
       "            for (int n = K, m; !w && n > 1; n = m) {\n                m = (n + 1) / 2;\n"
       "                for (int a = 0; a < n / 2; a++) buf[a] = buf[2 * a] + buf[2 * a + 1];\n"
       "                if (n & 1) buf[m - 1] = buf[n - 1];\n            }\n"
       "            if (!w) acc = acc + buf[0];\n"
       "            out[(int64_t)t * H + i] = orc_bf16_from_f32(acc);")],
     None,
     [lambda: pins.test_dispatch_backward_is_the_exact_sum_chain(oracle)]),
    ("dispatch-backward sum kept in bf16 between adds",
     "acc = acc + v;", "acc = orc_bf16_to_f32(orc_bf16_from_f32(acc + v));",
     [lambda: pins.test_dispatch_backward_is_the_exact_sum_chain(oracle)]),
    ("combine backward rounds the exact product straight to bf16",
     "                float prod = wk * orc_bf16_to_f32(g[(int64_t)t * H + i]);",
     "                int ex2;\n"
     "                double m2 = frexp((double)wk * (double)orc_bf16_to_f32(g[(int64_t)t * H + i]), &ex2);\n"
     "                float prod = (float)ldexp(nearbyint(m2 * 256.0) / 256.0, ex2);",
     [lambda: pins.test_combine_backward_is_one_fp32_product_then_bf16(oracle)]),
    ("combine backward multiplies in bf16",
     "float prod = wk * orc_bf16_to_f32(", "float prod = orc_bf16_to_f32(orc_bf16_from_f32(wk)) * orc_bf16_to_f32(",
     [lambda: pins.test_combine_backward_is_one_fp32_product_then_bf16(oracle)]),
]


@pytest.fixture
def mutant_lib(tmp_path):
    saved = oracle._lib
    src = open(SRC).read()

    def load(find, repl):
        # one (anchor, replacement) pair, or a list of pairs applied in turn
        edits = find if isinstance(find, list) else [(find, repl)]
        text = src
        for a, b in edits:
            assert text.count(a) == 1, f"mutation anchor not unique: {a!r}"
            text = text.replace(a, b)
        path = tmp_path / "mutant.c"
        path.write_text(text)
        so = oracle.compile_to(str(path), str(tmp_path / "libmutant.so"))
        oracle._lib = oracle.configure(ctypes.CDLL(so))

    yield load
    oracle._lib = saved


@pytest.mark.parametrize("name,find,repl,checks", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(mutant_lib, name, find, repl, checks):
    mutant_lib(find, repl)
    caught = 0
    for check in checks:
        try:
            with np.errstate(all="ignore"):
                check()
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin caught the planted mistake: {name}"


def test_real_oracle_passes_the_same_checks():
    oracle._lib = None  # the real library
    for _, _, _, checks in MUTANTS:
        for check in checks:
            check()
