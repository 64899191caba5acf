"""The oracle's pins catch plausible mistakes (CPU only).

Each case plants one mistake in a copy of the oracle's C source (compiled into
a temporary library; the oracle itself is untouched), points the oracle's
Python marshalling at that copy, and runs the pins of the affected function
(the same test functions the suite runs).  At least one of them must fail.
The unchanged copy passes them all.
"""
import os
import subprocess

import pytest

import oracle
import test_oracle_dispatch as tdisp
import test_oracle_plan as tplan
import test_oracle_plan_variants as tvar
import test_oracle_restore as trest
import test_oracle_steps as tsteps
from moe_expert_load_ue_b200 import inputs

SRC = os.path.join(os.path.dirname(oracle.__file__), "ue_oracle.c")


def _plan_pins():
    for case in tplan._cases():
        tplan.test_plan_hand_cases(case)
    for seed in range(40):
        tplan.test_plan_invariants_random(seed)
    tplan.test_plan_invariants_synthetic_workloads()
    tplan.test_brute_force_gap_report()


def _variant_pins():
    for case in tvar._cases():
        tvar.test_variant_hand_cases(case)
    for seed in range(40):
        tvar.test_variant_invariants_random(seed)
    tvar.test_spread_never_raises_the_max()
    tvar.test_variant_brute_force_gaps()


def _reroute_pins():
    for case in tsteps._golden():
        tsteps.test_reroute_hand_cases(case)
    tsteps.test_reroute_second_check_and_invariants(inputs.TINY)
    tsteps.test_reroute_bad_ids()


def _load_pins():
    tsteps.test_load_matches_bincount(inputs.TINY)
    tsteps.test_load_bad_ids_and_ragged_k()
    tsteps.test_rank_offsets_brute_force()


def _dispatch_pins():
    for case in tdisp._golden():
        tdisp.test_dispatch_hand_cases(case)
    tdisp.test_dispatch_matches_stable_argsort_and_quotas(inputs.TINY)
    tdisp.test_dispatch_drops_bad_ids()


def _sync_pins():
    for R in (1, 2):
        tsteps.test_sync_byte_map(R)
        tsteps.test_sync_delta_equals_full_sync_state(R)
    tsteps.test_sync_delta_same_plan_copies_nothing_and_none_is_full()


def _restore_pins():
    for E, N, R in ((16, 4, 1), (16, 4, 2), (12, 6, 3)):
        trest.test_restore_layer_stack(E, N, R)
    trest.test_restore_skips_slots_that_hold_the_expert()
    trest.test_restore_same_plan_copies_nothing_and_unknown_holder_is_full_sync()
    trest.test_restore_hand_case()


def _grad_pins():
    for bf16 in (False, True):
        tsteps.test_grad_reduce_exact_dyadic(bf16)
    tsteps.test_grad_reduce_zero_grads_identity_and_order()


# name: (pins, text in ue_oracle.c, planted replacement)
MUTANTS = {
    "Q rounded down": (_plan_pins, "(L + N - 1) / N;        /* Q = ceil(L / N) */", "L / N;"),
    "overflow smallest first": (_plan_pins, "return x->ovf > y->ovf ? -1 : 1;", "return x->ovf < y->ovf ? -1 : 1;"),
    "overflow ties to the higher id": (_plan_pins, "return x->e < y->e ? -1 : (x->e > y->e ? 1 : 0);",
                                       "return x->e > y->e ? -1 : (x->e < y->e ? 1 : 0);"),
    "spare ties to the highest rank": (_plan_pins, "if (best < 0 || Q - cur[r] > Q - cur[best]) best = r;",
                                       "if (best < 0 || Q - cur[r] >= Q - cur[best]) best = r;"),
    "home takes the whole load": (_plan_pins, "int64_t take = load[e] < Q - cur[h] ? load[e] : Q - cur[h];",
                                  "int64_t take = load[e];"),
    "chunk not capped by spare": (_plan_pins, "int64_t c = rem_e[e] < spare ? rem_e[e] : spare;",
                                  "int64_t c = rem_e[e];"),
    "requeue ties to the higher id": (_variant_pins, "if (rem_e[x] > 0 && (e < 0 || rem_e[x] > rem_e[e])) e = x;",
                                      "if (rem_e[x] > 0 && (e < 0 || rem_e[x] >= rem_e[e])) e = x;"),
    "spread ties to the later replica": (_variant_pins, "if (cur[r] < best_load) { best_load = cur[r]; best_a = a; }",
                                         "if (cur[r] <= best_load) { best_load = cur[r]; best_a = a; }"),
    "spread never back to the home": (_variant_pins, "int64_t best_load = cur[h];", "int64_t best_load = INT64_MAX;"),
    "inclusive cumulative quotas": (_reroute_pins, "rep_cum[pos] = (int32_t)cum;\n            cum += asg_c[a];",
                                    "cum += asg_c[a];\n            rep_cum[pos] = (int32_t)cum;"),
    "occurrences counted from 1": (_reroute_pins, "int64_t j = occ[e]++;", "int64_t j = ++occ[e];"),
    "quota range closed": (_reroute_pins, "if (lo <= j && j < lo + q)", "if (lo <= j && j <= lo + q)"),
    "tokens dealt round-robin to ranks": (_load_pins, "int64_t r = t / tokens_per_rank;", "int64_t r = t % N;"),
    "rank offsets inclusive": (_load_pins, "if (rank_off) rank_off[(int64_t)r * E + e] = (int32_t)run;\n"
                               "            run += counts[(int64_t)r * E + e];",
                               "run += counts[(int64_t)r * E + e];\n"
                               "            if (rank_off) rank_off[(int64_t)r * E + e] = (int32_t)run;"),
    "slot runs reversed": (_dispatch_pins, "int64_t p = cnt[s]++;",
                           "int64_t p = slot_off[s + 1] - 1 - (cnt[s]++ - slot_off[s]);"),
    "copy from the rank's first slot": (_sync_pins, "if (e >= E) return ORC_BAD_ARG;\n"
                                        "        int64_t home = (int64_t)(e / H) * HR + (e % H);\n"
                                        "        memcpy(W + (int64_t)s * slot_stride",
                                        "if (e >= E) return ORC_BAD_ARG;\n"
                                        "        int64_t home = (int64_t)(e / H) * HR;\n"
                                        "        memcpy(W + (int64_t)s * slot_stride"),
    "incremental skip inverted": (_sync_pins, "if (prev_slot_expert && prev_slot_expert[s] == e) continue;",
                                  "if (prev_slot_expert && prev_slot_expert[s] != e) continue;"),
    "restore skip inverted": (_restore_pins, "if (held_slot_expert && held_slot_expert[s] == e) continue;",
                              "if (held_slot_expert && held_slot_expert[s] != e) continue;"),
    "restore ignores the holder": (_restore_pins, "if (held_slot_expert && held_slot_expert[s] == e) continue;",
                                   "if (0) continue;"),
    "restore from the rank's first home slot": (_restore_pins,
                                                "const int64_t home_slot = (int64_t)(e / H) * HR + e % H;",
                                                "const int64_t home_slot = (int64_t)(e / H) * HR;"),
    "last replica's gradient dropped": (_grad_pins, "for (int i = rep_off[e] + 1; i < rep_off[e + 1]; ++i) {",
                                        "for (int i = rep_off[e] + 1; i < rep_off[e + 1] - 1; ++i) {"),
    "bf16 widened into the low half": (_grad_pins, "uint32_t u = (uint32_t)h << 16;", "uint32_t u = (uint32_t)h;"),
}


def _mutant(tmp_path, old, new):
    text = open(SRC).read()
    assert text.count(old) == 1, old
    src = tmp_path / "mutant.c"
    src.write_text(text.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-o", str(lib), str(src)],
                   check=True, capture_output=True)
    return oracle._open(str(lib))


def _passes(pins):
    try:
        pins()
    except (AssertionError, oracle.OracleError):
        return False
    return True


@pytest.mark.parametrize("pins", [_plan_pins, _variant_pins, _reroute_pins, _load_pins, _dispatch_pins, _sync_pins,
                                  _restore_pins, _grad_pins],
                         ids=lambda f: f.__name__)
def test_unchanged_copy_passes(tmp_path, monkeypatch, pins):
    monkeypatch.setattr(oracle, "_lib", _mutant(tmp_path, "int64_t j = occ[e]++;", "int64_t j = occ[e]++;"))
    assert _passes(pins)


@pytest.mark.parametrize("name", list(MUTANTS))
def test_mutant_is_caught(tmp_path, monkeypatch, name):
    pins, old, new = MUTANTS[name]
    monkeypatch.setattr(oracle, "_lib", _mutant(tmp_path, old, new))
    assert not _passes(pins), name
