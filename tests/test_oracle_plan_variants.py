"""Pins for the oracle's plan variants (CPU only).

REQUEUE re-queues a partly placed expert behind any expert with more overflow
left; SPREAD spreads a stuck expert's remainder over its replicas when slots
run out.  Checked by hand-worked cases (tests/golden/plan_variant_cases.json),
by every invariant of the base rule, by the brute-force optimum on tiny
inputs (no variant beats it; all reach it when slots do not run out), and by
a property of SPREAD: it never raises the busiest rank above the same greedy
without it (a stuck expert's home is full at Q and hosts no replica, so each
spread token lands on a rank no busier than that home would have been).
"""
import json
import os

import numpy as np
import pytest

import oracle
from test_oracle_plan import brute_force_optimum, check_plan_invariants

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "plan_variant_cases.json")
VARIANTS = (0, oracle.REQUEUE, oracle.SPREAD, oracle.REQUEUE | oracle.SPREAD)


def _cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _cases(), ids=lambda c: c["name"])
def test_variant_hand_cases(case):
    load = np.array(case["load"], np.int32)
    for v, exp in case["variants"].items():
        pl = oracle.plan(load, case["N"], case["R"], int(v))
        assert pl["slot_expert"].tolist() == exp["slot_expert"], v
        assert pl["slot_quota"].tolist() == exp["slot_quota"], v
        assert pl["rank_load_after"].tolist() == exp["rank_load_after"], v
        assert int(pl["info"][2] & 1) == exp["flag"], v
        check_plan_invariants(load, case["N"], case["R"], pl)


def _random_load(rng):
    N = int(rng.choice([1, 2, 3, 4, 8, 16, 32]))
    H = int(rng.integers(1, 6))
    R = int(rng.integers(0, 4))
    E = N * H
    s = float(rng.choice([0.0, 0.8, 1.2, 2.0, 3.0]))
    p = (rng.permutation(E) + 1.0) ** -s
    return rng.multinomial(int(rng.integers(0, 5000)), p / p.sum()).astype(np.int32), N, R


@pytest.mark.parametrize("seed", range(40))
def test_variant_invariants_random(seed):
    load, N, R = _random_load(np.random.default_rng(4321 + seed))
    for v in VARIANTS:
        check_plan_invariants(load, N, R, oracle.plan(load, N, R, v))


def test_variants_without_stuck_experts_match_the_base_loads():
    # with no slot running out, SPREAD changes nothing and every variant is optimal (max = Q)
    rng = np.random.default_rng(9)
    n = 0
    for _ in range(200):
        load, N, R = _random_load(rng)
        base = oracle.plan(load, N, R, 0)
        if base["info"][2] & 1:
            continue
        n += 1
        sp = oracle.plan(load, N, R, oracle.SPREAD)
        for f in oracle.PLAN_FIELDS:
            assert np.array_equal(sp[f], base[f]), f
    assert n > 20


def test_spread_never_raises_the_max():
    rng = np.random.default_rng(10)
    improved = 0
    for _ in range(400):
        load, N, R = _random_load(rng)
        for q in (0, oracle.REQUEUE):
            a = int(oracle.plan(load, N, R, q)["rank_load_after"].max())
            b = int(oracle.plan(load, N, R, q | oracle.SPREAD)["rank_load_after"].max())
            assert b <= a
            improved += b < a
    assert improved > 0


def test_variant_brute_force_gaps():
    """Every variant against the brute-force optimum on random tiny inputs:
    never better, equal whenever slots do not run out; the mean and worst
    gaps are printed (pytest -s) for the design notes."""
    rng = np.random.default_rng(77)
    gaps = {v: [] for v in VARIANTS}
    for trial in range(60):
        N = int(rng.choice([2, 3]))
        H = int(rng.integers(1, 3))
        R = 1 if N == 3 else int(rng.integers(1, 3))
        E = N * H
        load = rng.integers(0, 21, size=E).astype(np.int32)
        if trial % 3 == 0:
            load[rng.integers(E)] += 15
        opt = brute_force_optimum(load.tolist(), N, R)
        for v in VARIANTS:
            pl = oracle.plan(load, N, R, v)
            g = int(pl["rank_load_after"].max())
            assert g >= opt, v
            if not pl["info"][2] & 1:
                assert g == opt, v
            gaps[v].append(g / opt - 1.0 if opt else 0.0)
    for v in VARIANTS:
        print(f"variant {v}: mean gap {np.mean(gaps[v]):.4f}, worst {np.max(gaps[v]):.4f}")
    assert np.mean(gaps[oracle.REQUEUE | oracle.SPREAD]) <= np.mean(gaps[0])


def test_variant_rejects_bad_flags():
    with pytest.raises(oracle.OracleError):
        oracle.plan(np.ones(4, np.int32), 2, 1, 4)


def test_variant_brute_force_gaps_two_hot_experts():
    """Four ranks, one home expert and one redundant slot each, two hot
    experts competing for the slots: the variants' gaps to the optimum."""
    rng = np.random.default_rng(78)
    gaps = {v: [] for v in VARIANTS}
    for _ in range(60):
        load = rng.integers(0, 21, size=4).astype(np.int32)
        load[rng.integers(4, size=2)] += rng.integers(10, 30, size=2).astype(np.int32)
        opt = brute_force_optimum(load.tolist(), 4, 1)
        for v in VARIANTS:
            g = int(oracle.plan(load, 4, 1, v)["rank_load_after"].max())
            assert g >= opt, v
            gaps[v].append(g / opt - 1.0)
    for v in VARIANTS:
        print(f"two hot experts, variant {v}: mean gap {np.mean(gaps[v]):.4f}, worst {np.max(gaps[v]):.4f}")
    mean = {v: np.mean(gaps[v]) for v in VARIANTS}
    assert mean[oracle.REQUEUE | oracle.SPREAD] <= min(mean[oracle.REQUEUE], mean[oracle.SPREAD]) <= mean[0]
