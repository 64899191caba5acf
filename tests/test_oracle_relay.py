"""Pins for the oracle's weight sync across G GPUs with a relay tree (CPU only).

The relay mechanism against fan-out overload (UltraEP news summary, "Comment
fonctionne l'équilibrage en 300 microsecondes") is read as a doubling tree
over each expert's holder GPUs.  Checked by three hand-worked schedules
(tests/golden/relay_cases.json: every copy of every round and every GPU's
egress), and on random plans by properties that do not restate the schedule:
after all max(1, ceil(log2 G)) rounds (or the one direct round) the slots equal the single-GPU
sync on tagged bytes, so a copy taken from a GPU that had not yet received
its own copy would leave stale bytes; the rounds of one GPU's destinations
are independent of the other GPUs' within a round; each GPU sends at most one
copy of an expert per round; relay and direct move the same number of expert
copies between GPUs, and the relay never sends more from one GPU in a round.
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "relay_cases.json")


def _cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


def _tagged(S, nbytes, seed):
    return np.random.default_rng(seed).integers(0, 256, size=(S, nbytes), dtype=np.uint8)


def _apply(W, copies):
    # copies within one round read slots that no copy of that round writes
    for dst, src in copies:
        W[dst] = W[src]


@pytest.mark.parametrize("case", _cases(), ids=lambda c: c["name"])
def test_relay_hand_cases(case):
    E, N, R, G = case["E"], case["N"], case["R"], case["G"]
    se = np.array(case["slot_expert"], np.int32)
    S = se.size
    assert oracle.relay_rounds(G) == len(case["rounds"])
    W = _tagged(S, 48, 1)
    expect = W.copy()
    for rd in case["rounds"]:
        eg = oracle.sync_relay(W, 48, E, N, R, se, G, rd["round"])
        _apply(expect, rd["copies"])
        assert np.array_equal(W, expect), rd["round"]
        assert eg.tolist() == rd["egress"], rd["round"]
    full = _tagged(S, 48, 1)
    oracle.sync(full, 48, E, N, R, se)
    assert np.array_equal(W, full)
    Wd = _tagged(S, 48, 1)
    eg = oracle.sync_relay(Wd, 48, E, N, R, se, G, -1)
    expect = _tagged(S, 48, 1)
    _apply(expect, case["direct"]["copies"])
    assert np.array_equal(Wd, expect) and np.array_equal(Wd, full)
    assert eg.tolist() == case["direct"]["egress"]


def _random_plan(rng):
    N = int(rng.choice([2, 4, 8, 16, 32, 64]))
    H = int(rng.integers(1, 4))
    R = int(rng.integers(1, 4))
    E = N * H
    s = float(rng.choice([0.8, 1.2, 2.0]))
    p = (rng.permutation(E) + 1.0) ** -s
    load = rng.multinomial(int(rng.integers(100, 20000)), p / p.sum()).astype(np.int32)
    Gs = [g for g in (1, 2, 4, 8, 16, 32, 64) if N % g == 0]
    return E, N, R, int(rng.choice(Gs)), oracle.plan(load, N, R)["slot_expert"]


@pytest.mark.parametrize("seed", range(30))
def test_relay_rounds_reach_the_full_sync(seed):
    rng = np.random.default_rng(500 + seed)
    E, N, R, G, se = _random_plan(rng)
    S, nb = se.size, 32
    full = _tagged(S, nb, seed)
    oracle.sync(full, nb, E, N, R, se)
    W = _tagged(S, nb, seed)
    Wd = W.copy()
    total = np.zeros(G, np.int64)
    for k in range(oracle.relay_rounds(G)):
        # one GPU's destinations at a time, in reverse GPU order: a round has no
        # dependency between GPUs
        Wg = W.copy()
        eg = sum(oracle.sync_relay(Wg, nb, E, N, R, se, G, k, g) for g in reversed(range(G)))
        egall = oracle.sync_relay(W, nb, E, N, R, se, G, k)
        assert np.array_equal(W, Wg) and np.array_equal(eg, egall)
        total += egall
    assert np.array_equal(W, full)
    direct = oracle.sync_relay(Wd, nb, E, N, R, se, G, -1)
    assert np.array_equal(Wd, full)
    assert total.sum() == direct.sum()
    # rounds past the last one copy nothing new
    W2 = W.copy()
    assert oracle.sync_relay(W2, nb, E, N, R, se, G, oracle.relay_rounds(G)).sum() == 0
    assert np.array_equal(W2, full)


@pytest.mark.parametrize("seed", range(20))
def test_relay_egress_bounds(seed):
    rng = np.random.default_rng(900 + seed)
    E, N, R, G, se = _random_plan(rng)
    S = se.size
    H, HR = E // N, E // N + R
    SG = S // G
    held = np.zeros((G, E), bool)          # GPU g holds expert e (home or a filled redundant slot)
    for s in range(S):
        if se[s] >= 0:
            held[s // SG, se[s]] = True
    direct = oracle.sync_relay(_tagged(S, 16, 0), 16, E, N, R, se, G, -1)
    for k in range(oracle.relay_rounds(G)):
        eg = oracle.sync_relay(_tagged(S, 16, 0), 16, E, N, R, se, G, k)
        assert (eg <= held.sum(axis=1)).all()          # at most one copy per held expert per round
        assert eg.max() <= direct.max()
    # every GPU other than the home that holds a copy of e receives exactly one
    assert direct.sum() == int((held.sum(axis=0) - 1).sum())


def test_relay_single_gpu_is_one_local_round():
    E, N, R = 8, 4, 2
    se = oracle.plan(np.array([40, 1, 1, 1, 1, 1, 1, 2], np.int32), N, R)["slot_expert"]
    assert oracle.relay_rounds(1) == 1 and oracle.relay_rounds(2) == 1 and oracle.relay_rounds(5) == 3
    full = _tagged(se.size, 16, 3)
    oracle.sync(full, 16, E, N, R, se)
    for rd in (-1, 0):
        W = _tagged(se.size, 16, 3)
        assert oracle.sync_relay(W, 16, E, N, R, se, 1, rd).tolist() == [0]
        assert np.array_equal(W, full)


def test_relay_rejects_bad_arguments():
    se = np.full(12, -1, np.int32)
    W = np.zeros((12, 16), np.uint8)
    for G, rd, dst in ((3, 0, -1), (0, 0, -1), (4, -2, -1), (4, 0, 4)):
        with pytest.raises(oracle.OracleError):
            oracle.sync_relay(W, 16, 4, 4, 2, se, G, rd, dst)
