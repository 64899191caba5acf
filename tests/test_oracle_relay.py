"""Pins for the oracle's weight sync across G GPUs with a relay (CPU only).

The relay mechanism against fan-out overload (UltraEP news summary, "Comment
fonctionne l'équilibrage en 300 microsecondes") is read as a scatter of the
expert's parts from its home to its consumer GPUs, then an all-gather of the
parts among them.  Checked by three hand-worked schedules
(tests/golden/relay_cases.json: every byte range of every round and every
GPU's egress), and on random plans by properties that do not restate the
schedule: after the rounds (or the one direct round) the slots equal the
single-GPU sync on tagged bytes, so a range taken from a GPU that had not yet
received it would leave stale bytes; one GPU's destinations of a round do not
depend on another's; over the rounds every GPU receives exactly the bytes the
direct form sends it, and the home of an expert sends each byte once (its
egress is at most the direct form's and at most the slot size per expert it
homes).
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
    # copies within one round read byte ranges that no copy of that round writes
    for dst, src, lo, hi in copies:
        W[dst, lo:hi] = W[src, lo:hi]


@pytest.mark.parametrize("case", _cases(), ids=lambda c: c["name"])
def test_relay_hand_cases(case):
    E, N, R, G, nb = case["E"], case["N"], case["R"], case["G"], case["nbytes"]
    se = np.array(case["slot_expert"], np.int32)
    S = se.size
    assert oracle.relay_rounds(G) == len(case["rounds"])
    W = _tagged(S, nb, 1)
    expect = W.copy()
    for rd in case["rounds"]:
        eg = oracle.sync_relay(W, nb, E, N, R, se, G, rd["round"])
        _apply(expect, rd["copies"])
        assert np.array_equal(W, expect), rd["round"]
        assert eg.tolist() == rd["egress"], rd["round"]
    full = _tagged(S, nb, 1)
    oracle.sync(full, nb, E, N, R, se)
    assert np.array_equal(W, full)
    Wd = _tagged(S, nb, 1)
    eg = oracle.sync_relay(Wd, nb, E, N, R, se, G, -1)
    expect = _tagged(S, nb, 1)
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
    S, nb = se.size, int(rng.choice([16, 48, 160, 1008]))
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


@pytest.mark.parametrize("seed", range(20))
def test_relay_bytes(seed):
    rng = np.random.default_rng(900 + seed)
    E, N, R, G, se = _random_plan(rng)
    S, nb = se.size, int(rng.choice([16, 96, 4000]))
    H, HR = E // N, E // N + R
    SG = S // G
    homes = np.zeros(G, np.int64)              # slot bytes of the replicated experts each GPU homes
    for e in np.unique(se[(np.arange(S) % HR >= H) & (se >= 0)]):
        if any((s // SG) != ((e // H) * HR) // SG for s in np.nonzero((se == e) & (np.arange(S) % HR >= H))[0]):
            homes[((e // H) * HR) // SG] += nb
    direct = oracle.sync_relay(_tagged(S, nb, 0), nb, E, N, R, se, G, -1)
    relay = [oracle.sync_relay(_tagged(S, nb, 0), nb, E, N, R, se, G, k) for k in range(oracle.relay_rounds(G))]
    # round 0 sends only from homes, each byte of an expert once
    assert (relay[0] <= homes).all() and (relay[0] <= direct).all()
    # received bytes per GPU are the same in both forms: total sent equal
    assert sum(r.sum() for r in relay) == direct.sum()
    # per GPU and destination: each GPU's destinations taken alone receive the same bytes
    for g in range(G):
        a = sum(oracle.sync_relay(_tagged(S, nb, 0), nb, E, N, R, se, G, k, g).sum()
                for k in range(oracle.relay_rounds(G)))
        assert a == oracle.sync_relay(_tagged(S, nb, 0), nb, E, N, R, se, G, -1, g).sum()


def test_relay_single_gpu_is_one_local_round():
    E, N, R = 8, 4, 2
    se = oracle.plan(np.array([40, 1, 1, 1, 1, 1, 1, 2], np.int32), N, R)["slot_expert"]
    assert oracle.relay_rounds(1) == 1 and oracle.relay_rounds(2) == 1 and oracle.relay_rounds(3) == 2
    assert oracle.relay_rounds(128) == 2
    full = _tagged(se.size, 16, 3)
    oracle.sync(full, 16, E, N, R, se)
    for rd in (-1, 0):
        W = _tagged(se.size, 16, 3)
        assert oracle.sync_relay(W, 16, E, N, R, se, 1, rd).tolist() == [0]
        assert np.array_equal(W, full)


def test_relay_rejects_bad_arguments():
    se = np.full(12, -1, np.int32)
    W = np.zeros((12, 16), np.uint8)
    for G, rd, dst in ((3, 0, -1), (0, 0, -1), (4, -2, -1), (4, 2, -1), (4, 0, 4)):
        with pytest.raises(oracle.OracleError):
            oracle.sync_relay(W, 16, 4, 4, 2, se, G, rd, dst)
