"""Pins for the oracle's load, reroute, weight-sync and grad-reduce steps (CPU only).

Each check uses something other than the oracle's own arithmetic: numpy
library routines (bincount, stable argsort, searchsorted), brute-force
counting, hand-worked cases (tests/golden/reroute_cases.json), a byte-map
conservation replay for the copy, and exactly representable (dyadic) values
whose sums have a closed form for the reduction.
"""
import json
import os

import numpy as np
import pytest

import oracle
from moe_expert_load_ue_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "reroute_cases.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


# ---- load -------------------------------------------------------------------

@pytest.mark.parametrize("w", [inputs.TINY, inputs.CLASS_671B.with_(tokens_per_rank=128),
                               inputs.EXTREME.with_(tokens_per_rank=32)], ids=lambda w: w.name)
def test_load_matches_bincount(w):
    ids = inputs.topk_ids(w, 0)
    counts, bad = oracle.load(ids, w.E, w.N)
    assert counts.shape == (w.N, w.E)
    assert (bad == 0).all()
    assert counts.sum() == w.T * w.K
    flat = ids.reshape(w.N, -1)
    for r in range(w.N):
        assert np.array_equal(counts[r], np.bincount(flat[r], minlength=w.E))
    ld, off = oracle.expert_load(counts)
    assert np.array_equal(ld, np.bincount(ids.ravel(), minlength=w.E))


def test_load_bad_ids_and_ragged_k():
    rng = np.random.default_rng(5)
    T, K, E, N = 60, 3, 10, 4
    ids = rng.integers(-3, E + 3, size=(T, K)).astype(np.int32)
    counts, bad = oracle.load(ids, E, N)
    tpr = T // N
    for r in range(N):
        blk = ids[r * tpr:(r + 1) * tpr].ravel()
        ok = blk[(blk >= 0) & (blk < E)]
        assert np.array_equal(counts[r], np.bincount(ok, minlength=E))
        assert bad[r] == blk.size - ok.size


def test_rank_offsets_brute_force():
    w = inputs.CLASS_106B.with_(tokens_per_rank=64)
    ids = inputs.topk_ids(w, 3)
    counts, _ = oracle.load(ids, w.E, w.N)
    ld, off = oracle.expert_load(counts)
    tpr = w.tokens_per_rank
    for r in (0, 1, 7, w.N - 1):
        before = ids[:r * tpr].ravel()
        for e in range(w.E):
            assert off[r, e] == np.count_nonzero(before == e)


def test_load_empty():
    ids = np.zeros((0, 8), np.int32)
    counts, bad = oracle.load(ids, 16, 4)
    assert counts.sum() == 0 and bad.sum() == 0


def test_balls_in_bins_imbalance_at_s0():
    """At s=0 every token picks K distinct experts uniformly, so a rank's load
    over T tokens is a sum of hypergeometric draws.  The busiest rank's mean
    over seeds must match an independent simulation of that law."""
    w = inputs.Workload("uniform", E=256, K=8, N=64, R=1, tokens_per_rank=64, s=0.0)
    rng = np.random.default_rng(99)
    ours, sims = [], []
    for seed in range(8):
        ids = inputs.topk_ids(w.with_(base_seed=seed), 0)
        counts, _ = oracle.load(ids, w.E, w.N)
        ld, _ = oracle.expert_load(counts)
        pl = oracle.plan(ld, w.N, w.R)
        ours.append(pl["rank_load_before"].max() / (w.L / w.N))
        draws = rng.multivariate_hypergeometric([w.H] * w.N, w.K, size=w.T).sum(axis=0)
        sims.append(draws.max() / (w.L / w.N))
    assert abs(np.mean(ours) - np.mean(sims)) < 0.04, (np.mean(ours), np.mean(sims))
    assert np.mean(ours) > 1.05      # the busiest rank sits well above the mean


# ---- reroute ----------------------------------------------------------------

@pytest.mark.parametrize("case", _golden(), ids=lambda c: c["name"])
def test_reroute_hand_cases(case):
    ids = np.array(case["ids"], np.int32).reshape(-1, case["K"])
    counts, _ = oracle.load(ids, case["E"], case["N"])
    assert counts.tolist() == case["counts"]
    ld, off = oracle.expert_load(counts)
    assert off.tolist() == case["rank_off"]
    pl = oracle.plan(ld, case["N"], case["R"])
    assert oracle.reroute(ids, case["E"], pl).ravel().tolist() == case["phys"]


def reroute_by_sort(ids, E, pl):
    """Independent restatement with library routines: a stable argsort gives
    each (t, k) its occurrence index j; searchsorted finds the covering replica."""
    flat = ids.ravel()
    phys = np.full(flat.shape, -1, np.int32)
    valid = (flat >= 0) & (flat < E)
    idx = np.nonzero(valid)[0]
    order = idx[np.argsort(flat[idx], kind="stable")]
    sorted_e = flat[order]
    starts = np.searchsorted(sorted_e, np.arange(E), side="left")
    j = np.arange(order.size) - starts[sorted_e]
    off = pl["rep_off"]
    for e in np.unique(sorted_e):
        sel = sorted_e == e
        cum = pl["rep_cum"][off[e]:off[e + 1]]
        i = np.searchsorted(cum, j[sel], side="right") - 1
        phys[order[sel]] = pl["rep_slot"][off[e] + i]
    return phys.reshape(ids.shape)


@pytest.mark.parametrize("w", [inputs.TINY, inputs.CLASS_106B.with_(tokens_per_rank=512),
                               inputs.CLASS_671B.with_(tokens_per_rank=256),
                               inputs.EXTREME.with_(tokens_per_rank=64)], ids=lambda w: w.name)
def test_reroute_second_check_and_invariants(w):
    ids = inputs.topk_ids(w, 1)
    out = oracle.rebalance(ids, w.E, w.N, w.R)
    pl, phys = out["plan"], out["phys"]
    assert np.array_equal(phys, reroute_by_sort(ids, w.E, pl))
    # every (t, k) lands on a slot holding its expert
    assert np.array_equal(pl["slot_expert"][phys], ids)
    # per-slot token counts equal the plan's quotas exactly
    assert np.array_equal(np.bincount(phys.ravel(), minlength=w.S), pl["slot_quota"])


def test_reroute_bad_ids():
    rng = np.random.default_rng(8)
    E, N, R = 12, 3, 1
    ids = rng.integers(-2, E + 2, size=(30, 4)).astype(np.int32)
    out = oracle.rebalance(ids, E, N, R)
    bad = (ids < 0) | (ids >= E)
    assert (out["phys"][bad] == -1).all()
    good = ~bad
    assert np.array_equal(out["plan"]["slot_expert"][out["phys"][good]], ids[good])


# ---- weight sync ------------------------------------------------------------

def _byte_map_check(before, after, E, N, R, slot_expert):
    """Replay the copy as descriptors over a byte map: each byte of each filled
    redundant slot must be covered exactly once, from the same offset of the
    expert's home slot; every other byte must be unchanged."""
    H = E // N
    HR = H + R
    S, B = before.shape
    cover = np.zeros((S, B), np.int32)
    expect = before.copy()
    for s in range(S):
        e = slot_expert[s]
        if s % HR >= H and e >= 0:
            home = (e // H) * HR + e % H
            cover[s] += 1
            expect[s] = before[home]
    filled = cover.any(axis=1)
    assert (cover[filled] == 1).all()
    return np.array_equal(after, expect)


def _tagged_slots(S, B):
    # every byte names its slot and offset, so a transposed or shifted copy is visible
    s = np.arange(S, dtype=np.uint32)[:, None]
    x = np.arange(B, dtype=np.uint32)[None, :]
    return ((s * 2654435761 + x * 40503 + (x >> 8)) & 0xFF).astype(np.uint8)


@pytest.mark.parametrize("R", [1, 2])
def test_sync_byte_map(R):
    E, N = 12, 4
    rng = np.random.default_rng(R)
    ld = rng.multinomial(3000, np.r_[[0.5], np.full(E - 1, 0.5 / (E - 1))]).astype(np.int32)
    pl = oracle.plan(ld, N, R)
    assert pl["info"][4] > 0
    S, B = N * (E // N + R), 4096
    W = _tagged_slots(S, B)
    before = W.copy()
    oracle.sync(W, B, E, N, R, pl["slot_expert"])
    assert _byte_map_check(before, W, E, N, R, pl["slot_expert"])


def test_sync_byte_map_catches_wrong_source():
    """Plant a mistake on the CPU (a copy from the wrong home slot) and check
    that the byte-map test rejects it while a byte count would not."""
    E, N, R = 8, 4, 1
    ld = np.array([40, 1, 1, 1, 1, 1, 1, 1], np.int32)
    pl = oracle.plan(ld, N, R)
    S, B = N * (E // N + R), 1024
    W = _tagged_slots(S, B)
    before = W.copy()
    wrong = pl["slot_expert"].copy()
    H, HR = E // N, E // N + R
    for s in range(S):
        if s % HR >= H and wrong[s] >= 0:
            wrong[s] = (wrong[s] + 1) % E        # copy from the next expert's home
    oracle.sync(W, B, E, N, R, wrong)
    assert (W != before).sum() > 0
    assert not _byte_map_check(before, W, E, N, R, pl["slot_expert"])


def test_sync_partial_bytes_and_stride():
    E, N, R = 4, 2, 1
    pl = oracle.plan(np.array([10, 2, 1, 3], np.int32), N, R)
    S, B = 6, 256
    W = _tagged_slots(S, B)
    before = W.copy()
    oracle.sync(W, 64, E, N, R, pl["slot_expert"])
    assert np.array_equal(W[5, :64], before[0, :64])     # slot 5 replicates e0 (home slot 0)
    assert np.array_equal(W[5, 64:], before[5, 64:])
    assert np.array_equal(np.delete(W, 5, axis=0), np.delete(before, 5, axis=0))


# ---- grad reduce ------------------------------------------------------------

def _setup_grads(E, N, R, P, bf16, rng):
    ld = rng.multinomial(5000, np.r_[[0.3, 0.2], np.full(E - 2, 0.5 / (E - 2))]).astype(np.int32)
    pl = oracle.plan(ld, N, R)
    # dyadic values: multiples of 2^-8 below 2^4, so every fp32 partial sum is exact
    master = (rng.integers(-4096, 4096, size=(E, P)) / 256.0).astype(np.float32)
    lim = 256 if bf16 else 4096          # bf16 holds 8 significant bits: |k| < 256 is exact
    g = (rng.integers(-lim + 1, lim, size=(N * R, P)) / 256.0).astype(np.float32)
    if bf16:
        gb = (g.view(np.uint32) >> 16).astype(np.uint16)
        assert np.array_equal((gb.astype(np.uint32) << 16).view(np.float32), g)
        return pl, master, gb, g
    return pl, master, g, g


@pytest.mark.parametrize("bf16", [False, True])
def test_grad_reduce_exact_dyadic(bf16):
    E, N, R, P = 8, 4, 2, 1000
    rng = np.random.default_rng(11)
    pl, master, g_in, g_val = _setup_grads(E, N, R, P, bf16, rng)
    H, HR = E // N, E // N + R
    expect = master.astype(np.float64)
    for s in range(N * HR):
        e = pl["slot_expert"][s]
        if s % HR >= H and e >= 0:
            expect[e] += g_val[(s // HR) * R + (s % HR - H)]
    out = master.copy()
    oracle.grad_reduce(out, g_in, P, E, N, R, pl)
    assert np.array_equal(out.astype(np.float64), expect)
    # experts without replicas are untouched
    M = pl["info"][3]
    untouched = np.setdiff1d(np.arange(E), pl["rep_experts"][:M])
    assert np.array_equal(out[untouched], master[untouched])


def test_grad_reduce_zero_grads_identity_and_order():
    E, N, R, P = 8, 2, 3, 513
    rng = np.random.default_rng(12)
    ld = np.array([300, 1, 1, 1, 1, 1, 1, 1], np.int32)
    pl = oracle.plan(ld, N, R)
    master = rng.standard_normal((E, P)).astype(np.float32)
    out = master.copy()
    oracle.grad_reduce(out, np.zeros((N * R, P), np.float32), P, E, N, R, pl)
    assert np.array_equal(out, master)
    # non-dyadic values: the sum must follow replica order with fp32 rounding
    g = (rng.standard_normal((N * R, P)) * 1e-3).astype(np.float32)
    out = master.copy()
    oracle.grad_reduce(out, g, P, E, N, R, pl)
    H, HR = E // N, E // N + R
    ref = master.copy()
    off = pl["rep_off"]
    for e in range(E):
        for i in range(off[e] + 1, off[e + 1]):
            s = pl["rep_slot"][i]
            ref[e] = np.add(ref[e], g[(s // HR) * R + (s % HR - H)], dtype=np.float32)
    assert np.array_equal(out, ref)


# ---- weight sync, incremental form -----------------------------------------------

def _plans_sequence(E, N, R, n, seed):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        p = rng.permutation(E) + 1.0
        ld = rng.multinomial(4000, (p ** -1.5) / (p ** -1.5).sum()).astype(np.int32)
        out.append(oracle.plan(ld, N, R))
    return out


@pytest.mark.parametrize("R", [1, 2])
def test_sync_delta_equals_full_sync_state(R):
    """After a sync under plan A, the incremental sync under plan B (prev = A)
    must leave the bytes a full sync under B leaves; slots whose expert did not
    change are not written; the copy count is the numpy count of changed slots."""
    E, N = 16, 4
    H, HR = E // N, E // N + R
    S, B = N * HR, 512
    plans = _plans_sequence(E, N, R, 6, seed=R)
    W = _tagged_slots(S, B)
    assert oracle.sync_delta(W, B, E, N, R, plans[0]["slot_expert"], None) == plans[0]["info"][4]
    for a, b in zip(plans, plans[1:]):
        full = W.copy()
        oracle.sync(full, B, E, N, R, b["slot_expert"])
        before = W.copy()
        n = oracle.sync_delta(W, B, E, N, R, b["slot_expert"], a["slot_expert"])
        assert np.array_equal(W, full)
        red = (np.arange(S) % HR) >= H
        changed = red & (b["slot_expert"] >= 0) & (b["slot_expert"] != a["slot_expert"])
        assert n == int(changed.sum())
        assert np.array_equal(W[~changed], before[~changed])      # unchanged slots untouched


def test_sync_delta_same_plan_copies_nothing_and_none_is_full():
    E, N, R = 8, 4, 1
    pl = oracle.plan(np.array([40, 1, 1, 1, 1, 1, 1, 9], np.int32), N, R)
    S, B = N * (E // N + R), 256
    W = _tagged_slots(S, B)
    before = W.copy()
    assert oracle.sync_delta(W, B, E, N, R, pl["slot_expert"], pl["slot_expert"]) == 0
    assert np.array_equal(W, before)
    n = oracle.sync_delta(W, B, E, N, R, pl["slot_expert"], None)
    assert n == pl["info"][4] > 0
    assert _byte_map_check(before, W, E, N, R, pl["slot_expert"])
